"""GPU parity of fused_qk_norm_rope against the oracle.

The kernel computes in fp32 (the oracle in fp64, one rounding per output), so
the bar is the fused-op one of this library: at least 99.9% of the q/k
outputs bit-identical to the oracle, every other within one bf16 ulp, and the
v heads and every byte outside the qkv rows untouched.  Shapes: the Qwen3-8B
and Qwen3-32B attention layouts (32/64 q heads, 8 kv heads of 128), NeoX and
GPT-J pairing, head sizes 64 and 256, ragged token counts, padded rows,
positions across the whole cache.
"""
import numpy as np
import pytest
import torch

import fp8q_inputs as inp
import oracle
from helpers import to_dev_bf16

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import fp8_quantized_linear_rms_b200 as fq   # fails loudly if libfp8q.so is missing


def _cache(P, D):
    inv = 1.0 / (1e6 ** (np.arange(0, D, 2) / D))
    ang = np.arange(P)[:, None] * inv[None, :]
    return np.concatenate([np.cos(ang), np.sin(ang)], axis=1).astype(np.float32)


def _check(T, hq, hk, hv, D, neox, seed, pad=0, P=4096):
    g = np.random.default_rng(seed)
    W = (hq + hk + hv) * D
    qkv = inp.to_bf16_bits(g.uniform(-0.1, 0.1, size=(T, W)) * (1 + 30 * (g.random((T, W)) < 0.01)))
    qw, kw = inp.rms_weight_bf16(seed + 1, D), inp.rms_weight_bf16(seed + 2, D)
    cs = _cache(P, D)
    pos = g.integers(0, P, size=T).astype(np.int64)
    ref = oracle.qk_norm_rope(qkv, hq, hk, hv, D, 1e-6, qw, kw, cs, pos, neox)
    d = to_dev_bf16(qkv, ld=W + pad) if pad else to_dev_bf16(qkv)
    fq.fp8q_qk_norm_rope(d, hq, hk, hv, D, 1e-6, to_dev_bf16(qw[None, :])[0], to_dev_bf16(kw[None, :])[0],
                         torch.from_numpy(cs).cuda(), torch.from_numpy(pos).cuda(), neox)
    torch.cuda.synchronize()
    assert fq.fp8q_last_device_status() == fq.OK
    got = d.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    np.testing.assert_array_equal(got[:, (hq + hk) * D:], qkv[:, (hq + hk) * D:])     # v untouched
    qk, rq = got[:, :(hq + hk) * D], ref[:, :(hq + hk) * D]
    diff = qk != rq
    n = int(diff.sum())
    assert n <= 1e-3 * qk.size, f"{n} of {qk.size} outputs differ"
    if n:
        a = qk[diff].astype(np.int32)
        b = rq[diff].astype(np.int32)
        same_sign = (a & 0x8000) == (b & 0x8000)
        assert np.all(same_sign & (np.abs((a & 0x7FFF) - (b & 0x7FFF)) <= 1)), "an output moved by more than one ulp"
    return n


@pytest.mark.parametrize("neox", [True, False])
@pytest.mark.parametrize("T,hq,hk,hv", [(1, 32, 8, 8), (37, 32, 8, 8), (300, 64, 8, 8)])
def test_qk_norm_rope_qwen3_layouts(T, hq, hk, hv, neox):
    n = _check(T, hq, hk, hv, 128, neox, 100 + T + hq)
    print(f"T={T} hq={hq} neox={neox}: {n} outputs differ")


@pytest.mark.parametrize("D", [64, 256])
@pytest.mark.parametrize("neox", [True, False])
def test_qk_norm_rope_head_sizes(D, neox):
    _check(29, 6, 2, 2, D, neox, 200 + D)


def test_qk_norm_rope_padded_rows_and_canaries():
    # ld > width: the padding columns must stay as they are (NaN padding)
    T, hq, hk, hv, D = 17, 8, 2, 2, 128
    _check(T, hq, hk, hv, D, True, 300, pad=64)
    W = (hq + hk + hv) * D
    big = torch.full((T + 2, W + 64), 7.0, dtype=torch.bfloat16, device="cuda")
    view = big[1:T + 1, :W]
    cs = torch.from_numpy(_cache(16, D)).cuda()
    pos = torch.zeros(T, dtype=torch.int64, device="cuda")
    w = torch.ones(D, dtype=torch.bfloat16, device="cuda")
    fq.fp8q_qk_norm_rope(view, hq, hk, hv, D, 1e-6, w, w, cs, pos, True)
    torch.cuda.synchronize()
    assert torch.all(big[0] == 7.0) and torch.all(big[T + 1] == 7.0) and torch.all(big[:, W:] == 7.0)


def test_qk_norm_rope_full_size_qwen3_32b_prefill():
    # M = 8192 tokens of the Qwen3-32B qkv projection (64 q / 8 kv heads of 128)
    n = _check(8192, 64, 8, 8, 128, True, 400, P=32768)
    print(f"full size: {n} outputs differ")


def test_qk_norm_rope_bad_position_is_flagged():
    # a position outside the cache is not read: the token uses row 0 and the
    # device status word reports FP8Q_ERR_INVALID_ARG
    T, D = 3, 128
    x = torch.zeros((T, 3 * D), dtype=torch.bfloat16, device="cuda")
    w = torch.ones(D, dtype=torch.bfloat16, device="cuda")
    cs = torch.from_numpy(_cache(8, D)).cuda()
    pos = torch.tensor([0, 8, 2], dtype=torch.int64, device="cuda")
    fq.fp8q_qk_norm_rope(x, 1, 1, 1, D, 1e-6, w, w, cs, pos, True)
    assert fq.fp8q_last_device_status() == fq.ERR_INVALID_ARG
    assert fq.fp8q_last_device_status() == fq.OK
