"""GPU parity of the activation-quantization entry points against the oracle.

Standalone group / per-token quant must match the oracle bit for bit (codes
and scales).  The producer-fused ops (RMSNorm, SiLU*mul) must meet the fused
tolerance (>= 99.9% identical codes, the rest within one step, scales within
1e-5 relative); their kernels are designed to be exact as well, and the tests
report how many codes differ.  Shapes span several groups and CTAs, ragged M,
padded leading dimensions and the full Qwen3-8B / 32B row lengths.
"""
import numpy as np
import pytest
import torch

import fp8q_inputs as inp
import oracle
from helpers import assert_fused_quant_close, codes_np, fused_quant_exact, to_dev_bf16

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import fp8_quantized_linear_rms_b200 as fq   # fails loudly if libfp8q.so is missing


def _layout_scales(s_gpu: torch.Tensor, layout: str) -> np.ndarray:
    s = s_gpu.cpu().numpy()
    return s.T.copy() if layout == "group_major" else s


@pytest.mark.parametrize("ue8m0", [False, True])
@pytest.mark.parametrize("per_token", [False, True])
@pytest.mark.parametrize("M,K", [(1, 128), (3, 2048), (37, 4096), (130, 5120), (5, 12288),
                                 (2, 25600)])
def test_group_quant_bit_exact(M, K, per_token, ue8m0):
    x = inp.heavy_tailed_bf16(1000 + M + K, M, K)
    g = K if per_token else 128
    q_ref, s_ref = oracle.group_quant(x, g, ue8m0)
    q, s = fq.fp8q_group_quant(to_dev_bf16(x), g, ue8m0)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(codes_np(q), q_ref)
    np.testing.assert_array_equal(s.cpu().numpy(), s_ref)


@pytest.mark.parametrize("layout", ["row_major", "group_major"])
def test_group_quant_layouts_and_padding(layout):
    M, K = 19, 1024
    x = inp.normal_bf16(7, (M, K))
    q_ref, s_ref = oracle.group_quant(x, 128)
    xd = to_dev_bf16(x, ld=K + 64)                      # padded rows (NaN padding is never read)
    qbig = torch.full((M, K + 32), 0x5A, dtype=torch.uint8, device="cuda")
    q = qbig[:, :K].view(torch.float8_e4m3fn)
    _, s = fq.fp8q_group_quant(xd, 128, q=q, scale_layout=layout)
    torch.cuda.synchronize()
    got = qbig.cpu().numpy()
    np.testing.assert_array_equal(got[:, :K], q_ref)
    assert np.all(got[:, K:] == 0x5A), "wrote past the row"
    np.testing.assert_array_equal(_layout_scales(s, layout), s_ref)


@pytest.mark.parametrize("ue8m0", [False, True])
def test_group_quant_edge_values(ue8m0):
    K = 512
    rows = [np.zeros(K), np.full(K, -0.0), np.full(K, 1e-30), np.full(K, 3e38),
            np.linspace(-1e4, 1e4, K), np.where(np.arange(K) % 2, 1e-8, -1e-8)]
    rows.append(np.concatenate([np.zeros(K - 1), [448.0]]))
    x = inp.to_bf16_bits(np.stack(rows))
    for g in (128, K):
        q_ref, s_ref = oracle.group_quant(x, g, ue8m0)
        q, s = fq.fp8q_group_quant(to_dev_bf16(x), g, ue8m0)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(codes_np(q), q_ref)
        np.testing.assert_array_equal(s.cpu().numpy(), s_ref)


@pytest.mark.parametrize("ue8m0", [False, True])
@pytest.mark.parametrize("per_token", [False, True])
@pytest.mark.parametrize("M,H", [(16, 2048), (33, 4096), (129, 5120)])
def test_rmsnorm_quant(M, H, per_token, ue8m0):
    x = inp.heavy_tailed_bf16(2000 + M + H, M, H)
    w = inp.rms_weight_bf16(3000 + H, H)
    g = H if per_token else 128
    q_ref, s_ref = oracle.rmsnorm_quant(x, w, 1e-6, g, ue8m0)
    q, s = fq.fp8q_rmsnorm_quant(to_dev_bf16(x), to_dev_bf16(w[None, :])[0], 1e-6, g, ue8m0)
    torch.cuda.synchronize()
    n = assert_fused_quant_close(codes_np(q), s.cpu().numpy(), q_ref, s_ref, "rmsnorm")
    print(f"rmsnorm M={M} H={H} g={g} ue8m0={ue8m0}: {n} differing codes")


def test_rmsnorm_quant_closed_forms(golden):
    # The hand-derived 128/256-wide case of the golden file, through the GPU.
    c = [c for c in golden["rmsnorm_quant"]["cases"] if c["name"] == "row_norm_group_scales"][0]
    x = np.concatenate([np.full(n, v, np.float32) for v, n in c["x_fill"]])[None, :]
    w = np.full(x.shape[1], c["w_fill"], np.float32)
    q, s = fq.fp8q_rmsnorm_quant(to_dev_bf16(inp.to_bf16_bits(x)),
                                 to_dev_bf16(inp.to_bf16_bits(w)[None, :])[0], c["eps"], 128)
    torch.cuda.synchronize()
    assert np.all(codes_np(q) == 126)
    want = [np.float32(np.float32(a) / np.float32(448.0)) for a in c["scale_num"]]
    np.testing.assert_array_equal(s.cpu().numpy()[0], np.array(want, np.float32))


@pytest.mark.parametrize("ue8m0", [False, True])
@pytest.mark.parametrize("per_token", [False, True])
@pytest.mark.parametrize("M,I", [(16, 1024), (7, 12288), (65, 4096)])
def test_silu_mul_quant(M, I, per_token, ue8m0):
    x = inp.normal_bf16(4000 + M + I, (M, 2 * I), std=3.0)
    g = I if per_token else 128
    q_ref, s_ref = oracle.silu_mul_quant(x, g, ue8m0)
    q, s = fq.fp8q_silu_mul_quant(to_dev_bf16(x), g, ue8m0)
    torch.cuda.synchronize()
    n = assert_fused_quant_close(codes_np(q), s.cpu().numpy(), q_ref, s_ref, "silu")
    print(f"silu M={M} I={I} g={g} ue8m0={ue8m0}: {n} differing codes")


def test_silu_mul_extreme_gates():
    # gates far in both tails (exp overflow in fp32 below -88), zeros and signed zeros
    I = 256
    g = np.concatenate([np.linspace(-120, 120, I - 4), [0.0, -0.0, -85.5, -200.0]])
    u = np.concatenate([np.linspace(-3, 3, I - 4), [5.0, -5.0, 1e-3, 7.0]])
    x = inp.to_bf16_bits(np.stack([np.concatenate([g, u]), np.concatenate([u, g])]))
    for gs in (128, I):
        q_ref, s_ref = oracle.silu_mul_quant(x, gs)
        q, s = fq.fp8q_silu_mul_quant(to_dev_bf16(x), gs)
        torch.cuda.synchronize()
        assert_fused_quant_close(codes_np(q), s.cpu().numpy(), q_ref, s_ref, "silu tails")


@pytest.mark.parametrize("I", [256, 12288])
def test_silu_mul_tiny_gate_large_up(I):
    # A gate so small that g / (1 + e^-g) is an fp32 subnormal, times an up
    # value large enough to lift the product back into the normal range: each
    # row's amax comes from such an element, so its bf16 value decides the
    # scale.  Codes and scales must equal the definition bit for bit.
    rng = np.random.default_rng(77)
    g = rng.normal(0.0, 1e-3, size=(4, I))
    u = rng.normal(0.0, 1e-3, size=(4, I))
    for r, (gv, uv) in enumerate([(2.0 ** -133, 2.0 ** 120), (-(2.0 ** -128), 2.0 ** 115),
                                  (2.0 ** -110, 2.0 ** 100), (3 * 2.0 ** -131, -(2.0 ** 118))]):
        g[r, 5 + r] = gv
        u[r, 5 + r] = uv
    x = inp.to_bf16_bits(np.concatenate([g, u], axis=1))
    for gs in (I, 128):
        q_ref, s_ref = oracle.silu_mul_quant(x, gs)
        with fused_quant_exact(True):
            q, s = fq.fp8q_silu_mul_quant(to_dev_bf16(x), gs)
            torch.cuda.synchronize()
        np.testing.assert_array_equal(s.cpu().numpy(), s_ref)
        np.testing.assert_array_equal(codes_np(q), q_ref)
        # default (fast) mode: the deciding elements are exact, so are the scales
        q, s = fq.fp8q_silu_mul_quant(to_dev_bf16(x), gs)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(s.cpu().numpy(), s_ref)
        assert_fused_quant_close(codes_np(q), s.cpu().numpy(), q_ref, s_ref, "silu tiny gates, fast")


@pytest.mark.parametrize("op", ["rmsnorm", "silu"])
def test_full_size_qwen3_32b_prefill(op):
    # Config: Qwen3-32B prefill, M = 8192 tokens, H = 5120, I = 25600, heavy-tailed
    # activations; every row checked.
    M = 8192
    if op == "rmsnorm":
        H = 5120
        x = inp.heavy_tailed_bf16(5001, M, H)
        w = inp.rms_weight_bf16(5002, H)
        for g in (H, 128):
            q_ref, s_ref = oracle.rmsnorm_quant(x, w, 1e-6, g)
            q, s = fq.fp8q_rmsnorm_quant(to_dev_bf16(x), to_dev_bf16(w[None, :])[0], 1e-6, g)
            torch.cuda.synchronize()
            n = assert_fused_quant_close(codes_np(q), s.cpu().numpy(), q_ref, s_ref, op)
            print(f"{op} g={g}: {n} differing codes of {q_ref.size}")
    else:
        I = 25600
        x = inp.heavy_tailed_bf16(5003, M, 2 * I)
        for g in (I, 128):
            q_ref, s_ref = oracle.silu_mul_quant(x, g)
            q, s = fq.fp8q_silu_mul_quant(to_dev_bf16(x), g)
            torch.cuda.synchronize()
            n = assert_fused_quant_close(codes_np(q), s.cpu().numpy(), q_ref, s_ref, op)
            print(f"{op} g={g}: {n} differing codes of {q_ref.size}")


def test_quant_zero_rows_is_noop():
    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    q, s = fq.fp8q_group_quant(x, 128)
    assert q.shape == (0, 256) and s.shape == (0, 2)


def test_quant_deterministic():
    x = to_dev_bf16(inp.heavy_tailed_bf16(6001, 64, 4096))
    w = to_dev_bf16(inp.rms_weight_bf16(6002, 4096)[None, :])[0]
    a = fq.fp8q_rmsnorm_quant(x, w, 1e-6, 128)
    for _ in range(5):
        b = fq.fp8q_rmsnorm_quant(x, w, 1e-6, 128)
        assert torch.equal(a[0].view(torch.uint8), b[0].view(torch.uint8))
        assert torch.equal(a[1], b[1])


@pytest.mark.parametrize("ue8m0", [False, True])
def test_group_scale_for_every_bf16_amax(ue8m0):
    # Every positive finite bf16 value is the amax of one 128-group (plus one
    # all-zero group): the kernel's scale must equal the oracle's IEEE division
    # fl32(max(amax, 1e-10)/448) (and its UE8M0 rounding) for every one of them,
    # and the codes of the group's other, smaller random elements must match.
    amax_bits = np.arange(1, 0x7F80, dtype=np.int64)            # 1 .. largest finite
    G = amax_bits.size + 1                                       # + an all-zero group
    g = np.random.default_rng(99)
    groups = np.zeros((G, 128), np.int64)
    groups[:-1] = g.integers(0, amax_bits[:, None], size=(G - 1, 128))  # smaller magnitudes
    groups[:-1, :] |= g.integers(0, 2, size=(G - 1, 128)) << 15        # random signs
    pos = g.integers(0, 128, size=G - 1)
    groups[np.arange(G - 1), pos] = amax_bits | (g.integers(0, 2, size=G - 1) << 15)
    x = groups.astype(np.uint16).reshape(G // 8, 8 * 128)
    q_ref, s_ref = oracle.group_quant(x, 128, ue8m0)
    q, s = fq.fp8q_group_quant(to_dev_bf16(x), 128, ue8m0)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(s.cpu().numpy(), s_ref)
    np.testing.assert_array_equal(codes_np(q), q_ref)


@pytest.mark.parametrize("ue8m0", [False, True, "packed"])
@pytest.mark.parametrize("per_token", [False, True])
@pytest.mark.parametrize("M,H", [(16, 2048), (33, 4096), (129, 5120), (3, 20480)])
def test_add_rmsnorm_quant(M, H, per_token, ue8m0):
    # residual add + RMSNorm quant: the updated residual is bit-exact (one
    # bf16 rounding of the sum), codes and scales meet the fused tolerance;
    # H = 20480 takes the shared-memory ring kernel.
    x = inp.heavy_tailed_bf16(7000 + M + H, M, H)
    r = inp.normal_bf16(7100 + M + H, (M, H), std=2.0)
    w = inp.rms_weight_bf16(7200 + H, H)
    g = H if per_token else 128
    q_ref, s_ref, r_ref = oracle.add_rmsnorm_quant(x, r, w, 1e-6, g, ue8m0)
    rd = to_dev_bf16(r, ld=H + 64)                   # padded residual rows
    q, s = fq.fp8q_add_rmsnorm_quant(to_dev_bf16(x), rd, to_dev_bf16(w[None, :])[0], 1e-6, g, ue8m0)
    torch.cuda.synchronize()
    got_r = rd.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    np.testing.assert_array_equal(got_r, r_ref)
    if ue8m0 == "packed":
        np.testing.assert_array_equal(s.cpu().numpy(), s_ref)
        assert_fused_quant_close(codes_np(q), np.zeros(1), q_ref, np.zeros(1), "add+rms packed")
    else:
        n = assert_fused_quant_close(codes_np(q), s.cpu().numpy(), q_ref, s_ref, "add+rms")
        print(f"add+rms M={M} H={H} g={g} ue8m0={ue8m0}: {n} differing codes")


def test_add_rmsnorm_quant_full_size_qwen3_32b():
    # Qwen3-32B prefill: M = 8192 tokens, H = 5120; every row checked
    M, H = 8192, 5120
    x = inp.heavy_tailed_bf16(7301, M, H)
    r = inp.heavy_tailed_bf16(7302, M, H)
    w = inp.rms_weight_bf16(7303, H)
    for g in (H, 128):
        q_ref, s_ref, r_ref = oracle.add_rmsnorm_quant(x, r, w, 1e-6, g)
        rd = to_dev_bf16(r)
        q, s = fq.fp8q_add_rmsnorm_quant(to_dev_bf16(x), rd, to_dev_bf16(w[None, :])[0], 1e-6, g)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(rd.view(torch.int16).cpu().numpy().view(np.uint16), r_ref)
        n = assert_fused_quant_close(codes_np(q), s.cpu().numpy(), q_ref, s_ref, "add+rms full")
        print(f"add+rms full g={g}: {n} differing codes of {q_ref.size}")
