"""Host logic of the variant tuner (`fp8_quantized_linear_rms_b200/tune.py`), on
the CPU: every candidate it would time is a variant the library accepts for
that shape, the candidate set follows the shape (Swap-AB only for small M,
split-K only when the tiles do not fill the SMs, CTA pairs only for per-token
scales at M >= 256), ties go to the simplest variant, and the table it writes
parses back, row for row, in the layout the library compiles in."""
import os
import re

import fp8_quantized_linear_rms_b200 as fq
from fp8_quantized_linear_rms_b200 import tune

SMS = 148
ROW = re.compile(r"\{(-?\d+), (\d+), (\d+), (\d+), (\d+), (\d+), (\d+), (\d+)\},")


def test_every_candidate_is_accepted_by_the_library():
    for _, K, N in tune.SHAPES:
        for M in tune.M_BUCKETS:
            for bw in (False, True):
                cands = tune.candidates(M, N, K, SMS, bw)
                assert cands and len(set(cands)) == len(cands)
                try:
                    for v in cands:
                        fq.fp8q_force_gemm_variant(*v)
                        got = fq.fp8q_select_gemm_variant(M, N, K, bw)
                        assert got == dict(zip(("swap_ab", "split_k", "block_n", "cta_pair"), v))
                        fq.fp8q_workspace_bytes(M, N, K, bw)
                finally:
                    fq.fp8q_force_gemm_variant()


def test_candidate_sets_follow_the_shape():
    # decode: the warp-MMA weight-streaming variant, and Swap-AB with the token
    # count padded to 16, split-K / stream-K because 48 weight tiles do not
    # fill the SMs
    c = tune.candidates(1, 6144, 4096, SMS, True)
    assert (1, 1, 8, 0) in c and (1, 1, 8, 0) not in tune.candidates(9, 6144, 4096, SMS, True)
    assert all(v[0] == 1 for v in c) and {v[2] for v in c} == {8, 16, 32}
    assert {v[1] for v in c} >= {1, 0, 2, 3}
    assert all(v[3] == 0 for v in c)
    # large M: no swap, whole-K tiles only once they fill the SMs, pairs for
    # per-token scales only
    pt = tune.candidates(2048, 24576, 4096, SMS, False)
    bw = tune.candidates(2048, 24576, 4096, SMS, True)
    assert all(v[0] == 0 and v[1] == 1 for v in pt + bw)
    assert (0, 1, 256, 1) in pt and all(v[3] == 0 for v in bw)
    # split factors are ones the library runs as asked: never more than the
    # K blocks, never one whose last split would be empty (9 of 32 blocks
    # runs as 8 splits of 4)
    for v in tune.candidates(32, 4096, 512, SMS, False):
        assert v[1] <= 4
    assert tune._effective_split(9, 32) == 8 and tune._effective_split(8, 32) == 8
    for M in (1, 16, 64):
        for v in tune.candidates(M, 5120, 4096, SMS, True):
            assert v[1] in (0, 1) or tune._effective_split(v[1], 32) == v[1]


def test_ties_go_to_the_simplest_variant():
    whole, split, streamk = (0, 1, 128, 0), (0, 4, 128, 0), (0, 0, 128, 0)
    assert tune._complexity(whole) < tune._complexity(split) < tune._complexity(streamk)


def test_written_table_parses_back(tmp_path):
    rows = [
        {"shape": "a", "blockwise": 0, "m_max": 1, "N": 6144, "K": 4096, "variant": [1, 3, 16, 0],
         "us": 12.4},
        {"shape": "b", "blockwise": 1, "m_max": 2048, "N": 24576, "K": 4096,
         "variant": [0, 1, 256, 0], "us": 274.4},
        {"shape": "c", "blockwise": 0, "m_max": 8192, "N": 4096, "K": 4096,
         "variant": [0, 1, 256, 1], "us": 95.8},
    ]
    path = os.path.join(tmp_path, "table.inc")
    tune.write_table(rows, path, device="NVIDIA B200")
    parsed = [tuple(int(x) for x in m.groups()) for m in map(ROW.match, open(path)) if m]
    assert parsed == [(r["blockwise"], r["m_max"], r["N"], r["K"], *r["variant"]) for r in rows]


def test_trials_go_round_the_candidates():
    # every trial times each candidate once, starting one candidate further
    # along each time; the result is each candidate's median
    runs = [("a", None), ("b", None), ("c", None)]
    order, clock = [], iter(range(100))
    def time_one(v, fns):
        order.append(v)
        return {"a": 10.0, "b": 20.0, "c": 30.0}[v] + next(clock) * 0.001
    got = tune._round_robin(runs, 4, time_one)
    assert order == ["a", "b", "c", "b", "c", "a", "c", "a", "b", "a", "b", "c"]
    assert set(got) == {"a", "b", "c"}
    assert 10 < got["a"] < 11 and 20 < got["b"] < 21 and 30 < got["c"] < 31
