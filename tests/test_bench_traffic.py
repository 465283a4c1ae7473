"""The bench line's `roofline.traffic` rule, on the CPU: the DRAM bytes of an ncu
capture are reported only while the GEMM code they were taken on is unchanged.
The digest ignores comments and blank space and follows every code edit; the
algorithmic bytes beside it follow from the fused gate_up's operand sizes."""
import os
import shutil
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _copy_sources(tmp_path):
    dst = tmp_path / "fp8_quantized_linear_rms_b200" / "csrc"
    dst.mkdir(parents=True)
    for f in bench.GEMM_SOURCES:
        shutil.copy(os.path.join(ROOT, "fp8_quantized_linear_rms_b200", "csrc", f), dst / f)
    return dst


def test_digest_ignores_comments_and_follows_code(tmp_path, monkeypatch):
    dst = _copy_sources(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    base = bench.gemm_sources_digest()
    assert base == bench.gemm_sources_digest()            # deterministic
    p = dst / "fp8q_gemm.cu"
    src = p.read_text()
    p.write_text("// a comment line\n/* a block\n   comment */\n" + src.replace("\n", "\n\n", 3))
    assert bench.gemm_sources_digest() == base            # comments and blank lines only
    p.write_text(src.replace("constexpr int BK = 128;", "constexpr int BK = 64;", 1))
    assert bench.gemm_sources_digest() != base            # a code edit


def test_recorded_capture_is_for_the_bench_workload():
    (name, m), cap = next(iter(bench.TRAFFIC_CAPTURES.items()))
    assert name == "scaled_mm_blockwise_silu_quant" and m == bench.DEFAULT_M
    assert cap["read"] > 0 and cap["write"] > 0 and len(cap["sources_sha256"]) == 64
    # DRAM bytes within 1.5x of the algorithmic ones, not below the weights
    alg = bench.fused_gate_up_bytes(m)
    assert 2 * bench.I * bench.H <= cap["read"] + cap["write"] <= 1.5 * alg


def test_fused_gate_up_algorithmic_bytes():
    M, K, N2, I = 8192, bench.H, 2 * bench.I, bench.I
    want = M * K + N2 * K + 4 * M * (K // 128) + 4 * (N2 // 128) * (K // 128) + M * I + 4 * M * (I // 128)
    assert bench.fused_gate_up_bytes(M) == want == 521730560
