"""Host-side helpers of bench.py that decide what the bench line reports: the
source hash that ties a committed ncu summary to the kernel it measured (code
only, so that comments can be edited), and the look-up of that summary's DRAM
traffic, which must come back empty once the kernel's code has changed."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_code_only_drops_comments_and_blank_space_but_keeps_strings():
    src = 'int a;  // one\n/* two\n   lines */ asm("mov.u32 %0, %%smid; // kept");\n\n  int   b ;'
    assert bench.code_only(src) == 'int a; asm("mov.u32 %0, %%smid; // kept"); int b ;'
    assert bench.code_only('const char *s = "a \\" /* b */ c"; // tail') == 'const char *s = "a \\" /* b */ c";'
    assert bench.code_only("x = 1; /* unterminated") == "x = 1;"


def test_kernel_hash_ignores_comments_and_follows_code(tmp_path, monkeypatch):
    csrc = tmp_path / "nvfp4_w4a4_block_b200" / "csrc"
    csrc.mkdir(parents=True)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (csrc / "k.cuh").write_text("// a kernel\n__global__ void k() { int x = 1; }\n")
    h0 = bench.kernel_source_hash(("k.cuh",))
    (csrc / "k.cuh").write_text("// the same kernel, re-commented\n\n__global__ void k() {\n  int x = 1;  // one\n}\n")
    assert bench.kernel_source_hash(("k.cuh",)) == h0
    (csrc / "k.cuh").write_text("// a kernel\n__global__ void k() { int x = 2; }\n")
    assert bench.kernel_source_hash(("k.cuh",)) != h0


def test_committed_traffic_only_for_the_captured_code(tmp_path, monkeypatch):
    csrc = tmp_path / "nvfp4_w4a4_block_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (csrc / "k.cuh").write_text("__global__ void k() {}\n")
    h = bench.kernel_source_hash(("k.cuh",))
    (tmp_path / "profiles" / "k.md").write_text(f"dram bytes per launch: 1234\nkernel source hash: {h}\n")
    assert bench.committed_traffic("k.md", ("k.cuh",)) == 1234
    (csrc / "k.cuh").write_text("__global__ void k() { int y; }\n")
    assert bench.committed_traffic("k.md", ("k.cuh",)) is None
    assert bench.committed_traffic("missing.md", ("k.cuh",)) is None


def test_the_committed_decode_summary_matches_the_current_decode_kernel():
    """The decode GEMM's committed capture is the one the bench line's roofline
    traffic comes from; it must describe the kernel as it is now."""
    assert bench.committed_traffic("nvfp4_gemm_decode_kernel_m32.md", bench.DECODE_KERNEL_FILES) is not None
