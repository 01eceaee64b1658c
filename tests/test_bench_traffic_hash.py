"""bench.py reports a kernel's DRAM traffic from the committed ncu summary
only while the kernels it was taken from are the ones the sources compile
to.  The fingerprint is the GEMM translation unit with comments and blank
space left out: an edit to comments keeps it, an edit to code changes it.
Host logic only (no GPU)."""
import importlib
import os
import shutil

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    import bench
    return importlib.reload(bench)


def test_committed_traffic_matches_these_sources():
    bench = _bench()
    assert bench.ncu_traffic("llama3_8b_mlp", "F1_gate_up_swiglu") is not None
    assert bench.ncu_traffic("llama3_8b_mlp", "no_such_kernel") is None


def _copy_tree(tmp_path):
    for sub in ("lora_fine_tuning_mlp_b200/csrc", "include"):
        shutil.copytree(os.path.join(ROOT, sub), tmp_path / sub)
    return tmp_path / "lora_fine_tuning_mlp_b200" / "csrc" / "umma_gemm.cuh"


def test_comment_edits_keep_the_fingerprint_and_code_edits_change_it(tmp_path):
    bench = _bench()
    ref = bench.csrc_sha256()
    path = _copy_tree(tmp_path)
    bench.ROOT = str(tmp_path)
    try:
        assert bench.csrc_sha256() == ref
        text = path.read_text()
        path.write_text(text.replace("namespace lmlp {", "// a new comment line\nnamespace lmlp {  /* and one more */\n\n", 1))
        assert bench.csrc_sha256() == ref
        path.write_text(text.replace("constexpr int kBM = 128;", "constexpr int kBM = 64;", 1))
        assert bench.csrc_sha256() != ref
        # a header the translation unit includes counts as well
        hdr = tmp_path / "lora_fine_tuning_mlp_b200" / "csrc" / "ptx.cuh"
        path.write_text(text)
        assert bench.csrc_sha256() == ref
        hdr.write_text(hdr.read_text() + "\nnamespace lmlp { constexpr int kExtra = 1; }\n")
        assert bench.csrc_sha256() != ref
    finally:
        bench.ROOT = ROOT
