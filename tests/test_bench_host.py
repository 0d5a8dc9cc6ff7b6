"""Host logic of bench.py that needs no GPU: the roofline traffic record is
used only while the code of the kernel sources it was measured on is
unchanged (comment-only edits keep it)."""
import os

import bench


def test_recorded_traffic_matches_the_committed_tree():
    got = bench.recorded_traffic("s2_bwd_dkdv_kernel", "llama2-7b-n8192")
    assert got is None or got > 0
    assert bench.recorded_traffic("s2_bwd_dkdv_kernel", "no-such-workload") is None
    assert bench.recorded_traffic("no_such_kernel", "llama2-7b-n8192") is None


def test_recorded_traffic_follows_code_not_comments(tmp_path):
    root = tmp_path / "tree"
    (root / "profiles").mkdir(parents=True)
    csrc = root / "sparse_attention_attn_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text("// kernel\nint x = 1;  /* one */\n")
    digest = bench.source_digest(["k.cu"], str(csrc))
    (root / "profiles" / "dram_traffic_w.txt").write_text("# comment\n" f"kern w 100 23 {digest} k.cu\n")
    assert bench.recorded_traffic("kern", "w", root=str(root)) == 123
    # a comment-only edit: same code, the record stands
    (csrc / "k.cu").write_text("// the kernel, reworded\nint x = 1;\n")
    assert bench.recorded_traffic("kern", "w", root=str(root)) == 123
    # a code edit: the record no longer applies
    (csrc / "k.cu").write_text("// kernel\nint x = 2;\n")
    assert bench.recorded_traffic("kern", "w", root=str(root)) is None
    os.remove(csrc / "k.cu")
    assert bench.recorded_traffic("kern", "w", root=str(root)) is None
