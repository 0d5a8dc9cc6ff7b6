"""Host logic of bench.py that needs no GPU: the roofline traffic record is
used only while the kernel sources it was measured on are unchanged."""
import os

import bench


def test_recorded_traffic_matches_the_committed_tree():
    got = bench.recorded_traffic("s2_bwd_dkdv_kernel", "llama2-7b-n8192")
    assert got is None or got > 0
    assert bench.recorded_traffic("s2_bwd_dkdv_kernel", "no-such-workload") is None
    assert bench.recorded_traffic("no_such_kernel", "llama2-7b-n8192") is None


def test_recorded_traffic_is_dropped_when_a_source_changes(tmp_path):
    root = tmp_path / "tree"
    (root / "profiles").mkdir(parents=True)
    csrc = root / "sparse_attention_attn_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text("kernel v1\n")
    import hashlib
    h = hashlib.sha256()
    h.update(b"k.cu")
    h.update(b"kernel v1\n")
    (root / "profiles" / "dram_traffic_w.txt").write_text(
        "# comment\n" f"kern w 100 23 {h.hexdigest()} k.cu\n")
    assert bench.recorded_traffic("kern", "w", root=str(root)) == 123
    (csrc / "k.cu").write_text("kernel v2\n")
    assert bench.recorded_traffic("kern", "w", root=str(root)) is None
    os.remove(csrc / "k.cu")
    assert bench.recorded_traffic("kern", "w", root=str(root)) is None
