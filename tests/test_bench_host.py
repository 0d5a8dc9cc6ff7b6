"""Host logic of bench.py that needs no GPU: the roofline traffic record is
used only while the code of the kernel sources it was measured on is
unchanged (comment-only edits keep it); the clock sampler's summary of the
timed region (median SM clock, throttle reasons) from nvidia-smi samples."""
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


class _FakeSmi:
    """Stands in for the nvidia-smi sampler: writes fixed sample lines."""

    LINES = [
        "0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n",
        "0, 1800, 1965, 990.5, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n",
        "0, 1900, 1965, 980.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n",
        "garbled line\n",
    ]

    def __init__(self, cmd, stdout=None, stderr=None):
        assert cmd[0] == "nvidia-smi"
        stdout.writelines(self.LINES)
        stdout.flush()

    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def test_clock_sampler_summary(monkeypatch, tmp_path):
    monkeypatch.setattr(bench.subprocess, "Popen", _FakeSmi)
    c = bench.ClockSampler(0)
    c.start()
    got = c.stop()
    assert got == {"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}
    assert not os.path.exists(c.path)  # the temporary sample file is removed
    kept = bench.ClockSampler(0, str(tmp_path))
    kept.start()
    assert kept.stop()["samples"] == 3
    assert os.path.exists(tmp_path / "clocks_rank0.csv")


def test_clock_sampler_without_nvidia_smi(monkeypatch):
    def missing(*a, **k):
        raise FileNotFoundError("nvidia-smi")
    monkeypatch.setattr(bench.subprocess, "Popen", missing)
    c = bench.ClockSampler(0)
    c.start()
    assert c.stop() is None
    assert not os.path.exists(c.path)
