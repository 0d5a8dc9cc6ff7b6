"""Host logic of bench.py that needs no GPU: the roofline traffic record is
used only while the code of the kernel sources it was measured on is
unchanged (comment-only edits keep it); the clock sampler's summary of the
timed region (median SM clock, throttle reasons) from nvidia-smi samples; the
reference arm's JSON line (it runs the oracle on the host, no GPU needed)."""
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


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` (the fp64 oracle on the host cores) prints one
    JSON line with the keys the benchmark contract names."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--workload", "tiny",
                          "--steps", "2", "--warmup", "1", "--ref-step-seconds", "0.2"],
                         capture_output=True, text=True, timeout=300, cwd=root,
                         env={k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")})
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e", "gpu_launches"):
        assert key in d, key
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["steps"] == 2 and d["warmup"] == 1 and d["higher_is_better"] is True
    assert d["config"]["workload"] == "tiny"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["gpu_launches"] == 0
    # the per-step time is the measured time of the sampled steps, which fits
    # in the run's wall time; the extrapolated whole-workload step is separate
    assert 0 < d["ms_per_step"] * d["steps"] < 60_000
    assert d["full_workload_step_ms_extrapolated"] > 0
    # both arms print the same config object for a workload
    sys.path.insert(0, root)
    import bench
    from sparse_attention_attn_b200 import inputs as I
    assert d["config"] == bench.workload_config(I.TINY, 1)


def test_watchdog_sync_stops_a_stuck_device(monkeypatch):
    """bench.device_sync polls an event and raises once the limit passes
    (a fake event that never completes stands in for a stuck device); a
    device that finishes returns normally."""
    import pytest
    import torch

    import bench

    class Never:
        def record(self):
            pass

        def query(self):
            return False

    class After:
        n = 0

        def record(self):
            pass

        def query(self):
            After.n += 1
            return After.n > 3

    synced = []
    monkeypatch.setattr(torch.cuda, "synchronize", lambda: synced.append(1))
    monkeypatch.setattr(torch.cuda, "Event", lambda *a, **k: Never())
    with pytest.raises(RuntimeError, match="watchdog"):
        bench.device_sync(limit_s=0.05)
    assert not synced
    monkeypatch.setattr(torch.cuda, "Event", lambda *a, **k: After())
    bench.device_sync(limit_s=5)
    assert synced == [1]
