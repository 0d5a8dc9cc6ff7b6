"""Multi-process host logic of bench.py on CPU: two gloo ranks (world size 2).

Covers the parts of an N-GPU run that are not GPU work: rendezvous on
127.0.0.1, the barrier, the max-over-ranks reduction of the step time, the
weak-scaling aggregate, and the reference arm where only rank 0 measures and
prints while the other ranks exit without work.
"""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


WORKER = r'''
import json, os, sys
sys.path.insert(0, {root!r})
import torch
import bench
world, rank, local = bench.dist_setup()
assert world == 2
# max over ranks of a per-rank "step time"
t = bench.max_over_ranks(1.0 + rank * 2.5, world, torch.device("cpu"))
bench.barrier(world)
out = {{"rank": rank, "max": t}}
# reference arm: only rank 0 runs the (tiny) oracle sample and prints
class A: pass
a = A(); a.gpus = 2; a.steps = 1; a.warmup = 0; a.ref_step_seconds = 0.0
from sparse_attention_attn_b200 import inputs as I
bench.run_reference(a, I.TINY, world, rank)
print("RESULT " + json.dumps(out), flush=True)
import torch.distributed as dist
dist.destroy_process_group()
'''


def test_two_gloo_ranks():
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                   WORLD_SIZE="2", LOCAL_RANK=str(rank), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, "-c", WORKER.format(root=ROOT)], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=240)
        assert p.returncode == 0, err[-2000:]
        outs.append(out)
    results = [json.loads(line[7:]) for o in outs for line in o.splitlines() if line.startswith("RESULT ")]
    assert sorted(r["rank"] for r in results) == [0, 1]
    assert all(r["max"] == pytest.approx(3.5) for r in results)
    # the reference line comes from rank 0 only
    ref0 = [json.loads(l) for l in outs[0].splitlines() if l.startswith("{")]
    ref1 = [l for l in outs[1].splitlines() if l.startswith("{")]
    assert len(ref0) == 1 and ref0[0]["impl"] == "reference" and ref0[0]["n_gpus"] == 2
    assert ref0[0]["cpu_baseline"]["kind"] == "oracle" and ref0[0]["e2e"]["h2d_bytes_per_step"] == 0
    assert ref1 == []
