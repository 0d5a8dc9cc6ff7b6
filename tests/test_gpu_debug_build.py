"""The debug build (libs2attn_debug.so: every computed global index checked
against its tensor in the kernels) on the GPU: on valid calls no check fires
(device status 0) and the outputs are bit-identical to the default build's,
for the S2 forward and backward (planned kernels, and the selectable 64-key
forward, 128-query-tile dK/dV and ranged split-dS backward), the HGA lists and
the NF4 projection.  Each
build runs in its own process (S2ATTN_DEBUG selects the library at import)."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r'''
import hashlib, json, sys
import numpy as np, torch
sys.path.insert(0, sys.argv[1])
import sparse_attention_attn_b200 as s2
from sparse_attention_attn_b200 import _lib, inputs as I
dev = torch.device("cuda:0")
out = {"debug": _lib.load().s2attn_debug_checks()}
h = lambda *ts: hashlib.sha256(b"".join(t.detach().cpu().contiguous().view(torch.uint8).numpy().tobytes() for t in ts)).hexdigest()
shape = I.Shape("dbg", 1, 4, 2, 128, 1024, 256)
q, k, v, do = (t.to(dev) for t in I.make_inputs(shape))
o, lse = s2.s2attn_forward(q, k, v, shape.G)
dq, dk, dv = s2.s2attn_backward(q, k, v, o, lse, do, shape.G)
torch.cuda.synchronize()
out["s2"] = h(o, lse, dq, dk, dv)
out["status_fwd"] = s2.device_status()
# the selectable kernels: 64-key forward, dK/dV with 128-query tiles, split-dS in ranges
_lib.s2attn_set_tile_override("fwd_bn=64,bwd_qtile=128,ds_slots=2")
o3, l3 = s2.s2attn_forward(q, k, v, shape.G)
g3 = s2.s2attn_backward(q, k, v, o3, l3, do, shape.G)
_lib.s2attn_set_tile_override(None)
torch.cuda.synchronize()
out["variants"] = h(o3, l3, *g3)
out["status_variants"] = s2.device_status()
sel = -torch.ones((1, 4, 2), dtype=torch.int32)
sel[0, 2, 0] = 1
sel[0, 3, :] = torch.tensor([0, 3], dtype=torch.int32)
hist = sel.to(dev)
o2, l2 = s2.hga_forward(q, k, v, 512, hist)
g2 = s2.hga_backward(q, k, v, o2, l2, do, 512, hist)
torch.cuda.synchronize()
out["hga"] = h(o2, l2, *g2)
codes, sq, c2 = (t.to(dev) for t in I.make_nf4_weights(4 * 128, 512, seed=9))
x = I.randn_bf16((1, 300, 512), 19).to(dev)
qkv = s2.nf4_qkv(x, codes, sq, c2, 2, 1, 128)
torch.cuda.synchronize()
out["nf4"] = h(*qkv)
out["status"] = s2.device_status()
print(json.dumps(out))
'''


def _run(debug: bool):
    env = dict(os.environ)
    env.pop("S2ATTN_DEBUG", None)
    if debug:
        env["S2ATTN_DEBUG"] = "1"
    r = subprocess.run([sys.executable, "-c", SCRIPT, ROOT], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    return json.loads(r.stdout.strip().splitlines()[-1])


def test_debug_build_agrees_and_no_check_fires():
    from sparse_attention_attn_b200 import build
    build.build(debug=True)
    rel, dbg = _run(False), _run(True)
    assert rel["debug"] == 0 and dbg["debug"] == 1
    assert dbg["status_fwd"] == 0 and dbg["status_variants"] == 0 and dbg["status"] == 0, dbg
    for key in ("s2", "variants", "hga", "nf4"):
        assert dbg[key] == rel[key], f"{key}: the debug build's outputs differ from the default build's"
