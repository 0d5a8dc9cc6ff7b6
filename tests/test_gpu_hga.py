"""GPU parity of HGA-style block-sparse attention (through the C ABI) against
the fp64 oracle in oracle/hga_ref.py: each 256-row query block attends its
own segment causally plus the historical key tiles listed for it (detached).

Selections are seeded test inputs: random tiles of earlier segments, a
varying number per block, ended by -1.  Tolerances as in test_gpu_parity.py.
"""
import numpy as np
import pytest
import torch

import oracle.hga_ref as hr
from sparse_attention_attn_b200 import inputs as I
from tests.parity_util import check_grad, check_o, max_abs, to64

pytestmark = pytest.mark.gpu


def _selection(B, N, G, S, seed, fill=True):
    """int32 [B, N/256, S]: for each block up to S distinct tiles of earlier
    segments (sorted), the rest -1; some blocks get fewer than S."""
    rng = np.random.default_rng(seed)
    sel = -np.ones((B, N // 256, S), dtype=np.int32)
    if not fill:
        return sel
    for b in range(B):
        for qb in range(N // 256):
            prev = (qb * 256 // G) * G // 128
            n = min(S, prev, int(rng.integers(0, S + 1)) if qb % 3 == 0 else S)
            if n:
                sel[b, qb, :n] = np.sort(rng.choice(prev, size=n, replace=False))
    return sel


def _run(B, N, H, Hkv, D, G, sel, seed):
    import sparse_attention_attn_b200 as s2
    shape = I.Shape("hga", B, H, Hkv, D, N, G)
    q, k, v, do = I.make_inputs(shape, seed_offset=seed)
    dev = torch.device("cuda:0")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    hist = torch.from_numpy(sel).to(dev)
    o, lse = s2.hga_forward(qd, kd, vd, G, hist)
    dq, dk, dv = s2.hga_backward(qd, kd, vd, o, lse, dod, G, hist)
    torch.cuda.synchronize()
    assert s2.device_status() == 0
    return (q, k, v, do), (o, lse, dq, dk, dv)


HGA_SHAPES = [
    # (B, N, H, Hkv, D, G, S)
    (1, 1024, 4, 2, 128, 256, 3), (2, 2048, 4, 4, 128, 512, 4), (1, 1536, 6, 2, 64, 512, 5),
    (1, 2048, 2, 1, 128, 1024, 8),
]


@pytest.mark.parametrize("B,N,H,Hkv,D,G,S", HGA_SHAPES)
def test_whole_tensor(B, N, H, Hkv, D, G, S):
    sel = _selection(B, N, G, S, seed=N + S)
    (q, k, v, do), (o, lse, dq, dk, dv) = _run(B, N, H, Hkv, D, G, sel, 31)
    q64, k64, v64, do64 = (to64(t) for t in (q, k, v, do))
    o_ref, lse_ref = hr.hga_attention_fwd(q64, k64, v64, G, sel)
    dq_ref, dk_ref, dv_ref = hr.hga_attention_bwd(q64, k64, v64, do64, G, sel)
    check_o(to64(o), o_ref)
    assert max_abs(to64(lse), lse_ref) < 1e-3
    check_grad("dQ", to64(dq), dq_ref)
    check_grad("dK", to64(dk), dk_ref)
    check_grad("dV", to64(dv), dv_ref)


def test_empty_lists_and_out_of_range_entries():
    """All lists empty (-1) is local segment attention; entries that name a
    tile of the block's own or a later segment end its list (ignored)."""
    B, N, H, Hkv, D, G = 1, 1024, 4, 4, 128, 512
    sel = _selection(B, N, G, 2, 0, fill=False)
    (q, k, v, do), (o, lse, dq, dk, dv) = _run(B, N, H, Hkv, D, G, sel, 32)
    q64, k64, v64, do64 = (to64(t) for t in (q, k, v, do))
    o_ref, _ = hr.hga_attention_fwd(q64, k64, v64, G, sel)
    dq_ref, dk_ref, dv_ref = hr.hga_attention_bwd(q64, k64, v64, do64, G, sel)
    check_o(to64(o), o_ref)
    check_grad("dQ", to64(dq), dq_ref)
    check_grad("dK", to64(dk), dk_ref)
    sel2 = sel.copy()
    sel2[0, 2, 0] = 1                      # valid: tile 1 of segment 0 for block 2 (segment 1)
    sel2[0, 3, 0] = 6                      # own segment (tiles 4..7): ends block 3's list
    sel2[0, 3, 1] = 0
    (_, _, _, _), (o2, _, dq2, _, _) = _run(B, N, H, Hkv, D, G, sel2, 32)
    sel_eff = sel2.copy()
    sel_eff[0, 3, :] = -1                  # what the kernels are specified to use
    o_ref2, _ = hr.hga_attention_fwd(q64, k64, v64, G, sel_eff)
    dq_ref2, _, _ = hr.hga_attention_bwd(q64, k64, v64, do64, G, sel_eff)
    check_o(to64(o2), o_ref2, " [list ended by an own-segment tile]")
    check_grad("dQ", to64(dq2), dq_ref2)


def test_larger_selection_8k():
    """8192 tokens in 2048-row segments, 8 heads, up to 8 historical tiles
    (1024 tokens) per block; the LLaMA2-7B head layout."""
    B, N, H, Hkv, D, G, S = 1, 8192, 8, 8, 128, 2048, 8
    sel = _selection(B, N, G, S, seed=99)
    (q, k, v, do), (o, lse, dq, dk, dv) = _run(B, N, H, Hkv, D, G, sel, 33)
    q64, k64, v64, do64 = (to64(t) for t in (q, k, v, do))
    o_ref, lse_ref = hr.hga_attention_fwd(q64, k64, v64, G, sel)
    dq_ref, dk_ref, dv_ref = hr.hga_attention_bwd(q64, k64, v64, do64, G, sel)
    check_o(to64(o), o_ref)
    assert max_abs(to64(lse), lse_ref) < 1e-3
    check_grad("dQ", to64(dq), dq_ref)
    check_grad("dK", to64(dk), dk_ref)
    check_grad("dV", to64(dv), dv_ref)
