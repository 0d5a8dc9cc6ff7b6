"""Pins for the HGA block-sparse oracle (oracle/hga_ref.py):
* no selected history: plain causal attention inside each segment (s2_ref's
  group attention with no shift, itself pinned to torch SDPA);
* every earlier tile selected: dense causal attention over the whole
  sequence for o, lse, dq (s2_ref at G = N);
* torch autograd with the historical keys detached (an explicit additive mask
  and a detached copy of k, v for the historical part);
* the history piece merged with the local piece by log-sum-exp is the whole;
* a planted mistake (historical keys not detached) fails.
"""
import math

import numpy as np
import pytest
import torch

import oracle.chunk_ref as cr
import oracle.hga_ref as hr
import oracle.s2_ref as ref


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _qkvdo(B, N, H, Hkv, D, seed):
    return _rand((B, N, H, D), seed), _rand((B, N, Hkv, D), seed + 1), _rand((B, N, Hkv, D), seed + 2), \
        _rand((B, N, H, D), seed + 3)


def test_no_history_is_segment_causal():
    B, N, G, H, Hkv, D = 1, 1024, 512, 2, 1, 4
    q, k, v, do = _qkvdo(B, N, H, Hkv, D, 1)
    sel = -np.ones((B, N // 256, 3), dtype=int)
    o, lse = hr.hga_attention_fwd(q, k, v, G, sel)
    dq, dk, dv = hr.hga_attention_bwd(q, k, v, do, G, sel)
    scale = 1 / math.sqrt(D)
    for h in range(H):
        for g in range(N // G):
            sl = slice(g * G, (g + 1) * G)
            og, lg, _ = ref.group_causal_attention(q[0, sl, h], k[0, sl, 0], v[0, sl, 0], scale)
            np.testing.assert_allclose(o[0, sl, h], og, atol=1e-12, rtol=0)
            np.testing.assert_allclose(lse[0, h, sl], lg, atol=1e-12, rtol=0)
            dqg, _, _, _ = ref.group_causal_attention_grad(q[0, sl, h], k[0, sl, 0], v[0, sl, 0], do[0, sl, h], scale)
            np.testing.assert_allclose(dq[0, sl, h], dqg, atol=1e-12, rtol=0)


def test_full_history_is_dense_causal():
    B, N, G, H, Hkv, D = 1, 1024, 256, 2, 2, 4
    q, k, v, do = _qkvdo(B, N, H, Hkv, D, 2)
    sel = -np.ones((B, N // 256, N // 128), dtype=int)
    for qb in range(N // 256):
        prev = (qb * 256 // G) * G // 128                 # tiles of every earlier segment
        sel[0, qb, :prev] = np.arange(prev)
    o, lse = hr.hga_attention_fwd(q, k, v, G, sel)
    dq, _, _ = hr.hga_attention_bwd(q, k, v, do, G, sel)
    o_d, lse_d = ref.s2_attention_fwd(q, k, v, G=N)
    dq_d, _, _, _ = ref.s2_attention_bwd(q, k, v, do, G=N)
    np.testing.assert_allclose(o, o_d, atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, lse_d, atol=1e-12, rtol=0)
    np.testing.assert_allclose(dq, dq_d, atol=1e-11, rtol=0)


def _sel_example(B, N, G, seed):
    rng = np.random.default_rng(seed)
    S = 3
    sel = -np.ones((B, N // 256, S), dtype=int)
    for b in range(B):
        for qb in range(N // 256):
            prev = (qb * 256 // G) * G // 128
            if prev:
                pick = rng.choice(prev, size=min(S, prev), replace=False)
                sel[b, qb, :len(pick)] = np.sort(pick)
    return sel


def test_autograd_with_detached_history():
    B, N, G, H, Hkv, D = 1, 1024, 512, 2, 1, 4
    q, k, v, do = _qkvdo(B, N, H, Hkv, D, 3)
    sel = _sel_example(B, N, G, 4)
    local, hist = hr.hga_visible(N, G, sel[0])
    qt, kt, vt = (torch.from_numpy(x).requires_grad_(True) for x in (q, k, v))
    kd, vd = kt.detach(), vt.detach()
    loc = torch.from_numpy(local)
    his = torch.from_numpy(hist)
    scale = 1 / math.sqrt(D)
    outs = []
    for h in range(H):
        sl = scale * (qt[0, :, h] @ kt[0, :, 0].T)       # local scores (gradient to k)
        sh = scale * (qt[0, :, h] @ kd[0, :, 0].T)       # historical scores (k detached)
        s = torch.where(loc, sl, torch.where(his, sh, torch.full_like(sl, -math.inf)))
        p = torch.softmax(s, dim=1)
        outs.append(torch.where(loc, p, 0.0) @ vt[0, :, 0] + torch.where(his, p, 0.0) @ vd[0, :, 0])
    ot = torch.stack(outs, dim=1)[None]
    ot.backward(torch.from_numpy(do))
    o, _ = hr.hga_attention_fwd(q, k, v, G, sel)
    dq, dk, dv = hr.hga_attention_bwd(q, k, v, do, G, sel)
    np.testing.assert_allclose(o, ot.detach().numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(dq, qt.grad.numpy(), atol=1e-11, rtol=0)
    np.testing.assert_allclose(dk, kt.grad.numpy(), atol=1e-11, rtol=0)
    np.testing.assert_allclose(dv, vt.grad.numpy(), atol=1e-11, rtol=0)


def test_history_and_local_pieces_merge():
    B, N, G, H, Hkv, D = 1, 1024, 512, 2, 2, 6
    q, k, v, _ = _qkvdo(B, N, H, Hkv, D, 5)
    sel = _sel_example(B, N, G, 6)
    o, lse = hr.hga_attention_fwd(q, k, v, G, sel)
    qb = 3                                               # rows 768..1023, segment 1
    rows = slice(qb * 256, (qb + 1) * 256)
    tiles = [t for t in sel[0, qb] if t >= 0]
    kh = np.concatenate([k[:, t * 128:(t + 1) * 128] for t in tiles], axis=1)
    vh = np.concatenate([v[:, t * 128:(t + 1) * 128] for t in tiles], axis=1)
    o_h, l_h = cr.segment_attention_fwd(q[:, rows], kh, vh, None)
    o_l, l_l = cr.segment_attention_fwd(q[:, rows], k[:, G:(qb + 1) * 256], v[:, G:(qb + 1) * 256], qb * 256 - G)
    om, lm = cr.lse_merge(o_h, l_h, o_l, l_l)
    np.testing.assert_allclose(om, o[:, rows], atol=1e-12, rtol=0)
    np.testing.assert_allclose(lm, lse[:, :, rows], atol=1e-12, rtol=0)


def test_planted_mistake_undetached_history_fails():
    """Letting the historical keys take gradients too (a plausible slip: the
    whole visibility mask in the key gradients) must change dk, dv -- the
    autograd pin above fixes the detached form."""
    B, N, G, H, Hkv, D = 1, 1024, 512, 2, 1, 4
    q, k, v, do = _qkvdo(B, N, H, Hkv, D, 7)
    sel = _sel_example(B, N, G, 8)
    _, dk, dv = hr.hga_attention_bwd(q, k, v, do, G, sel)
    local, hist = hr.hga_visible(N, G, sel[0])
    vis = local | hist
    scale = 1 / math.sqrt(D)
    dk_bad = np.zeros_like(dk)
    for h in range(H):
        s = np.where(vis, scale * (q[0, :, h] @ k[0, :, 0].T), -np.inf)
        p = np.exp(s - s.max(1, keepdims=True))
        p /= p.sum(1, keepdims=True)
        o = p @ v[0, :, 0]
        ds = p * (do[0, :, h] @ v[0, :, 0].T - np.sum(do[0, :, h] * o, 1)[:, None])
        dk_bad[0, :, 0] += scale * (ds.T @ q[0, :, h])
    assert np.abs(dk_bad - dk).max() > 1e-3


def test_rejects_selection_from_own_segment():
    q, k, v, _ = _qkvdo(1, 1024, 1, 1, 4, 9)
    sel = -np.ones((1, 4, 1), dtype=int)
    sel[0, 3, 0] = 5            # tile 5 = rows 640..767: inside segment 1 of the block at rows 768..1023
    with pytest.raises(ValueError):
        hr.hga_attention_fwd(q, k, v, 512, sel)
