"""Pins for the chunk-wise attention oracle (oracle/chunk_ref.py), from facts
that do not come from it:
* a chunk with no earlier keys is plain dense causal attention (s2_ref at
  G = N, itself pinned to torch SDPA);
* the chunk's queries are the last rows of dense causal attention over the
  whole sequence, so o, lse and dq equal those rows of that attention, and dk,
  dv of the chunk's keys equal those rows when the earlier rows send no
  gradient (dO = 0 there);
* torch autograd with the earlier keys detached;
* merging the detached segment's and the chunk's own pieces by log-sum-exp
  gives the whole; merge is symmetric and a piece with lse = -inf is ignored.
"""
import numpy as np
import pytest
import torch

import oracle.chunk_ref as cr
import oracle.s2_ref as ref


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


@pytest.mark.parametrize("B,C,Nk,H,Hkv,D", [(1, 8, 8, 4, 4, 4), (2, 6, 20, 4, 2, 8), (1, 16, 48, 6, 3, 5)])
def test_chunk_is_the_tail_of_dense_causal(B, C, Nk, H, Hkv, D):
    q_all = _rand((B, Nk, H, D), 1)
    k, v = _rand((B, Nk, Hkv, D), 2), _rand((B, Nk, Hkv, D), 3)
    do_all = _rand((B, Nk, H, D), 4)
    do_all[:, : Nk - C] = 0.0                       # only the chunk's rows send gradient
    o_all, lse_all = ref.s2_attention_fwd(q_all, k, v, G=Nk)
    dq_all, dk_all, dv_all, _ = ref.s2_attention_bwd(q_all, k, v, do_all, G=Nk)
    q = q_all[:, Nk - C:]
    o, lse = cr.chunk_attention_fwd(q, k, v)
    np.testing.assert_allclose(o, o_all[:, Nk - C:], atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, lse_all[:, :, Nk - C:], atol=1e-12, rtol=0)
    dq, dk, dv = cr.chunk_attention_bwd(q, k, v, do_all[:, Nk - C:])
    np.testing.assert_allclose(dq, dq_all[:, Nk - C:], atol=1e-12, rtol=0)
    np.testing.assert_allclose(dk, dk_all[:, Nk - C:], atol=1e-12, rtol=0)
    np.testing.assert_allclose(dv, dv_all[:, Nk - C:], atol=1e-12, rtol=0)


def test_autograd_with_detached_past():
    B, C, Nk, H, Hkv, D = 1, 5, 12, 2, 1, 4
    q, k, v, do = _rand((B, C, H, D), 5), _rand((B, Nk, Hkv, D), 6), _rand((B, Nk, Hkv, D), 7), _rand((B, C, H, D), 8)
    qt = torch.from_numpy(q).requires_grad_(True)
    k_act = torch.from_numpy(k[:, Nk - C:].copy()).requires_grad_(True)
    v_act = torch.from_numpy(v[:, Nk - C:].copy()).requires_grad_(True)
    kk = torch.cat([torch.from_numpy(k[:, : Nk - C]), k_act], dim=1).repeat_interleave(H // Hkv, dim=2)
    vv = torch.cat([torch.from_numpy(v[:, : Nk - C]), v_act], dim=1).repeat_interleave(H // Hkv, dim=2)
    mask = torch.from_numpy(np.arange(Nk)[None, :] <= (Nk - C + np.arange(C))[:, None])
    ot = torch.nn.functional.scaled_dot_product_attention(qt.transpose(1, 2), kk.transpose(1, 2), vv.transpose(1, 2),
                                                          attn_mask=mask).transpose(1, 2)
    ot.backward(torch.from_numpy(do))
    o, _ = cr.chunk_attention_fwd(q, k, v)
    dq, dk, dv = cr.chunk_attention_bwd(q, k, v, do)
    np.testing.assert_allclose(o, ot.detach().numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(dq, qt.grad.numpy(), atol=1e-11, rtol=0)
    np.testing.assert_allclose(dk, k_act.grad.numpy(), atol=1e-11, rtol=0)
    np.testing.assert_allclose(dv, v_act.grad.numpy(), atol=1e-11, rtol=0)


def test_lse_merge_of_detached_and_own_segments():
    B, C, Nk, H, Hkv, D = 2, 7, 19, 4, 2, 6
    q, k, v = _rand((B, C, H, D), 9), _rand((B, Nk, Hkv, D), 10), _rand((B, Nk, Hkv, D), 11)
    c0 = Nk - C
    o_a, lse_a = cr.segment_attention_fwd(q, k[:, :c0], v[:, :c0], None)        # detached, all visible
    o_b, lse_b = cr.segment_attention_fwd(q, k[:, c0:], v[:, c0:], 0)           # own chunk, causal
    o, lse = cr.lse_merge(o_a, lse_a, o_b, lse_b)
    o_ref, lse_ref = cr.chunk_attention_fwd(q, k, v)
    np.testing.assert_allclose(o, o_ref, atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, lse_ref, atol=1e-12, rtol=0)
    o2, lse2 = cr.lse_merge(o_b, lse_b, o_a, lse_a)
    np.testing.assert_allclose(o2, o, atol=1e-14, rtol=0)
    o3, lse3 = cr.lse_merge(o_a, lse_a, o_b * 0 + 7.0, np.full_like(lse_b, -np.inf))
    np.testing.assert_allclose(o3, o_a, atol=0, rtol=0)
    np.testing.assert_allclose(lse3, lse_a, atol=0, rtol=0)


def test_planted_mistake_missing_past_fails():
    """Dropping the detached segment (attending the chunk's own keys only)
    must break the dense-tail pin."""
    B, C, Nk, H, D = 1, 6, 18, 2, 4
    q_all, k, v = _rand((B, Nk, H, D), 12), _rand((B, Nk, H, D), 13), _rand((B, Nk, H, D), 14)
    o_all, _ = ref.s2_attention_fwd(q_all, k, v, G=Nk)
    o_own, _ = cr.segment_attention_fwd(q_all[:, Nk - C:], k[:, Nk - C:], v[:, Nk - C:], 0)
    assert np.abs(o_own - o_all[:, Nk - C:]).max() > 1e-2
