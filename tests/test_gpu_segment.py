"""GPU parity of chunk-wise attention over detached earlier keys (segment
mode, through the C ABI) against the fp64 oracle in oracle/chunk_ref.py.

* one call over [earlier keys; own keys] (causal with a query offset):
  o, lse, dq and dk / dv of the chunk's own keys, whole tensors;
* the two-piece form: the detached segment (every key visible, dq only) and
  the chunk's own keys (causal), merged by log-sum-exp, dq summed;
* the merge itself element by element;
* a full-size chunk (the last 2048 rows of a 16384-token Qwen3-8B GQA
  sequence) on sampled heads.
Tolerances as in test_gpu_parity.py.
"""
import numpy as np
import pytest
import torch

import oracle.chunk_ref as cr
from sparse_attention_attn_b200 import inputs as I
from tests.parity_util import check_grad, check_o, max_abs, to64

pytestmark = pytest.mark.gpu


def _inputs(B, C, Nk, H, Hkv, D, seed):
    q = I.randn_bf16((B, C, H, D), seed)
    k = I.randn_bf16((B, Nk, Hkv, D), seed + 1)
    v = I.randn_bf16((B, Nk, Hkv, D), seed + 2)
    do = I.randn_bf16((B, C, H, D), seed + 3)
    return q, k, v, do


SHAPES = [
    # (B, C, Nk, H, Hkv, D): chunk rows, key rows
    (1, 512, 2048, 4, 4, 128), (2, 1024, 1536, 8, 2, 128), (1, 256, 256, 4, 2, 128),
    (1, 768, 4096, 4, 1, 64), (2, 384, 1152, 6, 3, 64),
]


@pytest.mark.parametrize("B,C,Nk,H,Hkv,D", SHAPES)
def test_one_call_whole_tensor(B, C, Nk, H, Hkv, D):
    import sparse_attention_attn_b200 as s2
    q, k, v, do = _inputs(B, C, Nk, H, Hkv, D, 50)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = s2.seg_forward(qd, kd, vd, causal=True)
    dq, dk, dv = s2.seg_backward(qd, kd, vd, o, lse, dod, causal=True)
    torch.cuda.synchronize()
    assert s2.device_status() == 0
    q64, k64, v64, do64 = (to64(t) for t in (q, k, v, do))
    o_ref, lse_ref = cr.chunk_attention_fwd(q64, k64, v64)
    dq_ref, dk_ref, dv_ref = cr.chunk_attention_bwd(q64, k64, v64, do64)
    check_o(to64(o), o_ref)
    assert max_abs(to64(lse), lse_ref) < 1e-3
    check_grad("dQ", to64(dq), dq_ref)
    check_grad("dK", to64(dk), dk_ref)
    check_grad("dV", to64(dv), dv_ref)


@pytest.mark.parametrize("B,C,Nk,H,Hkv,D", SHAPES[:2] + SHAPES[3:4])
def test_two_pieces_merged(B, C, Nk, H, Hkv, D):
    """The detached earlier keys and the chunk's own keys as separate pieces,
    merged by log-sum-exp (the autograd wrapper's path), against the one-call
    oracle."""
    import sparse_attention_attn_b200 as s2
    q, k, v, do = _inputs(B, C, Nk, H, Hkv, D, 60)
    c0 = Nk - C
    qd, dod = q.cuda(), do.cuda()
    kp, vp = k[:, :c0].contiguous().cuda(), v[:, :c0].contiguous().cuda()
    ka, va = k[:, c0:].contiguous().cuda(), v[:, c0:].contiguous().cuda()
    o_a, lse_a = s2.seg_forward(qd, kp, vp, causal=False)
    o_b, lse_b = s2.seg_forward(qd, ka, va, causal=True)
    o, lse = s2.lse_merge(o_a, lse_a, o_b, lse_b)
    dq, _, _ = s2.seg_backward(qd, kp, vp, o, lse, dod, causal=False)
    dq, dk, dv = s2.seg_backward(qd, ka, va, o, lse, dod, causal=True, dq=dq, dq_accumulate=True)
    torch.cuda.synchronize()
    assert s2.device_status() == 0
    q64, k64, v64, do64 = (to64(t) for t in (q, k, v, do))
    o_ref, lse_ref = cr.chunk_attention_fwd(q64, k64, v64)
    dq_ref, dk_ref, dv_ref = cr.chunk_attention_bwd(q64, k64, v64, do64)
    check_o(to64(o), o_ref, " [merged]")
    assert max_abs(to64(lse), lse_ref) < 1e-3
    check_grad("dQ", to64(dq), dq_ref, " [two pieces]")
    check_grad("dK", to64(dk), dk_ref)
    check_grad("dV", to64(dv), dv_ref)
    # each piece on its own against the oracle's segment attention
    oa_ref, la_ref = cr.segment_attention_fwd(q64, k64[:, :c0], v64[:, :c0], None)
    check_o(to64(o_a), oa_ref, " [detached piece]")
    assert max_abs(to64(lse_a), la_ref) < 1e-3
    # the autograd wrapper gives the same gradients
    qt = qd.clone().requires_grad_(True)
    kt, vt = ka.clone().requires_grad_(True), va.clone().requires_grad_(True)
    ot = s2.ChunkAttention.apply(qt, kt, vt, kp, vp)
    ot.backward(dod)
    check_o(to64(ot), o_ref, " [autograd]")
    check_grad("dQ", to64(qt.grad), dq_ref, " [autograd]")
    check_grad("dK", to64(kt.grad), dk_ref, " [autograd]")


@pytest.mark.parametrize("order", ["fwd_order=pairs", "fwd_order=snake"])
def test_odd_tile_chunk_both_orders(order):
    """A 9-tile chunk (the forward's last item has no second query tile) with
    enough units that the pairs order hands every CTA item 0 then that item:
    both pieces (detached keys, every key visible; own keys, causal) and the
    merge against the one-call oracle, under both forward work orders."""
    import sparse_attention_attn_b200 as s2
    from sparse_attention_attn_b200 import _lib
    B, C, Nk, H, Hkv, D = 2, 1152, 2304, 8, 2, 128
    q, k, v, do = _inputs(B, C, Nk, H, Hkv, D, 70)
    c0 = Nk - C
    qd = q.cuda()
    kp, vp = k[:, :c0].contiguous().cuda(), v[:, :c0].contiguous().cuda()
    ka, va = k[:, c0:].contiguous().cuda(), v[:, c0:].contiguous().cuda()
    _lib.s2attn_set_tile_override(order)
    try:
        o_a, lse_a = s2.seg_forward(qd, kp, vp, causal=False)
        o_b, lse_b = s2.seg_forward(qd, ka, va, causal=True)
        o, lse = s2.lse_merge(o_a, lse_a, o_b, lse_b)
        torch.cuda.synchronize()
        assert s2.device_status() == 0, f"device status [{order}]"
    finally:
        _lib.s2attn_set_tile_override(None)
    q64, k64, v64 = (to64(t) for t in (q, k, v))
    o_ref, lse_ref = cr.chunk_attention_fwd(q64, k64, v64)
    check_o(to64(o), o_ref, f" [merged, {order}]")
    assert max_abs(to64(lse), lse_ref) < 1e-3


def test_merge_elementwise():
    import sparse_attention_attn_b200 as s2
    B, N, H, D = 2, 256, 4, 128
    oa, ob = I.randn_bf16((B, N, H, D), 70), I.randn_bf16((B, N, H, D), 71)
    la = torch.randn(B, H, N, generator=torch.Generator().manual_seed(72)) * 3
    lb = torch.randn(B, H, N, generator=torch.Generator().manual_seed(73)) * 3
    lb[0, 0, :5] = float("-inf")                     # a piece with no visible key
    o, lse = s2.lse_merge(oa.cuda(), la.cuda(), ob.cuda(), lb.cuda())
    o_ref, lse_ref = cr.lse_merge(to64(oa), la.double().numpy(), to64(ob), lb.double().numpy())
    assert np.all(np.abs(to64(o) - o_ref) <= np.abs(o_ref) * 2.0 ** -8 + 1e-5)
    assert max_abs(to64(lse), lse_ref) < 1e-5
    # in place over the first piece
    oa_d, la_d = oa.cuda(), la.cuda()
    s2.lse_merge(oa_d, la_d, ob.cuda(), lb.cuda(), out=oa_d, lse=la_d)
    torch.cuda.synchronize()
    assert torch.equal(oa_d, o) and torch.equal(la_d, lse)


def test_full_size_chunk_sampled():
    """The last 2048 rows of a 16384-token Qwen3-8B GQA sequence (32 query
    heads, 8 kv heads): sampled heads against the oracle."""
    import sparse_attention_attn_b200 as s2
    B, C, Nk, H, Hkv, D = 1, 2048, 16384, 32, 8, 128
    q, k, v, do = _inputs(B, C, Nk, H, Hkv, D, 80)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = s2.seg_forward(qd, kd, vd, causal=True)
    dq, dk, dv = s2.seg_backward(qd, kd, vd, o, lse, dod, causal=True)
    torch.cuda.synchronize()
    assert s2.device_status() == 0
    rep = H // Hkv
    for kh in (0, Hkv - 1):
        hs = list(range(kh * rep, (kh + 1) * rep))
        q64 = to64(q[:, :, hs])
        k64, v64 = to64(k[:, :, kh:kh + 1]), to64(v[:, :, kh:kh + 1])
        o_ref, lse_ref = cr.chunk_attention_fwd(q64, k64, v64)
        dq_ref, dk_ref, dv_ref = cr.chunk_attention_bwd(q64, k64, v64, to64(do[:, :, hs]))
        check_o(to64(o[:, :, hs]), o_ref, f" [kvh{kh}]")
        assert max_abs(to64(lse[:, hs]), lse_ref) < 1e-3
        check_grad("dQ", to64(dq[:, :, hs]), dq_ref, f" [kvh{kh}]")
        check_grad("dK", to64(dk[:, :, kh:kh + 1]), dk_ref, f" [kvh{kh}]")
        check_grad("dV", to64(dv[:, :, kh:kh + 1]), dv_ref, f" [kvh{kh}]")
