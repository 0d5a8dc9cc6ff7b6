"""GPU parity of RoPE with Position Interpolation before S2 attention (through
the C ABI) against the fp64 oracle in oracle/rope_ref.py.

* the (cos, sin) table and the rotation pass, element by element;
* small shapes, whole tensors: o, lse, the rotated q / k, and the gradients
  with respect to the unrotated q, k (both backward paths at head dim 128);
* full size in the benchmark's launch configuration, sampled units (whole
  groups, or first / last rows of long groups) -- with Position Interpolation
  from 4096 tokens, and at 100K tokens also without it (angles up to 1e5 rad).
Tolerances as in test_gpu_parity.py.  The GPU stores the rotated q, k as bf16
(the activations' type) before attention; the oracle rotates in fp64, and the
extra rounding stays inside the tolerances.
"""
import numpy as np
import pytest
import torch

import oracle.rope_ref as rr
from sparse_attention_attn_b200 import inputs as I
from tests.parity_util import check_grad, check_o, max_abs, to64

pytestmark = pytest.mark.gpu

L_TRAIN = 4096  # LLaMA2's trained context: Position Interpolation scales positions by L_TRAIN / N
WHOLE_GROUP_MAX = 8192  # longer groups are compared on their first and last rows


def _pi(N):
    return min(1.0, L_TRAIN / N)


def _bf16_bound(ref):
    # one bf16 rounding (half an ulp, 2^-9 relative) plus fp32 arithmetic
    return np.abs(ref) * 2.0 ** -8 + 1e-6


@pytest.fixture
def bwd_path(request):
    from sparse_attention_attn_b200 import _lib
    _lib.s2attn_set_tile_override(f"bwd={request.param}")
    yield request.param
    _lib.s2attn_set_tile_override(None)


@pytest.mark.parametrize("N,D,s", [(8192, 128, 0.5), (102400, 128, 1.0), (102400, 128, 0.04), (1024, 64, 1.0)])
def test_table_against_oracle(N, D, s):
    import sparse_attention_attn_b200 as s2
    tab = s2.rope_table(N, D, s).cpu().double().numpy()
    a = rr.rope_angles(N, D, s)
    assert np.abs(tab[..., 0] - np.cos(a)).max() < 2e-7
    assert np.abs(tab[..., 1] - np.sin(a)).max() < 2e-7


@pytest.mark.parametrize("D", [64, 128])
def test_rotation_pass_against_oracle(D):
    import sparse_attention_attn_b200 as s2
    x = I.randn_bf16((2, 1024, 3, D), 40)
    xd = x.cuda()
    tab = s2.rope_table(1024, D, 0.5)
    y = s2.rope_apply(xd, tab)
    ref = rr.rope_rotate(to64(x), 0.5)
    assert np.all(np.abs(to64(y) - ref) <= _bf16_bound(ref))
    yi = s2.rope_apply(y, tab, inverse=True)
    ref_i = rr.rope_rotate(to64(y), 0.5, inverse=True)
    assert np.all(np.abs(to64(yi) - ref_i) <= _bf16_bound(ref_i))
    s2.rope_apply(xd, tab, out=xd)   # in place gives the same bits
    torch.cuda.synchronize()
    assert torch.equal(xd, y)


def _run(shape, s, seed_offset=0):
    import sparse_attention_attn_b200 as s2
    q, k, v, do = I.make_inputs(shape, seed_offset)
    dev = torch.device("cuda:0")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    tab = s2.rope_table(shape.N, shape.D, s)
    o, lse, qr, kr = s2.s2attn_forward_rope(qd, kd, vd, shape.G, tab)
    dq, dk, dv = s2.s2attn_backward_rope(qr, kr, vd, o, lse, dod, shape.G, tab)
    torch.cuda.synchronize()
    assert s2.device_status() == 0
    return (q, k, v, do), (o, lse, qr, kr, dq, dk, dv)


ROPE_SMALL = [
    # (B, N, H, Hkv, D, G, path)
    (2, 512, 4, 2, 128, 256, "fused"), (2, 512, 4, 2, 128, 256, "split"), (2, 512, 4, 2, 128, 256, "split_ds"),
    (1, 2048, 2, 2, 128, 2048, "fused"), (1, 1536, 6, 2, 128, 768, "fused"),
    (1, 1024, 4, 4, 64, 256, "split"), (1, 768, 6, 2, 64, 256, "split_ds"),
]


@pytest.mark.parametrize("B,N,H,Hkv,D,G,bwd_path", ROPE_SMALL, indirect=["bwd_path"])
def test_small_whole_tensor(B, N, H, Hkv, D, G, bwd_path):
    shape = I.Shape("rope", B, H, Hkv, D, N, G)
    s = 0.5
    (q, k, v, do), (o, lse, qr, kr, dq, dk, dv) = _run(shape, s, seed_offset=17)
    q64, k64, v64, do64 = (to64(t) for t in (q, k, v, do))
    o_ref, lse_ref, qr_ref, kr_ref = rr.s2_rope_attention_fwd(q64, k64, v64, G, s)
    dq_ref, dk_ref, dv_ref = rr.s2_rope_attention_bwd(q64, k64, v64, do64, G, s)
    assert np.all(np.abs(to64(qr) - qr_ref) <= _bf16_bound(qr_ref))
    assert np.all(np.abs(to64(kr) - kr_ref) <= _bf16_bound(kr_ref))
    check_o(to64(o), o_ref, f" [{bwd_path}]")
    assert max_abs(to64(lse), lse_ref) < 1e-3
    check_grad("dQ", to64(dq), dq_ref, f" [{bwd_path}]")
    check_grad("dK", to64(dk), dk_ref, f" [{bwd_path}]")
    check_grad("dV", to64(dv), dv_ref, f" [{bwd_path}]")


def _check_full_size(shape, s, m, units):
    (q, k, v, do), (o, lse, _, _, dq, dk, dv) = _run(shape, s)
    q, k, v, do = (t.float().numpy() for t in (q, k, v, do))
    o, lse = o.cpu(), lse.cpu()
    dq, dk, dv = (t.float().cpu().numpy() for t in (dq, dk, dv))
    rep = shape.H // shape.Hkv
    pieces = [("whole", None)] if shape.G <= WHOLE_GROUP_MAX else [("prefix", m), ("suffix", m)]
    msgs = []
    for b, h, g in units:
        kh = h // rep
        for piece, mm in pieces:
            dk_ref = dv_ref = 0.0
            for h2 in range(kh * rep, (kh + 1) * rep):
                u = rr.s2_rope_unit(q, k, v, do, shape.G, b, h2, g, s, piece=piece, m=mm)
                rows = u["rows"]
                tag = f"[{piece} b{b} h{h2} g{g} s={s}]"
                msgs.append(check_o(to64(o[b, rows, h2]), u["o"], tag))
                assert max_abs(to64(lse[b, h2, rows]), u["lse"]) < 1e-3, tag
                msgs.append(check_grad("dQ", dq[b, rows, h2].astype(np.float64), u["dq"], tag))
                dk_ref = dk_ref + u["dk_part"]
                dv_ref = dv_ref + u["dv_part"]
            tag = f"[{piece} b{b} kvh{kh} g{g} s={s}]"
            msgs.append(check_grad("dK", dk[b, rows, kh].astype(np.float64), dk_ref, tag))
            msgs.append(check_grad("dV", dv[b, rows, kh].astype(np.float64), dv_ref, tag))
    print("\n".join(msgs))


def test_llama2_7b_8k_sampled():
    shape = I.LLAMA2_7B_8K   # Position Interpolation 4096 -> 8192 (s = 0.5)
    _check_full_size(shape, _pi(shape.N), 2048, [(0, 0, 0), (0, shape.H - 1, shape.N // shape.G - 1)])


@pytest.mark.slow
@pytest.mark.parametrize("s", [L_TRAIN / 102400, 1.0], ids=["pi", "no-pi"])
def test_100k_sampled(s):
    shape = I.LLAMA2_7B_100K
    _check_full_size(shape, s, 1024, [(0, shape.H - 1, shape.N // shape.G - 1)])


def test_autograd_wrapper_matches_direct_calls():
    """S2RopeAttention through torch autograd equals the direct calls."""
    import sparse_attention_attn_b200 as s2
    shape = I.Shape("rope-ag", 1, 4, 2, 128, 1024, 256)
    q, k, v, do = (t.to("cuda:0") for t in I.make_inputs(shape, seed_offset=19))
    tab = s2.rope_table(shape.N, shape.D, 0.5)
    o_ref, lse, qr, kr = s2.s2attn_forward_rope(q, k, v, shape.G, tab)
    dq_ref, dk_ref, dv_ref = s2.s2attn_backward_rope(qr, kr, v, o_ref, lse, do, shape.G, tab)
    qt, kt, vt = (t.clone().requires_grad_(True) for t in (q, k, v))
    o = s2.S2RopeAttention.apply(qt, kt, vt, shape.G, tab)
    o.backward(do)
    torch.cuda.synchronize()
    assert torch.equal(o.detach(), o_ref)
    assert torch.equal(qt.grad, dq_ref) and torch.equal(kt.grad, dk_ref) and torch.equal(vt.grad, dv_ref)
