"""The 64-key forward (double-buffered scores, selected with the plan
override fwd_bn=64) against the fp64 oracle: the small whole-tensor shapes of
test_gpu_parity.py, the chunk-wise and HGA modes (their forwards run through
the same kernel), and the LLaMA2-7B workload at full size on sampled units.
Tolerances as in test_gpu_parity.py."""
import pytest

import oracle.s2_ref as ref
import tests.test_gpu_hga as thga
import tests.test_gpu_parity as tpar
import tests.test_gpu_segment as tseg
from sparse_attention_attn_b200 import inputs as I
from tests.parity_util import check_grad, check_o, max_abs, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(params=["fwd_bn=64", "fwd_bn=64,fwd_order=pairs"])
def fwd64(request):
    from sparse_attention_attn_b200 import _lib
    _lib.s2attn_set_tile_override(request.param)
    yield request.param
    _lib.s2attn_set_tile_override(None)


@pytest.mark.parametrize("B,N,H,Hkv,D,G", tpar.SMALL)
def test_small_whole_tensor(fwd64, B, N, H, Hkv, D, G):
    shape = I.Shape("small", B, H, Hkv, D, N, G)
    (q, k, v, do), (o, lse, dq, dk, dv) = tpar._run(shape, seed_offset=7)
    q64, k64, v64, do64 = (to64(t) for t in (q, k, v, do))
    o_ref, lse_ref = ref.s2_attention_fwd(q64, k64, v64, G)
    dq_ref, dk_ref, dv_ref, _ = ref.s2_attention_bwd(q64, k64, v64, do64, G)
    check_o(to64(o), o_ref, f" [{fwd64}]")
    assert max_abs(to64(lse), lse_ref) < 1e-3
    check_grad("dQ", to64(dq), dq_ref)
    check_grad("dK", to64(dk), dk_ref)
    check_grad("dV", to64(dv), dv_ref)


@pytest.mark.parametrize("B,C,Nk,H,Hkv,D", tseg.SHAPES)
def test_segment_one_call(fwd64, B, C, Nk, H, Hkv, D):
    tseg.test_one_call_whole_tensor(B, C, Nk, H, Hkv, D)


@pytest.mark.parametrize("B,C,Nk,H,Hkv,D", tseg.SHAPES[:2])
def test_segment_two_pieces(fwd64, B, C, Nk, H, Hkv, D):
    tseg.test_two_pieces_merged(B, C, Nk, H, Hkv, D)


@pytest.mark.parametrize("B,N,H,Hkv,D,G,S", thga.HGA_SHAPES)
def test_hga(fwd64, B, N, H, Hkv, D, G, S):
    thga.test_whole_tensor(B, N, H, Hkv, D, G, S)


def test_hga_empty_lists(fwd64):
    thga.test_empty_lists_and_out_of_range_entries()


def test_workload_llama2_7b_sampled(fwd64):
    tpar._check_full_size(I.LLAMA2_7B_8K, m=2048)
