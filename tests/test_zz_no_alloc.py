"""The backward variant that allocates nothing (s2attn_bwd_noalloc).

It exists for callers that cannot allocate device memory for a workspace (code
under another runtime's memory budget without an allocator handle, plugin
hosts that forbid cudaMalloc, programs that must not allocate once set up):
its scratch is a fixed array inside the library.  This file is collected last
so that a run stopping at its first failure has already run every other test;
it also passes when run alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import oracle.s2_ref as ref
from sparse_attention_attn_b200 import inputs as I
from tests.parity_util import GRAD_REL_FRO, check_grad, rel_fro, to64

pytestmark = pytest.mark.gpu


def test_bwd_noalloc_matches_bwd_twice():
    import sparse_attention_attn_b200 as s2
    from sparse_attention_attn_b200 import _lib

    shape = I.Shape("noalloc", 2, 8, 4, 128, 1024, 256)  # shifted heads, GQA, two batches
    q, k, v, do = (t.cuda() for t in I.make_inputs(shape, seed_offset=3))
    o, lse = s2.s2attn_forward(q, k, v, shape.G)
    # the fp64 oracle on the same inputs, independent of either entry point
    dq_or, dk_or, dv_or, _ = ref.s2_attention_bwd(to64(q), to64(k), to64(v), to64(do), shape.G)
    # the existing entry point, with a caller-provided workspace
    dq_ref, dk_ref, dv_ref = s2.s2attn_backward(q, k, v, o, lse, do, shape.G)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):  # the scratch array keeps the last call's contents: run twice
        dq, dk, dv = (torch.full_like(t, float("nan")) for t in (q, k, v))
        rc = _lib.s2attn_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                     lse.data_ptr(), do.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                     dv.data_ptr(), shape.B, shape.H, shape.Hkv, shape.N, shape.D,
                                     shape.G, stream)
        assert rc == 0, _lib.status_string(rc)
        assert _lib.s2attn_last_launch_count() == 3
        torch.cuda.synchronize()
        for name, got, other, oracle_grad in (("dq", dq, dq_ref, dq_or), ("dk", dk, dk_ref, dk_or),
                                              ("dv", dv, dv_ref, dv_or)):
            g, r = to64(got), to64(other)
            assert np.isfinite(g).all(), (call, name)
            assert rel_fro(g, r) <= GRAD_REL_FRO, (call, name, rel_fro(g, r))
            check_grad(name, g, oracle_grad, f" [no-alloc call {call}]")


def test_bwd_noalloc_rejects_oversize_shape():
    from sparse_attention_attn_b200 import _lib

    t = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    p = t.data_ptr()
    # 64 heads x 131072 rows need ~64 MiB of scratch, more than the array holds:
    # rejected before anything is launched (the pointers are never read)
    rc = _lib.s2attn_bwd_noalloc(p, p, p, p, p, p, p, p, p, 1, 64, 64, 131072, 128, 131072,
                                 torch.cuda.current_stream().cuda_stream)
    assert rc == _lib.S2ATTN_ERR_WORKSPACE
