"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

* a sweep of small shapes, whole tensors compared element by element;
* the five workload shapes and the dense (G = N) runs at full size, in the
  launch configuration the benchmark times: exact gradient identities on every
  (batch, kv-head, group) unit, and sampled units (for shifted heads including
  the wrap-around group) compared element by element with the oracle, every
  query head of the sampled kv-head included: whole groups up to 8192 rows,
  longer groups on their first rows (dK / dV with the longest accumulation) and
  last rows (O, lse, dQ of the rows with the most keys).

Tolerances: O max-abs 1e-2 and relative Frobenius 5e-3; dQ, dK, dV relative
Frobenius 1e-2 (bf16 inputs and outputs, fp32 accumulation).
"""
import numpy as np
import pytest
import torch

import oracle.s2_ref as ref
from sparse_attention_attn_b200 import inputs as I
from tests.parity_util import check_grad, check_identities, check_o, max_abs, rel_fro, report, to64

pytestmark = pytest.mark.gpu


def _run(shape: I.Shape, seed_offset=0):
    import sparse_attention_attn_b200 as s2
    q, k, v, do = I.make_inputs(shape, seed_offset)
    dev = torch.device("cuda:0")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o, lse = s2.s2attn_forward(qd, kd, vd, shape.G)
    dq, dk, dv = s2.s2attn_backward(qd, kd, vd, o, lse, dod, shape.G)
    assert s2.device_status() == 0
    torch.cuda.synchronize()
    return (q, k, v, do), (o, lse, dq, dk, dv)


SMALL = [
    # (B, N, H, Hkv, D, G)
    (1, 1024, 4, 4, 64, 256),     # the tiny workload shape
    (1, 128, 1, 1, 64, 128),      # one tile, dense
    (2, 512, 4, 2, 128, 256),     # GQA, shifted, two batches
    (1, 1024, 4, 1, 128, 1024),   # dense, one kv-head
    (1, 768, 6, 2, 64, 256),      # three query heads per kv-head, shifted
    (1, 512, 2, 2, 128, 512),     # dense, 4 tiles
    (1, 1024, 8, 4, 128, 512),    # shifted GQA, D=128
    (1, 512, 1, 1, 64, 256),      # H=1: every head shifted
    (1, 2048, 2, 2, 128, 2048),   # dense causal, 16 tiles
    (2, 1536, 4, 4, 64, 768),     # G/2 = 384: three-tile shift
    (1, 640, 2, 2, 64, 640),      # dense, 5 tiles: the last forward item has one query tile
    (1, 384, 3, 1, 128, 384),     # dense, 3 tiles, D=128, three query heads per kv-head
]


@pytest.fixture
def bwd_path(request):
    """Backward path forced through the plan override for the test's duration
    (head dim 128 has both; head dim 64 has the split path only)."""
    from sparse_attention_attn_b200 import _lib
    _lib.s2attn_set_tile_override(f"bwd={request.param}")
    yield request.param
    _lib.s2attn_set_tile_override(None)


SMALL_PATHS = [(*s, p) for s in SMALL
               for p in (("split_ds", "fused", "split") if s[4] == 128 else ("split_ds", "split"))]


@pytest.mark.parametrize("B,N,H,Hkv,D,G,bwd_path", SMALL_PATHS, indirect=["bwd_path"])
def test_small_whole_tensor(B, N, H, Hkv, D, G, bwd_path):
    shape = I.Shape("small", B, H, Hkv, D, N, G)
    (q, k, v, do), (o, lse, dq, dk, dv) = _run(shape, seed_offset=7)
    q64, k64, v64, do64 = (to64(t) for t in (q, k, v, do))
    o_ref, lse_ref = ref.s2_attention_fwd(q64, k64, v64, G)
    dq_ref, dk_ref, dv_ref, _ = ref.s2_attention_bwd(q64, k64, v64, do64, G)
    check_o(to64(o), o_ref)
    assert max_abs(to64(lse), lse_ref) < 1e-3
    check_grad("dQ", to64(dq), dq_ref)
    check_grad("dK", to64(dk), dk_ref)
    check_grad("dV", to64(dv), dv_ref)


# the split-dS backward with its dS workspace holding fewer (batch, kv head,
# group) units than there are: dK/dV in ranges of pairs (ranges that end inside
# a unit included), each followed by dQ for the units it completed, the slots
# reused from range to range
DS_RANGES = [
    ((2, 512, 4, 2, 128, 256), 2),    # 2 tiles a group: one pair a unit, 8 units
    ((1, 1024, 8, 4, 128, 512), 3),   # 4 tiles, 2 pairs a unit
    ((2, 1536, 4, 4, 64, 768), 2),    # 6 tiles, 3 pairs a unit: ranges of 4 pairs end inside units
    ((1, 640, 2, 2, 64, 640), 2),     # 5 tiles: the middle pair has one item
    ((1, 768, 6, 2, 64, 256), 4),     # three query heads per kv head
]


@pytest.mark.parametrize("shape,slots", DS_RANGES, ids=[f"{s}-slots{n}" for s, n in DS_RANGES])
def test_small_split_ds_ranges(shape, slots):
    from sparse_attention_attn_b200 import _lib
    B, N, H, Hkv, D, G = shape
    _lib.s2attn_set_tile_override(f"bwd=split_ds,ds_slots={slots}")
    try:
        assert _lib.s2attn_plan(B, H, Hkv, N, D, G, 148)["ds_slots"] == slots
        (q, k, v, do), (o, lse, dq, dk, dv) = _run(I.Shape("small", B, H, Hkv, D, N, G), seed_offset=11)
    finally:
        _lib.s2attn_set_tile_override(None)
    q64, k64, v64, do64 = (to64(t) for t in (q, k, v, do))
    dq_ref, dk_ref, dv_ref, _ = ref.s2_attention_bwd(q64, k64, v64, do64, G)
    tag = f" [ds_slots={slots}]"
    check_grad("dQ", to64(dq), dq_ref, tag)
    check_grad("dK", to64(dk), dk_ref, tag)
    check_grad("dV", to64(dv), dv_ref, tag)


PLAN_VARIANTS = [
    # every variant the per-shape plan can select, forced through the override
    (128, "fwd_order=pairs"), (128, "bwd=split,bwd_stages=2"), (128, "bwd=split,bwd_stages=3"),
    (128, "bwd=split_ds,bwd_stages=2"), (128, "bwd=fused"), (64, "fwd_order=pairs"), (64, "fwd_kv=4"),
    (64, "fwd_kv=6"), (64, "bwd=split,bwd_stages=4"), (64, "bwd=split_ds,bwd_stages=4"),
    (128, "fwd_bn=64"), (128, "fwd_bn=64,fwd_order=pairs"), (64, "fwd_bn=64"), (64, "fwd_bn=64,fwd_kv=12"),
    (128, "bwd=split_ds,ds_slots=2"), (128, "bwd=split_ds,ds_slots=3"), (64, "bwd=split_ds,ds_slots=2"),
    (128, "bwd_qtile=128"), (128, "bwd_qtile=128,bwd=split"), (64, "bwd_qtile=128"),
    (128, "bwd_qtile=128,ds_slots=3"),
]


@pytest.mark.parametrize("D,spec", PLAN_VARIANTS, ids=[f"d{d}-{s}" for d, s in PLAN_VARIANTS])
def test_plan_variants(D, spec):
    """Each selectable kernel variant (work order, K/V ring depth, backward path
    and stages) against the oracle on whole tensors: shifted GQA heads, two
    batches, groups of 16 tiles, more forward items (256) than a B200 has SMs
    and two or more backward items per CTA, so every CTA crosses from one item
    to the next (where the pipelines hand over between items)."""
    from sparse_attention_attn_b200 import _lib
    shape = I.Shape("plan", 2, 4, 2, D, 8192, 2048)
    _lib.s2attn_set_tile_override(spec)
    try:
        (q, k, v, do), (o, lse, dq, dk, dv) = _run(shape, seed_offset=13)
    finally:
        _lib.s2attn_set_tile_override(None)
    q64, k64, v64, do64 = (to64(t) for t in (q, k, v, do))
    o_ref, lse_ref = ref.s2_attention_fwd(q64, k64, v64, shape.G)
    dq_ref, dk_ref, dv_ref, _ = ref.s2_attention_bwd(q64, k64, v64, do64, shape.G)
    check_o(to64(o), o_ref, f" [{spec}]")
    assert max_abs(to64(lse), lse_ref) < 1e-3
    check_grad("dQ", to64(dq), dq_ref, f" [{spec}]")
    check_grad("dK", to64(dk), dk_ref, f" [{spec}]")
    check_grad("dV", to64(dv), dv_ref, f" [{spec}]")


@pytest.mark.parametrize("q_scale", [3.0, 0.0], ids=["large-scores", "equal-scores"])
def test_score_magnitudes(q_scale):
    """Scores three times larger than the N(0,1) workloads' (the running row
    maximum keeps growing, so the forward's lazy O rescale fires on many tiles)
    and all-equal scores (q = 0: uniform attention over each causal prefix).

    Peaked attention makes O close to single rows of V (|O| up to ~4), where one
    bf16 ulp of the output is 1/64: the element-wise bound is therefore 1e-2 plus
    half a bf16 ulp of the reference (2^-8 |ref|); the relative Frobenius bounds
    are the workloads' own.  A missed or doubled rescale would be off by a
    factor of 2^8 or more."""
    import sparse_attention_attn_b200 as s2
    shape = I.Shape("mag", 1, 4, 2, 128, 1024, 256)
    q, k, v, do = I.make_inputs(shape, seed_offset=11)
    q = (q.float() * q_scale).to(torch.bfloat16)
    dev = torch.device("cuda:0")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o, lse = s2.s2attn_forward(qd, kd, vd, shape.G)
    dq, dk, dv = s2.s2attn_backward(qd, kd, vd, o, lse, dod, shape.G)
    torch.cuda.synchronize()
    assert s2.device_status() == 0
    q64, k64, v64, do64 = (to64(t) for t in (q, k, v, do))
    o_ref, lse_ref = ref.s2_attention_fwd(q64, k64, v64, shape.G)
    dq_ref, dk_ref, dv_ref, _ = ref.s2_attention_bwd(q64, k64, v64, do64, shape.G)
    o64 = to64(o)
    assert rel_fro(o64, o_ref) <= 5e-3, report("O", o64, o_ref)
    assert np.all(np.abs(o64 - o_ref) <= 1e-2 + np.abs(o_ref) / 256), report("O", o64, o_ref)
    assert max_abs(to64(lse), lse_ref) < 1e-3 * max(1.0, q_scale)
    check_grad("dQ", to64(dq), dq_ref)
    check_grad("dK", to64(dk), dk_ref)
    check_grad("dV", to64(dv), dv_ref)


def _units(shape: I.Shape):
    """Sampled (b, h, g) units: an unshifted head's first group, the last head's
    last group (the wrap-around group when shifted), and a middle one.  Every
    query head of each sampled unit's kv-head is compared (all rep heads feed
    that kv-head's dK / dV)."""
    ng = shape.N // shape.G
    units = [(0, 0, 0), (shape.B - 1, shape.H - 1, ng - 1)]
    if shape.H > 2:
        units.append((0, shape.H // 2, ng // 2))
    return units


# Groups up to this many rows are compared whole (every row of every output);
# longer ones on their first and last m rows (prefix and suffix oracles).
WHOLE_GROUP_MAX = 8192


def _pieces(q, k, v, do, G, b, h, g, m):
    """Oracle pieces of unit (b, h, g): the whole group, or its first m rows
    (dK / dV of the keys with the longest accumulation: every later query row
    of the group reaches them) and its last m rows (O, lse, dQ of the query
    rows with the most keys)."""
    if G <= WHOLE_GROUP_MAX:
        return [("whole", ref.s2_unit(q, k, v, do, G, b, h, g))]
    return [("prefix", ref.s2_unit_prefix(q, k, v, do, G, b, h, g, m)),
            ("suffix", ref.s2_unit_suffix(q, k, v, do, G, b, h, g, m))]


def _check_full_size(shape: I.Shape, m: int, units=None):
    (q, k, v, do), (o, lse, dq, dk, dv) = _run(shape)
    # bf16 values are exact in float32; the oracle upcasts the slices it reads to float64
    q, k, v, do = (t.float().numpy() for t in (q, k, v, do))
    o, lse = o.cpu(), lse.cpu()
    dq, dk, dv = (t.float().cpu().numpy() for t in (dq, dk, dv))
    rep = shape.H // shape.Hkv
    msgs = [check_identities(shape, q, k, do, dq, dk, dv)]
    for b, h, g in (units or _units(shape)):
        kh = h // rep
        heads = range(kh * rep, (kh + 1) * rep)
        per_head = {h2: _pieces(q, k, v, do, shape.G, b, h2, g, m) for h2 in heads}
        for i, (what, u0) in enumerate(per_head[h]):
            rows = u0["rows"]
            dk_ref = np.zeros_like(u0["dk_part"])
            dv_ref = np.zeros_like(u0["dv_part"])
            for h2 in heads:
                u = per_head[h2][i][1]
                assert np.array_equal(u["rows"], rows)
                tag = f"[{what} {len(rows)} rows b{b} h{h2} g{g}]"
                msgs.append(check_o(to64(o[b, rows, h2]), u["o"], tag))
                assert max_abs(to64(lse[b, h2, rows]), u["lse"]) < 1e-3, tag
                msgs.append(check_grad("dQ", dq[b, rows, h2].astype(np.float64), u["dq"], tag))
                dk_ref += u["dk_part"]
                dv_ref += u["dv_part"]
            tag = f"[{what} {len(rows)} rows b{b} kvh{kh} g{g}, {rep} heads]"
            msgs.append(check_grad("dK", dk[b, rows, kh].astype(np.float64), dk_ref, tag))
            msgs.append(check_grad("dV", dv[b, rows, kh].astype(np.float64), dv_ref, tag))
    print("\n".join(msgs))


@pytest.mark.parametrize("shape", I.WORKLOADS[:4], ids=lambda s: s.name)
def test_workload_sampled(shape):
    _check_full_size(shape, m=2048)


@pytest.mark.parametrize("bwd_path", ["fused", "split"], indirect=True)
def test_workload_fused_backward_sampled(bwd_path):
    """The fused and the split (S and dP recomputed for dQ) backward paths,
    selectable through the plan, at full size."""
    _check_full_size(I.LLAMA2_7B_8K, m=2048)


@pytest.mark.slow
def test_workload_100k_sampled():
    _check_full_size(I.LLAMA2_7B_100K, m=1024)


@pytest.mark.parametrize("shape", [I.LLAMA2_7B_8K.dense()], ids=lambda s: s.name)
def test_dense_sampled(shape):
    _check_full_size(shape, m=1024)


@pytest.mark.slow
def test_dense_100k_sampled():
    # one unit: the prefix of a 102400-row group streams the whole group
    _check_full_size(I.LLAMA2_7B_100K.dense(), m=512, units=[(0, 0, 0)])


ODD_TILE_ORDERS = [(D, spec) for D in (128, 64) for spec in ("fwd_order=pairs", "fwd_order=snake",
                                                              "fwd_bn=64,fwd_order=pairs", "fwd_bn=64,fwd_order=snake")]


@pytest.mark.parametrize("D,spec", ODD_TILE_ORDERS, ids=[f"d{d}-{s}" for d, s in ODD_TILE_ORDERS])
def test_forward_orders_on_odd_tile_counts(D, spec):
    """Groups with an odd tile count end in an item without a second query
    tile.  In the equal-work pairs order every CTA takes such an item right
    after an item with two tiles (pair (0, last)), which once deadlocked the
    forward's issuer (it waited to release the missing tile's Q slot while
    that earlier item's second-tile work was still to issue).  Both orders
    and both key tiles against the oracle, several items per CTA."""
    import sparse_attention_attn_b200 as s2
    from sparse_attention_attn_b200 import _lib
    shape = I.Shape("odd", 2, 4, 2, D, 1152, 1152)  # dense, 9 tiles: items 0..4, item 4 without a second tile
    q, k, v, do = I.make_inputs(shape, seed_offset=21)
    _lib.s2attn_set_tile_override(spec)
    try:
        o, lse = s2.s2attn_forward(q.cuda(), k.cuda(), v.cuda(), shape.G)
        assert s2.device_status() == 0, f"device status after the forward [{spec}]"
    finally:
        _lib.s2attn_set_tile_override(None)
    o_ref, lse_ref = ref.s2_attention_fwd(to64(q), to64(k), to64(v), shape.G)
    check_o(to64(o), o_ref, f" [{spec}]")
    assert max_abs(to64(lse), lse_ref) < 1e-3


@pytest.mark.parametrize("shape", [I.Shape("agree", 2, 4, 2, 128, 2048, 512), I.Shape("agree64", 1, 6, 2, 64, 1536, 768),
                                   I.Shape("agree-odd-tiles", 1, 2, 2, 64, 640, 640),
                                   I.Shape("agree-odd-tiles-128", 2, 3, 1, 128, 640, 640),
                                   I.LLAMA2_7B_8K], ids=lambda s: s.name)
def test_backward_paths_agree_bitwise(shape):
    """The split backward (dQ recomputes S, P and dS), the split-dS backward
    (dQ from the dS the dK/dV kernel stored) and the split-dS backward in ranges
    (two units of dS at a time), each with 64-query sub-tiles or 128-query tiles
    in the dK/dV kernel, form every dS value with the same fp32 steps and bf16
    rounding and accumulate dK, dV and dQ over the same 16-deep steps in the
    same order: their gradients agree bit for bit."""
    import sparse_attention_attn_b200 as s2
    from sparse_attention_attn_b200 import _lib
    q, k, v, do = (t.cuda() for t in I.make_inputs(shape, 5))
    o, lse = s2.s2attn_forward(q, k, v, shape.G)
    outs = {}
    for spec in ("bwd=split", "bwd=split_ds", "bwd=split_ds,ds_slots=2", "bwd=split,bwd_qtile=128",
                 "bwd=split_ds,bwd_qtile=128", "bwd=split_ds,ds_slots=2,bwd_qtile=128"):
        _lib.s2attn_set_tile_override(spec)
        try:
            outs[spec] = s2.s2attn_backward(q, k, v, o, lse, do, shape.G)
            assert s2.device_status() == 0
        finally:
            _lib.s2attn_set_tile_override(None)
    ref_grads = outs.pop("bwd=split")
    for spec, grads in outs.items():
        for name, a, b in zip(("dq", "dk", "dv"), ref_grads, grads):
            assert torch.equal(a.view(torch.int16), b.view(torch.int16)), f"{name} differs under {spec}"


def test_launch_counts():
    from sparse_attention_attn_b200 import _lib
    import sparse_attention_attn_b200 as s2
    shape = I.Shape("lc", 1, 2, 2, 64, 512, 256)
    q, k, v, do = (t.cuda() for t in I.make_inputs(shape))
    o, lse = s2.s2attn_forward(q, k, v, shape.G)
    assert _lib.s2attn_last_launch_count() == 1
    s2.s2attn_backward(q, k, v, o, lse, do, shape.G)
    assert _lib.s2attn_last_launch_count() == 3
    # dS of 2 of the 4 units at once: two ranges of 2 pairs, each dK/dV + dQ
    _lib.s2attn_set_tile_override("ds_slots=2")
    try:
        s2.s2attn_backward(q, k, v, o, lse, do, shape.G)
        assert _lib.s2attn_last_launch_count() == 5
    finally:
        _lib.s2attn_set_tile_override(None)


def test_bounded_wait_times_out_cleanly():
    """A wait on an mbarrier nothing arrives at gives up after its limit and
    reports S2ATTN_ERR_DEVICE_TIMEOUT; the context stays usable."""
    from sparse_attention_attn_b200 import _lib
    st = torch.zeros(2, dtype=torch.int32, device="cuda")
    rc = _lib.s2attn_selftest_wait_timeout(st.data_ptr(), 20_000_000, torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert int(st[0]) == _lib.S2ATTN_ERR_DEVICE_TIMEOUT and int(st[1]) == 999
    # the context still works afterwards
    x = torch.ones(1024, device="cuda")
    assert float(x.sum()) == 1024.0


def test_forward_output_only_16_byte_aligned():
    """An output buffer that is 16- but not 32-byte aligned takes the 16-byte
    store path of the epilogue; it must give the same bits as the aligned one."""
    import sparse_attention_attn_b200 as s2
    shape = I.Shape("align", 1, 4, 2, 128, 1024, 256)
    q, k, v, _ = (t.to("cuda:0") for t in I.make_inputs(shape, seed_offset=3))
    o_ref, lse_ref = s2.s2attn_forward(q, k, v, shape.G)
    n = q.numel()
    buf = torch.empty(n + 64, dtype=torch.bfloat16, device="cuda:0")
    off = next(i for i in range(16) if (buf.data_ptr() + 2 * i) % 32 == 16)
    o16 = buf[off:off + n].view_as(q)
    assert o16.data_ptr() % 16 == 0 and o16.data_ptr() % 32 == 16
    o_got, lse_got = s2.s2attn_forward(q, k, v, shape.G, out=o16)
    torch.cuda.synchronize()
    assert s2.device_status() == 0
    assert torch.equal(o_got, o_ref) and torch.equal(lse_got, lse_ref)


def test_backward_gradients_only_16_byte_aligned():
    """dk / dv buffers that are 16- but not 32-byte aligned take the 16-byte
    store path of the dK/dV epilogue; the bits must match the aligned run."""
    import sparse_attention_attn_b200 as s2
    shape = I.Shape("align", 1, 4, 2, 128, 1024, 256)
    q, k, v, do = (t.to("cuda:0") for t in I.make_inputs(shape, seed_offset=5))
    o, lse = s2.s2attn_forward(q, k, v, shape.G)
    dq_ref, dk_ref, dv_ref = s2.s2attn_backward(q, k, v, o, lse, do, shape.G)

    def offset16(like):
        n = like.numel()
        buf = torch.empty(n + 64, dtype=like.dtype, device=like.device)
        off = next(i for i in range(16) if (buf.data_ptr() + 2 * i) % 32 == 16)
        return buf[off:off + n].view_as(like)

    dk16, dv16 = offset16(k), offset16(v)
    assert dk16.data_ptr() % 32 == 16 and dv16.data_ptr() % 32 == 16
    dq, dk, dv = s2.s2attn_backward(q, k, v, o, lse, do, shape.G, dk=dk16, dv=dv16)
    torch.cuda.synchronize()
    assert s2.device_status() == 0
    assert torch.equal(dq, dq_ref) and torch.equal(dk, dk_ref) and torch.equal(dv, dv_ref)


def test_binding_rejects_bad_operands():
    """Wrong dtypes, shapes, strides, group sizes, alignment and workspaces are
    refused before any launch, and the library stays usable afterwards."""
    import sparse_attention_attn_b200 as s2
    from sparse_attention_attn_b200 import _lib
    shape = I.Shape("reject", 1, 4, 2, 64, 512, 256)
    q, k, v, do = (t.to("cuda:0") for t in I.make_inputs(shape, seed_offset=7))
    with pytest.raises(ValueError, match="must be torch.bfloat16"):
        s2.s2attn_forward(q.float(), k, v, shape.G)
    with pytest.raises(ValueError, match="has shape"):
        s2.s2attn_forward(q, k[:, :256], v, shape.G)
    with pytest.raises(ValueError, match="contiguous"):
        s2.s2attn_forward(q.transpose(1, 2).contiguous().transpose(1, 2), k, v, shape.G)
    with pytest.raises(ValueError, match="CUDA tensor"):
        s2.s2attn_forward(q, k.cpu(), v, shape.G)
    with pytest.raises(_lib.S2AttnError) as e:
        s2.s2attn_forward(q, k, v, 192)  # N % G != 0
    assert e.value.status == _lib.S2ATTN_ERR_INVALID_ARG
    with pytest.raises(_lib.S2AttnError) as e:
        s2.s2attn_forward(q, k, v, 128)  # shifted groups need G % 256 == 0
    assert e.value.status == _lib.S2ATTN_ERR_UNSUPPORTED
    n = q.numel()
    buf = torch.empty(n + 8, dtype=torch.bfloat16, device="cuda:0")
    off = next(i for i in range(8) if (buf.data_ptr() + 2 * i) % 16 == 8)
    with pytest.raises(_lib.S2AttnError) as e:
        s2.s2attn_forward(q, k, v, shape.G, out=buf[off:off + n].view_as(q))
    assert e.value.status == _lib.S2ATTN_ERR_MISALIGNED
    o, lse = s2.s2attn_forward(q, k, v, shape.G)
    with pytest.raises(ValueError, match="workspace"):
        s2.s2attn_backward(q, k, v, o, lse, do, shape.G, workspace=torch.empty(1 << 20, dtype=torch.uint8))
    with pytest.raises(_lib.S2AttnError) as e:
        s2.s2attn_backward(q, k, v, o, lse, do, shape.G,
                           workspace=torch.empty(16, dtype=torch.uint8, device="cuda:0"))
    assert e.value.status == _lib.S2ATTN_ERR_WORKSPACE
    dq, dk, dv = s2.s2attn_backward(q, k, v, o, lse, do, shape.G)
    torch.cuda.synchronize()
    assert s2.device_status() == 0
    o_ref, _ = ref.s2_attention_fwd(to64(q), to64(k), to64(v), shape.G)
    assert rel_fro(to64(o), o_ref) <= 5e-3


def test_autograd_wrapper_matches_direct_calls():
    """S2Attention through torch autograd (its backward runs on autograd's
    worker thread) gives the direct calls' results bit for bit."""
    import sparse_attention_attn_b200 as s2
    shape = I.Shape("autograd", 1, 4, 2, 128, 1024, 256)
    q, k, v, do = (t.to("cuda:0") for t in I.make_inputs(shape, seed_offset=9))
    o_ref, lse = s2.s2attn_forward(q, k, v, shape.G)
    dq_ref, dk_ref, dv_ref = s2.s2attn_backward(q, k, v, o_ref, lse, do, shape.G)
    qt, kt, vt = (t.clone().requires_grad_(True) for t in (q, k, v))
    o = s2.s2_attn(qt, kt, vt, shape.G)
    o.backward(do)
    torch.cuda.synchronize()
    assert torch.equal(o.detach(), o_ref)
    assert torch.equal(qt.grad, dq_ref) and torch.equal(kt.grad, dk_ref) and torch.equal(vt.grad, dv_ref)
