"""Host-only checks of the C ABI (no GPU needed, nothing is launched).

* libs2attn.so loads and exports every function include/s2attn.h declares;
* status codes and their names;
* argument validation: every invalid argument returns its status code before
  any CUDA call is made (fake, never-dereferenced pointers are passed);
* workspace sizing.
"""
import ctypes
import os
import re

import pytest

from sparse_attention_attn_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "s2attn.h")

P = 0x10000  # a 16-byte aligned fake device address (never dereferenced)


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"S2ATTN_API\s+[\w\s\*]+?\b(s2attn_\w+)\s*\(", text)))


def test_header_declares_the_documented_entry_points():
    names = declared_functions()
    for required in ("s2attn_fwd", "s2attn_bwd", "s2attn_bwd_workspace_bytes", "s2attn_device_status",
                     "s2attn_status_string", "s2attn_bwd_noalloc"):
        assert required in names


def test_library_exports_every_declared_symbol():
    lib = _lib.load()
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert name in _lib.SIGNATURES, f"binding lacks {name}"


def test_status_strings():
    for code, name in ((0, "S2ATTN_OK"), (1, "S2ATTN_ERR_INVALID_ARG"), (2, "S2ATTN_ERR_UNSUPPORTED"),
                       (3, "S2ATTN_ERR_MISALIGNED"), (4, "S2ATTN_ERR_CUDA"), (5, "S2ATTN_ERR_DEVICE_TIMEOUT"),
                       (6, "S2ATTN_ERR_WORKSPACE")):
        assert _lib.status_string(code) == name
    assert _lib.status_string(99) == "S2ATTN_UNKNOWN_STATUS"


def fwd(q=P, k=P, v=P, o=P, lse=P, B=1, H=4, Hkv=4, N=1024, D=64, G=256):
    return _lib.s2attn_fwd(q, k, v, o, lse, B, H, Hkv, N, D, G, None)


def bwd(ptr=P, B=1, H=4, Hkv=4, N=1024, D=64, G=256, ws=P, wsb=1 << 30):
    return _lib.s2attn_bwd(ptr, ptr, ptr, ptr, ptr, ptr, ptr, ptr, ptr, B, H, Hkv, N, D, G, ws, wsb, None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), _lib.S2ATTN_ERR_INVALID_ARG),
    (dict(lse=None), _lib.S2ATTN_ERR_INVALID_ARG),
    (dict(B=0), _lib.S2ATTN_ERR_INVALID_ARG),          # empty batch is rejected, not a no-op
    (dict(N=0), _lib.S2ATTN_ERR_INVALID_ARG),
    (dict(H=-4), _lib.S2ATTN_ERR_INVALID_ARG),
    (dict(H=4, Hkv=3), _lib.S2ATTN_ERR_INVALID_ARG),   # H % Hkv
    (dict(N=1024, G=384), _lib.S2ATTN_ERR_INVALID_ARG),  # N % G
    (dict(N=1024, G=2048), _lib.S2ATTN_ERR_INVALID_ARG),  # G > N
    (dict(D=96), _lib.S2ATTN_ERR_UNSUPPORTED),
    (dict(D=256), _lib.S2ATTN_ERR_UNSUPPORTED),
    (dict(N=1000, G=1000), _lib.S2ATTN_ERR_UNSUPPORTED),  # ragged length (not a tile multiple)
    (dict(N=1536, G=384), _lib.S2ATTN_ERR_UNSUPPORTED),  # shift G/2 = 192 is not a whole tile
    (dict(H=6, Hkv=3, N=1024, G=256), _lib.S2ATTN_ERR_UNSUPPORTED),  # kv-head would mix shifts
    (dict(q=P + 8), _lib.S2ATTN_ERR_MISALIGNED),
    (dict(o=P + 4), _lib.S2ATTN_ERR_MISALIGNED),
])
def test_forward_argument_validation(kw, status):
    assert fwd(**kw) == status
    assert _lib.s2attn_last_launch_count() == 0


def test_backward_argument_validation():
    assert bwd(ptr=None) == _lib.S2ATTN_ERR_INVALID_ARG
    assert bwd(D=80) == _lib.S2ATTN_ERR_UNSUPPORTED
    assert bwd(ptr=P + 2) == _lib.S2ATTN_ERR_MISALIGNED
    need = _lib.s2attn_bwd_workspace_bytes(1, 4, 4, 1024, 64, 256)
    assert bwd(ws=None) == _lib.S2ATTN_ERR_WORKSPACE
    assert bwd(wsb=need - 1) == _lib.S2ATTN_ERR_WORKSPACE
    assert bwd(ws=P + 16) == _lib.S2ATTN_ERR_WORKSPACE  # workspace must be 256-byte aligned
    assert _lib.s2attn_last_launch_count() == 0


def test_workspace_bytes():
    # status block + two fp32 [B, H, N] row-statistics arrays, each rounded to 256 bytes;
    # on the split-dS path (the default while its blocks fit 4 GiB) also the dS
    # blocks: B H (N/G) T (T+1)/2 blocks of 128 x 128 bf16, T = G/128; on the
    # fused backward the fp32 [B, H, N, D] dq accumulator instead
    ds = 32 * 4 * (16 * 17 // 2) * 128 * 128 * 2
    assert _lib.s2attn_bwd_workspace_bytes(1, 32, 32, 8192, 128, 2048) == 256 + 2 * 32 * 8192 * 4 + ds
    assert _lib.s2attn_bwd_workspace_bytes(1, 1, 1, 128, 64, 128) == 256 + 2 * 512 + 128 * 128 * 2
    assert _lib.s2attn_bwd_workspace_bytes(1, 4, 3, 1024, 64, 256) == 0  # invalid shape
    # LLaMA2-70B at 32K tokens: 17 GB of dS blocks in all, over the budget: the
    # workspace holds the dS of 7 (batch, kv head, group) units of 8 query heads
    # each (545 MB a unit), the backward running in ranges
    unit = 8 * (64 * 65 // 2) * 128 * 128 * 2
    assert _lib.s2attn_bwd_workspace_bytes(1, 64, 8, 32768, 128, 8192) == 256 + 2 * 64 * 32768 * 4 + 7 * unit
    # 100K tokens, 32 heads: 6 units of 643 MB
    unit = (200 * 201 // 2) * 128 * 128 * 2
    assert _lib.s2attn_bwd_workspace_bytes(1, 32, 32, 102400, 128, 25600) == 256 + 2 * 32 * 102400 * 4 + 6 * unit
    # the split path, forced through the override, needs no accumulator
    try:
        _lib.s2attn_set_tile_override("bwd=split")
        assert _lib.s2attn_bwd_workspace_bytes(1, 32, 32, 8192, 128, 2048) == 256 + 2 * 32 * 8192 * 4
        _lib.s2attn_set_tile_override("ds_slots=3")  # dS of 3 of the 128 units
        assert _lib.s2attn_bwd_workspace_bytes(1, 32, 32, 8192, 128, 2048) == \
            256 + 2 * 32 * 8192 * 4 + 3 * (16 * 17 // 2) * 128 * 128 * 2
        _lib.s2attn_set_tile_override("fwd_order=pairs,bwd=fused")
        assert _lib.s2attn_bwd_workspace_bytes(1, 32, 32, 8192, 128, 2048) == 256 + 2 * 32 * 8192 * 4 + 32 * 8192 * 128 * 4
    finally:
        _lib.s2attn_set_tile_override(None)


def test_noalloc_rejects_oversize_before_launch():
    # 64 heads x 131072 rows need ~64 MiB of scratch: rejected without touching the device
    assert _lib.s2attn_bwd_noalloc(P, P, P, P, P, P, P, P, P, 1, 64, 64, 131072, 128, 131072, None) == \
        _lib.S2ATTN_ERR_WORKSPACE
    assert _lib.s2attn_bwd_noalloc(P, P, P, P, P, P, P, P, P, 1, 4, 3, 1024, 64, 256, None) == \
        _lib.S2ATTN_ERR_INVALID_ARG  # invalid shape: reported by the backward's own validation


def test_profile_api_host_side():
    assert _lib.s2attn_profile_start(0) == _lib.S2ATTN_ERR_INVALID_ARG
    assert _lib.s2attn_profile_stop(None, None, 0) == 0  # not started: nothing recorded


def test_plan_selection_table():
    """The per-shape plan (host logic, no GPU): the split-dS backward, its
    workspace holding every unit's dS blocks while they fit 4 GiB and as many
    units as fit beyond that; the forward's work order following the K/V size;
    the selected depths."""
    from sparse_attention_attn_b200 import inputs as I
    expect = {
        "tiny": ("snake", 8, "split_ds", 3, 16),
        "llama2-7b-n8192": ("snake", 4, "split_ds", 3, 128),
        "qwen3-8b-gqa-n16384": ("snake", 4, "split_ds", 3, 32),
        "llama2-70b-gqa-n32768": ("snake", 4, "split_ds", 3, 7),
        "llama2-7b-n102400": ("pairs", 4, "split_ds", 3, 6),
    }
    for s in I.WORKLOADS:
        p = _lib.s2attn_plan(s.B, s.H, s.Hkv, s.N, s.D, s.G, 148)
        got = (p["fwd_order"], p["fwd_kv_slots"], p["bwd_path"], p["bwd_stages"], p["ds_slots"])
        assert got == expect[s.name], s.name
        assert p["fwd_bn"] == 128
    # a unit whose dS alone passes half the budget leaves no room for two: the split path
    p = _lib.s2attn_plan(1, 64, 1, 65536, 128, 65536, 148)
    assert (p["bwd_path"], p["ds_slots"]) == ("split", 0)
    with pytest.raises(_lib.S2AttnError):
        _lib.s2attn_plan(1, 4, 3, 1024, 64, 256, 148)


def test_plan_override_parsing():
    """S2ATTN_TILE-style overrides force existing variants and ignore values
    that do not exist for the call's head dim."""
    try:
        _lib.s2attn_set_tile_override("fwd_order=pairs,fwd_kv=2,bwd=split,bwd_stages=2")
        p = _lib.s2attn_plan(1, 32, 32, 8192, 128, 2048, 148)   # a 2-slot K/V ring does not exist
        assert p == {"fwd_order": "pairs", "fwd_bn": 128, "fwd_kv_slots": 4, "bwd_path": "split", "bwd_stages": 2,
                     "ds_slots": 0, "bwd_qtile": 64}
        p = _lib.s2attn_plan(1, 4, 4, 1024, 64, 256, 148)   # head dim 64: kv 2 and stages 2 do not exist
        assert p == {"fwd_order": "pairs", "fwd_bn": 128, "fwd_kv_slots": 8, "bwd_path": "split", "bwd_stages": 3,
                     "ds_slots": 0, "bwd_qtile": 64}
        _lib.s2attn_set_tile_override("bwd=fused,fwd_kv=6,bwd_stages=4,junk,=,x=y")  # no fused path at D = 64
        assert _lib.s2attn_plan(1, 4, 4, 1024, 64, 256, 148) == \
            {"fwd_order": "snake", "fwd_bn": 128, "fwd_kv_slots": 6, "bwd_path": "split_ds", "bwd_stages": 4,
             "ds_slots": 16, "bwd_qtile": 64}
        assert _lib.s2attn_plan(1, 32, 32, 8192, 128, 2048, 148) == \
            {"fwd_order": "snake", "fwd_bn": 128, "fwd_kv_slots": 4, "bwd_path": "fused", "bwd_stages": 4,
             "ds_slots": 0, "bwd_qtile": 64}
        _lib.s2attn_set_tile_override("bwd_stages=5")  # 5 stages exist for neither head dim
        assert _lib.s2attn_plan(1, 32, 32, 8192, 128, 2048, 148)["bwd_stages"] == 3
        assert _lib.s2attn_plan(1, 4, 4, 1024, 64, 256, 148)["bwd_stages"] == 3
        _lib.s2attn_set_tile_override("ds_slots=2")
        assert _lib.s2attn_plan(1, 32, 32, 8192, 128, 2048, 148)["ds_slots"] == 2
        _lib.s2attn_set_tile_override("ds_slots=1000,bwd_stages=2")  # more slots than units: every unit
        assert _lib.s2attn_plan(1, 32, 32, 8192, 128, 2048, 148)["ds_slots"] == 128
        _lib.s2attn_set_tile_override("ds_slots=1")  # fewer than 2 slots do not exist
        assert _lib.s2attn_plan(1, 64, 8, 32768, 128, 8192, 148)["ds_slots"] == 7
        _lib.s2attn_set_tile_override("fwd_bn=64,fwd_kv=4")  # 4 slots do not exist for 64-key tiles
        assert _lib.s2attn_plan(1, 32, 32, 8192, 128, 2048, 148)["fwd_bn"] == 64
        assert _lib.s2attn_plan(1, 32, 32, 8192, 128, 2048, 148)["fwd_kv_slots"] == 8
        assert _lib.s2attn_plan(1, 4, 4, 1024, 64, 256, 148)["fwd_kv_slots"] == 8
        _lib.s2attn_set_tile_override("fwd_bn=64,fwd_kv=12")
        assert _lib.s2attn_plan(1, 4, 4, 1024, 64, 256, 148)["fwd_kv_slots"] == 12
        assert _lib.s2attn_plan(1, 32, 32, 8192, 128, 2048, 148)["fwd_kv_slots"] == 8
        _lib.s2attn_set_tile_override("bwd=split_ds")  # forced where not even 2 units fit: 2 slots
        assert _lib.s2attn_plan(1, 64, 1, 65536, 128, 65536, 148)["bwd_path"] == "split_ds"
        assert _lib.s2attn_plan(1, 64, 1, 65536, 128, 65536, 148)["ds_slots"] == 1  # one unit: all of them
        assert _lib.s2attn_plan(2, 64, 1, 65536, 128, 65536, 148)["ds_slots"] == 2
    finally:
        _lib.s2attn_set_tile_override(None)
    assert _lib.s2attn_plan(1, 32, 32, 8192, 128, 2048, 148)["bwd_path"] == "split_ds"
    assert _lib.s2attn_plan(1, 64, 8, 32768, 128, 8192, 148)["ds_slots"] == 7


def test_nf4_levels_and_argument_checks_on_the_host():
    """The library's NF4 levels (host computation: bisection on erfc) against
    the oracle's (scipy's inverse normal CDF), and the projection's argument
    checks, which return before any CUDA call."""
    import numpy as np
    import oracle.nf4_ref as nr
    from sparse_attention_attn_b200 import _lib
    np.testing.assert_allclose(np.array(_lib.s2attn_nf4_levels()), nr.nf4_levels(), rtol=0, atol=6e-8)
    lib = _lib.load()
    p = 1 << 20  # fake, 16-byte aligned device addresses: nothing is dereferenced
    args = dict(x=p, codes=p, sq=p, c2=p, q=p, k=p, v=p)

    def call(M=16, K=256, H=2, Hkv=1, D=128, **over):
        a = dict(args, **over)
        return lib.s2attn_nf4_qkv(a["x"], a["codes"], a["sq"], a["c2"], a["q"], a["k"], a["v"], M, K, H, Hkv, D,
                                  None)
    assert call(x=None) == _lib.S2ATTN_ERR_INVALID_ARG
    assert call(M=0) == _lib.S2ATTN_ERR_INVALID_ARG
    assert call(K=96) == _lib.S2ATTN_ERR_UNSUPPORTED          # not a whole number of 64-element blocks
    assert call(H=1, Hkv=1, D=64) == _lib.S2ATTN_ERR_UNSUPPORTED  # 64 features: not a whole 128-row tile
    assert call(x=p + 8) == _lib.S2ATTN_ERR_MISALIGNED
    assert call(q=p + 2) == _lib.S2ATTN_ERR_MISALIGNED
    assert lib.s2attn_nf4_dequant(p, p, p, p, 4, 100, None) == _lib.S2ATTN_ERR_UNSUPPORTED
    assert lib.s2attn_nf4_dequant(p, p, p, p + 8, 4, 128, None) == _lib.S2ATTN_ERR_MISALIGNED


def test_debug_build_exports_the_same_symbols():
    """libs2attn_debug.so (kernels with index checks) builds and exports every
    entry point of the header, and says it is the debug build."""
    import ctypes

    from sparse_attention_attn_b200 import build
    path = build.build(debug=True)
    lib = ctypes.CDLL(path)
    for name in declared_functions():
        assert hasattr(lib, name), name
    lib.s2attn_debug_checks.restype = ctypes.c_int
    assert lib.s2attn_debug_checks() == 1
