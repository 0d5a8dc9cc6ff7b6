"""ctypes binding of libs2attn.so: the C ABI of include/s2attn.h, same names.

Argument marshalling only.  Every step of the attention runs in the library's
CUDA kernels; there is no Python or CPU fallback: if the library is missing or
the device is not a B200, calls raise.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# S2ATTN_DEBUG=1 selects the debug build (in-kernel index checks; built by
# `python -m sparse_attention_attn_b200.build --debug`)
LIB_PATH = os.path.join(_HERE, "libs2attn_debug.so" if os.environ.get("S2ATTN_DEBUG") == "1" else "libs2attn.so")

S2ATTN_OK = 0
S2ATTN_ERR_INVALID_ARG = 1
S2ATTN_ERR_UNSUPPORTED = 2
S2ATTN_ERR_MISALIGNED = 3
S2ATTN_ERR_CUDA = 4
S2ATTN_ERR_DEVICE_TIMEOUT = 5
S2ATTN_ERR_WORKSPACE = 6
S2ATTN_ERR_DEVICE_BOUNDS = 7

_vp = ctypes.c_void_p
_i = ctypes.c_int

# name -> (restype, argtypes); mirrors include/s2attn.h
SIGNATURES = {
    "s2attn_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp]),
    "s2attn_bwd_workspace_bytes": (ctypes.c_size_t, [_i, _i, _i, _i, _i, _i]),
    "s2attn_bwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i,
                        _vp, ctypes.c_size_t, _vp]),
    "s2attn_device_status": (_i, [_vp, _vp]),
    "s2attn_status_string": (ctypes.c_char_p, [_i]),
    "s2attn_selftest_wait_timeout": (_i, [_vp, ctypes.c_uint64, _vp]),
    "s2attn_last_launch_count": (_i, []),
    "s2attn_debug_checks": (_i, []),
    "s2attn_last_cuda_error": (_i, []),
    "s2attn_cuda_error_string": (ctypes.c_char_p, [_i]),
    "s2attn_profile_start": (_i, [_i]),
    "s2attn_profile_stop": (_i, [_vp, _vp, _i]),
    "s2attn_set_tile_override": (_i, [ctypes.c_char_p]),
    "s2attn_seg_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp]),
    "s2attn_seg_bwd_workspace_bytes": (ctypes.c_size_t, [_i, _i, _i, _i, _i, _i]),
    "s2attn_seg_bwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _vp,
                            ctypes.c_size_t, _vp]),
    "s2attn_lse_merge": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _vp]),
    "s2attn_hga_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp]),
    "s2attn_hga_bwd_workspace_bytes": (ctypes.c_size_t, [_i, _i, _i, _i, _i, _i]),
    "s2attn_hga_bwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp,
                            ctypes.c_size_t, _vp]),
    "s2attn_rope_table_bytes": (ctypes.c_size_t, [_i, _i]),
    "s2attn_rope_table": (_i, [_vp, _i, _i, ctypes.c_double, ctypes.c_double, _vp]),
    "s2attn_rope_apply": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _vp]),
    "s2attn_fwd_rope": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp]),
    "s2attn_bwd_rope": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp,
                             ctypes.c_size_t, _vp]),
    "s2attn_plan": (_i, [_i, _i, _i, _i, _i, _i, _i, _vp]),
    "s2attn_nf4_levels": (_i, [_vp]),
    "s2attn_nf4_qkv": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp]),
    "s2attn_nf4_dequant": (_i, [_vp, _vp, _vp, _vp, _i, _i, _vp]),
    "s2attn_bwd_noalloc": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i,
                                _vp]),
}

_lib = None


class S2AttnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        msg = f"{fn} failed: {status_string(status)} ({status})"
        if status == S2ATTN_ERR_CUDA:
            err = load().s2attn_last_cuda_error()
            msg += f"; CUDA: {load().s2attn_cuda_error_string(err).decode()} ({err})"
        super().__init__(msg)


def load() -> ctypes.CDLL:
    """Load libs2attn.so (built in-tree).  Raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing; build it with `python -m sparse_attention_attn_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().s2attn_status_string(int(status)).decode()


def _check(fn: str, status: int) -> None:
    if status != S2ATTN_OK:
        raise S2AttnError(fn, status)


def s2attn_fwd(q, k, v, o, lse, B, H, Hkv, N, D, G, stream) -> int:
    """Raw C call with integer device pointers; returns the status code."""
    return load().s2attn_fwd(q, k, v, o, lse, B, H, Hkv, N, D, G, stream)


def s2attn_bwd_workspace_bytes(B, H, Hkv, N, D, G) -> int:
    return load().s2attn_bwd_workspace_bytes(B, H, Hkv, N, D, G)


def s2attn_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, H, Hkv, N, D, G, workspace, workspace_bytes,
               stream) -> int:
    return load().s2attn_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, H, Hkv, N, D, G, workspace,
                             workspace_bytes, stream)


def s2attn_device_status(workspace, stream) -> int:
    return load().s2attn_device_status(workspace, stream)


def s2attn_selftest_wait_timeout(status_out, limit_ns, stream) -> int:
    return load().s2attn_selftest_wait_timeout(status_out, limit_ns, stream)


def s2attn_last_launch_count() -> int:
    return load().s2attn_last_launch_count()


def s2attn_profile_start(max_launches) -> int:
    return load().s2attn_profile_start(max_launches)


def s2attn_profile_stop(ms, kernel_ids, capacity) -> int:
    return load().s2attn_profile_stop(ms, kernel_ids, capacity)


def s2attn_seg_fwd(q, k, v, o, lse, B, H, Hkv, N, Nk, D, causal, stream) -> int:
    return load().s2attn_seg_fwd(q, k, v, o, lse, B, H, Hkv, N, Nk, D, causal, stream)


def s2attn_seg_bwd_workspace_bytes(B, H, Hkv, N, Nk, D) -> int:
    return load().s2attn_seg_bwd_workspace_bytes(B, H, Hkv, N, Nk, D)


def s2attn_seg_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, H, Hkv, N, Nk, D, causal, dq_accumulate, workspace,
                   workspace_bytes, stream) -> int:
    return load().s2attn_seg_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, H, Hkv, N, Nk, D, causal, dq_accumulate,
                                 workspace, workspace_bytes, stream)


def s2attn_lse_merge(o_a, lse_a, o_b, lse_b, o, lse, B, H, N, D, stream) -> int:
    return load().s2attn_lse_merge(o_a, lse_a, o_b, lse_b, o, lse, B, H, N, D, stream)


def s2attn_hga_fwd(q, k, v, o, lse, hist, S, B, H, Hkv, N, D, G, stream) -> int:
    return load().s2attn_hga_fwd(q, k, v, o, lse, hist, S, B, H, Hkv, N, D, G, stream)


def s2attn_hga_bwd_workspace_bytes(B, H, Hkv, N, D, G) -> int:
    return load().s2attn_hga_bwd_workspace_bytes(B, H, Hkv, N, D, G)


def s2attn_hga_bwd(q, k, v, o, lse, dO, dq, dk, dv, hist, S, B, H, Hkv, N, D, G, workspace, workspace_bytes,
                   stream) -> int:
    return load().s2attn_hga_bwd(q, k, v, o, lse, dO, dq, dk, dv, hist, S, B, H, Hkv, N, D, G, workspace,
                                 workspace_bytes, stream)


def s2attn_rope_table_bytes(N, D) -> int:
    return load().s2attn_rope_table_bytes(N, D)


def s2attn_rope_table(table, N, D, pos_scale, rope_base, stream) -> int:
    return load().s2attn_rope_table(table, N, D, pos_scale, rope_base, stream)


def s2attn_rope_apply(x, out, table, B, N, heads, D, inverse, stream) -> int:
    return load().s2attn_rope_apply(x, out, table, B, N, heads, D, inverse, stream)


def s2attn_fwd_rope(q, k, v, o, lse, q_rot, k_rot, table, B, H, Hkv, N, D, G, stream) -> int:
    return load().s2attn_fwd_rope(q, k, v, o, lse, q_rot, k_rot, table, B, H, Hkv, N, D, G, stream)


def s2attn_bwd_rope(q_rot, k_rot, v, o, lse, dO, dq, dk, dv, table, B, H, Hkv, N, D, G, workspace,
                    workspace_bytes, stream) -> int:
    return load().s2attn_bwd_rope(q_rot, k_rot, v, o, lse, dO, dq, dk, dv, table, B, H, Hkv, N, D, G, workspace,
                                  workspace_bytes, stream)


def s2attn_plan(B, H, Hkv, N, D, G, num_sms):
    """The per-shape plan as a dict (host only), or raises on an invalid shape."""
    out = (ctypes.c_int * 7)()
    _check("s2attn_plan", load().s2attn_plan(B, H, Hkv, N, D, G, num_sms, ctypes.addressof(out)))
    return {"fwd_order": "snake" if out[0] else "pairs", "fwd_bn": out[4], "fwd_kv_slots": out[1],
            "bwd_path": {0: "split", 1: "fused", 2: "split_ds"}[out[2]], "bwd_stages": out[3],
            "ds_slots": out[5], "bwd_qtile": out[6]}


def s2attn_nf4_levels():
    """The library's 16 NF4 levels (host computation) as a list of floats."""
    out = (ctypes.c_float * 16)()
    _check("s2attn_nf4_levels", load().s2attn_nf4_levels(ctypes.addressof(out)))
    return list(out)


def s2attn_nf4_qkv(x, codes, scale_codes, c2, q, k, v, M, K, H, Hkv, D, stream) -> int:
    return load().s2attn_nf4_qkv(x, codes, scale_codes, c2, q, k, v, M, K, H, Hkv, D, stream)


def s2attn_nf4_dequant(codes, scale_codes, c2, w, rows, K, stream) -> int:
    return load().s2attn_nf4_dequant(codes, scale_codes, c2, w, rows, K, stream)


def s2attn_set_tile_override(spec) -> int:
    """Test / sweep hook: force a kernel variant (None restores S2ATTN_TILE)."""
    return load().s2attn_set_tile_override(None if spec is None else spec.encode())


def s2attn_bwd_noalloc(q, k, v, o, lse, dO, dq, dk, dv, B, H, Hkv, N, D, G, stream) -> int:
    """Backward with the library's built-in scratch, for callers that cannot allocate."""
    return load().s2attn_bwd_noalloc(q, k, v, o, lse, dO, dq, dk, dv, B, H, Hkv, N, D, G, stream)
