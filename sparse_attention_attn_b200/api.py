"""PyTorch-facing calls of the S2-Attn library (device memory and streams only).

Each function checks tensor placement, dtype, layout and shape, then calls the
C ABI through ctypes on torch's current CUDA stream.  The arithmetic happens
only in the CUDA kernels of libs2attn.so; a missing library or a non-B200
device raises instead of falling back to anything else.

Shift rule (LongQLoRA community post, section 03, Shift Short Attention; the
LongLoRA abstract): with group size G < N, query heads h >= H/2 attend inside
groups of the sequence rolled by G/2 rows (wrap-around); G == N is dense causal
attention.  Training uses the shifted groups, inference the dense path.
"""
from __future__ import annotations

import torch

from . import _lib


def _stream(device=None) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _need(name: str, t: torch.Tensor, shape, dtype=torch.bfloat16, device=None) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device} (all operands on one device)")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _dims(q: torch.Tensor, k: torch.Tensor):
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q must be [B, N, H, D] and k [B, N, Hkv, D]")
    B, N, H, D = q.shape
    return B, N, H, k.shape[2], D


def s2attn_forward(q, k, v, group_size: int, out=None, lse=None):
    """S2-Attn forward.  q [B,N,H,D], k/v [B,N,Hkv,D] bf16 CUDA tensors.

    Returns (o [B,N,H,D] bf16, lse [B,H,N] fp32 natural-log log-sum-exp).
    """
    B, N, H, Hkv, D = _dims(q, k)
    _need("q", q, (B, N, H, D))
    dev = q.device
    _need("k", k, (B, N, Hkv, D), device=dev)
    _need("v", v, (B, N, Hkv, D), device=dev)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    _need("out", out, (B, N, H, D), device=dev)
    _need("lse", lse, (B, H, N), torch.float32, device=dev)
    with torch.cuda.device(dev):  # the C ABI launches on the current device
        st = _lib.s2attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                             B, H, Hkv, N, D, int(group_size), _stream(dev))
    _lib._check("s2attn_fwd", st)
    return out, lse


def bwd_workspace_bytes(B, H, Hkv, N, D, group_size) -> int:
    n = _lib.s2attn_bwd_workspace_bytes(B, H, Hkv, N, D, int(group_size))
    if n == 0:
        raise _lib.S2AttnError("s2attn_bwd_workspace_bytes", _lib.S2ATTN_ERR_INVALID_ARG)
    return n


def s2attn_backward(q, k, v, o, lse, do, group_size: int, dq=None, dk=None, dv=None,
                    workspace=None):
    """S2-Attn backward.  Returns (dq, dk, dv); dk/dv summed over shared query heads."""
    B, N, H, Hkv, D = _dims(q, k)
    _need("q", q, (B, N, H, D))
    dev = q.device
    for name, t, shp in (("k", k, (B, N, Hkv, D)), ("v", v, (B, N, Hkv, D)),
                         ("o", o, (B, N, H, D)), ("do", do, (B, N, H, D))):
        _need(name, t, shp, device=dev)
    _need("lse", lse, (B, H, N), torch.float32, device=dev)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _need("dq", dq, (B, N, H, D), device=dev)
    _need("dk", dk, (B, N, Hkv, D), device=dev)
    _need("dv", dv, (B, N, Hkv, D), device=dev)
    wsb = bwd_workspace_bytes(B, H, Hkv, N, D, group_size)
    if workspace is None:
        workspace = torch.empty(wsb, dtype=torch.uint8, device=dev)
    if not isinstance(workspace, torch.Tensor) or workspace.device != dev or not workspace.is_contiguous():
        raise ValueError(f"workspace must be a contiguous tensor on {dev}")
    if workspace.numel() * workspace.element_size() < wsb:
        raise _lib.S2AttnError("s2attn_bwd", _lib.S2ATTN_ERR_WORKSPACE)
    with torch.cuda.device(dev):  # the C ABI launches on the current device
        st = _lib.s2attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                             do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                             B, H, Hkv, N, D, int(group_size), workspace.data_ptr(),
                             workspace.numel() * workspace.element_size(), _stream(dev))
    _lib._check("s2attn_bwd", st)
    return dq, dk, dv


def device_status(workspace=None) -> int:
    """Synchronise the current stream and return (and clear) the device status."""
    ptr = workspace.data_ptr() if workspace is not None else None
    return _lib.s2attn_device_status(ptr, _stream())


def rope_table(N: int, D: int, pos_scale: float, rope_base: float = 10000.0, device=None):
    """fp32 (cos, sin) table [N, D/2, 2] of RoPE with Position Interpolation:
    pair i at token t turns by t * pos_scale * rope_base^(-2i/D) (LongQLoRA
    post section 04: Position Interpolation shrinks RoPE's angles; pos_scale =
    L_train / L_target).  Built on the GPU; reuse it across layers and steps."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    nbytes = _lib.s2attn_rope_table_bytes(N, D)
    if nbytes == 0:
        raise _lib.S2AttnError("s2attn_rope_table_bytes", _lib.S2ATTN_ERR_UNSUPPORTED)
    table = torch.empty((N, D // 2, 2), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        st = _lib.s2attn_rope_table(table.data_ptr(), N, D, float(pos_scale), float(rope_base), _stream(dev))
    _lib._check("s2attn_rope_table", st)
    return table


def rope_apply(x, table, inverse: bool = False, out=None):
    """x [B, N, heads, D] bf16 rotated by the table (the opposite way when
    `inverse`); out may be x (in place)."""
    B, N, Hx, D = x.shape
    _need("x", x, (B, N, Hx, D))
    _need("table", table, (N, D // 2, 2), torch.float32, device=x.device)
    out = torch.empty_like(x) if out is None else out
    _need("out", out, (B, N, Hx, D), device=x.device)
    with torch.cuda.device(x.device):
        st = _lib.s2attn_rope_apply(x.data_ptr(), out.data_ptr(), table.data_ptr(), B, N, Hx, D, int(inverse),
                                    _stream(x.device))
    _lib._check("s2attn_rope_apply", st)
    return out


def s2attn_forward_rope(q, k, v, group_size: int, table, out=None, lse=None, q_rot=None, k_rot=None):
    """S2 attention on RoPE-rotated q and k.  Returns (o, lse, q_rot, k_rot);
    q_rot and k_rot are what the backward takes."""
    B, N, H, Hkv, D = _dims(q, k)
    _need("q", q, (B, N, H, D))
    dev = q.device
    _need("k", k, (B, N, Hkv, D), device=dev)
    _need("v", v, (B, N, Hkv, D), device=dev)
    _need("table", table, (N, D // 2, 2), torch.float32, device=dev)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev) if lse is None else lse
    q_rot = torch.empty_like(q) if q_rot is None else q_rot
    k_rot = torch.empty_like(k) if k_rot is None else k_rot
    _need("out", out, (B, N, H, D), device=dev)
    _need("lse", lse, (B, H, N), torch.float32, device=dev)
    _need("q_rot", q_rot, (B, N, H, D), device=dev)
    _need("k_rot", k_rot, (B, N, Hkv, D), device=dev)
    with torch.cuda.device(dev):
        st = _lib.s2attn_fwd_rope(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                  q_rot.data_ptr(), k_rot.data_ptr(), table.data_ptr(), B, H, Hkv, N, D,
                                  int(group_size), _stream(dev))
    _lib._check("s2attn_fwd_rope", st)
    return out, lse, q_rot, k_rot


def s2attn_backward_rope(q_rot, k_rot, v, o, lse, do, group_size: int, table, dq=None, dk=None, dv=None,
                         workspace=None):
    """Backward of s2attn_forward_rope: gradients with respect to the
    unrotated q and k, and v.  Returns (dq, dk, dv)."""
    B, N, H, Hkv, D = _dims(q_rot, k_rot)
    _need("q_rot", q_rot, (B, N, H, D))
    dev = q_rot.device
    for name, t, shp in (("k_rot", k_rot, (B, N, Hkv, D)), ("v", v, (B, N, Hkv, D)),
                         ("o", o, (B, N, H, D)), ("do", do, (B, N, H, D))):
        _need(name, t, shp, device=dev)
    _need("lse", lse, (B, H, N), torch.float32, device=dev)
    _need("table", table, (N, D // 2, 2), torch.float32, device=dev)
    dq = torch.empty_like(q_rot) if dq is None else dq
    dk = torch.empty_like(k_rot) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for name, t, shp in (("dq", dq, (B, N, H, D)), ("dk", dk, (B, N, Hkv, D)), ("dv", dv, (B, N, Hkv, D))):
        _need(name, t, shp, device=dev)
    wsb = bwd_workspace_bytes(B, H, Hkv, N, D, group_size)
    if workspace is None:
        workspace = torch.empty(wsb, dtype=torch.uint8, device=dev)
    if workspace.numel() * workspace.element_size() < wsb:
        raise _lib.S2AttnError("s2attn_bwd_rope", _lib.S2ATTN_ERR_WORKSPACE)
    with torch.cuda.device(dev):
        st = _lib.s2attn_bwd_rope(q_rot.data_ptr(), k_rot.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                  do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), table.data_ptr(),
                                  B, H, Hkv, N, D, int(group_size), workspace.data_ptr(),
                                  workspace.numel() * workspace.element_size(), _stream(dev))
    _lib._check("s2attn_bwd_rope", st)
    return dq, dk, dv


class S2RopeAttention(torch.autograd.Function):
    """Autograd wrapper: RoPE with Position Interpolation, then S2 attention."""

    @staticmethod
    def forward(ctx, q, k, v, group_size, table):
        o, lse, q_rot, k_rot = s2attn_forward_rope(q, k, v, group_size, table)
        ctx.save_for_backward(q_rot, k_rot, v, o, lse, table)
        ctx.group_size = group_size
        return o

    @staticmethod
    def backward(ctx, do):
        q_rot, k_rot, v, o, lse, table = ctx.saved_tensors
        dq, dk, dv = s2attn_backward_rope(q_rot, k_rot, v, o, lse, do.contiguous(), ctx.group_size, table)
        return dq, dk, dv, None, None


def seg_forward(q, k, v, causal: bool = True, out=None, lse=None):
    """Attention of a chunk's queries q [B, N, H, D] over keys k, v [B, Nk, Hkv, D]:
    causal -- row i sees keys [0, Nk - N + i] (the earlier keys, then its own
    chunk causally); not causal -- every key (a detached segment as a piece).
    Returns (o, lse) of that attention."""
    B, N, H, Hkv, D = _dims(q, k)
    Nk = k.shape[1]
    _need("q", q, (B, N, H, D))
    dev = q.device
    _need("k", k, (B, Nk, Hkv, D), device=dev)
    _need("v", v, (B, Nk, Hkv, D), device=dev)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev) if lse is None else lse
    _need("out", out, (B, N, H, D), device=dev)
    _need("lse", lse, (B, H, N), torch.float32, device=dev)
    with torch.cuda.device(dev):
        st = _lib.s2attn_seg_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                 B, H, Hkv, N, Nk, D, int(causal), _stream(dev))
    _lib._check("s2attn_seg_fwd", st)
    return out, lse


def seg_backward(q, k, v, o, lse, do, causal: bool = True, dq=None, dk=None, dv=None, dq_accumulate=False,
                 workspace=None):
    """Backward of seg_forward given the chunk rows' final o and lse: dq, and
    (causal) dk, dv of the chunk's own keys -- the last N key rows.  Not
    causal: dq only (dk, dv returned as None).  dq_accumulate adds into dq."""
    B, N, H, Hkv, D = _dims(q, k)
    Nk = k.shape[1]
    _need("q", q, (B, N, H, D))
    dev = q.device
    for name, t, shp in (("k", k, (B, Nk, Hkv, D)), ("v", v, (B, Nk, Hkv, D)), ("o", o, (B, N, H, D)),
                         ("do", do, (B, N, H, D))):
        _need(name, t, shp, device=dev)
    _need("lse", lse, (B, H, N), torch.float32, device=dev)
    if dq is None:
        if dq_accumulate:
            raise ValueError("dq_accumulate needs dq")
        dq = torch.empty_like(q)
    _need("dq", dq, (B, N, H, D), device=dev)
    if causal:
        dk = torch.empty((B, N, Hkv, D), dtype=k.dtype, device=dev) if dk is None else dk
        dv = torch.empty((B, N, Hkv, D), dtype=v.dtype, device=dev) if dv is None else dv
        _need("dk", dk, (B, N, Hkv, D), device=dev)
        _need("dv", dv, (B, N, Hkv, D), device=dev)
    else:
        dk = dv = None
    wsb = _lib.s2attn_seg_bwd_workspace_bytes(B, H, Hkv, N, Nk, D)
    if wsb == 0:
        raise _lib.S2AttnError("s2attn_seg_bwd_workspace_bytes", _lib.S2ATTN_ERR_INVALID_ARG)
    if workspace is None:
        workspace = torch.empty(wsb, dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        st = _lib.s2attn_seg_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                 do.data_ptr(), dq.data_ptr(), None if dk is None else dk.data_ptr(),
                                 None if dv is None else dv.data_ptr(), B, H, Hkv, N, Nk, D, int(causal),
                                 int(dq_accumulate), workspace.data_ptr(),
                                 workspace.numel() * workspace.element_size(), _stream(dev))
    _lib._check("s2attn_seg_bwd", st)
    return dq, dk, dv


def lse_merge(o_a, lse_a, o_b, lse_b, out=None, lse=None):
    """Attention over the union of two disjoint key sets from the two pieces'
    (o, lse); out / lse may be o_a / lse_a (in place)."""
    B, N, H, D = o_a.shape
    dev = o_a.device
    _need("o_a", o_a, (B, N, H, D))
    _need("o_b", o_b, (B, N, H, D), device=dev)
    _need("lse_a", lse_a, (B, H, N), torch.float32, device=dev)
    _need("lse_b", lse_b, (B, H, N), torch.float32, device=dev)
    out = torch.empty_like(o_a) if out is None else out
    lse = torch.empty_like(lse_a) if lse is None else lse
    _need("out", out, (B, N, H, D), device=dev)
    _need("lse", lse, (B, H, N), torch.float32, device=dev)
    with torch.cuda.device(dev):
        st = _lib.s2attn_lse_merge(o_a.data_ptr(), lse_a.data_ptr(), o_b.data_ptr(), lse_b.data_ptr(),
                                   out.data_ptr(), lse.data_ptr(), B, H, N, D, _stream(dev))
    _lib._check("s2attn_lse_merge", st)
    return out, lse


def _need_hist(hist, B, N, dev):
    if not isinstance(hist, torch.Tensor) or hist.dtype != torch.int32 or hist.dim() != 3:
        raise ValueError("hist must be an int32 tensor [B, N/256, S]")
    if hist.device != dev or not hist.is_contiguous() or tuple(hist.shape[:2]) != (B, N // 256):
        raise ValueError(f"hist must be a contiguous [B, N/256, S] tensor on {dev}")


def hga_forward(q, k, v, group_size: int, hist, out=None, lse=None):
    """HGA-style block-sparse attention: each row attends its own segment
    (group_size rows, no shift) causally and the historical key tiles listed
    for its 256-row query block in hist (int32 [B, N/256, S], tile indices of
    earlier segments; a list ends at its first other entry, e.g. -1)."""
    B, N, H, Hkv, D = _dims(q, k)
    _need("q", q, (B, N, H, D))
    dev = q.device
    _need("k", k, (B, N, Hkv, D), device=dev)
    _need("v", v, (B, N, Hkv, D), device=dev)
    _need_hist(hist, B, N, dev)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev) if lse is None else lse
    _need("out", out, (B, N, H, D), device=dev)
    _need("lse", lse, (B, H, N), torch.float32, device=dev)
    with torch.cuda.device(dev):
        st = _lib.s2attn_hga_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                 hist.data_ptr(), hist.shape[2], B, H, Hkv, N, D, int(group_size), _stream(dev))
    _lib._check("s2attn_hga_fwd", st)
    return out, lse


def hga_backward(q, k, v, o, lse, do, group_size: int, hist, dq=None, dk=None, dv=None, workspace=None):
    """Backward of hga_forward: dq through every attended key; dk, dv through
    the local attention only (the historical keys are detached)."""
    B, N, H, Hkv, D = _dims(q, k)
    _need("q", q, (B, N, H, D))
    dev = q.device
    for name, t, shp in (("k", k, (B, N, Hkv, D)), ("v", v, (B, N, Hkv, D)), ("o", o, (B, N, H, D)),
                         ("do", do, (B, N, H, D))):
        _need(name, t, shp, device=dev)
    _need("lse", lse, (B, H, N), torch.float32, device=dev)
    _need_hist(hist, B, N, dev)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    wsb = _lib.s2attn_hga_bwd_workspace_bytes(B, H, Hkv, N, D, int(group_size))
    if wsb == 0:
        raise _lib.S2AttnError("s2attn_hga_bwd_workspace_bytes", _lib.S2ATTN_ERR_INVALID_ARG)
    if workspace is None:
        workspace = torch.empty(wsb, dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        st = _lib.s2attn_hga_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                 do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), hist.data_ptr(),
                                 hist.shape[2], B, H, Hkv, N, D, int(group_size), workspace.data_ptr(),
                                 workspace.numel() * workspace.element_size(), _stream(dev))
    _lib._check("s2attn_hga_bwd", st)
    return dq, dk, dv


class ChunkAttention(torch.autograd.Function):
    """Chunk-wise training step: the chunk's queries attend its own keys
    causally and the detached earlier keys fully; the two pieces are merged by
    log-sum-exp and only q, k_act, v_act receive gradients."""

    @staticmethod
    def forward(ctx, q, k_act, v_act, k_past, v_past):
        o_a, lse_a = seg_forward(q, k_past, v_past, causal=False)
        o_b, lse_b = seg_forward(q, k_act, v_act, causal=True)
        o, lse = lse_merge(o_a, lse_a, o_b, lse_b, out=o_a, lse=lse_a)
        ctx.save_for_backward(q, k_act, v_act, k_past, v_past, o, lse)
        return o

    @staticmethod
    def backward(ctx, do):
        q, k_act, v_act, k_past, v_past, o, lse = ctx.saved_tensors
        do = do.contiguous()
        dq, _, _ = seg_backward(q, k_past, v_past, o, lse, do, causal=False)
        dq, dk, dv = seg_backward(q, k_act, v_act, o, lse, do, causal=True, dq=dq, dq_accumulate=True)
        return dq, dk, dv, None, None


class S2Attention(torch.autograd.Function):
    """Autograd wrapper: the drop-in attention call of a training step."""

    @staticmethod
    def forward(ctx, q, k, v, group_size):
        o, lse = s2attn_forward(q, k, v, group_size)
        ctx.save_for_backward(q, k, v, o, lse)
        ctx.group_size = group_size
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse = ctx.saved_tensors
        dq, dk, dv = s2attn_backward(q, k, v, o, lse, do.contiguous(), ctx.group_size)
        return dq, dk, dv, None


def s2_attn(q, k, v, group_size: int):
    """Shifted sparse attention with autograd (training path)."""
    return S2Attention.apply(q, k, v, group_size)


def dense_causal_attn(q, k, v):
    """Dense causal attention through the same kernels (G = N, no shift)."""
    return S2Attention.apply(q, k, v, q.shape[1])


# ---------------------------------------------------------------- NF4 QKV projection

def _need_nf4(codes, scale_codes, c2, rows: int, K: int, dev) -> None:
    _need("codes", codes, (rows, K // 2), torch.uint8, device=dev)
    _need("scale_codes", scale_codes, (rows * (K // 64),), torch.int8, device=dev)
    _need("c2", c2, ((rows * (K // 64) + 255) // 256,), torch.float32, device=dev)


def nf4_levels():
    """The 16 NF4 levels the kernels use (ascending; index = 4-bit code)."""
    return _lib.s2attn_nf4_levels()


def nf4_qkv(x, codes, scale_codes, c2, n_heads: int, n_kv_heads: int, head_dim: int, q=None, k=None, v=None):
    """q, k, v = the QKV projection of x (bf16 [B, N, K]) through NF4 weights
    with double quantization, dequantized inside the tensor-core GEMM.  The
    weight is [(H + 2 Hkv) D, K]: codes uint8 [rows, K/2] (two 4-bit codes a
    byte, the even element in the low nibble), scale_codes int8 [rows K/64],
    c2 fp32 [ceil(rows K/64 / 256)].  Returns bf16 [B, N, H, D], [B, N, Hkv, D],
    [B, N, Hkv, D]."""
    if not isinstance(x, torch.Tensor) or x.dim() != 3:
        raise ValueError("x must be a [B, N, K] tensor")
    B, N, K = x.shape
    H, Hkv, D = int(n_heads), int(n_kv_heads), int(head_dim)
    dev = x.device
    _need("x", x, (B, N, K))
    rows = (H + 2 * Hkv) * D
    _need_nf4(codes, scale_codes, c2, rows, K, dev)
    q = torch.empty((B, N, H, D), dtype=torch.bfloat16, device=dev) if q is None else q
    k = torch.empty((B, N, Hkv, D), dtype=torch.bfloat16, device=dev) if k is None else k
    v = torch.empty((B, N, Hkv, D), dtype=torch.bfloat16, device=dev) if v is None else v
    _need("q", q, (B, N, H, D), device=dev)
    _need("k", k, (B, N, Hkv, D), device=dev)
    _need("v", v, (B, N, Hkv, D), device=dev)
    with torch.cuda.device(dev):
        st = _lib.s2attn_nf4_qkv(x.data_ptr(), codes.data_ptr(), scale_codes.data_ptr(), c2.data_ptr(), q.data_ptr(),
                                 k.data_ptr(), v.data_ptr(), B * N, K, H, Hkv, D, _stream(dev))
    _lib._check("s2attn_nf4_qkv", st)
    return q, k, v


def nf4_dequantize(codes, scale_codes, c2, out=None):
    """The dequantized weight W' (bf16 [rows, K]) of NF4 codes [rows, K/2]."""
    if not isinstance(codes, torch.Tensor) or codes.dim() != 2:
        raise ValueError("codes must be a [rows, K/2] tensor")
    rows, K = codes.shape[0], 2 * codes.shape[1]
    dev = codes.device
    _need_nf4(codes, scale_codes, c2, rows, K, dev)
    out = torch.empty((rows, K), dtype=torch.bfloat16, device=dev) if out is None else out
    _need("out", out, (rows, K), device=dev)
    with torch.cuda.device(dev):
        st = _lib.s2attn_nf4_dequant(codes.data_ptr(), scale_codes.data_ptr(), c2.data_ptr(), out.data_ptr(), rows, K,
                                     _stream(dev))
    _lib._check("s2attn_nf4_dequant", st)
    return out
