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
