"""fp64 CPU oracle for chunk-wise attention over detached earlier KV.

TEST INFRASTRUCTURE ONLY: imported by the test suite, the package smoke check
and the benchmark's CPU-baseline leg, never by the product path; it shares no
code with the CUDA kernels.

What the pages state:
* HGA digest (arXiv 2607.15105, English abstract): segment-wise
  backpropagation -- only the active segment stays differentiable, older KV is
  detached (kept in RAM or NVMe) and attended without gradient;
* SeCO / SpaCO digest (arXiv 2505.16710, abstract): the long input is split
  into chunks, each chunk builds its own graph and backpropagates locally, so
  only one chunk's activations are stored.

Readings taken where the pages are silent (listed in the design notes):
* the active chunk holds the last C rows of a sequence of Nk rows; its query
  row i (sequence position c0 + i, c0 = Nk - C) attends keys [0, c0 + i]:
  every earlier key, and its own chunk's keys causally;
* gradients: dq for the chunk's queries (through every key it attends), dk and
  dv for the chunk's own keys only -- the earlier keys are detached;
* softmax over keys processed in separate pieces (the earlier KV fetched from
  another memory tier, the chunk's own KV) is recovered exactly by merging the
  pieces' outputs through their log-sum-exps:
  lse = log(exp(lse_a) + exp(lse_b)), o = exp(lse_a - lse) o_a + exp(lse_b - lse) o_b;
* scale 1/sqrt(D), lse natural log, grouped-query heads as in s2_ref.

All arithmetic is float64 numpy.  q, o, do, dq: [B, C, H, D]; k, v: [B, Nk, Hkv, D];
dk, dv: [B, C, Hkv, D]; lse: [B, H, C].
"""

from __future__ import annotations

import math

import numpy as np

__all__ = ["chunk_attention_fwd", "chunk_attention_bwd", "lse_merge", "segment_attention_fwd"]


def _visible(C: int, Nk: int) -> np.ndarray:
    c0 = Nk - C
    return np.arange(Nk)[None, :] <= (c0 + np.arange(C))[:, None]


def chunk_attention_fwd(q, k, v, scale: float | None = None):
    """Returns (o [B,C,H,D], lse [B,H,C])."""
    q, k, v = (np.asarray(t, dtype=np.float64) for t in (q, k, v))
    B, C, H, D = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    vis = _visible(C, Nk)
    o = np.zeros_like(q)
    lse = np.zeros((B, H, C))
    for b in range(B):
        for h in range(H):
            kh = h // (H // Hkv)
            s = np.where(vis, scale * (q[b, :, h] @ k[b, :, kh].T), -np.inf)
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            l = e.sum(axis=1, keepdims=True)
            o[b, :, h] = (e / l) @ v[b, :, kh]
            lse[b, h] = (m + np.log(l))[:, 0]
    return o, lse


def chunk_attention_bwd(q, k, v, do, scale: float | None = None):
    """Returns (dq [B,C,H,D], dk [B,C,Hkv,D], dv [B,C,Hkv,D]): the gradients
    of the chunk's queries and of its own keys and values (the last C key
    rows); the earlier keys are detached and get none."""
    q, k, v, do = (np.asarray(t, dtype=np.float64) for t in (q, k, v, do))
    B, C, H, D = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    vis = _visible(C, Nk)
    dq = np.zeros_like(q)
    dk = np.zeros((B, C, Hkv, D))
    dv = np.zeros((B, C, Hkv, D))
    for b in range(B):
        for h in range(H):
            kh = h // (H // Hkv)
            s = np.where(vis, scale * (q[b, :, h] @ k[b, :, kh].T), -np.inf)
            p = np.exp(s - s.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            o = p @ v[b, :, kh]
            dp = do[b, :, h] @ v[b, :, kh].T
            delta = np.sum(do[b, :, h] * o, axis=1)
            ds = p * (dp - delta[:, None])
            dq[b, :, h] = scale * (ds @ k[b, :, kh])
            dk[b, :, kh] += scale * (ds.T @ q[b, :, h])[Nk - C:]
            dv[b, :, kh] += (p.T @ do[b, :, h])[Nk - C:]
    return dq, dk, dv


def segment_attention_fwd(q, k, v, causal_offset: int | None, scale: float | None = None):
    """Attention of q over one segment of keys: all of them (causal_offset
    None: the earlier, detached segment) or causally with query row i seeing
    keys [0, causal_offset + i] of the segment.  Returns (o, lse) of that
    segment alone, the pieces lse_merge combines."""
    q, k, v = (np.asarray(t, dtype=np.float64) for t in (q, k, v))
    B, C, H, D = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    vis = np.ones((C, Nk), dtype=bool) if causal_offset is None else \
        np.arange(Nk)[None, :] <= (causal_offset + np.arange(C))[:, None]
    o = np.zeros_like(q)
    lse = np.zeros((B, H, C))
    for b in range(B):
        for h in range(H):
            kh = h // (H // Hkv)
            s = np.where(vis, scale * (q[b, :, h] @ k[b, :, kh].T), -np.inf)
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            l = e.sum(axis=1, keepdims=True)
            o[b, :, h] = (e / l) @ v[b, :, kh]
            lse[b, h] = (m + np.log(l))[:, 0]
    return o, lse


def lse_merge(o_a, lse_a, o_b, lse_b):
    """Softmax attention over the union of two disjoint key sets from the two
    pieces: o [B,C,H,D], lse [B,H,C]."""
    o_a, lse_a, o_b, lse_b = (np.asarray(t, dtype=np.float64) for t in (o_a, lse_a, o_b, lse_b))
    lse = np.logaddexp(lse_a, lse_b)
    wa = np.exp(lse_a - lse).transpose(0, 2, 1)[..., None]
    wb = np.exp(lse_b - lse).transpose(0, 2, 1)[..., None]
    return wa * o_a + wb * o_b, lse
