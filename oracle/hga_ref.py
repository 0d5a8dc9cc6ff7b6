"""fp64 CPU oracle for HGA-style block-sparse attention over gathered history.

TEST INFRASTRUCTURE ONLY: imported by the test suite, the package smoke check
and the benchmark's CPU-baseline leg, never by the product path; it shares no
code with the CUDA kernels.

What the page states (HGA digest, arXiv 2607.15105, English abstract):
Hierarchical Global Attention loads, for each query block, a bounded set of
exact historical tokens; with segment-wise backpropagation only the active
segment stays differentiable and older KV is detached.

Readings taken where the page is silent (listed in the design notes):
* the sequence is cut into segments of G rows; a query row attends its own
  segment's keys causally (local attention, no shift) plus the historical
  keys selected for its query block;
* a query block is 256 rows (two 128-row tiles) and selections are whole
  128-row key tiles from earlier segments: sel[b, qb, :] lists tile indices
  (-1 = unused slot), shared by all heads; how they are chosen (chunk
  summaries) is the model's business, so the oracle takes them as input;
* the historical keys are detached: dq flows through every attended key,
  dk and dv only to keys through the local (same-segment) attention;
* scale 1/sqrt(D), lse natural log, grouped-query heads as in s2_ref.

All arithmetic is float64 numpy.  q, o, do, dq: [B, N, H, D]; k, v, dk, dv:
[B, N, Hkv, D]; sel: int [B, N/256, S]; lse: [B, H, N].
"""

from __future__ import annotations

import math

import numpy as np

__all__ = ["QBLOCK", "hga_visible", "hga_attention_fwd", "hga_attention_bwd"]

QBLOCK = 256


def hga_visible(N: int, G: int, sel_b) -> tuple[np.ndarray, np.ndarray]:
    """Masks [N, N] for one batch entry: `local` (same segment, key not after
    the query) and `hist` (key in a tile selected for the query's block)."""
    t = np.arange(N)
    local = (t[:, None] // G == t[None, :] // G) & (t[None, :] <= t[:, None])
    hist = np.zeros((N, N), dtype=bool)
    for qb in range(N // QBLOCK):
        for tile in np.asarray(sel_b[qb]):
            if tile >= 0:
                hist[qb * QBLOCK:(qb + 1) * QBLOCK, tile * 128:(tile + 1) * 128] = True
    return local, hist & ~local


def _check(q, k, G, sel):
    B, N, H, D = q.shape
    if N % G or G % QBLOCK or np.asarray(sel).shape[:2] != (B, N // QBLOCK):
        raise ValueError("need N % G == 0, G % 256 == 0 and sel of shape [B, N/256, S]")
    for b in range(B):
        for qb in range(N // QBLOCK):
            for tile in np.asarray(sel[b][qb]):
                if tile >= 0 and tile * 128 >= (qb * QBLOCK // G) * G:
                    raise ValueError("selected tiles must lie in earlier segments")
    return B, N, H, k.shape[2], D


def hga_attention_fwd(q, k, v, G: int, sel, scale: float | None = None):
    """Returns (o, lse): softmax over the union of local and selected keys."""
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    B, N, H, Hkv, D = _check(q, k, G, sel)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    o = np.zeros_like(q)
    lse = np.zeros((B, H, N))
    for b in range(B):
        local, hist = hga_visible(N, G, sel[b])
        vis = local | hist
        for h in range(H):
            kh = h // (H // Hkv)
            s = np.where(vis, scale * (q[b, :, h] @ k[b, :, kh].T), -np.inf)
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            l = e.sum(axis=1, keepdims=True)
            o[b, :, h] = (e / l) @ v[b, :, kh]
            lse[b, h] = (m + np.log(l))[:, 0]
    return o, lse


def hga_attention_bwd(q, k, v, do, G: int, sel, scale: float | None = None):
    """Returns (dq, dk, dv): dq through every attended key; dk, dv through
    the local attention only (historical keys are detached)."""
    q, k, v, do = (np.asarray(x, dtype=np.float64) for x in (q, k, v, do))
    B, N, H, Hkv, D = _check(q, k, G, sel)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        local, hist = hga_visible(N, G, sel[b])
        vis = local | hist
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
            dsl = np.where(local, ds, 0.0)                 # gradient reaches keys only through local attention
            dk[b, :, kh] += scale * (dsl.T @ q[b, :, h])
            dv[b, :, kh] += np.where(local, p, 0.0).T @ do[b, :, h]
    return dq, dk, dv
