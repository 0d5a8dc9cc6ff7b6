"""fp64 CPU oracle for shifted sparse attention (S2-Attn), forward and backward.

TEST INFRASTRUCTURE ONLY.  This module is the slow, obviously-correct statement
of what the CUDA path computes.  Only the test suite, the package smoke check and
the benchmark's CPU-baseline leg may import it; the product path never does, and
it shares no code with the CUDA kernels or their host library.

What is computed, and where it is stated
----------------------------------------
* LongQLoRA community post ("LongQLoRA: 单卡高效扩展 LLaMA2-13B 的上下文长度"),
  §03 Method, Background, the Shift Short Attention paragraphs: the input is
  split into groups, self-attention runs only inside each group, and attention
  is also computed "between groups" so that quality approaches global attention.
* Same post, §04 Setup: the group size is a quarter of the target length, S2 is
  used only during training, global attention at inference; the model is
  trained with next-token prediction (so attention is causal).
* LongLoRA abstract ("LongLoRA: Efficient Fine-tuning of Long-Context Large
  Language Models", chatpaper.ai page): "shift short attention", dense global
  attention needed at inference, a drop-in change of two lines in training.

Readings taken where the pages are silent (each listed in the design notes):
* the shifted heads are h >= H//2 (integer division), shifted by G//2 rows with
  wrap-around, and only when G < N; G == N is plain dense causal attention;
* rolled row r of a shifted head holds original row (r + s) mod N, i.e. the
  roll is numpy's ``roll(x, -s)``; for s = G/2 with G | N the other direction
  yields the same set of ordered groups (tested);
* causality is taken in rolled order inside a group;
* grouped-query heads: query head h reads kv-head h // (H // Hkv); the query
  heads of one kv-head must share one shift;
* scale 1/sqrt(D); lse is the natural-log log-sum-exp, stored at original
  positions;
* the backward is the analytic gradient of softmax attention:
  dP = dO V^T, Delta_i = sum_d dO_id O_id, dS = P * (dP - Delta),
  dQ = scale dS K, dK = scale dS^T Q, dV = P^T dO, with dK and dV summed over
  the query heads that share a kv-head.

All arithmetic is float64 numpy (matmuls through numpy/BLAS).  Inputs are the
exact values the GPU sees (bf16 values upcast to float64 by the caller).
Tensors use the (batch, sequence, heads, head_dim) layout: q, o, do, dq are
[B, N, H, D]; k, v, dk, dv are [B, N, Hkv, D]; lse and delta are [B, H, N].
"""

from __future__ import annotations

import math

import numpy as np

__all__ = [
    "shift_of_head",
    "kv_head_of",
    "roll_to_groups",
    "roll_back",
    "group_causal_attention",
    "group_causal_attention_grad",
    "s2_attention_fwd",
    "s2_attention_bwd",
    "s2_attention_fwd_maskform",
    "s2_unit",
    "group_suffix_attention",
    "s2_unit_suffix",
    "group_prefix_attention",
    "s2_unit_prefix",
    "s2_effective_flops",
]


# ---------------------------------------------------------------------------
# index map: which heads shift, by how much, which kv-head they read
# ---------------------------------------------------------------------------

def shift_of_head(h: int, H: int, N: int, G: int) -> int:
    """Roll amount for query head h.

    LongQLoRA post §03 (Background) says attention is also computed between
    groups; the mechanism read here is the LongLoRA one: the second half of the
    heads (h >= H//2) is rolled by half a group.  With G == N there is a single
    group and the call is dense causal attention (post §03/§04: global attention
    at inference), so nothing is shifted.
    """
    if G >= N:
        return 0
    return G // 2 if h >= H // 2 else 0


def kv_head_of(h: int, H: int, Hkv: int) -> int:
    """Grouped-query mapping: contiguous blocks of H // Hkv query heads."""
    return h // (H // Hkv)


def roll_to_groups(x: np.ndarray, s: int) -> np.ndarray:
    """Rolled sequence along axis 0: out[r] = x[(r + s) mod N]."""
    return np.roll(x, -s, axis=0)


def roll_back(x: np.ndarray, s: int) -> np.ndarray:
    """Inverse of roll_to_groups: out[(r + s) mod N] = x[r]."""
    return np.roll(x, s, axis=0)


# ---------------------------------------------------------------------------
# one group: plain causal softmax attention and its analytic gradient
# ---------------------------------------------------------------------------

def group_causal_attention(qg: np.ndarray, kg: np.ndarray, vg: np.ndarray,
                           scale: float):
    """Causal softmax attention over one group (rows in rolled order).

    S = scale * Qg Kg^T, S_ij = -inf for j > i, P = row softmax (max
    subtracted), Og = P Vg, lse_i = m_i + ln sum_j exp(S_ij - m_i).
    Returns (Og, lse, P).
    """
    n = qg.shape[0]
    s = scale * (qg @ kg.T)
    s = np.where(np.tril(np.ones((n, n), dtype=bool)), s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    p = e / l
    og = p @ vg
    lse = (m + np.log(l))[:, 0]
    return og, lse, p


def group_causal_attention_grad(qg, kg, vg, dog, scale: float):
    """Analytic backward of group_causal_attention.

    Recomputes P and O, then dP = dO V^T, Delta = rowsum(dO * O),
    dS = P * (dP - Delta), dQ = scale dS K, dK = scale dS^T Q, dV = P^T dO.
    Returns (dQg, dKg, dVg, Delta).
    """
    og, _, p = group_causal_attention(qg, kg, vg, scale)
    dp = dog @ vg.T
    delta = np.sum(dog * og, axis=1)
    ds = p * (dp - delta[:, None])
    dqg = scale * (ds @ kg)
    dkg = scale * (ds.T @ qg)
    dvg = p.T @ dog
    return dqg, dkg, dvg, delta


# ---------------------------------------------------------------------------
# whole tensors: literal roll, split, attend, unroll
# ---------------------------------------------------------------------------

def _check(q, k, v, G):
    B, N, H, D = q.shape
    Hkv = k.shape[2]
    if k.shape != (B, N, Hkv, D) or v.shape != k.shape:
        raise ValueError("k, v must be [B, N, Hkv, D] matching q")
    if H % Hkv or N % G:
        raise ValueError("need H % Hkv == 0 and N % G == 0")
    kvh = [kv_head_of(h, H, Hkv) for h in range(H)]
    for kh in range(Hkv):
        shifts = {shift_of_head(h, H, N, G) for h in range(H) if kvh[h] == kh}
        if len(shifts) != 1:
            raise ValueError("query heads of one kv-head must share a shift")
    return B, N, H, Hkv, D


def s2_attention_fwd(q, k, v, G: int, scale: float | None = None):
    """S2-Attn forward.  Returns (o [B,N,H,D], lse [B,H,N]) in float64."""
    q, k, v = (np.asarray(t, dtype=np.float64) for t in (q, k, v))
    B, N, H, Hkv, D = _check(q, k, v, G)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    o = np.zeros_like(q)
    lse = np.zeros((B, H, N))
    for b in range(B):
        for h in range(H):
            s = shift_of_head(h, H, N, G)
            kh = kv_head_of(h, H, Hkv)
            qr = roll_to_groups(q[b, :, h], s)
            kr = roll_to_groups(k[b, :, kh], s)
            vr = roll_to_groups(v[b, :, kh], s)
            orr = np.zeros((N, D))
            lr = np.zeros(N)
            for g in range(N // G):
                sl = slice(g * G, (g + 1) * G)
                orr[sl], lr[sl], _ = group_causal_attention(qr[sl], kr[sl], vr[sl], scale)
            o[b, :, h] = roll_back(orr, s)
            lse[b, h] = roll_back(lr, s)
    return o, lse


def s2_attention_bwd(q, k, v, do, G: int, scale: float | None = None):
    """S2-Attn backward.  Returns (dq, dk, dv, delta[B,H,N]) in float64.

    dk and dv of a kv-head are summed over the query heads that read it.
    """
    q, k, v, do = (np.asarray(t, dtype=np.float64) for t in (q, k, v, do))
    B, N, H, Hkv, D = _check(q, k, v, G)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    delta = np.zeros((B, H, N))
    for b in range(B):
        for h in range(H):
            s = shift_of_head(h, H, N, G)
            kh = kv_head_of(h, H, Hkv)
            qr = roll_to_groups(q[b, :, h], s)
            kr = roll_to_groups(k[b, :, kh], s)
            vr = roll_to_groups(v[b, :, kh], s)
            dor = roll_to_groups(do[b, :, h], s)
            dqr = np.zeros((N, D))
            dkr = np.zeros((N, D))
            dvr = np.zeros((N, D))
            der = np.zeros(N)
            for g in range(N // G):
                sl = slice(g * G, (g + 1) * G)
                dqr[sl], dkr[sl], dvr[sl], der[sl] = group_causal_attention_grad(
                    qr[sl], kr[sl], vr[sl], dor[sl], scale)
            dq[b, :, h] = roll_back(dqr, s)
            dk[b, :, kh] += roll_back(dkr, s)
            dv[b, :, kh] += roll_back(dvr, s)
            delta[b, h] = roll_back(der, s)
    return dq, dk, dv, delta


# ---------------------------------------------------------------------------
# an independent formulation: one N x N visibility mask per head
# ---------------------------------------------------------------------------

def s2_attention_fwd_maskform(q, k, v, G: int, scale: float | None = None):
    """Same forward written without any roll: key t' is visible to query t iff
    both fall in the same group of the head's rolled order and t' does not come
    after t in that order.  Plain dense softmax over the masked N x N scores.
    Used only to cross-check s2_attention_fwd on small inputs.
    """
    q, k, v = (np.asarray(t, dtype=np.float64) for t in (q, k, v))
    B, N, H, Hkv, D = _check(q, k, v, G)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    o = np.zeros_like(q)
    lse = np.zeros((B, H, N))
    t = np.arange(N)
    for h in range(H):
        s = shift_of_head(h, H, N, G)
        kh = kv_head_of(h, H, Hkv)
        pos = (t - s) % N               # rolled position of original row t
        grp = pos // G
        vis = (grp[:, None] == grp[None, :]) & (pos[None, :] <= pos[:, None])
        for b in range(B):
            sc = scale * (q[b, :, h] @ k[b, :, kh].T)
            sc = np.where(vis, sc, -np.inf)
            m = sc.max(axis=1, keepdims=True)
            e = np.exp(sc - m)
            l = e.sum(axis=1, keepdims=True)
            o[b, :, h] = (e / l) @ v[b, :, kh]
            lse[b, h] = (m + np.log(l))[:, 0]
    return o, lse


# ---------------------------------------------------------------------------
# one (batch, query head, group) unit at original positions, for sampling
# ---------------------------------------------------------------------------

def s2_unit(q, k, v, do, G: int, b: int, h: int, g: int,
            scale: float | None = None, backward: bool = True):
    """Oracle for one unit: batch b, query head h, rolled group g.

    Takes full tensors (any array-like, upcast to float64 for the slice only)
    and returns a dict with ``rows`` (original positions of the group's rows,
    in rolled order) and the unit's o, lse and, if ``backward``, delta, dq and
    this head's contribution dk_part / dv_part to its kv-head at those rows.
    """
    B, N, H, D = q.shape
    Hkv = k.shape[2]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    s = shift_of_head(h, H, N, G)
    kh = kv_head_of(h, H, Hkv)
    rows = (np.arange(g * G, (g + 1) * G) + s) % N
    qg = np.asarray(q[b, rows, h], dtype=np.float64)
    kg = np.asarray(k[b, rows, kh], dtype=np.float64)
    vg = np.asarray(v[b, rows, kh], dtype=np.float64)
    og, lse, _ = group_causal_attention(qg, kg, vg, scale)
    out = {"rows": rows, "o": og, "lse": lse, "kv_head": kh, "shift": s}
    if backward:
        dog = np.asarray(do[b, rows, h], dtype=np.float64)
        dqg, dkg, dvg, delta = group_causal_attention_grad(qg, kg, vg, dog, scale)
        out.update(dq=dqg, dk_part=dkg, dv_part=dvg, delta=delta)
    return out


def group_suffix_attention(qg, kg, vg, dog, i0: int, scale: float):
    """Causal attention of one group restricted to its last rows [i0, n).

    Query rows i >= i0 see keys [0, i], so their o, lse and dq are exactly
    those of the whole group; and key rows j >= i0 are seen only by query rows
    i >= j >= i0, so dk and dv of rows [i0, n) are exact as well.  Same
    definitions as group_causal_attention(_grad), evaluated on the
    (n - i0) x n block of scores only.  Returns (o, lse, dq, dk, dv, delta)
    for rows [i0, n).
    """
    n = qg.shape[0]
    qs, dos = qg[i0:], dog[i0:]
    s = scale * (qs @ kg.T)
    vis = np.arange(n)[None, :] <= np.arange(i0, n)[:, None]
    s = np.where(vis, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    p = e / l
    o = p @ vg
    lse = (m + np.log(l))[:, 0]
    dp = dos @ vg.T
    delta = np.sum(dos * o, axis=1)
    ds = p * (dp - delta[:, None])
    dq = scale * (ds @ kg)
    dk = scale * (ds.T @ qs)
    dv = p.T @ dos
    return o, lse, dq, dk[i0:], dv[i0:], delta


def s2_unit_suffix(q, k, v, do, G: int, b: int, h: int, g: int, m: int,
                   scale: float | None = None):
    """Oracle for the last m rolled rows of unit (b, h, g), at original positions.

    Returns a dict like s2_unit: rows, o, lse, dq, delta, and this head's
    contribution dk_part / dv_part to its kv-head at those rows.
    """
    B, N, H, D = q.shape
    Hkv = k.shape[2]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    s = shift_of_head(h, H, N, G)
    kh = kv_head_of(h, H, Hkv)
    rows_all = (np.arange(g * G, (g + 1) * G) + s) % N
    qg = np.asarray(q[b, rows_all, h], dtype=np.float64)
    kg = np.asarray(k[b, rows_all, kh], dtype=np.float64)
    vg = np.asarray(v[b, rows_all, kh], dtype=np.float64)
    dog = np.asarray(do[b, rows_all, h], dtype=np.float64)
    o, lse, dq, dk, dv, delta = group_suffix_attention(qg, kg, vg, dog, G - m, scale)
    return {"rows": rows_all[G - m:], "o": o, "lse": lse, "dq": dq, "dk_part": dk,
            "dv_part": dv, "delta": delta, "kv_head": kh, "shift": s}


def group_prefix_attention(qg, kg, vg, dog, m: int, scale: float, block: int = 1024):
    """Causal attention of one group, the outputs that belong to its first rows [0, m).

    Key rows j < m are read by every query row i >= j of the group, so their dk
    and dv need the whole group: the query rows are streamed in blocks of
    `block` rows.  Each block's softmax is taken over all the keys its rows see
    (keys [0, i]), its O (for Delta = rowsum(dO * O)) over all of them too, and
    only the score columns of keys [0, m) feed dk, dv.  Query rows i < m see
    only keys [0, i], so their o, lse and dq come out of the first block whole.
    Same definitions as group_causal_attention(_grad).  Returns
    (o, lse, dq, dk, dv, delta) for rows [0, m).
    """
    n, D = qg.shape
    dk = np.zeros((m, D))
    dv = np.zeros((m, D))
    o_pre = np.zeros((m, D))
    lse_pre = np.zeros(m)
    dq_pre = np.zeros((m, D))
    delta_pre = np.zeros(m)
    for i0 in range(0, n, block):
        i1 = min(n, i0 + block)
        s = scale * (qg[i0:i1] @ kg[:i1].T)
        vis = np.arange(i1)[None, :] <= np.arange(i0, i1)[:, None]
        s = np.where(vis, s, -np.inf)
        mx = s.max(axis=1, keepdims=True)
        e = np.exp(s - mx)
        l = e.sum(axis=1, keepdims=True)
        p = e / l
        o = p @ vg[:i1]
        dp = dog[i0:i1] @ vg[:i1].T
        delta = np.sum(dog[i0:i1] * o, axis=1)
        ds = p * (dp - delta[:, None])
        kc = min(m, i1)                      # key columns of the prefix this block sees
        dk[:kc] += scale * (ds[:, :kc].T @ qg[i0:i1])
        dv[:kc] += p[:, :kc].T @ dog[i0:i1]
        if i0 < m:                           # query rows of the prefix in this block
            r1 = min(m, i1)
            o_pre[i0:r1] = o[:r1 - i0]
            lse_pre[i0:r1] = (mx + np.log(l))[:r1 - i0, 0]
            dq_pre[i0:r1] = scale * (ds[:r1 - i0] @ kg[:i1])
            delta_pre[i0:r1] = delta[:r1 - i0]
    return o_pre, lse_pre, dq_pre, dk, dv, delta_pre


def s2_unit_prefix(q, k, v, do, G: int, b: int, h: int, g: int, m: int,
                   scale: float | None = None, block: int = 1024):
    """Oracle for the first m rolled rows of unit (b, h, g), at original positions.

    The counterpart of s2_unit_suffix for the start of a group: dk_part and
    dv_part of its first m key rows (the rows every later query row of the
    group contributes to), and o, lse, dq, delta of its first m query rows.
    """
    B, N, H, D = q.shape
    Hkv = k.shape[2]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    s = shift_of_head(h, H, N, G)
    kh = kv_head_of(h, H, Hkv)
    rows_all = (np.arange(g * G, (g + 1) * G) + s) % N
    qg = np.asarray(q[b, rows_all, h], dtype=np.float64)
    kg = np.asarray(k[b, rows_all, kh], dtype=np.float64)
    vg = np.asarray(v[b, rows_all, kh], dtype=np.float64)
    dog = np.asarray(do[b, rows_all, h], dtype=np.float64)
    o, lse, dq, dk, dv, delta = group_prefix_attention(qg, kg, vg, dog, m, scale, block)
    return {"rows": rows_all[:m], "o": o, "lse": lse, "dq": dq, "dk_part": dk,
            "dv_part": dv, "delta": delta, "kv_head": kh, "shift": s}


def s2_effective_flops(B: int, H: int, N: int, G: int, D: int):
    """Effective FLOPs counted the way the performance target states them:
    forward 4*B*H*N*G*D/2 (two matmuls over a causal half of each G x G
    block), backward 2.5x the forward.  Returns (fwd, bwd)."""
    fwd = 4.0 * B * H * N * G * D * 0.5
    return fwd, 2.5 * fwd
