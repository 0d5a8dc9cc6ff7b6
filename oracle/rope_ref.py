"""fp64 CPU oracle for rotary position embedding with Position Interpolation.

TEST INFRASTRUCTURE ONLY: imported by the test suite, the package smoke check
and the benchmark's CPU-baseline leg, never by the product path; it shares no
code with the CUDA kernels.

What the pages state (LongQLoRA community post):
* §02 Introduction: LLaMA models use RoPE, rotary position encoding, so their
  context can be extended by adjusting the rotation;
* §03 Method, Background: Position Interpolation (from Meta) extends the
  context length by interpolating positions, then a short fine-tune;
* §04 Setup: Position Interpolation shrinks RoPE's rotation angles to extend
  LLaMA2 from 4096 to 8192 tokens, before S2 attention is applied.

Readings taken where the pages are silent (listed in the design notes):
* the rotary pairs are (i, i + D/2) for i < D/2 (the "rotate half" layout);
* the frequency of pair i is base^(-2i/D) with base 10000;
* Position Interpolation multiplies every position by s = L_train / L_target
  (0.5 for 4096 -> 8192), so the angle of pair i at token t is t * s * base^(-2i/D);
* the rotation is applied to q and k at their original token positions,
  before the shift and grouping of S2 attention, and not to v;
* the rotated q and k are bf16 tensors, like every activation at the call
  boundary (the forward returns them and the backward takes them), so the
  attention sees them rounded to bf16 (round to nearest even); the gradients
  pass through that rounding unchanged;
* the backward of a rotation is the rotation by the opposite angle.

All arithmetic is float64 numpy.  Layout: x is [B, N, heads, D].
"""

from __future__ import annotations

import numpy as np

from .s2_ref import s2_attention_bwd, s2_attention_fwd

__all__ = ["rope_angles", "rope_rotate", "rope_rotate_rows", "round_bf16", "s2_rope_attention_fwd",
           "s2_rope_attention_bwd", "s2_rope_unit"]


def round_bf16(x) -> np.ndarray:
    """Values rounded to bfloat16 (8 significant bits, round to nearest even),
    returned as float64: first to float32 (nearest), then the low 16 bits of
    the float32 pattern are rounded away, ties to even."""
    u = np.ascontiguousarray(np.asarray(x, dtype=np.float64).astype(np.float32)).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def rope_angles(N: int, D: int, pos_scale: float, base: float = 10000.0) -> np.ndarray:
    """[N, D/2] rotation angles: angle[t, i] = t * pos_scale * base^(-2i/D)."""
    i = np.arange(D // 2, dtype=np.float64)
    freq = base ** (-2.0 * i / D)
    t = np.arange(N, dtype=np.float64) * pos_scale
    return t[:, None] * freq[None, :]


def rope_rotate(x, pos_scale: float, base: float = 10000.0, inverse: bool = False) -> np.ndarray:
    """Rotate each pair (x_i, x_{i+D/2}) of every row t by angle[t, i]
    (by -angle[t, i] when `inverse`):
        y_i        = x_i cos a - x_{i+D/2} sin a
        y_{i+D/2}  = x_i sin a + x_{i+D/2} cos a
    x is [B, N, heads, D]; returns a float64 array of the same shape."""
    x = np.asarray(x, dtype=np.float64)
    B, N, Hx, D = x.shape
    a = rope_angles(N, D, pos_scale, base)
    if inverse:
        a = -a
    c = np.cos(a)[None, :, None, :]
    s = np.sin(a)[None, :, None, :]
    x1, x2 = x[..., : D // 2], x[..., D // 2:]
    return np.concatenate([x1 * c - x2 * s, x1 * s + x2 * c], axis=-1)


def rope_rotate_rows(x, t, pos_scale: float, base: float = 10000.0, inverse: bool = False) -> np.ndarray:
    """The same rotation for rows x [n, D] at token positions t [n] (for
    sampling single units of long sequences)."""
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[-1]
    i = np.arange(D // 2, dtype=np.float64)
    a = (np.asarray(t, dtype=np.float64) * pos_scale)[:, None] * (base ** (-2.0 * i / D))[None, :]
    if inverse:
        a = -a
    c, s = np.cos(a), np.sin(a)
    x1, x2 = x[:, : D // 2], x[:, D // 2:]
    return np.concatenate([x1 * c - x2 * s, x1 * s + x2 * c], axis=-1)


def s2_rope_unit(q, k, v, do, G: int, b: int, h: int, g: int, pos_scale: float, base: float = 10000.0,
                 piece: str = "whole", m: int | None = None, bf16_boundary: bool = True):
    """One (batch b, query head h, rolled group g) unit of S2 attention on
    rotated q and k, at original positions.  piece = "whole" (every row of the
    group), "prefix" or "suffix" (its first / last m rows, as s2_unit_prefix /
    s2_unit_suffix).  dq and this head's dk_part are rotated back (gradients
    with respect to the unrotated q and k); o, lse, dv_part as in s2_ref."""
    from .s2_ref import group_causal_attention, group_causal_attention_grad, group_prefix_attention, \
        group_suffix_attention, kv_head_of, shift_of_head
    B, N, H, D = q.shape
    Hkv = k.shape[2]
    scale = 1.0 / np.sqrt(D)
    s = shift_of_head(h, H, N, G)
    kh = kv_head_of(h, H, Hkv)
    rows = (np.arange(g * G, (g + 1) * G) + s) % N
    qg = _boundary(rope_rotate_rows(q[b, rows, h], rows, pos_scale, base), bf16_boundary)
    kg = _boundary(rope_rotate_rows(k[b, rows, kh], rows, pos_scale, base), bf16_boundary)
    vg = np.asarray(v[b, rows, kh], dtype=np.float64)
    dog = np.asarray(do[b, rows, h], dtype=np.float64)
    if piece == "whole":
        og, lse, _ = group_causal_attention(qg, kg, vg, scale)
        dq, dk, dv, _ = group_causal_attention_grad(qg, kg, vg, dog, scale)
        r = rows
    elif piece == "prefix":
        og, lse, dq, dk, dv, _ = group_prefix_attention(qg, kg, vg, dog, m, scale)
        r = rows[:m]
    else:
        og, lse, dq, dk, dv, _ = group_suffix_attention(qg, kg, vg, dog, G - m, scale)
        r = rows[G - m:]
    return {"rows": r, "o": og, "lse": lse, "kv_head": kh,
            "dq": rope_rotate_rows(dq, r, pos_scale, base, inverse=True),
            "dk_part": rope_rotate_rows(dk, r, pos_scale, base, inverse=True), "dv_part": dv}


def _boundary(x, bf16: bool):
    return round_bf16(x) if bf16 else x


def s2_rope_attention_fwd(q, k, v, G: int, pos_scale: float, base: float = 10000.0, bf16_boundary: bool = True):
    """S2 attention of rotated q and k: returns (o, lse, q_rot, k_rot), q_rot
    and k_rot as the exact rotation (fp64).  With bf16_boundary the attention
    reads them rounded to bf16 (the call boundary's dtype); without, it reads
    the exact values (the plain composite function, for the gradient pins)."""
    qr = rope_rotate(q, pos_scale, base)
    kr = rope_rotate(k, pos_scale, base)
    o, lse = s2_attention_fwd(_boundary(qr, bf16_boundary), _boundary(kr, bf16_boundary), v, G)
    return o, lse, qr, kr


def s2_rope_attention_bwd(q, k, v, do, G: int, pos_scale: float, base: float = 10000.0, bf16_boundary: bool = True):
    """Gradients with respect to the unrotated q and k (and v): the S2
    backward on the rotated inputs, then dq and dk rotated back.
    Returns (dq, dk, dv)."""
    qr = _boundary(rope_rotate(q, pos_scale, base), bf16_boundary)
    kr = _boundary(rope_rotate(k, pos_scale, base), bf16_boundary)
    dqr, dkr, dv, _ = s2_attention_bwd(qr, kr, v, do, G)
    return rope_rotate(dqr, pos_scale, base, inverse=True), rope_rotate(dkr, pos_scale, base, inverse=True), dv
