"""fp64 CPU oracle for 4-bit NormalFloat (NF4) weights with double
quantization, and the QKV projection that dequantizes them.

TEST INFRASTRUCTURE ONLY: imported by the test suite, the package smoke check
and the benchmark's CPU-baseline leg, never by the product path; it shares no
code with the CUDA kernels.

What the pages state (LongQLoRA community post, section 03, QLoRA): the
pretrained weights are quantized to 4 bits with the 4-bit NormalFloat data
type ("theoretically optimal", better than FP4 and Int4); Double
Quantization saves 0.37 bit per parameter on average; LongQLoRA quantizes the
whole model this way (section 04) and the attention's q, k, v come from the
quantized projections.

Readings taken where the pages are silent (listed in the design notes):
* NF4 levels (the QLoRA construction): 16 values, quantiles of the standard
  normal distribution normalised to [-1, 1] with an exact zero -- 8 positive
  levels Phi^-1(p) for p evenly spaced from 1/2 to 1 - delta (the zero is the
  first), 7 negative ones the same way with 8 points, delta = (1/30 + 1/32)/2,
  each side divided by Phi^-1(1 - delta);
* first-level blocks of 64 consecutive weights of a row with an absmax scale;
  those scales quantized to 8 bits in blocks of 256 with an fp32 second-level
  scale: 4 + 8/64 + 32/(64*256) = 4.127 bits per weight against 4.5 with fp32
  scales, the 0.37 bit the post states;
* the second level is symmetric int8 absmax: scale' = round(127 scale / c) c / 127
  with c the block's largest scale; codes are chosen against the exact
  first-level scale (nearest level of w / absmax);
* the GEMM's operand: W' in bf16, formed as level * (code * c2 / 127) with
  each operation a float32 rounding, then rounded to bf16 (a bitsandbytes-like
  fp32 dequantization feeding a bf16 GEMM);
* the projection: [q | k | v] = X W^T with W [(H + 2 Hkv) D, d_model] the
  dequantized NF4 weight (level * scale'), X bf16 activations; q, k, v come
  out in the (batch, sequence, heads, head_dim) layout as row blocks of W.

All arithmetic float64 numpy (scipy for the normal quantiles).
"""

from __future__ import annotations

import numpy as np

from oracle.rope_ref import round_bf16

__all__ = ["NF4_DELTA", "nf4_levels", "quantize_nf4", "dequantize_nf4", "nf4_qkv_projection",
           "bits_per_weight", "round_bf16", "unpack_codes", "dequantize_nf4_bf16"]

NF4_DELTA = 0.5 * (1.0 / 30.0 + 1.0 / 32.0)
BLOCK = 64
DQ_BLOCK = 256


def nf4_levels() -> np.ndarray:
    """The 16 NF4 levels, ascending (index = code)."""
    from scipy.special import ndtri
    top = ndtri(1.0 - NF4_DELTA)
    pos = ndtri(np.linspace(0.5, 1.0 - NF4_DELTA, 9)) / top          # 0 and 8 positive levels
    neg = -ndtri(np.linspace(0.5, 1.0 - NF4_DELTA, 8)[1:]) / top     # 7 negative levels
    return np.sort(np.concatenate([neg, pos]))


def bits_per_weight(double_quant: bool = True) -> float:
    return 4.0 + (8.0 / BLOCK + 32.0 / (BLOCK * DQ_BLOCK) if double_quant else 32.0 / BLOCK)


def quantize_nf4(w):
    """w [rows, K] (K % 64 == 0) -> (codes uint8 [rows, K], scale codes int8
    [rows * K / 64], second-level scales float32 [ceil(rows * K / 64 / 256)];
    the last second-level block may hold fewer than 256 first-level scales)."""
    w = np.asarray(w, dtype=np.float64)
    rows, K = w.shape
    lv = nf4_levels()
    blocks = w.reshape(-1, BLOCK)
    absmax = np.abs(blocks).max(axis=1)
    safe = np.where(absmax > 0, absmax, 1.0)
    x = blocks / safe[:, None]
    codes = np.abs(x[..., None] - lv[None, None, :]).argmin(axis=-1).astype(np.uint8)
    grp = np.arange(absmax.size) // DQ_BLOCK
    c2 = np.zeros(grp[-1] + 1)
    np.maximum.at(c2, grp, absmax)
    c2s = np.where(c2 > 0, c2, 1.0)
    sq = np.rint(absmax / c2s[grp] * 127.0).astype(np.int8)
    return codes.reshape(rows, K), sq, c2.astype(np.float32)


def dequantize_nf4(codes, scale_codes, c2) -> np.ndarray:
    """float64 [rows, K]: level[code] * scale_code * c2 / 127 per 64-block,
    c2 of the block's second-level block (first-level block index // 256)."""
    codes = np.asarray(codes)
    rows, K = codes.shape
    lv = nf4_levels()
    sq = np.asarray(scale_codes, dtype=np.float64)
    scale = sq * np.asarray(c2, dtype=np.float64)[np.arange(sq.size) // DQ_BLOCK] / 127.0
    return (lv[codes.reshape(-1, BLOCK)] * scale[:, None]).reshape(rows, K)


def dequantize_nf4_bf16(codes, scale_codes, c2) -> np.ndarray:
    """The dequantized weight as the GEMM's bf16 operand, in the precision the
    design states for it (float64 result holding bf16 values): the level table
    rounded to float32; s = float32(code) * c2 then / 127, each step a float32
    operation rounded to nearest; level * s in float32; then rounded to the
    nearest bf16 (ties to even).  Within one bf16 ulp of dequantize_nf4."""
    codes = np.asarray(codes)
    rows, K = codes.shape
    lv32 = nf4_levels().astype(np.float32)
    sq = np.asarray(scale_codes).astype(np.float32)
    c2_32 = np.asarray(c2, dtype=np.float32)[np.arange(sq.size) // DQ_BLOCK]
    s32 = (sq * c2_32) / np.float32(127.0)
    w32 = lv32[codes.reshape(-1, BLOCK)] * s32[:, None]
    assert w32.dtype == np.float32
    return round_bf16(w32).reshape(rows, K)


def unpack_codes(packed) -> np.ndarray:
    """uint8 [rows, K/2] with two codes a byte (element 2j in the low nibble)
    -> uint8 [rows, K]."""
    packed = np.asarray(packed, dtype=np.uint8)
    out = np.empty((packed.shape[0], 2 * packed.shape[1]), dtype=np.uint8)
    out[:, 0::2] = packed & 15
    out[:, 1::2] = packed >> 4
    return out


def nf4_qkv_projection(x, codes, scale_codes, c2, H: int, Hkv: int, D: int, bf16_weights: bool = False):
    """x [B, N, d_model] -> (q [B,N,H,D], k [B,N,Hkv,D], v [B,N,Hkv,D]) with
    the dequantized weight W [(H + 2 Hkv) D, d_model]: [q | k | v] = x W^T.
    bf16_weights takes W as the GEMM's bf16 operand (dequantize_nf4_bf16, the
    tensor cores' operand type) instead of the exact dequantized values."""
    x = np.asarray(x, dtype=np.float64)
    B, N, _ = x.shape
    w = dequantize_nf4_bf16(codes, scale_codes, c2) if bf16_weights else dequantize_nf4(codes, scale_codes, c2)
    y = x @ w.T
    q = y[..., : H * D].reshape(B, N, H, D)
    k = y[..., H * D:(H + Hkv) * D].reshape(B, N, Hkv, D)
    v = y[..., (H + Hkv) * D:].reshape(B, N, Hkv, D)
    return q, k, v
