"""GPU parity of the NF4 kernels (through the C ABI) against the fp64 oracle
in oracle/nf4_ref.py.

* dequantization alone: bit-exact against the oracle's bf16 operand in the
  stated precision (float32 steps, then bf16), within one bf16 ulp of the
  exact level * scale everywhere and equal to its nearest bf16 for all but a
  tiny fraction;
* the fused QKV projection against the oracle's x W'^T with that bf16
  operand: element-wise within half a bf16 ulp of the result (|y| 2^-8) plus
  2e-4 of the result's rms (fp32 accumulation order), relative Frobenius error
  within 3e-3; shapes with ragged token tails, one token, GQA
  head counts, head dim 64, and weights quantized by the oracle from normal
  draws as well as random storage;
* the full-size projection of a LLaMA2-7B layer at 8192 tokens on sampled
  tokens.
"""
import numpy as np
import pytest
import torch

import oracle.nf4_ref as nr
from sparse_attention_attn_b200 import inputs as I

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _pack(codes_u8: np.ndarray) -> np.ndarray:
    return (codes_u8[:, 0::2] | (codes_u8[:, 1::2] << 4)).astype(np.uint8)


def _to64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def _check_proj(name, got, ref):
    rms = float(np.sqrt(np.mean(ref ** 2)))
    err = np.abs(got - ref)
    bound = np.abs(ref) * 2.0 ** -8 + 2e-4 * rms
    worst = float(np.max(err - bound))
    frob = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    print(f"{name}: max_abs {err.max():.3e} rms {rms:.3e} rel_frob {frob:.2e}")
    over = np.argwhere((err - bound).reshape(-1) > 0).reshape(-1)
    if over.size:
        g, r = got.reshape(-1), ref.reshape(-1)
        print(f"  {over.size} elements over the bound; first: " + ", ".join(
            f"[{i}] ref {r[i]:.6f} got {g[i]:.6f} rn(ref) {float(nr.round_bf16(r[i])):.6f}" for i in over[:6]))
    assert worst <= 0, f"{name}: element error exceeds half an ulp + 1e-3 rms by {worst:.3e}"
    assert frob <= 3e-3, f"{name}: relative Frobenius error {frob:.2e}"


def _run_proj(B, N, K, H, Hkv, D, codes, sq, c2, seed):
    import sparse_attention_attn_b200 as s2
    x = I.randn_bf16((B, N, K), seed)
    q, k, v = s2.nf4_qkv(x.to(DEV), codes.to(DEV), sq.to(DEV), c2.to(DEV), H, Hkv, D)
    torch.cuda.synchronize()
    assert s2.device_status() == 0
    return x, q, k, v


def test_library_levels_match_oracle():
    import sparse_attention_attn_b200 as s2
    np.testing.assert_allclose(np.array(s2.nf4_levels(), dtype=np.float64), nr.nf4_levels(), rtol=0, atol=6e-8)


@pytest.mark.parametrize("rows,K", [(128, 64), (384, 1024), (1000, 512)])
def test_dequant_against_oracle(rows, K):
    import sparse_attention_attn_b200 as s2
    codes, sq, c2 = I.make_nf4_weights(rows, K, seed=rows + K)
    w = s2.nf4_dequantize(codes.to(DEV), sq.to(DEV), c2.to(DEV))
    torch.cuda.synchronize()
    c = nr.unpack_codes(codes.numpy())
    exact = nr.dequantize_nf4(c, sq.numpy(), c2.numpy())
    got = _to64(w)
    # the stated precision (float32 steps, then bf16): bit-exact
    np.testing.assert_array_equal(got, nr.dequantize_nf4_bf16(c, sq.numpy(), c2.numpy()))
    rn = nr.round_bf16(exact)
    ulp = np.maximum(np.abs(rn), 1e-30) * 2.0 ** -7
    assert np.all(np.abs(got - exact) <= ulp), "an element is more than one bf16 ulp from level * scale"
    frac_equal = float(np.mean(got == rn))
    print(f"dequant {rows}x{K}: {frac_equal:.6f} equal to RNE(level * scale)")
    assert frac_equal >= 0.999


PROJ_SHAPES = [
    # (B, N, K, H, Hkv, D)
    (1, 300, 256, 2, 1, 128),     # ragged token tail, 4 weight tiles
    (2, 512, 1024, 4, 2, 64),     # head dim 64, GQA
    (1, 1, 512, 2, 2, 64),        # a single token
    (1, 257, 4096, 8, 8, 128),    # model width 4096, one token past a tile
    (1, 1024, 2048, 8, 2, 128),   # several token tiles, GQA
]


@pytest.mark.parametrize("B,N,K,H,Hkv,D", PROJ_SHAPES)
def test_projection_random_storage(B, N, K, H, Hkv, D):
    rows = (H + 2 * Hkv) * D
    codes, sq, c2 = I.make_nf4_weights(rows, K, seed=7 + N)
    x, q, k, v = _run_proj(B, N, K, H, Hkv, D, codes, sq, c2, seed=40 + N)
    rq, rk, rv = nr.nf4_qkv_projection(x.float().numpy(), nr.unpack_codes(codes.numpy()), sq.numpy(), c2.numpy(),
                                       H, Hkv, D, bf16_weights=True)
    for name, got, ref in (("q", q, rq), ("k", k, rk), ("v", v, rv)):
        _check_proj(f"{name} {B}x{N}x{K}", _to64(got), ref)


def test_projection_of_quantized_normal_weights():
    B, N, K, H, Hkv, D = 1, 640, 1024, 4, 2, 128
    rows = (H + 2 * Hkv) * D
    rng = np.random.default_rng(5)
    w = rng.standard_normal((rows, K)) * 0.02
    codes_u8, sq, c2 = nr.quantize_nf4(w)
    codes = torch.from_numpy(_pack(codes_u8))
    x, q, k, v = _run_proj(B, N, K, H, Hkv, D, codes, torch.from_numpy(sq), torch.from_numpy(c2), seed=77)
    rq, rk, rv = nr.nf4_qkv_projection(x.float().numpy(), codes_u8, sq, c2, H, Hkv, D, bf16_weights=True)
    for name, got, ref in (("q", q, rq), ("k", k, rk), ("v", v, rv)):
        _check_proj(f"{name} quantized normal", _to64(got), ref)
    # and against the unquantized weight: the NF4 error stays at the level the
    # 4-bit type allows (relative Frobenius well under 0.2)
    full = x.float().numpy().astype(np.float64) @ w.T
    got = np.concatenate([_to64(t).reshape(B, N, -1) for t in (q, k, v)], axis=-1)
    rel = np.linalg.norm(got - full) / np.linalg.norm(full)
    print(f"NF4 projection vs unquantized weights: rel_frob {rel:.3f}")
    assert rel < 0.2


def test_full_size_llama2_7b_sampled_tokens():
    c = I.NF4_LLAMA2_7B_8K
    M, K, H, Hkv, D = c["M"], c["K"], c["H"], c["Hkv"], c["D"]
    rows = (H + 2 * Hkv) * D
    codes, sq, c2 = I.make_nf4_weights(rows, K, seed=3)
    x, q, k, v = _run_proj(1, M, K, H, Hkv, D, codes, sq, c2, seed=90)
    toks = np.sort(np.random.default_rng(11).choice(M, size=48, replace=False))
    toks[-1] = M - 1
    xs = x.float().numpy()[:, toks]
    rq, rk, rv = nr.nf4_qkv_projection(xs, nr.unpack_codes(codes.numpy()), sq.numpy(), c2.numpy(), H, Hkv, D,
                                       bf16_weights=True)
    for name, got, ref in (("q", q, rq), ("k", k, rk), ("v", v, rv)):
        _check_proj(f"{name} llama2-7b sampled", _to64(got[:, toks]), ref)


def test_rejections():
    import sparse_attention_attn_b200 as s2
    codes, sq, c2 = (t.to(DEV) for t in I.make_nf4_weights(384, 128, seed=1))
    x = torch.zeros((1, 4, 128), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(ValueError):  # 384 weight rows, 3 * 256 = 768 expected
        s2.nf4_qkv(x, codes, sq, c2, 1, 1, 256)
    codes, sq, c2 = (t.to(DEV) for t in I.make_nf4_weights(192, 128, seed=2))
    with pytest.raises(s2.S2AttnError):  # H D = 64 is not a multiple of 128
        s2.nf4_qkv(x, codes, sq, c2, 1, 1, 64)


@pytest.mark.parametrize("spec", ["nf4_stages=4", "nf4_dq=12"])
def test_projection_variants(spec):
    """Each selectable variant of the NF4 kernel (pipeline depth, dequantization
    warps) on a shape with more tiles than a B200 has SMs (every CTA crosses
    tiles) and a ragged token tail."""
    from sparse_attention_attn_b200 import _lib
    B, N, K, H, Hkv, D = 1, 2600, 1024, 16, 8, 128
    rows = (H + 2 * Hkv) * D
    codes, sq, c2 = I.make_nf4_weights(rows, K, seed=21)
    _lib.s2attn_set_tile_override(spec)
    try:
        x, q, k, v = _run_proj(B, N, K, H, Hkv, D, codes, sq, c2, seed=22)
    finally:
        _lib.s2attn_set_tile_override(None)
    rq, rk, rv = nr.nf4_qkv_projection(x.float().numpy(), nr.unpack_codes(codes.numpy()), sq.numpy(), c2.numpy(),
                                       H, Hkv, D, bf16_weights=True)
    for name, got, ref in (("q", q, rq), ("k", k, rk), ("v", v, rv)):
        _check_proj(f"{name} [{spec}]", _to64(got), ref)
