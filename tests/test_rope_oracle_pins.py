"""Pins for the RoPE + Position Interpolation oracle (oracle/rope_ref.py), from
facts that do not come from the oracle itself:

* a hand-worked example (tests/golden/rope_pi_d4.json);
* the complex-number form of the rotation (numpy complex exponentials);
* relative-position invariance: <R(m) u, R(n) w> depends only on m - n;
* Position Interpolation: scale s at token t equals scale 1 at position t*s;
* rotations keep norms, position 0 is the identity, the inverse undoes it;
* central finite differences of S2 attention on rotated inputs.
Planted mistakes (on the CPU, in copies of the oracle) must break a pin.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle.rope_ref as rr

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_bf16_rounding_matches_torch_and_ties():
    """round_bf16 against torch's float32 -> bfloat16 cast (a library
    routine), and hand-picked ties: 1 + 2^-8 (halfway, even below) rounds down,
    1 + 3*2^-8 (halfway, odd below) rounds up."""
    import torch
    x = np.random.default_rng(30).standard_normal(100_000).astype(np.float32) * 10.0
    ref = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(rr.round_bf16(x), ref)
    np.testing.assert_array_equal(rr.round_bf16([1 + 2**-8, 1 + 3 * 2**-8, -(1 + 2**-8)]), [1.0, 1 + 2**-6, -1.0])


def test_golden_hand_example():
    gd = json.load(open(os.path.join(GOLDEN, "rope_pi_d4.json")))
    x = np.zeros((1, gd["t"] + 1, 1, gd["D"]))
    x[0, gd["t"], 0] = gd["x"]
    y = rr.rope_rotate(x, gd["pos_scale"], gd["base"])
    np.testing.assert_allclose(y[0, gd["t"], 0], gd["y"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(rr.rope_angles(gd["t"] + 1, gd["D"], gd["pos_scale"], gd["base"])[gd["t"]],
                               gd["angles"], rtol=1e-15, atol=0)


def test_complex_form():
    B, N, H, D = 2, 37, 3, 16
    x = _rand((B, N, H, D), 1)
    y = rr.rope_rotate(x, 0.25, 500.0)
    z = x[..., : D // 2] + 1j * x[..., D // 2:]
    t = np.arange(N)[:, None] * 0.25
    a = t * 500.0 ** (-np.arange(D // 2) * 2.0 / D)[None, :]
    zr = z * np.exp(1j * a)[None, :, None, :]
    np.testing.assert_allclose(y[..., : D // 2], zr.real, rtol=0, atol=1e-12)
    np.testing.assert_allclose(y[..., D // 2:], zr.imag, rtol=0, atol=1e-12)


def test_relative_position_invariance():
    N, D = 64, 32
    u, w = _rand(D, 2), _rand(D, 3)
    q = np.tile(u, (1, N, 1, 1))
    k = np.tile(w, (1, N, 1, 1))
    qr, kr = rr.rope_rotate(q, 0.5), rr.rope_rotate(k, 0.5)
    for m, n in ((10, 3), (40, 33), (63, 56)):           # all at distance 7
        np.testing.assert_allclose(qr[0, m, 0] @ kr[0, n, 0], qr[0, 10, 0] @ kr[0, 3, 0], rtol=0, atol=1e-12)
    assert abs(qr[0, 10, 0] @ kr[0, 3, 0] - qr[0, 10, 0] @ kr[0, 4, 0]) > 1e-6


def test_position_interpolation_is_scaled_positions():
    N, D = 48, 8
    x = np.tile(_rand(D, 4), (1, N, 1, 1))
    half = rr.rope_rotate(x, 0.5)
    full = rr.rope_rotate(x, 1.0)
    np.testing.assert_allclose(half[0, 0::2], full[0, : N // 2], rtol=0, atol=1e-12)   # token 2j at s=1/2 == position j
    # PI keeps every angle of an 8192-token sequence below 4096 * frequency,
    # the range of positions a 4096-token model was trained on
    a = rr.rope_angles(8192, 128, 4096 / 8192)
    freq = 10000.0 ** (-2.0 * np.arange(64) / 128)
    assert np.all(a.max(axis=0) < 4096 * freq)
    assert np.any(rr.rope_angles(8192, 128, 1.0).max(axis=0) >= 4096 * freq)


def test_norms_identity_and_inverse():
    x = _rand((2, 40, 4, 32), 5)
    y = rr.rope_rotate(x, 0.5)
    np.testing.assert_allclose(np.linalg.norm(y[..., :16] + 0j, axis=-1) ** 2 + np.linalg.norm(y[..., 16:], axis=-1) ** 2,
                               np.linalg.norm(x, axis=-1) ** 2, rtol=1e-12)
    np.testing.assert_array_equal(y[:, 0], x[:, 0])
    np.testing.assert_allclose(rr.rope_rotate(y, 0.5, inverse=True), x, rtol=0, atol=1e-12)


@pytest.mark.parametrize("Hkv", [4, 2])
def test_backward_finite_differences(Hkv):
    B, N, G, H, D = 1, 16, 8, 4, 4
    q, k, v = _rand((B, N, H, D), 6), _rand((B, N, Hkv, D), 7), _rand((B, N, Hkv, D), 8)
    w = _rand((B, N, H, D), 9)
    dq, dk, dv = rr.s2_rope_attention_bwd(q, k, v, w, G, 0.5, 100.0, bf16_boundary=False)
    eps = 1e-6

    def loss(qq, kk, vv):
        return float(np.sum(rr.s2_rope_attention_fwd(qq, kk, vv, G, 0.5, 100.0, bf16_boundary=False)[0] * w))

    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = {"q": q, "k": k, "v": v, name: xp}
            args_m = {"q": q, "k": k, "v": v, name: xm}
            num[idx] = (loss(args_p["q"], args_p["k"], args_p["v"]) - loss(args_m["q"], args_m["k"], args_m["v"])) / (2 * eps)
        assert np.linalg.norm(num - g) / np.linalg.norm(g) < 1e-6, name


def test_planted_mistakes_fail(monkeypatch):
    gd = json.load(open(os.path.join(GOLDEN, "rope_pi_d4.json")))

    def interleaved(x, pos_scale, base=10000.0, inverse=False):      # pairs (2i, 2i+1) instead of (i, i+D/2)
        x = np.asarray(x, dtype=np.float64)
        a = rr.rope_angles(x.shape[1], x.shape[3], pos_scale, base) * (-1 if inverse else 1)
        c, s = np.cos(a)[None, :, None, :], np.sin(a)[None, :, None, :]
        y = x.copy()
        y[..., 0::2] = x[..., 0::2] * c - x[..., 1::2] * s
        y[..., 1::2] = x[..., 0::2] * s + x[..., 1::2] * c
        return y

    x = np.zeros((1, 2, 1, 4))
    x[0, 1, 0] = gd["x"]
    assert np.abs(interleaved(x, 0.5)[0, 1, 0] - gd["y"]).max() > 1e-2

    # forgetting to rotate the gradients back breaks the finite-difference pin
    q, k, v, w = _rand((1, 8, 2, 4), 10), _rand((1, 8, 2, 4), 11), _rand((1, 8, 2, 4), 12), _rand((1, 8, 2, 4), 13)
    good = rr.rope_rotate
    monkeypatch.setattr(rr, "rope_rotate", lambda x, s, base=10000.0, inverse=False: good(x, s, base, False))
    dq_bad, _, _ = rr.s2_rope_attention_bwd(q, k, v, w, 8, 0.5, 100.0, bf16_boundary=False)
    monkeypatch.setattr(rr, "rope_rotate", good)
    dq_good, _, _ = rr.s2_rope_attention_bwd(q, k, v, w, 8, 0.5, 100.0, bf16_boundary=False)
    eps = 1e-6
    qp, qm = q.copy(), q.copy()
    qp[0, 5, 1, 2] += eps
    qm[0, 5, 1, 2] -= eps
    num = (np.sum(rr.s2_rope_attention_fwd(qp, k, v, 8, 0.5, 100.0, bf16_boundary=False)[0] * w)
           - np.sum(rr.s2_rope_attention_fwd(qm, k, v, 8, 0.5, 100.0, bf16_boundary=False)[0] * w)) / (2 * eps)
    assert abs(num - dq_good[0, 5, 1, 2]) < 1e-6
    assert abs(num - dq_bad[0, 5, 1, 2]) > 1e-4


def test_rows_and_unit_match_whole_tensor():
    """The row-sampling forms equal the whole-tensor oracle on their rows."""
    import oracle.s2_ref as ref
    B, N, G, H, Hkv, D = 1, 64, 32, 4, 2, 6
    q, k, v, do = _rand((B, N, H, D), 20), _rand((B, N, Hkv, D), 21), _rand((B, N, Hkv, D), 22), _rand((B, N, H, D), 23)
    rows = np.array([5, 63, 0, 17])
    np.testing.assert_allclose(rr.rope_rotate_rows(q[0, rows, 1], rows, 0.5, 100.0),
                               rr.rope_rotate(q, 0.5, 100.0)[0, rows, 1], rtol=0, atol=1e-13)
    o, lse, _, _ = rr.s2_rope_attention_fwd(q, k, v, G, 0.5, 100.0)
    dq, dk, dv = rr.s2_rope_attention_bwd(q, k, v, do, G, 0.5, 100.0)
    # the bf16 boundary is a rounding of the exact rotation, and moves o by a bf16 ulp's worth
    o_exact, _, _, _ = rr.s2_rope_attention_fwd(q, k, v, G, 0.5, 100.0, bf16_boundary=False)
    assert 0 < np.abs(o - o_exact).max() < 1e-2
    for h, g in ((0, 1), (3, 1), (2, 0)):
        kh = h // (H // Hkv)
        parts = {}
        for piece, m in (("whole", None), ("prefix", 12), ("suffix", 12)):  # noqa: B007
            u = rr.s2_rope_unit(q, k, v, do, G, 0, h, g, 0.5, 100.0, piece, m)
            np.testing.assert_allclose(u["o"], o[0, u["rows"], h], atol=1e-12, rtol=0)
            np.testing.assert_allclose(u["lse"], lse[0, h, u["rows"]], atol=1e-12, rtol=0)
            np.testing.assert_allclose(u["dq"], dq[0, u["rows"], h], atol=1e-12, rtol=0)
            parts[piece] = u
        # the kv-head's dk / dv are the sums of its query heads' parts
        h2 = kh * (H // Hkv) + (1 - h % 2)
        u2 = rr.s2_rope_unit(q, k, v, do, G, 0, h2, g, 0.5, 100.0)
        np.testing.assert_allclose(parts["whole"]["dk_part"] + u2["dk_part"], dk[0, u2["rows"], kh], atol=1e-12, rtol=0)
        np.testing.assert_allclose(parts["whole"]["dv_part"] + u2["dv_part"], dv[0, u2["rows"], kh], atol=1e-12, rtol=0)
