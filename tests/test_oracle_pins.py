"""Pins for the fp64 oracle: checks against facts that do not come from the oracle itself.

* a hand-derived worked example (all-zero scores) in tests/golden/;
* the G == N special case against torch's scaled_dot_product_attention
  (causal, float64, autograd for the backward);
* an independent N x N-mask formulation of the same forward;
* central finite differences of the backward;
* closed-form invariants: softmax rows sum to one, the first row of a group
  copies its value row, shift equivariance, group locality, the gradient
  identities, and the roll-direction invariance of the shift;
* the cost ratio printed in the LongLoRA abstract.
A few tests plant a mistake in a copy of the oracle and check that a pin fails.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle.s2_ref as ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _qkvdo(B, N, H, Hkv, D, seed=0):
    return (_rand((B, N, H, D), seed), _rand((B, N, Hkv, D), seed + 1),
            _rand((B, N, Hkv, D), seed + 2), _rand((B, N, H, D), seed + 3))


# ---------------------------------------------------------------- golden example

def test_golden_uniform_scores():
    gd = json.load(open(os.path.join(GOLDEN, "uniform_scores_n8_g4.json")))
    N, G, H, Hkv, D = gd["N"], gd["G"], gd["H"], gd["Hkv"], gd["D"]
    vals = np.array(gd["v_values"], dtype=np.float64)
    q = np.zeros((1, N, H, D))
    k = np.tile(vals[None, :, None, None], (1, 1, Hkv, D))
    v = k.copy()
    do = np.ones((1, N, H, D))
    o, lse = ref.s2_attention_fwd(q, k, v, G)
    dq, dk, dv, _ = ref.s2_attention_bwd(q, k, v, do, G)
    for h in range(H):
        np.testing.assert_allclose(o[0, :, h, 0], gd["o"][h], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[0, h], np.log(gd["lse_count"][h]), rtol=0, atol=1e-12)
        np.testing.assert_allclose(dv[0, :, h, 0], gd["dv"][h], rtol=0, atol=1e-12)
        np.testing.assert_allclose(dq[0, :, h, 0], gd["dq"][h], rtol=0, atol=1e-12)
    assert np.all(dk == 0.0)


def test_cost_model_matches_page():
    gd = json.load(open(os.path.join(GOLDEN, "cost_ratio.json")))
    f8k = sum(ref.s2_effective_flops(1, 32, 8192, 8192, 128))
    f2k = sum(ref.s2_effective_flops(1, 32, 2048, 2048, 128))
    assert f8k / f2k == gd["dense_8192_over_2048"]
    fs2 = sum(ref.s2_effective_flops(1, 32, 8192, 2048, 128))
    assert f8k / fs2 == gd["dense_over_s2_at_group_quarter"]


# ---------------------------------------------------------- dense special case

def _sdpa(q, k, v, Hkv_rep):
    # q,k,v as [B,N,H,D] float64 torch tensors; causal SDPA on [B,H,N,D]
    kk = k.repeat_interleave(Hkv_rep, dim=2)
    vv = v.repeat_interleave(Hkv_rep, dim=2)
    o = torch.nn.functional.scaled_dot_product_attention(
        q.transpose(1, 2), kk.transpose(1, 2), vv.transpose(1, 2), is_causal=True)
    return o.transpose(1, 2)


@pytest.mark.parametrize("B,N,H,Hkv,D", [(1, 32, 4, 4, 8), (2, 48, 4, 2, 16), (1, 64, 6, 1, 4)])
def test_dense_equals_sdpa_forward(B, N, H, Hkv, D):
    q, k, v, _ = _qkvdo(B, N, H, Hkv, D, seed=11)
    o, lse = ref.s2_attention_fwd(q, k, v, G=N)
    ot = _sdpa(torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), H // Hkv).numpy()
    np.testing.assert_allclose(o, ot, rtol=0, atol=1e-12)
    # lse against torch.logsumexp over the causal scores (a library reduction)
    scale = 1.0 / math.sqrt(D)
    for h in range(H):
        kh = h // (H // Hkv)
        s = scale * torch.einsum("bnd,bmd->bnm", torch.from_numpy(q[:, :, h]), torch.from_numpy(k[:, :, kh]))
        s = s.masked_fill(~torch.ones(N, N, dtype=torch.bool).tril(), float("-inf"))
        np.testing.assert_allclose(lse[:, h], torch.logsumexp(s, dim=-1).numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("B,N,H,Hkv,D", [(1, 32, 4, 4, 8), (2, 40, 4, 2, 16)])
def test_dense_equals_sdpa_backward(B, N, H, Hkv, D):
    q, k, v, do = _qkvdo(B, N, H, Hkv, D, seed=21)
    dq, dk, dv, delta = ref.s2_attention_bwd(q, k, v, do, G=N)
    qt, kt, vt = (torch.from_numpy(x).requires_grad_(True) for x in (q, k, v))
    ot = _sdpa(qt, kt, vt, H // Hkv)
    ot.backward(torch.from_numpy(do))
    np.testing.assert_allclose(dq, qt.grad.numpy(), rtol=0, atol=1e-11)
    np.testing.assert_allclose(dk, kt.grad.numpy(), rtol=0, atol=1e-11)
    np.testing.assert_allclose(dv, vt.grad.numpy(), rtol=0, atol=1e-11)
    np.testing.assert_allclose(delta, np.einsum("bnhd,bnhd->bhn", do, ot.detach().numpy()), rtol=0, atol=1e-11)


# ------------------------------------------------------- independent formulation

@pytest.mark.parametrize("B,N,G,H,Hkv,D", [
    (1, 16, 8, 4, 4, 4), (2, 32, 8, 4, 2, 8), (1, 64, 16, 8, 4, 8), (1, 48, 16, 2, 2, 4),
    (1, 64, 64, 4, 1, 8), (1, 24, 12, 6, 2, 5),
])
def test_mask_formulation_agrees(B, N, G, H, Hkv, D):
    q, k, v, _ = _qkvdo(B, N, H, Hkv, D, seed=N + G)
    o1, l1 = ref.s2_attention_fwd(q, k, v, G)
    o2, l2 = ref.s2_attention_fwd_maskform(q, k, v, G)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-12)


def test_roll_direction_is_immaterial():
    """Rolling by +G/2 instead of -G/2 yields the same ordered groups."""
    B, N, G, H, Hkv, D = 1, 32, 8, 2, 2, 4
    q, k, v, _ = _qkvdo(B, N, H, Hkv, D, seed=5)
    o, _ = ref.s2_attention_fwd(q, k, v, G)
    h, s = 1, G // 2
    # opposite direction written out: rolled position of row t is (t + s) mod N
    t = np.arange(N)
    pos = (t + s) % N
    vis = (pos[:, None] // G == pos[None, :] // G) & (pos[None, :] <= pos[:, None])
    sc = (q[0, :, h] @ k[0, :, h].T) / math.sqrt(D)
    sc = np.where(vis, sc, -np.inf)
    p = np.exp(sc - sc.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    np.testing.assert_allclose(o[0, :, h], p @ v[0, :, h], rtol=0, atol=1e-12)


# --------------------------------------------------------- finite differences

@pytest.mark.parametrize("Hkv", [4, 2])
def test_backward_finite_differences(Hkv):
    B, N, G, H, D = 1, 16, 8, 4, 4
    q, k, v, _ = _qkvdo(B, N, H, Hkv, D, seed=7)
    w = _rand((B, N, H, D), 99)        # loss L = sum(O * W), so dO = W
    dq, dk, dv, _ = ref.s2_attention_bwd(q, k, v, w, G)
    eps = 1e-6

    def loss(qq, kk, vv):
        return float(np.sum(ref.s2_attention_fwd(qq, kk, vv, G)[0] * w))

    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp = x.copy(); xp[idx] += eps
            xm = x.copy(); xm[idx] -= eps
            args_p = {"q": q, "k": k, "v": v}; args_p[name] = xp
            args_m = {"q": q, "k": k, "v": v}; args_m[name] = xm
            num[idx] = (loss(**{"qq": args_p["q"], "kk": args_p["k"], "vv": args_p["v"]})
                        - loss(**{"qq": args_m["q"], "kk": args_m["k"], "vv": args_m["v"]})) / (2 * eps)
        rel = np.linalg.norm(num - g) / np.linalg.norm(g)
        assert rel < 1e-6, (name, rel)


# ------------------------------------------------------------ invariants

def test_softmax_rows_and_first_row():
    G, D = 12, 5
    qg, kg, vg = _rand((G, D), 1), _rand((G, D), 2), _rand((G, D), 3)
    og, lse, p = ref.group_causal_attention(qg, kg, vg, 1.0 / math.sqrt(D))
    np.testing.assert_allclose(p.sum(1), 1.0, rtol=0, atol=1e-14)
    assert np.all(p[np.triu_indices(G, 1)] == 0.0)
    np.testing.assert_array_equal(og[0], vg[0])      # first row sees only itself
    assert lse[0] == pytest.approx(float(qg[0] @ kg[0]) / math.sqrt(D), abs=1e-14)


def test_shift_equivariance():
    """A shifted head equals an unshifted head run on inputs rolled by G/2, rolled back."""
    B, N, G, H, D = 2, 32, 8, 2, 4
    q, k, v, _ = _qkvdo(B, N, H, H, D, seed=3)
    o, lse = ref.s2_attention_fwd(q, k, v, G)
    s = G // 2
    rq = np.roll(q, -s, axis=1); rk = np.roll(k, -s, axis=1); rv = np.roll(v, -s, axis=1)
    # put the rolled head-1 data into head 0 (never shifted) of a fresh call
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    q2[:, :, 0], k2[:, :, 0], v2[:, :, 0] = rq[:, :, 1], rk[:, :, 1], rv[:, :, 1]
    o2, lse2 = ref.s2_attention_fwd(q2, k2, v2, G)
    np.testing.assert_allclose(np.roll(o2[:, :, 0], s, axis=1), o[:, :, 1], rtol=0, atol=1e-13)
    np.testing.assert_allclose(np.roll(lse2[:, 0], s, axis=1), lse[:, 1], rtol=0, atol=1e-13)


def test_group_locality():
    B, N, G, H, D = 1, 32, 8, 4, 4
    q, k, v, _ = _qkvdo(B, N, H, H, D, seed=4)
    o, _ = ref.s2_attention_fwd(q, k, v, G)
    for h in (0, 3):
        s = ref.shift_of_head(h, H, N, G)
        rows = (np.arange(G, 2 * G) + s) % N          # rolled group 1 of head h
        outside = np.setdiff1d(np.arange(N), rows)
        q2, k2, v2 = q.copy(), k.copy(), v.copy()
        for x in (q2, k2, v2):
            x[:, outside, h] += 5.0 * _rand((B, outside.size, D), h)
        o2, _ = ref.s2_attention_fwd(q2, k2, v2, G)
        np.testing.assert_array_equal(o2[:, rows, h], o[:, rows, h])


@pytest.mark.parametrize("Hkv", [4, 2, 1])
def test_gradient_identities(Hkv):
    B, N, G, H, D = 1, 32, 8, 4, 6
    if Hkv == 1:
        G = N      # a single kv-head can only serve heads that share one shift
    q, k, v, do = _qkvdo(B, N, H, Hkv, D, seed=8)
    dq, dk, dv, _ = ref.s2_attention_bwd(q, k, v, do, G)
    rep = H // Hkv
    for kh in range(Hkv):
        s = ref.shift_of_head(kh * rep, H, N, G)
        for g in range(N // G):
            rows = (np.arange(g * G, (g + 1) * G) + s) % N
            np.testing.assert_allclose(dk[0, rows, kh].sum(0), 0.0, atol=1e-12)
            hs = list(range(kh * rep, (kh + 1) * rep))
            np.testing.assert_allclose(dv[0, rows, kh].sum(0), do[0][np.ix_(rows, hs)].sum((0, 1)), atol=1e-12)
    assert np.sum(q * dq) == pytest.approx(np.sum(k * dk), abs=1e-10)


def test_unit_matches_full():
    B, N, G, H, Hkv, D = 2, 32, 8, 4, 2, 4
    q, k, v, do = _qkvdo(B, N, H, Hkv, D, seed=9)
    o, lse = ref.s2_attention_fwd(q, k, v, G)
    dq, dk, dv, delta = ref.s2_attention_bwd(q, k, v, do, G)
    u = ref.s2_unit(q, k, v, do, G, b=1, h=3, g=3)
    np.testing.assert_allclose(u["o"], o[1, u["rows"], 3], atol=1e-13, rtol=0)
    np.testing.assert_allclose(u["lse"], lse[1, 3, u["rows"]], atol=1e-13, rtol=0)
    np.testing.assert_allclose(u["dq"], dq[1, u["rows"], 3], atol=1e-13, rtol=0)
    np.testing.assert_allclose(u["delta"], delta[1, 3, u["rows"]], atol=1e-13, rtol=0)
    # kv-head 1 serves heads 2 and 3, which share the shift: parts sum to dk/dv
    u2 = ref.s2_unit(q, k, v, do, G, b=1, h=2, g=3)
    np.testing.assert_allclose(u["dk_part"] + u2["dk_part"], dk[1, u["rows"], 1], atol=1e-13, rtol=0)
    np.testing.assert_allclose(u["dv_part"] + u2["dv_part"], dv[1, u["rows"], 1], atol=1e-13, rtol=0)


def test_suffix_matches_full_unit():
    """The suffix oracle (used to sample long groups) equals the whole-group oracle on its rows."""
    B, N, G, H, Hkv, D = 1, 64, 32, 4, 2, 6
    q, k, v, do = _qkvdo(B, N, H, Hkv, D, seed=12)
    for h, g in ((0, 1), (3, 1), (2, 0)):
        full = ref.s2_unit(q, k, v, do, G, b=0, h=h, g=g)
        suf = ref.s2_unit_suffix(q, k, v, do, G, b=0, h=h, g=g, m=12)
        np.testing.assert_array_equal(suf["rows"], full["rows"][-12:])
        for key in ("o", "lse", "dq", "dk_part", "dv_part", "delta"):
            np.testing.assert_allclose(suf[key], full[key][-12:], rtol=0, atol=1e-12, err_msg=key)


@pytest.mark.parametrize("m,block", [(12, 5), (12, 64), (32, 7), (1, 3), (20, 20)])
def test_prefix_matches_full_unit(m, block):
    """The prefix oracle (dk/dv of a group's first key rows, which every later
    query row reaches) equals the whole-group oracle on its rows, for query
    blocks that do not divide the group, blocks smaller and larger than the
    prefix, and the whole group as the prefix."""
    B, N, G, H, Hkv, D = 1, 64, 32, 4, 2, 6
    q, k, v, do = _qkvdo(B, N, H, Hkv, D, seed=14)
    for h, g in ((0, 1), (3, 1), (2, 0)):
        full = ref.s2_unit(q, k, v, do, G, b=0, h=h, g=g)
        pre = ref.s2_unit_prefix(q, k, v, do, G, b=0, h=h, g=g, m=m, block=block)
        np.testing.assert_array_equal(pre["rows"], full["rows"][:m])
        for key in ("o", "lse", "dq", "dk_part", "dv_part", "delta"):
            np.testing.assert_allclose(pre[key], full[key][:m], rtol=0, atol=1e-12, err_msg=key)


def test_prefix_and_suffix_cover_whole_tensor_gradients():
    """dk/dv of a kv-head assembled from prefix (first half) and suffix (second
    half) pieces, summed over the kv-head's query heads, equal the whole-tensor
    backward: the two sampling oracles together reach every key row."""
    B, N, G, H, Hkv, D = 1, 48, 16, 4, 2, 5
    q, k, v, do = _qkvdo(B, N, H, Hkv, D, seed=15)
    _, dk, dv, _ = ref.s2_attention_bwd(q, k, v, do, G)
    rep = H // Hkv
    for kh in range(Hkv):
        for g in range(N // G):
            pk, pv = 0.0, 0.0
            sk, sv = 0.0, 0.0
            for h in range(kh * rep, (kh + 1) * rep):
                pre = ref.s2_unit_prefix(q, k, v, do, G, 0, h, g, m=G // 2, block=5)
                suf = ref.s2_unit_suffix(q, k, v, do, G, 0, h, g, m=G // 2)
                pk, pv = pk + pre["dk_part"], pv + pre["dv_part"]
                sk, sv = sk + suf["dk_part"], sv + suf["dv_part"]
            np.testing.assert_allclose(pk, dk[0, pre["rows"], kh], rtol=0, atol=1e-12)
            np.testing.assert_allclose(pv, dv[0, pre["rows"], kh], rtol=0, atol=1e-12)
            np.testing.assert_allclose(sk, dk[0, suf["rows"], kh], rtol=0, atol=1e-12)
            np.testing.assert_allclose(sv, dv[0, suf["rows"], kh], rtol=0, atol=1e-12)


def test_prefix_planted_mistake_fails():
    """Taking Delta from the prefix's key columns only (a plausible shortcut:
    O restricted to keys [0, m)) must break the prefix pin."""
    B, N, G, H, Hkv, D = 1, 32, 32, 2, 2, 4
    q, k, v, do = _qkvdo(B, N, H, Hkv, D, seed=16)
    full = ref.s2_unit(q, k, v, do, G, b=0, h=0, g=0)
    m = 8
    qg, kg, vg, dog = (x[0, :, 0] for x in (q, k, v, do))
    scale = 1.0 / math.sqrt(D)

    def prefix_only_delta(qg, kg, vg, dog, m, scale, block=1024):
        n = qg.shape[0]
        s = scale * (qg @ kg.T)
        s = np.where(np.tril(np.ones((n, n), dtype=bool)), s, -np.inf)
        p = np.exp(s - s.max(1, keepdims=True))
        p /= p.sum(1, keepdims=True)
        delta = np.sum(dog * (p[:, :m] @ vg[:m]), axis=1)
        ds = p * (dog @ vg.T - delta[:, None])
        return None, None, None, scale * ds[:, :m].T @ qg, p[:, :m].T @ dog, delta

    good = ref.group_prefix_attention(qg, kg, vg, dog, m, scale, block=7)
    np.testing.assert_allclose(good[3], full["dk_part"][:m], atol=1e-12, rtol=0)
    bad = prefix_only_delta(qg, kg, vg, dog, m, scale)
    assert np.abs(bad[3] - full["dk_part"][:m]).max() > 1e-3


def test_rejects_mixed_shift_kv_head():
    q, k, v, _ = _qkvdo(1, 16, 4, 1, 4)
    with pytest.raises(ValueError):
        ref.s2_attention_fwd(q, k, v, G=8)


# ------------------------------------------------- planted mistakes are caught

def test_planted_mistakes_fail_the_pins(monkeypatch):
    """Each planted mistake (in the oracle, on the CPU) must break a pin above."""
    B, N, H, D = 1, 16, 2, 4
    q, k, v, do = _qkvdo(B, N, H, H, D, seed=31)
    qt, kt, vt = (torch.from_numpy(x).requires_grad_(True) for x in (q, k, v))
    ot = _sdpa(qt, kt, vt, 1)
    ot.backward(torch.from_numpy(do))
    good = ref.group_causal_attention_grad

    def drop_delta(qg, kg, vg, dog, scale):
        og, _, p = ref.group_causal_attention(qg, kg, vg, scale)
        ds = p * (dog @ vg.T)
        return scale * ds @ kg, scale * ds.T @ qg, p.T @ dog, np.zeros(len(qg))

    def transposed_dv(qg, kg, vg, dog, scale):
        dq_, dk_, _, de = good(qg, kg, vg, dog, scale)
        _, _, p = ref.group_causal_attention(qg, kg, vg, scale)
        return dq_, dk_, p @ dog, de

    for bad in (drop_delta, transposed_dv):
        monkeypatch.setattr(ref, "group_causal_attention_grad", bad)
        dq, dk, dv, _ = ref.s2_attention_bwd(q, k, v, do, G=N)
        err = max(np.abs(dq - qt.grad.numpy()).max(), np.abs(dv - vt.grad.numpy()).max())
        assert err > 1e-3, bad.__name__
    monkeypatch.setattr(ref, "group_causal_attention_grad", good)

    # shifting the first half of the heads instead of the second breaks the golden example
    monkeypatch.setattr(ref, "shift_of_head", lambda h, H, N, G: 0 if G >= N else (G // 2 if h < H // 2 else 0))
    gd = json.load(open(os.path.join(GOLDEN, "uniform_scores_n8_g4.json")))
    vals = np.array(gd["v_values"], dtype=np.float64)
    kk = np.tile(vals[None, :, None, None], (1, 1, 2, 1))
    o, _ = ref.s2_attention_fwd(np.zeros((1, 8, 2, 1)), kk, kk, 4)
    assert np.abs(o[0, :, 1, 0] - gd["o"][1]).max() > 0.1
