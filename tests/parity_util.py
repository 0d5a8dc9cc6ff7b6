"""Comparison helpers shared by the GPU parity tests (no attention arithmetic here:
the gradient identities below are sums over given outputs)."""
from __future__ import annotations

import numpy as np
import torch

# Tolerances of the GPU path against the fp64 oracle (bf16 inputs, fp32 accumulate):
O_MAX_ABS = 1e-2
O_REL_FRO = 5e-3
GRAD_REL_FRO = 1e-2


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def rel_fro(got: np.ndarray, ref: np.ndarray) -> float:
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / (den if den > 0 else 1.0))


def max_abs(got: np.ndarray, ref: np.ndarray) -> float:
    return float(np.max(np.abs(got - ref))) if got.size else 0.0


def report(name: str, got: np.ndarray, ref: np.ndarray) -> str:
    idx = np.unravel_index(np.argmax(np.abs(got - ref)), got.shape) if got.size else ()
    return (f"{name}: max_abs={max_abs(got, ref):.3e} rel_fro={rel_fro(got, ref):.3e} "
            f"worst@{tuple(int(i) for i in idx)} got={got[idx] if got.size else 0:.5f} "
            f"ref={ref[idx] if got.size else 0:.5f}")


def check_o(got, ref, what=""):
    msg = report("O" + what, got, ref)
    assert max_abs(got, ref) <= O_MAX_ABS and rel_fro(got, ref) <= O_REL_FRO, msg
    return msg


def check_grad(name, got, ref, what=""):
    msg = report(name + what, got, ref)
    assert rel_fro(got, ref) <= GRAD_REL_FRO, msg
    return msg


def check_identities(shape, q, k, do, dq, dk, dv):
    """Exact identities of the backward, checked on EVERY (batch, kv-head, group)
    unit at full size (the oracle itself satisfies them to ~1e-15):
      sum_j dK_j = 0        (softmax is unchanged when a constant is added to all keys),
      sum_j dV_j = sum_i dO_i over the kv-head's query heads   (rows of P sum to one),
      sum_i q_i . dQ_i = sum_j k_j . dK_j   (S is bilinear in q and k).
    The GPU's outputs are bf16-rounded results of fp32 arithmetic; independent
    errors of relative size e add up to about e * sqrt(G) * (rms row norm), so
    each residual is normalised by sqrt(G) * rms and must stay below 2e-2,
    twice the gradients' relative Frobenius tolerance.  A missed tile, head or
    group leaves a residual of order one."""
    G, rep = shape.G, shape.H // shape.Hkv
    worst = {"dK": 0.0, "dV": 0.0, "qdQ": 0.0}
    for b in range(shape.B):
        for kh in range(shape.Hkv):
            h0 = kh * rep
            s = G // 2 if (G < shape.N and h0 >= shape.H // 2) else 0
            for g in range(shape.N // G):
                rows = (np.arange(g * G, (g + 1) * G) + s) % shape.N
                dkg = dk[b, rows, kh].astype(np.float64)
                dvg = dv[b, rows, kh].astype(np.float64)
                kg = k[b, rows, kh].astype(np.float64)
                rms_k = np.sqrt(np.mean(np.sum(dkg * dkg, axis=1)))
                rms_v = np.sqrt(np.mean(np.sum(dvg * dvg, axis=1)))
                rk = np.linalg.norm(dkg.sum(0)) / (np.sqrt(G) * rms_k)
                target = do[b][np.ix_(rows, range(h0, h0 + rep))].astype(np.float64).sum((0, 1))
                rv = np.linalg.norm(dvg.sum(0) - target) / (np.sqrt(G) * rms_v)
                qdq = np.einsum("nhd,nhd->nh", q[b][np.ix_(rows, range(h0, h0 + rep))].astype(np.float64),
                                dq[b][np.ix_(rows, range(h0, h0 + rep))].astype(np.float64))
                kdk = np.einsum("nd,nd->n", kg, dkg)
                rq = abs(qdq.sum() - kdk.sum()) / (np.sqrt(G * rep) * np.sqrt(np.mean(qdq * qdq)))
                for key, r in (("dK", rk), ("dV", rv), ("qdQ", rq)):
                    assert r <= 2e-2, f"identity {key} at b{b} kvh{kh} g{g}: residual {r:.3e}"
                    worst[key] = max(worst[key], r)
    return "identities over all units, worst normalised residual: " + \
        " ".join(f"{k_}={v_:.2e}" for k_, v_ in worst.items())
