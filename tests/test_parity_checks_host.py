"""CPU checks of the GPU parity machinery itself (no GPU needed).

The full-size parity tests check exact gradient identities on every unit.  Here
the same check is fed the oracle's own gradients, rounded to bf16 like the
GPU's outputs (it must pass), and the same gradients with a planted mistake of
the kind a kernel could make (it must fail).
"""
import numpy as np
import pytest
import torch

import oracle.s2_ref as ref
from sparse_attention_attn_b200 import inputs as I
from tests.parity_util import check_identities


def _bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).float().numpy()


@pytest.fixture(scope="module")
def grads():
    shape = I.Shape("ident", 1, 4, 2, 64, 512, 256)   # shifted heads 2-3, two query heads per kv-head
    q, k, v, do = (t.float().numpy() for t in I.make_inputs(shape, seed_offset=21))
    dq, dk, dv, _ = ref.s2_attention_bwd(q, k, v, do, shape.G)
    return shape, q, k, v, do, _bf16(dq), _bf16(dk), _bf16(dv)


def test_identities_hold_for_rounded_oracle(grads):
    shape, q, k, v, do, dq, dk, dv = grads
    msg = check_identities(shape, q, k, do, dq, dk, dv)
    print(msg)
    assert "worst" in msg


@pytest.mark.parametrize("plant", ["dk_tile_lost", "dv_head_lost", "dq_tile_lost", "dk_wrong_group"])
def test_identities_catch_planted_mistakes(grads, plant):
    shape, q, k, v, do, dq, dk, dv = grads
    dq, dk, dv = dq.copy(), dk.copy(), dv.copy()
    G, N = shape.G, shape.N
    if plant == "dk_tile_lost":          # one 128-row tile of kv-head 0 never written
        dk[0, 128:256, 0] = 0.0
    elif plant == "dv_head_lost":        # the second query head of kv-head 1 not summed in
        for g in range(N // G):
            u = ref.s2_unit(q, k, v, do, G, 0, 3, g)
            dv[0, u["rows"], 1] -= u["dv_part"]
    elif plant == "dq_tile_lost":
        dq[0, 0:128, 1] = 0.0
    else:                                # a shifted kv-head's rows written one group too early
        dk[0, :, 1] = np.roll(dk[0, :, 1], -G // 2, axis=0)
    with pytest.raises(AssertionError, match="identity"):
        check_identities(shape, q, k, do, dq, dk, dv)
