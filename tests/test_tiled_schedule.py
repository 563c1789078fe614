"""Block-size and split invariance: the tiled schedule the kernels follow
(``tiled_ref``) equals the oracle's token-by-token recurrence for every block
size C and chunk count S, ragged tails included (CPU only)."""
import numpy as np
import pytest

import pins
import tiled_ref


@pytest.mark.parametrize("C", [1, 2, 3, 4, 8, 16, 37])
@pytest.mark.parametrize("S", [1, 2, 3, 5])
def test_forward_tiled_matches_oracle(orc, C, S):
    q, k, v, dO, lam, s0 = pins.small_case(L=37, kv0=True, lams=(1.0, 0.9, 0.0))
    o_ref, st_ref = orc.forward(q, k, v, lam, s0, want_state=True)
    o, st = tiled_ref.forward(q, k, v, lam, s0, C, S)
    pins.assert_close(o, o_ref, 1e-12, f"tiled o C={C} S={S}")
    pins.assert_close(st, st_ref, 1e-12, f"tiled state C={C} S={S}")


@pytest.mark.parametrize("C", [1, 2, 4, 8, 16, 37])
@pytest.mark.parametrize("S", [1, 2, 3])
def test_backward_tiled_matches_oracle(orc, C, S):
    q, k, v, dO, lam, s0 = pins.small_case(L=37, kv0=True, lams=(1.0, 0.9, 0.0))
    ref = orc.backward(q, k, v, lam, dO, s0)
    got = tiled_ref.backward(q, k, v, lam, dO, s0, C, S)
    for name, x, r in zip(("dq", "dk", "dv", "dkv0"), got, ref):
        pins.assert_close(x, r, 1e-12, f"tiled {name} C={C} S={S}")


def test_tiled_no_state(orc):
    q, k, v, dO, lam, _ = pins.small_case(L=20, kv0=False)
    o_ref = orc.forward(q, k, v, lam)
    o, _ = tiled_ref.forward(q, k, v, lam, None, 8, 2)
    pins.assert_close(o, o_ref, 1e-12, "tiled o, no kv0")
    ref = orc.backward(q, k, v, lam, dO)
    got = tiled_ref.backward(q, k, v, lam, dO, None, 8, 2)
    for name, x, r in zip(("dq", "dk", "dv", "dkv0"), got, ref):
        pins.assert_close(x, r, 1e-12, f"tiled {name}, no kv0")
