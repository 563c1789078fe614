"""The pins bite: each plausible mistake planted in a copy of the oracle
(on the CPU, in a temporary build) must make at least one pin fail."""
import os

import pytest

import oracle
import pins

# (name, original text, planted mistake)
MUTANTS = [
    ("forward_no_decay",
     "kv[i * e + j] = lam * kv[i * e + j] + (double)kt[i] * (double)vt[j];",
     "kv[i * e + j] = kv[i * e + j] + (double)kt[i] * (double)vt[j];"),
    ("forward_diagonal_decayed",
     "kv[i * e + j] = lam * kv[i * e + j] + (double)kt[i] * (double)vt[j];",
     "kv[i * e + j] = lam * (kv[i * e + j] + (double)kt[i] * (double)vt[j]);"),
    ("forward_ignores_kv0",
     "if (kv0) memcpy(kv, kv0 + bh * d * e, sizeof(double) * d * e);",
     "if (0) memcpy(kv, kv0 + bh * d * e, sizeof(double) * d * e);"),
    ("forward_wrong_operand",
     "acc += (double)qt[i] * kv[i * e + j];",
     "acc += (double)kt[i] * kv[i * e + j];"),
    ("backward_dq_stale_state",
     "st[i * e + j] = lam * st[i * e + j] + (double)kt[i] * (double)vt[j];",
     "st[i * e + j] = lam * (st[i * e + j] + (double)kt[i] * (double)vt[j]);"),
    ("backward_dq_sign",
     "dq[(bh * L + t) * d + i] = acc;",
     "dq[(bh * L + t) * d + i] = -acc;"),
    ("backward_reverse_no_decay",
     "st[i * e + j] = lam * st[i * e + j] + (double)qt[i] * (double)gt[j];",
     "st[i * e + j] = st[i * e + j] + (double)qt[i] * (double)gt[j];"),
    ("backward_reverse_off_by_one",
     "st[i * e + j] = lam * st[i * e + j] + (double)qt[i] * (double)gt[j];",
     "st[i * e + j] = lam * (st[i * e + j] + (double)qt[i] * (double)gt[j]);"),
    ("backward_dk_wrong_operand",
     "acc += (double)vt[j] * st[i * e + j];",
     "acc += (double)gt[j] * st[i * e + j];"),
    ("backward_dv_wrong_operand",
     "acc += (double)kt[i] * st[i * e + j];",
     "acc += (double)qt[i] * st[i * e + j];"),
    ("backward_dkv0_missing_lambda",
     "dkv0[bh * d * e + i] = lam * st[i];",
     "dkv0[bh * d * e + i] = st[i];"),
    ("backward_ignores_terminal_adjoint",
     "if (gend) memcpy(st, gend + bh * d * e, sizeof(double) * d * e);",
     "if (0) memcpy(st, gend + bh * d * e, sizeof(double) * d * e);"),
    ("backward_terminal_adjoint_wrong_head",
     "if (gend) memcpy(st, gend + bh * d * e, sizeof(double) * d * e);",
     "if (gend) memcpy(st, gend + (bh % H) * d * e, sizeof(double) * d * e);"),
    ("dlambda_derivative_missing_decay",
     "rt[i * e + j] = st[i * e + j] + lam * rt[i * e + j];",
     "rt[i * e + j] = st[i * e + j] + rt[i * e + j];"),
    ("dlambda_sign",
     "part[bh] = acc;",
     "part[bh] = -acc;"),
    ("decode_drops_new_token",
     "s[i * e + j] = lam * s[i * e + j] + (double)kt[i] * (double)vt[j];",
     "s[i * e + j] = lam * s[i * e + j] + (double)kt[i] * (double)vt[j] * (double)(lam != lam);"),
    ("feature_map_drops_one",
     "y[i] = elu + 1.0;",
     "y[i] = elu;"),
    ("feature_map_branches_swapped",
     "double elu = xi > 0.0 ? xi : expm1(xi);",
     "double elu = xi > 0.0 ? expm1(xi) : xi;"),
    ("feature_map_exp_not_expm1",
     "double elu = xi > 0.0 ? xi : expm1(xi);",
     "double elu = xi > 0.0 ? xi : exp(xi);"),
    ("feature_map_grad_branches_swapped",
     "double delu = xi > 0.0 ? 1.0 : exp(xi);",
     "double delu = xi > 0.0 ? exp(xi) : 1.0;"),
    ("feature_map_grad_ignores_upstream",
     "dx[i] = dy[i] * delu;",
     "dx[i] = delu;"),
    ("feature_map_grad_is_the_map",
     "double delu = xi > 0.0 ? 1.0 : exp(xi);",
     "double delu = xi > 0.0 ? xi + 1.0 : exp(xi);"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    with open(oracle.SRC) as f:
        src = f.read()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    mutated = src.replace(old, new, 1)
    cpath = os.path.join(tmp_path, f"{name}.c")
    with open(cpath, "w") as f:
        f.write(mutated)
    lib = oracle.build(src=cpath, out=os.path.join(tmp_path, f"lib{name}.so"), force=True)
    orc = oracle.Oracle(lib)
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin(orc)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"no pin caught mutant {name}"
