"""The backward oracle against its pins, and planted mistakes in a copy of
its C source that the pins must reject (CPU only)."""
import os

import pytest

import oracle
import oracle_bwd_pins as bpins

MUTANTS = {
    # the normalisation Jacobian without its -sum_k dw_k w_k term
    "drop_dot": ("double ds = sum > ORACLE_EPS ? (dw[k] - dot) / sum : dw[k] / ORACLE_EPS;",
                 "double ds = sum > ORACLE_EPS ? dw[k] / sum : dw[k] / ORACLE_EPS;"),
    # clamped positions differentiated as if unclamped
    "clamp_branch": ("double ds = sum > ORACLE_EPS ? (dw[k] - dot) / sum : dw[k] / ORACLE_EPS;",
                     "double ds = (dw[k] - dot) / (sum > ORACLE_EPS ? sum : ORACLE_EPS);"),
    # sigmoid derivative taken at the normalised weight
    "sigmoid_deriv_of_w": ("+= ds * s[k] * (1.0 - s[k]);", "+= ds * w[k] * (1.0 - w[k]);"),
    # adjoint carried with the mirrored slot's weight (mutants must stay in
    # bounds: they run inside the test process)
    "carry_slot_swap": ("carry_next[q + k - 1] += w[k] * adj[q];",
                        "carry_next[q + k - 1] += w[2 - k] * adj[q];"),
    # adjoint not carried to the previous line
    "no_carry": ("double *t = carry; carry = carry_next; carry_next = t;", ";"),
    # du from the adjoint instead of the output gradient
    "du_from_adjoint": ("du[e] += gyv * hl[q];", "du[e] += adj[q] * hl[q];"),
    # dlambda from the output gradient instead of the adjoint
    "dlambda_from_gy": ("dlambda[e] += adj[q] * x[at(xpl, H, W, i, j)];",
                        "dlambda[e] += gyv * x[at(xpl, H, W, i, j)];"),
    # dw taken against the current line instead of the previous one
    "dw_current_line": ("dw[k] = hprv ? adj[q] * hprv[q + k - 1] : 0.0;",
                        "dw[k] = adj[q] * hl[q + k - 1];"),
    # shared logit gradients overwritten per channel instead of summed
    "share_w_overwrite": ("dwlogit[at(wpl + k, H, W, i, j)] += ds", "dwlogit[at(wpl + k, H, W, i, j)] = ds"),
    # the adjoint gated by u twice
    "u_on_carry": ("adj[q] = u[e] * gyv + carry[q];", "adj[q] = u[e] * (gyv + carry[q]);"),
}


@pytest.mark.parametrize("check", bpins.BWD_CHECKS, ids=lambda c: c.__name__)
def test_backward_pin(check):
    check(oracle.default())


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_backward_mutant_is_caught(name, tmp_path):
    src = open(oracle.SOURCE).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    mpath = os.path.join(tmp_path, f"mut_{name}.c")
    with open(mpath, "w") as f:
        f.write(src.replace(old, new))
    orc = oracle.Oracle(oracle.compile_oracle(mpath, os.path.join(tmp_path, f"libmut_{name}.so")))
    caught = []
    for check in bpins.BWD_CHECKS:
        try:
            check(orc)
        except AssertionError:
            caught.append(check.__name__)
    assert caught, f"no pin rejects backward mutant {name}"
