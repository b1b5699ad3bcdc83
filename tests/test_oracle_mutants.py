"""Are the oracle's pins sharp?  Plant one plausible mistake at a time in a
copy of the oracle's C source (on the CPU, in a temporary directory),
compile it, and require that at least one pin rejects it."""
import os

import pytest

import oracle
import oracle_pins as pins

MUTANTS = {
    # slot k read as offset 1-k instead of k-1 (neighbour orientation)
    "slot_orientation": ("acc += w[k] * hprev[q + k - 1];", "acc += w[k] * hprev[q - k + 1];"),
    # lambda dropped from the input term
    "drop_lambda": ("acc += lambda[at(gp, H, W, i, j)] * x[at(xp, H, W, i, j)];",
                    "acc += x[at(xp, H, W, i, j)];"),
    # u dropped from the output gate
    "drop_u": ("out[at(xp, H, W, i, j)] += u[at(gp, H, W, i, j)] * hcur[q];",
               "out[at(xp, H, W, i, j)] += hcur[q];"),
    # sigmoid with the wrong sign
    "sigmoid_sign": ("return 1.0 / (1.0 + exp(-z));", "return 1.0 / (1.0 + exp(z));"),
    # clamp removed
    "no_clamp": ("double denom = sum > ORACLE_EPS ? sum : ORACLE_EPS;", "double denom = sum;"),
    # clamp replaced by an additive epsilon
    "eps_added": ("double denom = sum > ORACLE_EPS ? sum : ORACLE_EPS;",
                  "double denom = sum + ORACLE_EPS;"),
    # backward directions swept forward
    "no_reverse": ("int line = (d % 2 == 0) ? step : L - 1 - step;", "int line = step;"),
    # hidden line never carried to the next step
    "no_carry": ("double *t = hprev; hprev = hcur; hcur = t;", ";"),
    # all channels read and write channel 0's plane of x and y
    "channel_zero": ("size_t xp = (size_t)b * (size_t)Cc + (size_t)c;", "size_t xp = (size_t)b * (size_t)Cc;"),
    # an extra off-grid slot counted on the far edge
    "edge_slot": ("valid[k] = (q + k - 1 >= 0) && (q + k - 1 < M);\n                            lg[k] = valid[k] ? wlogit[at(wp",
                  "valid[k] = (q + k - 1 >= 0) && (q + k - 1 <= M);\n                            lg[k] = valid[k] ? wlogit[at(wp"),
    # every direction gated by direction 0's lambda and u
    "gates_of_slot0": ("size_t gp = ((size_t)b * 4 + (size_t)d) * (size_t)Cc + (size_t)c;",
                       "size_t gp = ((size_t)b * 4 + 0) * (size_t)Cc + (size_t)c;"),
    # logits of the wrong direction
    "logits_of_next_dir": ("size_t wp = (((size_t)b * 4 + (size_t)d) * (size_t)Cw +",
                           "size_t wp = (((size_t)b * 4 + (size_t)((d + 1) % 4)) * (size_t)Cw +"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    src = open(oracle.SOURCE).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    mpath = os.path.join(tmp_path, f"mut_{name}.c")
    with open(mpath, "w") as f:
        f.write(src.replace(old, new))
    lib = oracle.compile_oracle(mpath, os.path.join(tmp_path, f"libmut_{name}.so"))
    orc = oracle.Oracle(lib)
    caught = []
    for check in pins.ALL_CHECKS:
        try:
            check(orc)
        except AssertionError:
            caught.append(check.__name__)
    assert caught, f"no pin rejects mutant {name}"
