"""Pins that tie the Prop2D oracle to something other than itself.

Each ``check_*`` takes an oracle object (``prop2d`` and ``weights`` methods)
and raises AssertionError when the oracle disagrees with:
  * the hand-derived examples in ``golden/hand_examples.txt``;
  * a dense brute force: the line scan unrolled into products of explicit
    tridiagonal matrices, and the whole map as one N x N matrix (the
    "attention view" of Sec. 3 "Complexity and the attention analogy");
  * invariants the pages fix (row-stochastic weights; constant input gives
    (i+1)*c on the top->bottom scan; flipping the grid swaps scans);
  * special cases that reduce to library routines (numpy.cumsum,
    scipy.special.expit) and structural laws (linearity, direction
    additivity, transpose symmetry, channel sharing).

They are written as plain functions so that the mutation test can run them
against deliberately broken copies of the oracle.
"""
from __future__ import annotations

import os

import numpy as np
from scipy.special import expit

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
EPS = 1e-6  # denominator clamp of the normalisation (reading of Sec. 5.1)


# ----------------------------------------------------------------------------
# helpers
# ----------------------------------------------------------------------------

def rand_inputs(rng, B, Cc, H, W, share_w=0, sigma=1.0):
    Cw = 1 if share_w else Cc
    x = rng.standard_normal((B, Cc, H, W))
    lam = rng.uniform(0, 1, (B, 4, Cc, H, W))
    wl = rng.standard_normal((B, 4, Cw, 3, H, W)) * sigma
    u = rng.uniform(0, 1, (B, 4, Cc, H, W))
    return x, lam, wl, u


def parse_hand_examples(path=None):
    path = path or os.path.join(GOLDEN, "hand_examples.txt")
    examples, cur = [], None
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, *vals = line.split()
            if key == "name":
                cur = {"name": vals[0]}
                examples.append(cur)
            elif key in ("shape", "dirs"):
                cur[key] = [int(v) for v in vals]
            else:
                cur[key] = np.array([float(v) for v in vals])
    return examples


def hand_example_inputs(ex):
    """Broadcast one hand example to the C-ABI layouts (B = Cc = 1)."""
    H, W = ex["shape"]
    x = ex["x"].reshape(1, 1, H, W)
    lam = np.broadcast_to(ex["lambda"].reshape(1, 1, 1, H, W), (1, 4, 1, H, W)).copy()
    u = np.broadcast_to(ex["u"].reshape(1, 1, 1, H, W), (1, 4, 1, H, W)).copy()
    wl = np.broadcast_to(ex["logit"].reshape(1, 1, 1, 3, 1, 1), (1, 4, 1, 3, H, W)).copy()
    return x, lam, wl, u


def line_weight_matrix(wl_plane3, d, line, H, W):
    """Dense tridiagonal T (M x M) for line `line` of direction d, built from
    library sigmoid values: T[q, q+k-1] = s_k / max(sum of on-grid s, eps)."""
    M = W if d < 2 else H
    T = np.zeros((M, M))
    for q in range(M):
        i, j = (line, q) if d < 2 else (q, line)
        s = np.zeros(3)
        for k in range(3):
            if 0 <= q + k - 1 < M:
                s[k] = expit(wl_plane3[k, i, j])
        den = max(s.sum(), EPS)
        for k in range(3):
            if 0 <= q + k - 1 < M:
                T[q, q + k - 1] = s[k] / den
    return T


def direction_operator(wl_plane3, d, H, W):
    """The whole scan of direction d as one (H*W) x (H*W) matrix A with
    vec(h) = A vec(lambda * x), built from products of tridiagonals:
    block (l, t) = T_l T_{l-1} ... T_{t+1} for t <= l in scan order."""
    L, M = (H, W) if d < 2 else (W, H)
    order = list(range(L)) if d % 2 == 0 else list(range(L - 1, -1, -1))
    Ts = [line_weight_matrix(wl_plane3, d, line, H, W) for line in order]

    def flat(line, q):
        i, j = (line, q) if d < 2 else (q, line)
        return i * W + j

    N = H * W
    A = np.zeros((N, N))
    for a, la in enumerate(order):
        for b in range(a + 1):
            P = np.eye(M)
            for t in range(b + 1, a + 1):
                P = Ts[t] @ P
            lb = order[b]
            for q in range(M):
                for r in range(M):
                    A[flat(la, q), flat(lb, r)] = P[q, r]
    return A


def brute_force_prop2d(x, lam, wl, u, dirs=15, share_w=0):
    B, Cc, H, W = x.shape
    y = np.zeros_like(x)
    for b in range(B):
        for c in range(Cc):
            for d in range(4):
                if not dirs & (1 << d):
                    continue
                cw = 0 if share_w else c
                A = direction_operator(wl[b, d, cw], d, H, W)
                v = (lam[b, d, c] * x[b, c]).reshape(-1)
                y[b, c] += u[b, d, c] * (A @ v).reshape(H, W)
    return y


def assert_close(a, b, rel=1e-12, what=""):
    scale = max(1.0, float(np.max(np.abs(b))) if b.size else 1.0)
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= rel * scale, f"{what}: max abs err {err:.3e} > {rel:.1e} * {scale:.3e}"


# ----------------------------------------------------------------------------
# pins
# ----------------------------------------------------------------------------

def check_hand_examples(orc):
    for ex in parse_hand_examples():
        x, lam, wl, u = hand_example_inputs(ex)
        H, W = ex["shape"]
        y = orc.prop2d(x, lam, wl, u, dirs=ex["dirs"][0])
        assert_close(y.reshape(-1), ex["y"], 1e-13, ex["name"])


def check_weights_row_stochastic(orc):
    rng = np.random.default_rng(1)
    for (H, W) in [(1, 1), (1, 5), (5, 1), (4, 7), (6, 6)]:
        wl = rng.standard_normal((2, 4, 3, 3, H, W)) * 2.0
        w = orc.weights(wl)
        for d in range(4):
            s = w[:, d].sum(axis=2)
            assert np.all(np.abs(s - 1.0) < 4e-16), f"rows do not sum to 1 (d={d}, {H}x{W})"
            # off-grid slots are exactly zero
            if d < 2:
                assert np.all(w[:, d, :, 0, :, 0] == 0) and np.all(w[:, d, :, 2, :, W - 1] == 0)
            else:
                assert np.all(w[:, d, :, 0, 0, :] == 0) and np.all(w[:, d, :, 2, H - 1, :] == 0)
        assert np.all(w >= 0)


def check_weights_expit(orc):
    """Normalised weights equal library sigmoid over the on-grid slots, divided by their sum."""
    rng = np.random.default_rng(2)
    H, W = 4, 5
    wl = rng.standard_normal((1, 4, 2, 3, H, W)) * 3.0
    w = orc.weights(wl)
    for d in range(4):
        M = W if d < 2 else H
        for c in range(2):
            for i in range(H):
                for j in range(W):
                    q = j if d < 2 else i
                    valid = np.array([0 <= q + k - 1 < M for k in range(3)])
                    s = np.where(valid, expit(wl[0, d, c, :, i, j]), 0.0)
                    want = s / s.sum()
                    got = w[0, d, c, :, i, j]
                    assert np.max(np.abs(got - want)) < 1e-15, (d, c, i, j, got, want)


def check_weights_clamp(orc):
    """Logits of -40: the on-grid sigmoids sum below eps, so the denominator is eps."""
    wl = np.full((1, 4, 1, 3, 3, 3), -40.0)
    w = orc.weights(wl)
    s = expit(-40.0)
    # interior position of a row line: all three slots on the grid
    assert abs(w[0, 0, 0, 1, 1, 1] - s / EPS) < 1e-24
    assert abs(w[0, 0, 0, 0, 1, 1] - s / EPS) < 1e-24
    assert w[0, 0, 0, :, 1, 1].sum() < 1e-10  # far from row-stochastic: the clamp binds


def check_brute_force(orc):
    rng = np.random.default_rng(3)
    for (B, Cc, H, W, dirs, sw) in [(1, 2, 3, 4, 15, 0), (2, 1, 5, 3, 15, 0), (1, 2, 6, 6, 15, 0),
                                    (1, 3, 4, 4, 15, 1), (1, 1, 1, 5, 15, 0), (1, 1, 5, 1, 15, 0),
                                    (1, 2, 4, 5, 5, 0), (1, 2, 5, 4, 10, 0), (1, 1, 2, 2, 9, 1)]:
        x, lam, wl, u = rand_inputs(rng, B, Cc, H, W, sw, sigma=2.0)
        y = orc.prop2d(x, lam, wl, u, dirs=dirs, share_w=sw)
        yb = brute_force_prop2d(x, lam, wl, u, dirs=dirs, share_w=sw)
        assert_close(y, yb, 1e-12, f"brute force {B}x{Cc}x{H}x{W} dirs={dirs} share_w={sw}")


def check_constant_input(orc):
    """lambda = u = 1, x = c: every row-stochastic line map preserves constants,
    so the top->bottom scan holds (i+1)*c at row i (and likewise per direction)."""
    rng = np.random.default_rng(4)
    H, W, c = 7, 5, 1.75
    x = np.full((1, 1, H, W), c)
    one = np.ones((1, 4, 1, H, W))
    wl = rng.standard_normal((1, 4, 1, 3, H, W)) * 2.0
    i = np.arange(H)[:, None] * np.ones((1, W))
    j = np.ones((H, 1)) * np.arange(W)[None, :]
    expect = {1: (i + 1) * c, 2: (H - i) * c, 4: (j + 1) * c, 8: (W - j) * c}
    for dirs, want in expect.items():
        y = orc.prop2d(x, one, wl, one, dirs=dirs)[0, 0]
        assert_close(y, want, 1e-13, f"constant input dirs={dirs}")


def check_flip_h(orc):
    """Flipping the grid along H swaps top->bottom and bottom->top (slots unchanged);
    left->right / right->left swap their neighbour slots (k -> 2-k)."""
    rng = np.random.default_rng(5)
    x, lam, wl, u = rand_inputs(rng, 1, 2, 5, 4, sigma=2.0)
    y = orc.prop2d(x, lam, wl, u)
    perm = [1, 0, 2, 3]
    xf = x[:, :, ::-1]
    lamf = lam[:, perm][:, :, :, ::-1]
    uf = u[:, perm][:, :, :, ::-1]
    wlf = wl[:, perm][:, :, :, :, ::-1].copy()
    wlf[:, 2:] = wlf[:, 2:, :, ::-1]   # column lines: up <-> down neighbour slots
    yf = orc.prop2d(xf, lamf, wlf, uf)
    assert_close(yf, y[:, :, ::-1], 1e-12, "flip along H")


def check_flip_w(orc):
    rng = np.random.default_rng(6)
    x, lam, wl, u = rand_inputs(rng, 1, 2, 4, 6, sigma=2.0)
    y = orc.prop2d(x, lam, wl, u)
    perm = [0, 1, 3, 2]
    xf = x[..., ::-1]
    lamf = lam[:, perm][..., ::-1]
    uf = u[:, perm][..., ::-1]
    wlf = wl[:, perm][..., ::-1].copy()
    wlf[:, :2] = wlf[:, :2, :, ::-1]   # row lines: left <-> right neighbour slots
    yf = orc.prop2d(xf, lamf, wlf, uf)
    assert_close(yf, y[..., ::-1], 1e-12, "flip along W")


def check_transpose(orc):
    """Transposing H <-> W maps top->bottom to left->right and bottom->top to right->left."""
    rng = np.random.default_rng(7)
    x, lam, wl, u = rand_inputs(rng, 1, 2, 3, 6, sigma=2.0)
    y = orc.prop2d(x, lam, wl, u)
    perm = [2, 3, 0, 1]
    xt = x.transpose(0, 1, 3, 2)
    lamt = lam[:, perm].transpose(0, 1, 2, 4, 3)
    ut = u[:, perm].transpose(0, 1, 2, 4, 3)
    wlt = wl[:, perm].transpose(0, 1, 2, 3, 5, 4)
    yt = orc.prop2d(xt, lamt, wlt, ut)
    assert_close(yt, y.transpose(0, 1, 3, 2), 1e-12, "transpose")


def check_identity_weights_cumsum(orc):
    """Side logits of -1e4 make every line map the identity; each scan is then a
    cumulative sum of lambda * x along its direction (numpy.cumsum)."""
    rng = np.random.default_rng(8)
    H, W = 5, 6
    x, lam, _, u = rand_inputs(rng, 1, 1, H, W)
    wl = np.zeros((1, 4, 1, 3, H, W))
    wl[:, :, :, 0] = -1e4
    wl[:, :, :, 2] = -1e4
    for d, axis, rev in [(0, 0, False), (1, 0, True), (2, 1, False), (3, 1, True)]:
        v = lam[0, d, 0] * x[0, 0]
        if rev:
            cs = np.flip(np.cumsum(np.flip(v, axis), axis), axis)
        else:
            cs = np.cumsum(v, axis)
        y = orc.prop2d(x, lam, wl, u, dirs=1 << d)[0, 0]
        assert_close(y, u[0, d, 0] * cs, 1e-13, f"identity weights d={d}")


def check_single_pixel(orc):
    rng = np.random.default_rng(9)
    x, lam, wl, u = rand_inputs(rng, 2, 3, 1, 1)
    y = orc.prop2d(x, lam, wl, u)
    want = (u * lam).sum(axis=1) * x
    assert_close(y, want, 1e-14, "H = W = 1")


def check_linearity(orc):
    rng = np.random.default_rng(10)
    x1, lam, wl, u = rand_inputs(rng, 1, 2, 4, 5, sigma=2.0)
    x2 = rng.standard_normal(x1.shape)
    a, b = 0.7, -1.3
    y = orc.prop2d(a * x1 + b * x2, lam, wl, u)
    want = a * orc.prop2d(x1, lam, wl, u) + b * orc.prop2d(x2, lam, wl, u)
    assert_close(y, want, 1e-12, "linearity in x")


def check_direction_additivity(orc):
    rng = np.random.default_rng(11)
    x, lam, wl, u = rand_inputs(rng, 1, 2, 4, 5, sigma=2.0)
    y = orc.prop2d(x, lam, wl, u, dirs=15)
    parts = sum(orc.prop2d(x, lam, wl, u, dirs=1 << d) for d in range(4))
    assert_close(y, parts, 1e-13, "sum over directions")


def check_share_w(orc):
    """share_w = 1 is per-channel logits with the one field copied to every channel."""
    rng = np.random.default_rng(12)
    x, lam, wl, u = rand_inputs(rng, 2, 3, 4, 4, share_w=1, sigma=2.0)
    y = orc.prop2d(x, lam, wl, u, share_w=1)
    wl_full = np.repeat(wl, 3, axis=2)
    y_full = orc.prop2d(x, lam, wl_full, u, share_w=0)
    assert_close(y, y_full, 0.0, "share_w broadcast")


def check_stored_regression(orc):
    """Values written by tests/golden/make_golden.py (which calls only the oracle)."""
    path = os.path.join(GOLDEN, "oracle_tiny_seed0.txt")
    from spatial_propagation_vision_b200.workloads import WORKLOADS, workload_inputs
    inp = workload_inputs(WORKLOADS["tiny"], seed=0)
    t = {k: v.double().numpy() for k, v in inp.items()}
    y = orc.prop2d(t["x"], t["lam"], t["wlogit"], t["u"])
    rows = np.loadtxt(path)
    for b, c, i, j, val in rows:
        got = y[int(b), int(c), int(i), int(j)]
        assert abs(got - val) <= 1e-12 * max(1.0, abs(val)), (b, c, i, j, got, val)


ALL_CHECKS = [
    check_hand_examples, check_weights_row_stochastic, check_weights_expit,
    check_weights_clamp, check_brute_force, check_constant_input, check_flip_h,
    check_flip_w, check_transpose, check_identity_weights_cumsum, check_single_pixel,
    check_linearity, check_direction_additivity, check_share_w,
]
