"""Pins that tie the backward oracle (oracle_prop2d_bwd_f64) to something
other than itself.

Each ``check_bwd_*`` takes an oracle object (``prop2d``, ``prop2d_bwd``) and
raises AssertionError when the backward disagrees with:
  * fp64 central finite differences of the FORWARD oracle, element by
    element, on tiny grids (the definition of a gradient);
  * the transpose of the dense brute-force operator of each direction
    (y = sum_d u_d * A_d (lambda_d * x), built from library sigmoids), which
    fixes dx, dlambda and du exactly;
  * the normalisation's scale invariance: w(a s) = w(s) for any a > 0, so at
    every position where the clamp does not bind, sum_j s_j dL/ds_j = 0,
    i.e. sum_j dwt_j / (1 - s_j) = 0 over the on-grid slots;
  * zeros for the slots of directions that are not enabled.
"""
from __future__ import annotations

import numpy as np
from scipy.special import expit

import oracle_pins as pins


def _loss(orc, gy, x, lam, wl, u, dirs, share_w):
    return float(np.sum(gy * orc.prop2d(x, lam, wl, u, dirs=dirs, share_w=share_w)))


def _fd_check(orc, x, lam, wl, u, gy, dirs, share_w, what, h=1e-6, rel=1e-7):
    g = orc.prop2d_bwd(x, lam, wl, u, gy, dirs=dirs, share_w=share_w)
    args = {"x": x, "lam": lam, "wlogit": wl, "u": u}
    for name, arr in args.items():
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            a = arr.copy()
            a[idx] += h
            kw = dict(args, **{name: a})
            lp = _loss(orc, gy, kw["x"], kw["lam"], kw["wlogit"], kw["u"], dirs, share_w)
            a[idx] -= 2 * h
            kw = dict(args, **{name: a})
            lm = _loss(orc, gy, kw["x"], kw["lam"], kw["wlogit"], kw["u"], dirs, share_w)
            fd[idx] = (lp - lm) / (2 * h)
        scale = max(1.0, float(np.max(np.abs(fd))))
        err = float(np.max(np.abs(g[name] - fd)))
        assert err <= rel * scale, f"{what}: d{name} differs from finite differences by {err:.3e}"


def check_bwd_finite_differences(orc):
    rng = np.random.default_rng(21)
    for (B, Cc, H, W, dirs, sw) in [(1, 2, 3, 4, 15, 0), (1, 2, 4, 3, 15, 1), (1, 1, 2, 5, 6, 0),
                                    (1, 1, 5, 2, 9, 0), (1, 1, 1, 4, 15, 0)]:
        x, lam, wl, u = pins.rand_inputs(rng, B, Cc, H, W, sw, sigma=2.0)
        gy = rng.standard_normal(x.shape)
        _fd_check(orc, x, lam, wl, u, gy, dirs, sw, f"{B}x{Cc}x{H}x{W} dirs={dirs} share_w={sw}")


def check_bwd_clamped_finite_differences(orc):
    """Logits near -15: the on-grid sigmoids (about 3e-7 each) sum just below
    eps = 1e-6, the clamp holds the denominator and the weights (about 0.3)
    are far from row-stochastic; the forward is then linear in each sigmoid."""
    rng = np.random.default_rng(22)
    x, lam, _, u = pins.rand_inputs(rng, 1, 1, 3, 3)
    wl = -15.0 + 0.05 * rng.uniform(-1, 1, (1, 4, 1, 3, 3, 3))
    s = expit(wl)
    assert np.all(3 * s.max() < 1e-6)
    gy = rng.standard_normal(x.shape)
    _fd_check(orc, x, lam, wl, u, gy, 15, 0, "clamped", h=1e-5, rel=1e-6)


def check_bwd_dense_transpose(orc):
    rng = np.random.default_rng(23)
    for (B, Cc, H, W, dirs, sw) in [(1, 2, 3, 4, 15, 0), (2, 1, 4, 4, 15, 1), (1, 2, 5, 3, 10, 0)]:
        x, lam, wl, u = pins.rand_inputs(rng, B, Cc, H, W, sw, sigma=2.0)
        gy = rng.standard_normal(x.shape)
        g = orc.prop2d_bwd(x, lam, wl, u, gy, dirs=dirs, share_w=sw)
        dx = np.zeros_like(x)
        dlam = np.zeros_like(lam)
        du = np.zeros_like(u)
        for b in range(B):
            for c in range(Cc):
                for d in range(4):
                    if not dirs & (1 << d):
                        continue
                    A = pins.direction_operator(wl[b, d, 0 if sw else c], d, H, W)
                    v = (lam[b, d, c] * x[b, c]).reshape(-1)
                    h = (A @ v).reshape(H, W)
                    adj = (A.T @ (u[b, d, c] * gy[b, c]).reshape(-1)).reshape(H, W)
                    du[b, d, c] = gy[b, c] * h
                    dlam[b, d, c] = x[b, c] * adj
                    dx[b, c] += lam[b, d, c] * adj
        pins.assert_close(g["x"], dx, 1e-12, "dx vs dense transpose")
        pins.assert_close(g["lam"], dlam, 1e-12, "dlambda vs dense transpose")
        pins.assert_close(g["u"], du, 1e-12, "du vs dense operator")


def check_bwd_scale_invariance(orc):
    rng = np.random.default_rng(24)
    H, W = 4, 5
    x, lam, wl, u = pins.rand_inputs(rng, 1, 2, H, W, sigma=1.5)
    gy = rng.standard_normal(x.shape)
    g = orc.prop2d_bwd(x, lam, wl, u, gy)["wlogit"]
    for d in range(4):
        M = W if d < 2 else H
        for c in range(2):
            for i in range(H):
                for j in range(W):
                    q = j if d < 2 else i
                    on = np.array([0 <= q + k - 1 < M for k in range(3)])
                    s = expit(wl[0, d, c, :, i, j])
                    tot = float(np.sum(np.where(on, g[0, d, c, :, i, j] / (1.0 - s), 0.0)))
                    ref = float(np.max(np.abs(g[0, d, c, :, i, j]))) + 1e-300
                    assert abs(tot) <= 1e-10 * max(ref, 1e-12), (d, c, i, j, tot)
                    assert np.all(g[0, d, c, ~on, i, j] == 0.0), "off-grid slot has a gradient"


def check_bwd_disabled_directions_zero(orc):
    rng = np.random.default_rng(25)
    x, lam, wl, u = pins.rand_inputs(rng, 1, 2, 3, 4, sigma=2.0)
    gy = rng.standard_normal(x.shape)
    g = orc.prop2d_bwd(x, lam, wl, u, gy, dirs=5)
    for d in (1, 3):
        assert np.all(g["lam"][:, d] == 0) and np.all(g["u"][:, d] == 0)
        assert np.all(g["wlogit"][:, d] == 0)
    assert np.any(g["lam"][:, 0] != 0) and np.any(g["wlogit"][:, 2] != 0)


BWD_CHECKS = [check_bwd_finite_differences, check_bwd_clamped_finite_differences,
              check_bwd_dense_transpose, check_bwd_scale_invariance,
              check_bwd_disabled_directions_zero]
