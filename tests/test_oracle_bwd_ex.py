"""The backward of the sharing variants (oracle_prop2d_bwd_ex_f64) against
what fixes it: finite differences of the sharing-variant forward, and the
pinned per-direction backward on broadcast inputs, whose gradients the shared
inputs must sum (CPU only)."""
import numpy as np
import pytest

import oracle


def _inputs(shape, gate_dirs, G, seed):
    B, Cc, H, W = shape
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((B, Cc, H, W))
    lam = rng.uniform(0.1, 1.0, (B, gate_dirs, Cc, H, W))
    u = rng.uniform(0.1, 1.0, (B, gate_dirs, Cc, H, W))
    wl = rng.standard_normal((B, 4, G, 3, H, W)) * 1.5
    gy = rng.standard_normal((B, Cc, H, W))
    return x, lam, wl, u, gy


@pytest.mark.parametrize("shape", [(1, 4, 3, 5), (2, 2, 4, 4), (1, 6, 1, 5), (1, 2, 5, 1)])
@pytest.mark.parametrize("gate_dirs", [4, 1])
@pytest.mark.parametrize("groups", ["all", "one", "some"])
@pytest.mark.parametrize("dirs", [15, 6, 9])
def test_shared_gradients_sum_the_per_direction_ones(shape, gate_dirs, groups, dirs):
    B, Cc, H, W = shape
    G = {"all": Cc, "one": 1, "some": Cc // 2 if Cc % 2 == 0 and Cc > 2 else 1}[groups]
    x, lam, wl, u, gy = _inputs(shape, gate_dirs, G, hash((shape, gate_dirs, G, dirs)) % 2**32)
    g = oracle.prop2d_bwd_ex(x, lam, wl, u, gy, dirs=dirs, gate_dirs=gate_dirs, w_groups=G)
    lam4 = np.broadcast_to(lam, (B, 4, Cc, H, W)).copy()
    u4 = np.broadcast_to(u, (B, 4, Cc, H, W)).copy()
    cpg = Cc // G
    gf = oracle.prop2d_bwd(x, lam4, np.repeat(wl, cpg, axis=2), u4, gy, dirs=dirs)
    np.testing.assert_allclose(g["x"], gf["x"], rtol=1e-13, atol=1e-13)
    want_lam = gf["lam"].sum(axis=1, keepdims=True) if gate_dirs == 1 else gf["lam"]
    want_u = gf["u"].sum(axis=1, keepdims=True) if gate_dirs == 1 else gf["u"]
    np.testing.assert_allclose(g["lam"], want_lam, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(g["u"], want_u, rtol=1e-13, atol=1e-13)
    want_wl = gf["wlogit"].reshape(B, 4, G, cpg, 3, H, W).sum(axis=3)
    np.testing.assert_allclose(g["wlogit"], want_wl, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("gate_dirs,G", [(1, 1), (1, 2), (4, 1)])
def test_shared_gradients_match_finite_differences(gate_dirs, G):
    """Central differences of the sharing-variant forward, element by element."""
    shape = (1, 2, 3, 4)
    x, lam, wl, u, gy = _inputs(shape, gate_dirs, G, 17 + gate_dirs + G)
    g = oracle.prop2d_bwd_ex(x, lam, wl, u, gy, gate_dirs=gate_dirs, w_groups=G)
    args = {"x": x, "lam": lam, "wlogit": wl, "u": u}

    def loss(a):
        return float(np.sum(gy * oracle.prop2d_ex(a["x"], a["lam"], a["wlogit"], a["u"],
                                                   gate_dirs=gate_dirs, w_groups=G)))

    h = 1e-6
    for name, arr in args.items():
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            a = dict(args)
            p = arr.copy(); p[idx] += h; a[name] = p
            lp = loss(a)
            m = arr.copy(); m[idx] -= h; a[name] = m
            lm = loss(a)
            fd[idx] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(g[name], fd, rtol=1e-6, atol=1e-7, err_msg=name)


@pytest.mark.parametrize("gate_dirs,G", [(2, 1), (4, 3), (4, 0)])
def test_bwd_ex_rejects_bad_sharing(gate_dirs, G):
    x = np.zeros((1, 4, 2, 2))
    lam = np.zeros((1, max(gate_dirs, 1), 4, 2, 2))
    wl = np.zeros((1, 4, max(G, 1), 3, 2, 2))
    with pytest.raises((ValueError, AssertionError)):
        oracle.prop2d_bwd_ex(x, lam, wl, lam, x, gate_dirs=gate_dirs, w_groups=G)
