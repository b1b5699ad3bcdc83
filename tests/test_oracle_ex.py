"""The sharing variants of the oracle (oracle_prop2d_ex_f64) reduce to the
pinned forward: shared gates are per-direction gates that are equal, grouped
logits are per-channel logits repeated over each group (CPU only)."""
import numpy as np
import pytest

import oracle
import oracle_pins as pins


@pytest.mark.parametrize("shape", [(1, 4, 3, 5), (2, 6, 4, 4), (1, 2, 1, 6), (1, 3, 6, 1)])
@pytest.mark.parametrize("gate_dirs", [4, 1])
@pytest.mark.parametrize("groups", ["all", "one", "some"])
@pytest.mark.parametrize("dirs", [15, 5, 10])
def test_ex_reduces_to_forward(shape, gate_dirs, groups, dirs):
    B, Cc, H, W = shape
    G = {"all": Cc, "one": 1, "some": Cc // 2 if Cc % 2 == 0 and Cc > 2 else 1}[groups]
    rng = np.random.default_rng(hash((shape, gate_dirs, groups, dirs)) % 2**32)
    x = rng.standard_normal((B, Cc, H, W))
    lam = rng.uniform(0, 1, (B, gate_dirs, Cc, H, W))
    u = rng.uniform(0, 1, (B, gate_dirs, Cc, H, W))
    wl = rng.standard_normal((B, 4, G, 3, H, W)) * 2.0
    y = oracle.prop2d_ex(x, lam, wl, u, dirs=dirs, gate_dirs=gate_dirs, w_groups=G)
    lam4 = np.broadcast_to(lam, (B, 4, Cc, H, W)).copy()
    u4 = np.broadcast_to(u, (B, 4, Cc, H, W)).copy()
    wl_full = np.repeat(wl, Cc // G, axis=2)
    want = oracle.prop2d(x, lam4, wl_full, u4, dirs=dirs)
    pins.assert_close(y, want, 1e-15, f"ex {shape} gates={gate_dirs} G={G}")
    if G == 1:
        pins.assert_close(y, oracle.prop2d(x, lam4, wl, u4, dirs=dirs, share_w=1), 1e-15, "G=1")


def test_ex_brute_force_shared_gates():
    """Shared gates against the dense brute force directly."""
    rng = np.random.default_rng(31)
    B, Cc, H, W = 1, 2, 4, 3
    x = rng.standard_normal((B, Cc, H, W))
    lam = rng.uniform(0, 1, (B, 1, Cc, H, W))
    u = rng.uniform(0, 1, (B, 1, Cc, H, W))
    wl = rng.standard_normal((B, 4, 1, 3, H, W)) * 2.0
    y = oracle.prop2d_ex(x, lam, wl, u, gate_dirs=1, w_groups=1)
    yb = pins.brute_force_prop2d(x, np.repeat(lam, 4, axis=1), wl, np.repeat(u, 4, axis=1),
                                 share_w=1)
    pins.assert_close(y, yb, 1e-12, "brute force, shared gates")


@pytest.mark.parametrize("gate_dirs,G", [(2, 1), (4, 3), (4, 0)])
def test_ex_rejects_bad_sharing(gate_dirs, G):
    x = np.zeros((1, 4, 2, 2))
    lam = np.zeros((1, max(gate_dirs, 1), 4, 2, 2))
    wl = np.zeros((1, 4, max(G, 1), 3, 2, 2))
    with pytest.raises((ValueError, AssertionError)):
        oracle.prop2d_ex(x, lam, wl, lam, gate_dirs=gate_dirs, w_groups=G)
