"""GPU parity of the backward (gspn_prop2d_bwd) against the fp64 backward
oracle, gradient by gradient: max |g_gpu - g_oracle| <= tol * max |g_oracle|
with tol = 1e-4 for fp32 inputs and 2e-2 for bf16 inputs (the oracle sees the
same bf16-rounded inputs and upstream gradient)."""
import numpy as np
import pytest
import torch

import oracle
from spatial_propagation_vision_b200.workloads import WORKLOADS, make_inputs, workload_inputs

pytestmark = pytest.mark.gpu

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


@pytest.fixture(scope="module")
def gspn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from spatial_propagation_vision_b200 import prop2d
    return prop2d


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def check_bwd(gspn, inp, dirs=15, share_w=0, seed=0, what=""):
    g = torch.Generator().manual_seed(seed)
    gy = torch.randn(inp["x"].shape, generator=g).to(inp["x"].dtype)
    d = {k: v.cuda() for k, v in inp.items()}
    got = gspn.prop2d_bwd(d["x"], d["lam"], d["wlogit"], d["u"], gy.cuda(), dirs=dirs,
                          share_w=share_w)
    torch.cuda.synchronize()
    assert gspn.launch_info()["path"] == "bwd"
    want = oracle.prop2d_bwd(f64(inp["x"]), f64(inp["lam"]), f64(inp["wlogit"]), f64(inp["u"]),
                             f64(gy), dirs=dirs, share_w=share_w)
    tol = TOL[inp["x"].dtype]
    worst = 0.0
    for k in ("x", "lam", "wlogit", "u"):
        a, b = f64(got[k]), want[k]
        assert np.all(np.isfinite(a)), f"{what}: d{k} not finite"
        scale = float(np.max(np.abs(b)))
        err = float(np.max(np.abs(a - b)))
        assert err <= tol * max(scale, 1e-30), f"{what}: d{k} err {err:.3e} > {tol} * {scale:.3e}"
        worst = max(worst, err / max(scale, 1e-30))
    return worst


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [(1, 1, 1, 1), (1, 2, 5, 7), (2, 3, 16, 16), (1, 2, 37, 38),
                                   (1, 2, 33, 17), (2, 2, 74, 74), (1, 1, 100, 130),
                                   (1, 1, 256, 256)], ids=lambda s: "x".join(map(str, s)))
def test_backward_shapes(gspn, shape, dtype):
    B, Cc, H, W = shape
    inp = make_inputs(B, Cc, H, W, sigma_w=2.0, dtype=dtype, seed=sum(shape))
    check_bwd(gspn, inp, seed=1, what=f"{shape} {dtype}")


@pytest.mark.parametrize("dirs", [1, 2, 4, 8, 5, 10, 3, 12])
def test_backward_direction_masks(gspn, dirs):
    inp = make_inputs(1, 2, 19, 22, sigma_w=2.0, dtype="f32", seed=dirs)
    check_bwd(gspn, inp, dirs=dirs, seed=2, what=f"dirs={dirs}")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_backward_share_w(gspn, dtype):
    inp = make_inputs(2, 3, 19, 24, share_w=1, sigma_w=1.5, dtype=dtype, seed=5)
    check_bwd(gspn, inp, share_w=1, seed=3, what=f"share_w {dtype}")


def test_backward_clamped(gspn):
    """Logits near -15: the clamp holds the local sum's denominator."""
    inp = make_inputs(1, 2, 9, 10, sigma_w=1.0, dtype="f32", seed=6)
    g = torch.Generator().manual_seed(7)
    inp["wlogit"] = -15.0 + 0.05 * (2 * torch.rand(inp["wlogit"].shape, generator=g) - 1)
    check_bwd(gspn, inp, seed=4, what="clamped")


@pytest.mark.parametrize("name", ["1k", "2k", "mid"])
def test_backward_workload(gspn, name):
    """A benchmark workload's shape (1k: B=32, Cc=64, 74x74 bf16; 2k: 8x64x148x148
    bf16 with logits shared by the channels; mid: 8x64x37x37 fp32), every plane."""
    w = WORKLOADS[name]
    rel = check_bwd(gspn, workload_inputs(w, seed=0), share_w=w.share_w, seed=9, what=name)
    print(f"\n{name} backward: worst max|err| / max|g| = {rel:.3e}")


@pytest.mark.parametrize("dtype,shape", [("f32", (1, 2, 19, 23)), ("bf16", (2, 3, 74, 74)),
                                         ("f32", (1, 1, 100, 130))],
                         ids=lambda v: "x".join(map(str, v)) if isinstance(v, tuple) else str(v))
def test_backward_nan_in_off_grid_slots(gspn, dtype, shape):
    """Off-grid logit slots (slot 0 of a line's first position, slot 2 of its
    last) carry no weight; filled with NaN they must reach no gradient, and
    their own gradient is zero (the oracle never reads them)."""
    B, Cc, H, W = shape
    inp = make_inputs(B, Cc, H, W, sigma_w=2.0, dtype=dtype, seed=23)
    wl = inp["wlogit"].clone()
    nan = float("nan")
    wl[:, 0:2, :, 0, :, 0] = nan
    wl[:, 0:2, :, 2, :, W - 1] = nan
    wl[:, 2:4, :, 0, 0, :] = nan
    wl[:, 2:4, :, 2, H - 1, :] = nan
    inp["wlogit"] = wl
    check_bwd(gspn, inp, seed=5, what=f"NaN edge slots {shape} {dtype}")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [(1, 4, 16, 20), (2, 6, 37, 38), (1, 4, 74, 74)],
                         ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("gate_dirs,groups", [(1, "all"), (4, "half"), (1, "one"), (1, "half")])
def test_backward_sharing_variants(gspn, shape, dtype, gate_dirs, groups):
    """Gradients of the sharing variants (shared gates sum over the
    directions, grouped logits over their channels) against the oracle."""
    B, Cc, H, W = shape
    G = {"all": Cc, "half": Cc // 2, "one": 1}[groups]
    g = torch.Generator().manual_seed(hash((shape, gate_dirs, G)) % 2**31)
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    x = torch.randn((B, Cc, H, W), generator=g)
    lam = torch.rand((B, gate_dirs, Cc, H, W), generator=g)
    wl = torch.randn((B, 4, G, 3, H, W), generator=g) * 2.0
    u = torch.rand((B, gate_dirs, Cc, H, W), generator=g)
    gy = torch.randn((B, Cc, H, W), generator=g)
    inp = {k: v.to(td) for k, v in {"x": x, "lam": lam, "wlogit": wl, "u": u, "gy": gy}.items()}
    d = {k: v.cuda() for k, v in inp.items()}
    got = gspn.prop2d_bwd_ex(d["x"], d["lam"], d["wlogit"], d["u"], d["gy"], gate_dirs=gate_dirs,
                             w_groups=G)
    torch.cuda.synchronize()
    assert gspn.launch_info()["path"] == "bwd"
    f64 = lambda t: t.detach().to("cpu", torch.float64).numpy()
    want = oracle.prop2d_bwd_ex(f64(inp["x"]), f64(inp["lam"]), f64(inp["wlogit"]), f64(inp["u"]),
                                f64(inp["gy"]), gate_dirs=gate_dirs, w_groups=G)
    tol = 1e-4 if dtype == "f32" else 2e-2
    for k in ("x", "lam", "wlogit", "u"):
        scale = float(np.max(np.abs(want[k])))
        err = float(np.max(np.abs(f64(got[k]) - want[k])))
        assert err <= tol * max(scale, 1e-30), f"{k}: {err:.3e} > {tol} * {scale:.3e}"


@pytest.mark.parametrize("gate_dirs,groups", [(4, "all"), (1, "one")])
def test_autograd_function(gspn, gate_dirs, groups):
    """Prop2DFunction: torch autograd through the library's forward and
    backward matches the oracle's gradients of L = sum(gy * y)."""
    B, Cc, H, W = 2, 4, 20, 18
    G = Cc if groups == "all" else 1
    g = torch.Generator().manual_seed(7)
    x = torch.randn((B, Cc, H, W), generator=g)
    lam = torch.rand((B, gate_dirs, Cc, H, W), generator=g)
    wl = torch.randn((B, 4, G, 3, H, W), generator=g) * 2.0
    u = torch.rand((B, gate_dirs, Cc, H, W), generator=g)
    gy = torch.randn((B, Cc, H, W), generator=g)
    leaves = [t.cuda().requires_grad_() for t in (x, lam, wl, u)]
    y = gspn.prop2d_autograd(*leaves, gate_dirs=gate_dirs, w_groups=G)
    (y * gy.cuda()).sum().backward()
    f64 = lambda t: t.detach().to("cpu", torch.float64).numpy()
    want = oracle.prop2d_bwd_ex(f64(x), f64(lam), f64(wl), f64(u), f64(gy), gate_dirs=gate_dirs,
                                w_groups=G)
    for leaf, k in zip(leaves, ("x", "lam", "wlogit", "u")):
        scale = float(np.max(np.abs(want[k])))
        err = float(np.max(np.abs(f64(leaf.grad) - want[k])))
        assert err <= 1e-4 * max(scale, 1e-30), f"{k}: {err:.3e} vs {scale:.3e}"
