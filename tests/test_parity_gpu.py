"""GPU parity: the CUDA library (through its C ABI) against the fp64 oracle.

Bar: max |y_gpu - y_oracle| <= tol * max |y_oracle| with tol = 1e-4 for fp32
inputs and 2e-2 for bf16 inputs (fp32 state in both cases).  The oracle sees
exactly the values the GPU sees (bf16 inputs widened exactly to fp64).
"""
import numpy as np
import pytest
import torch

import oracle
import oracle_pins as pins
from spatial_propagation_vision_b200.workloads import WORKLOADS, make_inputs, workload_inputs

pytestmark = pytest.mark.gpu

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


@pytest.fixture(scope="module")
def gspn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from spatial_propagation_vision_b200 import prop2d
    return prop2d


def to_dev(inp):
    return {k: v.cuda() for k, v in inp.items()}


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def oracle_planes(inp, planes, dirs, share_w):
    """Oracle output of the listed (b, c) planes (planes are independent)."""
    out = []
    for b, c in planes:
        cw = 0 if share_w else c
        x = f64(inp["x"][b:b + 1, c:c + 1])
        lam = f64(inp["lam"][b:b + 1, :, c:c + 1])
        u = f64(inp["u"][b:b + 1, :, c:c + 1])
        wl = f64(inp["wlogit"][b:b + 1, :, cw:cw + 1])
        out.append(oracle.prop2d(x, lam, wl, u, dirs=dirs, share_w=0)[0, 0])
    return np.stack(out)


def workspace(gspn, inp, dirs=15, share_w=1):
    B, Cc, H, W = inp["x"].shape
    n = gspn.workspace_bytes(B, Cc, H, W, dirs, share_w, inp["x"].dtype)
    return torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")


def check(gspn, inp, dirs=15, share_w=0, planes=None, what="", ws=False):
    d = to_dev(inp)
    kw = {"workspace": workspace(gspn, inp, dirs, share_w)} if ws else {}
    y = gspn.prop2d_fwd(d["x"], d["lam"], d["wlogit"], d["u"], dirs=dirs, share_w=share_w, **kw)
    torch.cuda.synchronize()
    yg = f64(y)
    if planes is None:
        yo = oracle.prop2d(f64(inp["x"]), f64(inp["lam"]), f64(inp["wlogit"]), f64(inp["u"]),
                           dirs=dirs, share_w=share_w)
    else:
        yo = oracle_planes(inp, planes, dirs, share_w)
        yg = np.stack([yg[b, c] for b, c in planes])
    tol = TOL[inp["x"].dtype]
    scale = float(np.max(np.abs(yo))) if yo.size else 0.0
    err = float(np.max(np.abs(yg - yo))) if yo.size else 0.0
    assert np.all(np.isfinite(yg)), f"{what}: non-finite output"
    assert err <= tol * max(scale, 1e-30), f"{what}: max err {err:.3e} > {tol:.0e} * {scale:.3e}"
    return err / max(scale, 1e-30)


# --------------------------------------------------------------------------
# the five workloads
# --------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_workload_full(gspn, name):
    w = WORKLOADS[name]
    rel = check(gspn, workload_inputs(w, seed=0), share_w=w.share_w, what=name)
    print(f"\n{name}: max|err| / max|y| = {rel:.3e}")


@pytest.mark.parametrize("name", ["1k", "2k", "orig"])
def test_workload_sampled_planes(gspn, name):
    """Full-size workload in the launch the benchmark times; the oracle checks
    sampled planes one by one (first, last, and random ones)."""
    w = WORKLOADS[name]
    inp = workload_inputs(w, seed=0)
    rng = np.random.default_rng(0)
    n = 3 if name == "orig" else 8
    planes = [(0, 0), (w.B - 1, w.Cc - 1)]
    planes += [(int(rng.integers(w.B)), int(rng.integers(w.Cc))) for _ in range(n)]
    rel = check(gspn, inp, share_w=w.share_w, planes=planes, what=name)
    print(f"\n{name} (sampled planes): max|err| / max|y| = {rel:.3e}")


# --------------------------------------------------------------------------
# shapes, ragged tails, masks, dtypes, channel sharing
# --------------------------------------------------------------------------

SHAPES = [
    (1, 1, 1, 1), (1, 2, 1, 7), (1, 2, 7, 1), (2, 3, 2, 2), (1, 2, 3, 5), (1, 2, 31, 33),
    (2, 2, 33, 31), (1, 3, 32, 32), (1, 2, 64, 65), (2, 2, 74, 74), (1, 2, 16, 100),
    (1, 1, 100, 16), (1, 2, 97, 129), (1, 1, 129, 97), (1, 1, 148, 148), (1, 1, 256, 256),
    (1, 1, 255, 3), (1, 1, 3, 255),
]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_shapes(gspn, shape, dtype):
    B, Cc, H, W = shape
    inp = make_inputs(B, Cc, H, W, sigma_w=2.0, dtype=dtype, seed=hash(shape) % 1000)
    check(gspn, inp, what=f"{shape} {dtype}")


@pytest.mark.parametrize("dirs", [1, 2, 4, 8, 3, 12, 5, 10, 6, 9, 7, 11, 13, 14, 15])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_direction_masks(gspn, dirs, dtype):
    inp = make_inputs(2, 3, 21, 18, sigma_w=2.0, dtype=dtype, seed=dirs)
    check(gspn, inp, dirs=dirs, what=f"dirs={dirs}")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [(2, 5, 16, 16), (3, 4, 37, 38), (1, 3, 148, 148)],
                         ids=lambda s: "x".join(map(str, s)))
def test_share_w(gspn, shape, dtype):
    B, Cc, H, W = shape
    inp = make_inputs(B, Cc, H, W, share_w=1, sigma_w=1.0, dtype=dtype, seed=7)
    check(gspn, inp, share_w=1, what=f"share_w {shape}")


# --------------------------------------------------------------------------
# compact mode with a workspace: the shared weights normalised once
# --------------------------------------------------------------------------

def test_workload_2k_workspace(gspn):
    """The 2k compact workload through gspn_prop2d_fwd_ws (sampled planes)."""
    w = WORKLOADS["2k"]
    inp = workload_inputs(w, seed=0)
    rng = np.random.default_rng(1)
    planes = [(0, 0), (w.B - 1, w.Cc - 1)] + [(int(rng.integers(w.B)), int(rng.integers(w.Cc)))
                                              for _ in range(8)]
    rel = check(gspn, inp, share_w=1, planes=planes, what="2k ws", ws=True)
    print(f"\n2k with workspace (sampled planes): max|err| / max|y| = {rel:.3e}")
    assert gspn.launch_info()["launches"] == 2


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [(1, 1, 1, 1), (2, 5, 16, 16), (3, 4, 37, 38), (2, 3, 74, 74),
                                   (1, 3, 148, 148), (1, 2, 31, 97), (1, 2, 256, 256),
                                   (1, 2, 2, 40), (1, 3, 17, 1)],
                         ids=lambda s: "x".join(map(str, s)))
def test_share_w_workspace(gspn, shape, dtype):
    B, Cc, H, W = shape
    inp = make_inputs(B, Cc, H, W, share_w=1, sigma_w=2.0, dtype=dtype, seed=17)
    check(gspn, inp, share_w=1, what=f"share_w ws {shape} {dtype}", ws=True)


@pytest.mark.parametrize("dirs", [1, 2, 4, 8, 5, 10, 15])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_share_w_workspace_masks(gspn, dirs, dtype):
    inp = make_inputs(2, 3, 21, 18, share_w=1, sigma_w=2.0, dtype=dtype, seed=dirs)
    check(gspn, inp, dirs=dirs, share_w=1, what=f"ws dirs={dirs}", ws=True)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("mode", ["clamp_binds", "all_very_negative", "saturated_positive"])
def test_share_w_workspace_extremes(gspn, mode, dtype):
    """The clamp (sum of the weights below 1) and saturated logits through the
    weights normalised ahead."""
    inp = make_inputs(2, 3, 19, 23, share_w=1, sigma_w=1.0, dtype="f32", seed=3)
    g = torch.Generator().manual_seed(6)
    shape = inp["wlogit"].shape
    if mode == "clamp_binds":
        wl = -16.0 - 4.0 * torch.rand(shape, generator=g)
    elif mode == "all_very_negative":
        wl = -40.0 - 20.0 * torch.rand(shape, generator=g)
    else:
        wl = 30.0 + 60.0 * torch.rand(shape, generator=g)
    inp["wlogit"] = wl
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    inp = {k: v.to(td) for k, v in inp.items()}
    check(gspn, inp, share_w=1, what=f"ws {mode} {dtype}", ws=True)


def test_workspace_unused_without_share_w(gspn):
    inp = make_inputs(2, 3, 30, 30, sigma_w=2.0, dtype="bf16", seed=2)
    d = to_dev(inp)
    y0 = gspn.prop2d_fwd(d["x"], d["lam"], d["wlogit"], d["u"])
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    y1 = gspn.prop2d_fwd(d["x"], d["lam"], d["wlogit"], d["u"], workspace=ws)
    torch.cuda.synchronize()
    assert gspn.launch_info()["launches"] == 1
    assert torch.equal(y0, y1)


# --------------------------------------------------------------------------
# numerics edge cases
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_hand_examples(gspn, dtype):
    for ex in pins.parse_hand_examples():
        x, lam, wl, u = pins.hand_example_inputs(ex)
        inp = {"x": torch.tensor(x, dtype=dtype), "lam": torch.tensor(lam, dtype=dtype),
               "wlogit": torch.tensor(wl, dtype=dtype), "u": torch.tensor(u, dtype=dtype)}
        check(gspn, inp, dirs=ex["dirs"][0], what=ex["name"])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("mode", ["all_very_negative", "clamp_binds", "overflow_pairs",
                                  "saturated_positive", "mixed_extremes"])
def test_extreme_logits(gspn, mode, dtype):
    """Logit ranges where the denominator clamp binds (all on-grid logits
    below about -14) or where a product form of the normalisation would
    overflow (two logits below about -44)."""
    B, Cc, H, W = 1, 2, 19, 23
    inp = make_inputs(B, Cc, H, W, sigma_w=1.0, dtype="f32", seed=3)
    g = torch.Generator().manual_seed(5)
    wl = inp["wlogit"]
    if mode == "all_very_negative":
        wl = -40.0 - 20.0 * torch.rand(wl.shape, generator=g)
    elif mode == "clamp_binds":
        wl = -16.0 - 4.0 * torch.rand(wl.shape, generator=g)
    elif mode == "overflow_pairs":
        wl = wl.clone()
        wl[:, :, :, 0] = -60.0
        wl[:, :, :, 2] = -50.0
    elif mode == "saturated_positive":
        wl = 30.0 + 60.0 * torch.rand(wl.shape, generator=g)
    else:
        pick = torch.randint(0, 4, wl.shape, generator=g)
        vals = torch.tensor([-90.0, -14.5, 0.0, 90.0])
        wl = vals[pick] + 0.1 * torch.randn(wl.shape, generator=g)
    inp["wlogit"] = wl
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    inp = {k: v.to(td) for k, v in inp.items()}
    check(gspn, inp, what=f"{mode} {dtype}")


# --------------------------------------------------------------------------
# launch paths, host entry point, streams, errors
# --------------------------------------------------------------------------

@pytest.mark.parametrize("shape,dtype,path", [
    ((2, 3, 74, 74), "bf16", "dir-shared"),
    ((2, 3, 74, 74), "f32", "dir"),
    ((1, 2, 160, 160), "f32", "dir-shared"),   # two output planes do not fit
    ((1, 2, 256, 256), "f32", "dir-yglobal"),
    ((1, 2, 256, 256), "bf16", "dir-banded"),
    ((1, 2, 148, 148), "bf16", "dir-shared"),
    ((1, 2, 20, 33), "bf16", "generic"),       # odd bf16 row width
    ((1, 1, 300, 40), "f32", "generic"),       # line longer than 256
    ((2, 2, 1, 40), "bf16", "generic"),        # lines of one position
    ((1, 3, 17, 1), "f32", "generic"),
])
def test_launch_paths(gspn, shape, dtype, path):
    B, Cc, H, W = shape
    inp = make_inputs(B, Cc, H, W, sigma_w=2.0, dtype=dtype, seed=11)
    check(gspn, inp, what=path)
    assert gspn.launch_info()["path"] == path


def test_host_entry_point(gspn):
    inp = make_inputs(2, 3, 37, 40, sigma_w=2.0, dtype="bf16", seed=4)
    h = {k: v.pin_memory() for k, v in inp.items()}
    h["out"] = torch.empty_like(inp["x"]).pin_memory()
    d = {k: torch.empty_like(v, device="cuda") for k, v in h.items()}
    y = gspn.prop2d_fwd_host(h, d)
    dd = to_dev(inp)
    y_dev = gspn.prop2d_fwd(dd["x"], dd["lam"], dd["wlogit"], dd["u"])
    torch.cuda.synchronize()
    yo = oracle.prop2d(f64(inp["x"]), f64(inp["lam"]), f64(inp["wlogit"]), f64(inp["u"]))
    scale = np.max(np.abs(yo))
    assert np.max(np.abs(f64(y) - yo)) <= 2e-2 * scale
    assert np.max(np.abs(f64(y) - f64(y_dev))) <= 1e-2 * scale


def test_side_stream(gspn):
    inp = to_dev(make_inputs(1, 4, 30, 30, dtype="f32", seed=9))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        y = gspn.prop2d_fwd(inp["x"], inp["lam"], inp["wlogit"], inp["u"], stream=s)
    s.synchronize()
    y0 = gspn.prop2d_fwd(inp["x"], inp["lam"], inp["wlogit"], inp["u"])
    torch.cuda.synchronize()
    assert torch.allclose(y, y0, rtol=1e-5, atol=1e-5 * float(y0.abs().max()))


def test_misaligned_pointer_rejected(gspn):
    buf = torch.zeros(4 * 1 * 1 * 8 * 8 + 1, device="cuda")
    x = buf[1:65].view(1, 1, 8, 8)   # 4-byte offset: not 16-byte aligned
    inp = to_dev(make_inputs(1, 1, 8, 8, dtype="f32", seed=1))
    with pytest.raises(gspn.GspnError) as e:
        gspn.prop2d_fwd(x, inp["lam"], inp["wlogit"], inp["u"])
    assert e.value.status == 5


def test_output_fully_overwritten(gspn):
    inp = to_dev(make_inputs(2, 2, 24, 24, dtype="f32", seed=2))
    out = torch.full((2, 2, 24, 24), float("nan"), device="cuda")
    gspn.prop2d_fwd(inp["x"], inp["lam"], inp["wlogit"], inp["u"], out=out)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()
