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


def oracle_all(inp, dirs, share_w):
    """Oracle output of every plane, computed in (batch, channel-chunk) slices
    so that the fp64 copies stay small."""
    B, Cc, H, W = inp["x"].shape
    chunk = max(1, (1 << 20) // (H * W))
    out = np.empty(tuple(inp["x"].shape), dtype=np.float64)
    for b in range(B):
        for c0 in range(0, Cc, chunk):
            c1 = min(Cc, c0 + chunk)
            wl = inp["wlogit"][b:b + 1] if share_w else inp["wlogit"][b:b + 1, :, c0:c1]
            out[b:b + 1, c0:c1] = oracle.prop2d(
                f64(inp["x"][b:b + 1, c0:c1]), f64(inp["lam"][b:b + 1, :, c0:c1]), f64(wl),
                f64(inp["u"][b:b + 1, :, c0:c1]), dirs=dirs, share_w=share_w)
    return out


def workspace(gspn, inp, dirs=15, share_w=1):
    B, Cc, H, W = inp["x"].shape
    n = gspn.workspace_bytes(B, Cc, H, W, dirs, share_w, inp["x"].dtype)
    return torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")


# the kernel (gspn_prop2d_fwd_algo) behind each launch path
ALGO_OF_PATH = {"dir": "direction", "dir-shared": "direction", "dir-yglobal": "direction",
                "dir-half": "direction",
                "dir-banded": "direction", "pair": "sweep_pair", "split": "split",
                "generic": "generic"}


def check(gspn, inp, dirs=15, share_w=0, planes=None, what="", ws=False, path=None, algo=None,
          skip_refused=False):
    """Run the library and compare with the oracle; `path`, when given, is the
    launch path the call must have taken (gspn_last_launch_info).  The kernel
    is pinned to the path's (gspn_prop2d_fwd_algo) unless `algo` says
    otherwise ("auto": the library's own choice, which `path` then checks);
    calls with a workspace always make the library's choice.  With
    `skip_refused`, a kernel that refuses the sizes (GSPN_ERR_ALGO) skips the
    test."""
    d = to_dev(inp)
    if algo is None and path is not None and not ws:
        algo = ALGO_OF_PATH[path]
    if ws or algo is None:
        kw = {"workspace": workspace(gspn, inp, dirs, share_w)} if ws else {}
        y = gspn.prop2d_fwd(d["x"], d["lam"], d["wlogit"], d["u"], dirs=dirs, share_w=share_w, **kw)
    else:
        G = 1 if share_w else inp["x"].shape[1]
        try:
            y = gspn.prop2d_fwd_ex(d["x"], d["lam"], d["wlogit"], d["u"], dirs=dirs, w_groups=G,
                                   algo=algo)
        except gspn.GspnError as e:
            if skip_refused and e.status == 11:
                pytest.skip(f"{algo} does not take {tuple(inp['x'].shape)}")
            raise
    torch.cuda.synchronize()
    if path is not None:
        assert gspn.launch_info()["path"] == path, (what, gspn.launch_info())
    yg = f64(y)
    if planes == "all":
        yo = oracle_all(inp, dirs, share_w)
    elif planes is None:
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


@pytest.mark.parametrize("name,path", [("1k", "dir-half"), ("2k", "dir-half"),
                                       ("orig", "dir-yglobal")])
def test_workload_all_planes(gspn, name, path):
    """Full-size workload in the launch the benchmark times, every plane
    compared with the oracle (every item of every persistent CTA, the last
    partial round included)."""
    w = WORKLOADS[name]
    inp = workload_inputs(w, seed=0)
    rel = check(gspn, inp, share_w=w.share_w, planes="all", what=name, path=path)
    print(f"\n{name} (all planes): max|err| / max|y| = {rel:.3e}")


# --------------------------------------------------------------------------
# shapes, ragged tails, masks, dtypes, channel sharing
# --------------------------------------------------------------------------

SHAPES = [
    (1, 1, 1, 1), (1, 2, 1, 7), (1, 2, 7, 1), (2, 3, 2, 2), (1, 2, 3, 5), (1, 2, 31, 33),
    (2, 2, 33, 31), (1, 3, 32, 32), (1, 2, 64, 65), (2, 2, 74, 74), (1, 2, 16, 100),
    (1, 1, 100, 16), (1, 2, 97, 129), (1, 1, 129, 97), (1, 1, 148, 148), (1, 1, 256, 256),
    (1, 1, 255, 3), (1, 1, 3, 255),
    # every lane layout of the sweep-pair kernel, odd line counts (the two
    # sweeps meet on the middle line), non-square grids
    (2, 2, 2, 2), (2, 3, 5, 6), (1, 2, 37, 38), (1, 2, 38, 36), (1, 2, 50, 50), (1, 2, 81, 82),
    (1, 2, 112, 112), (1, 2, 128, 128), (1, 2, 40, 64), (1, 2, 96, 80), (3, 5, 74, 74),
]


# every kernel on every shape it takes (refusals skip), and the library's choice
ALGOS = ["auto", "direction", "sweep_pair", "split", "generic"]


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_shapes(gspn, shape, dtype, algo):
    B, Cc, H, W = shape
    inp = make_inputs(B, Cc, H, W, sigma_w=2.0, dtype=dtype, seed=hash(shape) % 1000)
    check(gspn, inp, what=f"{shape} {dtype} {algo}", algo=algo, skip_refused=True)


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("dirs", [1, 2, 4, 8, 3, 12, 5, 10, 6, 9, 7, 11, 13, 14, 15])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_direction_masks(gspn, dirs, dtype, algo):
    inp = make_inputs(2, 3, 21, 18, sigma_w=2.0, dtype=dtype, seed=dirs)
    check(gspn, inp, dirs=dirs, what=f"dirs={dirs} {algo}", algo=algo, skip_refused=True)


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [(2, 5, 16, 16), (3, 4, 37, 38), (1, 3, 148, 148)],
                         ids=lambda s: "x".join(map(str, s)))
def test_share_w(gspn, shape, dtype, algo):
    B, Cc, H, W = shape
    inp = make_inputs(B, Cc, H, W, share_w=1, sigma_w=1.0, dtype=dtype, seed=7)
    check(gspn, inp, share_w=1, what=f"share_w {shape} {algo}", algo=algo, skip_refused=True)


# --------------------------------------------------------------------------
# compact mode with a workspace: the shared weights normalised once
# --------------------------------------------------------------------------

def test_workload_2k_workspace(gspn):
    """The 2k compact workload through gspn_prop2d_fwd_ws (every plane)."""
    w = WORKLOADS["2k"]
    inp = workload_inputs(w, seed=0)
    rel = check(gspn, inp, share_w=1, planes="all", what="2k ws", ws=True, path="dir-half")
    print(f"\n2k with workspace (all planes): max|err| / max|y| = {rel:.3e}")
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


@pytest.mark.parametrize("dtype,W", [("f32", 23), ("bf16", 24)])
@pytest.mark.parametrize("mode", ["clamp_binds", "all_very_negative", "saturated_positive"])
def test_share_w_workspace_extremes(gspn, mode, dtype, W):
    """The clamp (sum of the weights below 1) and saturated logits through the
    weights normalised ahead (fp16 weights for bf16 inputs), on the direction
    kernel that reads them (even width for bf16)."""
    inp = make_inputs(2, 3, 19, W, share_w=1, sigma_w=1.0, dtype="f32", seed=3)
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
    check(gspn, inp, share_w=1, what=f"ws {mode} {dtype}", ws=True,
          path="dir-half" if dtype == "bf16" else "dir")
    assert gspn.launch_info()["launches"] == 2


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

@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_hand_examples(gspn, dtype, algo):
    ran = 0
    for ex in pins.parse_hand_examples():
        x, lam, wl, u = pins.hand_example_inputs(ex)
        inp = {"x": torch.tensor(x, dtype=dtype), "lam": torch.tensor(lam, dtype=dtype),
               "wlogit": torch.tensor(wl, dtype=dtype), "u": torch.tensor(u, dtype=dtype)}
        try:
            check(gspn, inp, dirs=ex["dirs"][0], what=f"{ex['name']} {algo}", algo=algo,
                  skip_refused=True)
            ran += 1
        except pytest.skip.Exception:
            pass
    if not ran:
        pytest.skip(f"{algo} takes none of the hand examples")


@pytest.mark.parametrize("dtype,shape,path", [
    ("f32", (1, 2, 19, 23), "dir"), ("bf16", (1, 2, 19, 24), "dir-half"),
    ("bf16", (1, 2, 19, 2), "dir-shared"),
    ("f32", (1, 2, 19, 23), "split"), ("bf16", (1, 2, 19, 24), "split"),
    ("bf16", (1, 2, 74, 74), "dir-half"), ("f32", (1, 2, 16, 16), "pair"),
    ("bf16", (1, 2, 16, 16), "pair"), ("f32", (1, 2, 19, 150), "dir"),
    ("bf16", (1, 2, 19, 150), "dir-half"), ("bf16", (1, 2, 19, 23), "generic")],
    ids=lambda v: "x".join(map(str, v)) if isinstance(v, tuple) else str(v))
@pytest.mark.parametrize("mode", ["all_very_negative", "clamp_binds", "overflow_pairs",
                                  "saturated_positive", "mixed_extremes"])
def test_extreme_logits(gspn, mode, dtype, shape, path):
    """Logit ranges where the denominator clamp binds (all on-grid logits
    below about -14) or where a product form of the normalisation would
    overflow (two logits below about -44), on each kernel that normalises in
    the scan (the launch path is asserted)."""
    B, Cc, H, W = shape
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
    check(gspn, inp, what=f"{mode} {dtype} {shape}", path=path)


@pytest.mark.parametrize("dtype,shape,path", [
    ("f32", (1, 2, 16, 15), "pair"), ("bf16", (2, 3, 74, 74), "dir-half"),
    ("bf16", (2, 3, 21, 2), "dir-shared"), ("bf16", (2, 3, 21, 4), "dir-half"),
    ("f32", (1, 2, 16, 15), "split"), ("bf16", (2, 3, 74, 74), "split"),
    ("f32", (1, 2, 60, 100), "split"),
    ("f32", (1, 2, 37, 38), "dir"), ("f32", (1, 2, 19, 150), "dir"),
    ("bf16", (1, 2, 148, 148), "dir-half"), ("f32", (1, 1, 256, 256), "dir-yglobal"),
    ("bf16", (1, 2, 19, 23), "generic")],
    ids=lambda v: "x".join(map(str, v)) if isinstance(v, tuple) else str(v))
def test_nan_in_off_grid_slots(gspn, dtype, shape, path):
    """Off-grid logit slots (slot 0 of a line's first position, slot 2 of its
    last) carry no weight and are never needed; filled with NaN they must not
    reach the output (the oracle never reads them)."""
    B, Cc, H, W = shape
    inp = make_inputs(B, Cc, H, W, sigma_w=2.0, dtype=dtype, seed=13)
    wl = inp["wlogit"].clone()
    nan = float("nan")
    wl[:, 0:2, :, 0, :, 0] = nan          # row lines: left end, slot 0
    wl[:, 0:2, :, 2, :, W - 1] = nan      # row lines: right end, slot 2
    wl[:, 2:4, :, 0, 0, :] = nan          # column lines: top end, slot 0
    wl[:, 2:4, :, 2, H - 1, :] = nan      # column lines: bottom end, slot 2
    inp["wlogit"] = wl
    check(gspn, inp, what=f"NaN edge slots {shape} {dtype}", path=path)


# --------------------------------------------------------------------------
# launch paths, host entry point, streams, errors
# --------------------------------------------------------------------------

@pytest.mark.parametrize("shape,dtype,path", [
    ((2, 3, 74, 74), "bf16", "split"),         # few planes: at most two waves of four CTAs
    ((2, 64, 74, 74), "bf16", "split"),
    ((4, 64, 74, 74), "bf16", "dir-half"),     # four waves
    ((8, 32, 37, 37), "f32", "split"),
    ((8, 64, 37, 37), "f32", "dir"),           # three waves
    ((2, 3, 74, 74), "f32", "split"),
    ((4, 4, 37, 37), "f32", "split"),
    ((1, 4, 16, 16), "f32", "split"),
    ((2, 2, 16, 14), "bf16", "split"),
    ((1, 2, 20, 33), "bf16", "split"),         # odd bf16 row width
    ((8, 24, 16, 16), "f32", "pair"),          # lines of up to 16
    ((8, 24, 16, 14), "bf16", "pair"),
    ((8, 40, 37, 37), "f32", "dir"),
    ((8, 40, 74, 74), "bf16", "dir-half"),
    ((8, 40, 20, 33), "bf16", "generic"),      # odd bf16 row width
    ((1, 2, 160, 160), "f32", "dir-shared"),   # lines over 128; two output planes do not fit
    ((1, 2, 256, 256), "f32", "dir-yglobal"),
    ((1, 1, 256, 250), "f32", "dir-yglobal"),   # width not a multiple of 4: scalar column flush
    ((1, 1, 231, 253), "f32", "dir-yglobal"),   # odd width: a last column chunk of one column
    ((1, 2, 256, 256), "bf16", "dir-banded"),
    ((1, 2, 148, 148), "bf16", "dir-half"),
    ((1, 1, 300, 40), "f32", "generic"),       # line longer than 256
    ((2, 2, 1, 40), "bf16", "generic"),        # lines of one position
    ((1, 3, 17, 1), "f32", "generic"),
], ids=lambda v: "x".join(map(str, v)) if isinstance(v, tuple) else str(v))
def test_launch_paths(gspn, shape, dtype, path):
    """The library's own choice of kernel (and its parity there)."""
    B, Cc, H, W = shape
    inp = make_inputs(B, Cc, H, W, sigma_w=2.0, dtype=dtype, seed=11)
    check(gspn, inp, what=path, path=path, algo="auto")


@pytest.mark.parametrize("shape,dtype,algo", [
    ((1, 2, 200, 40), "f32", "split"),        # line over 128
    ((1, 2, 15, 15), "bf16", "split"),        # plane of an odd number of bf16 elements
    ((1, 2, 200, 40), "f32", "sweep_pair"),   # line over 128
    ((1, 2, 16, 15), "bf16", "sweep_pair"),   # odd bf16 row width
    ((1, 2, 100, 16), "f32", "sweep_pair"),   # rows shorter than the lanes' pair blocks
    ((1, 2, 20, 33), "bf16", "direction"),    # odd bf16 row width
    ((1, 2, 1, 40), "f32", "direction"),      # lines of one position
    ((1, 2, 300, 40), "bf16", "direction")],  # line over 256
    ids=lambda v: "x".join(map(str, v)) if isinstance(v, tuple) else str(v))
def test_algo_refused_when_out_of_range(gspn, shape, dtype, algo):
    """A named kernel whose limits the sizes exceed is refused (GSPN_ERR_ALGO)
    before anything runs: the output is left untouched."""
    B, Cc, H, W = shape
    inp = to_dev(make_inputs(B, Cc, H, W, sigma_w=2.0, dtype=dtype, seed=5))
    out = torch.full_like(inp["x"], 7.0)
    with pytest.raises(gspn.GspnError) as e:
        gspn.prop2d_fwd_ex(inp["x"], inp["lam"], inp["wlogit"], inp["u"], algo=algo, out=out)
    torch.cuda.synchronize()
    assert e.value.status == 11
    assert bool((out == 7.0).all())


@pytest.mark.parametrize("shape,dtype", [((2, 3, 37, 40), "bf16"), ((1, 1, 5, 5), "f32"),
                                         ((5, 1, 5, 5), "f32"), ((7, 2, 9, 6), "bf16"),
                                         ((3, 1, 3, 3), "bf16")],
                         ids=lambda v: "x".join(map(str, v)) if isinstance(v, tuple) else str(v))
def test_host_entry_point(gspn, shape, dtype):
    """Pipelined batch chunks, also when a batch element's bytes are not a
    multiple of 16 (chunks then start at aligned batch indices)."""
    B, Cc, H, W = shape
    inp = make_inputs(B, Cc, H, W, sigma_w=2.0, dtype=dtype, seed=4)
    h = {k: v.pin_memory() for k, v in inp.items()}
    h["out"] = torch.empty_like(inp["x"]).pin_memory()
    d = {k: torch.empty_like(v, device="cuda") for k, v in h.items()}
    y = gspn.prop2d_fwd_host(h, d)
    dd = to_dev(inp)
    y_dev = gspn.prop2d_fwd(dd["x"], dd["lam"], dd["wlogit"], dd["u"])
    torch.cuda.synchronize()
    yo = oracle.prop2d(f64(inp["x"]), f64(inp["lam"]), f64(inp["wlogit"]), f64(inp["u"]))
    scale = np.max(np.abs(yo))
    tol = TOL[inp["x"].dtype]
    assert np.max(np.abs(f64(y) - yo)) <= tol * scale
    assert np.max(np.abs(f64(y) - f64(y_dev))) <= tol * scale


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


# --------------------------------------------------------------------------
# sharing variants: lambda/u shared by the directions, logits by channel groups
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dtype,shape,path", [
    ("bf16", (2, 4, 74, 74), "dir-half"), ("f32", (1, 6, 16, 16), "pair"),
    ("bf16", (2, 4, 74, 74), "split"), ("f32", (1, 4, 37, 38), "split"),
    ("f32", (1, 4, 19, 150), "dir"), ("bf16", (1, 4, 19, 150), "dir-half"),
    ("bf16", (1, 4, 20, 33), "generic")],
    ids=lambda v: "x".join(map(str, v)) if isinstance(v, tuple) else str(v))
@pytest.mark.parametrize("gate_dirs,groups", [(1, "all"), (4, "half"), (1, "one"), (4, "one")])
def test_sharing_variants(gspn, dtype, shape, path, gate_dirs, groups):
    B, Cc, H, W = shape
    G = {"all": Cc, "half": Cc // 2, "one": 1}[groups]
    g = torch.Generator().manual_seed(41)
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    x = torch.randn((B, Cc, H, W), generator=g)
    lam = torch.rand((B, gate_dirs, Cc, H, W), generator=g)
    wl = torch.randn((B, 4, G, 3, H, W), generator=g) * 2.0
    u = torch.rand((B, gate_dirs, Cc, H, W), generator=g)
    inp = {k: v.to(td) for k, v in {"x": x, "lam": lam, "wlogit": wl, "u": u}.items()}
    d = to_dev(inp)
    y = gspn.prop2d_fwd_ex(d["x"], d["lam"], d["wlogit"], d["u"], gate_dirs=gate_dirs, w_groups=G,
                           algo=ALGO_OF_PATH[path])
    torch.cuda.synchronize()
    assert gspn.launch_info()["path"] == path
    yo = oracle.prop2d_ex(f64(inp["x"]), f64(inp["lam"]), f64(inp["wlogit"]), f64(inp["u"]),
                          gate_dirs=gate_dirs, w_groups=G)
    scale = float(np.max(np.abs(yo)))
    err = float(np.max(np.abs(f64(y) - yo)))
    assert err <= TOL[td] * scale, f"{err:.3e} vs {scale:.3e}"


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [(2, 3, 74, 74), (1, 2, 37, 38), (1, 2, 50, 50), (1, 2, 81, 82),
                                   (1, 2, 112, 112), (1, 2, 128, 128), (1, 2, 40, 64),
                                   (1, 2, 96, 80), (1, 2, 16, 100), (3, 5, 21, 18)],
                         ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("dirs", [1, 2, 3])
def test_row_directions_on_the_sweep_pair_kernel(gspn, shape, dtype, dirs):
    """Row directions alone run on the sweep-pair kernel for lines up to 128
    (every lane layout: pairs plus one or two singles per lane)."""
    B, Cc, H, W = shape
    if dtype == "bf16" and W % 2:
        pytest.skip("odd bf16 rows go to the general kernel")
    inp = make_inputs(B, Cc, H, W, sigma_w=2.0, dtype=dtype, seed=dirs + sum(shape))
    want = "pair" if W >= 32 * (((max(H, W) + 15) // 16 - 1) // 2) else None
    check(gspn, inp, dirs=dirs, what=f"rows {shape} {dtype} dirs={dirs}", path=want)
