"""gspn_prop2d_fwd_noalloc: the compact mode for callers that cannot allocate.

Some callers cannot hand the library a workspace: they run inside a host
framework that owns all device memory and forbids allocating while it
executes, so they cannot call cudaMalloc (or an allocating library routine)
to make one.  gspn_prop2d_fwd_noalloc keeps the compact mode's normalised
weights in a scratch array built into the library instead.  These tests call
it through the C ABI and compare it with gspn_prop2d_fwd_ws, which takes a
caller workspace, on two calls in a row (the array keeps the first call's
contents when the second starts), and check that sizes beyond the array are
rejected before anything is launched.

This file is named so that pytest collects it last.
"""
import ctypes

import pytest
import torch

from spatial_propagation_vision_b200.workloads import make_inputs

pytestmark = pytest.mark.gpu

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


@pytest.fixture(scope="module")
def gspn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from spatial_propagation_vision_b200 import prop2d
    return prop2d


def _noalloc(gspn, d, share_w, out):
    """One call of the C entry point on the current stream; returns the status."""
    B, Cc, H, W = d["x"].shape
    dt = 1 if d["x"].dtype == torch.bfloat16 else 0
    return gspn.lib.gspn_prop2d_fwd_noalloc(
        d["x"].data_ptr(), d["lam"].data_ptr(), d["wlogit"].data_ptr(), d["u"].data_ptr(),
        B, Cc, H, W, 15, share_w, dt, out.data_ptr(),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("dtype,shape", [("bf16", (4, 8, 148, 148)), ("f32", (2, 5, 37, 38)),
                                         ("bf16", (2, 3, 74, 74))])
def test_noalloc_matches_workspace_entry_point(gspn, dtype, shape):
    B, Cc, H, W = shape
    # two different inputs, run back to back through the shared scratch array
    seeds = (21, 22)
    for seed in seeds:
        inp = make_inputs(B, Cc, H, W, share_w=1, sigma_w=1.0, dtype=dtype, seed=seed)
        d = {k: v.cuda() for k, v in inp.items()}
        n = gspn.workspace_bytes(B, Cc, H, W, 15, 1, d["x"].dtype)
        assert 0 < n <= gspn.NOALLOC_WORKSPACE_BYTES
        ws = torch.empty(n, dtype=torch.uint8, device="cuda")
        ref = gspn.prop2d_fwd(d["x"], d["lam"], d["wlogit"], d["u"], share_w=1, workspace=ws)
        out = torch.full_like(d["x"], float("nan"))
        assert _noalloc(gspn, d, 1, out) == 0
        assert gspn.launch_info()["launches"] == 2
        torch.cuda.synchronize()
        scale = float(ref.double().abs().max())
        err = float((out.double() - ref.double()).abs().max())
        assert torch.isfinite(out).all()
        assert err <= TOL[d["x"].dtype] * scale, f"seed {seed}: {err:.3e} vs {scale:.3e}"


def test_noalloc_without_share_w_is_the_plain_call(gspn):
    inp = make_inputs(2, 3, 30, 32, sigma_w=2.0, dtype="bf16", seed=5)
    d = {k: v.cuda() for k, v in inp.items()}
    ref = gspn.prop2d_fwd(d["x"], d["lam"], d["wlogit"], d["u"])
    out = torch.empty_like(ref)
    assert _noalloc(gspn, d, 0, out) == 0
    torch.cuda.synchronize()
    assert torch.equal(out, ref)


def test_noalloc_rejects_sizes_beyond_the_array(gspn):
    # B = 16 grids of 148 x 148 bf16 need 8.4 MB of weights: more than the array
    B, Cc, H, W = 16, 1, 148, 148
    assert gspn.workspace_bytes(B, Cc, H, W, 15, 1, torch.bfloat16) > gspn.NOALLOC_WORKSPACE_BYTES
    x = torch.zeros((B, Cc, H, W), dtype=torch.bfloat16, device="cuda")
    g = torch.zeros((B, 4, Cc, H, W), dtype=torch.bfloat16, device="cuda")
    wl = torch.zeros((B, 4, 1, 3, H, W), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros_like(x)
    st = _noalloc(gspn, {"x": x, "lam": g, "wlogit": wl, "u": g}, 1, out)
    assert st == 9
    assert gspn.lib.gspn_status_str(st).decode().startswith("GSPN_ERR_NOALLOC_LIMIT")
