"""The Python binding without a GPU: it loads the library, sizes the compact
mode's workspace through the C ABI, and rejects tensors it cannot pass on
(before any CUDA call)."""
import pytest
import torch

from spatial_propagation_vision_b200 import build


@pytest.fixture(scope="module")
def prop2d():
    build.build_library()
    from spatial_propagation_vision_b200 import prop2d as m
    return m


def test_workspace_bytes(prop2d):
    # [B][4][3][H][W]: fp16 weights for bf16 inputs, fp32 for fp32 inputs
    assert prop2d.workspace_bytes(8, 64, 148, 148, 15, 1, torch.bfloat16) == 8 * 4 * 3 * 148 * 148 * 2
    assert prop2d.workspace_bytes(2, 5, 16, 16, 15, 1, torch.float32) == 2 * 4 * 3 * 16 * 16 * 4
    assert prop2d.workspace_bytes(8, 64, 148, 148, 15, 0, torch.bfloat16) == 0


def test_rejects_cpu_tensors(prop2d):
    x = torch.zeros(1, 2, 4, 4)
    lam = u = torch.zeros(1, 4, 2, 4, 4)
    wl = torch.zeros(1, 4, 2, 3, 4, 4)
    with pytest.raises(ValueError, match="CUDA"):
        prop2d.prop2d_fwd(x, lam, wl, u)


def test_rejects_unsupported_dtype_and_rank(prop2d):
    lam = u = torch.zeros(1, 4, 2, 4, 4, dtype=torch.float16)
    wl = torch.zeros(1, 4, 2, 3, 4, 4, dtype=torch.float16)
    with pytest.raises(ValueError, match="dtype"):
        prop2d.prop2d_fwd(torch.zeros(1, 2, 4, 4, dtype=torch.float16), lam, wl, u)
    with pytest.raises(ValueError, match="B, Cc, H, W"):
        prop2d.prop2d_fwd(torch.zeros(2, 4, 4), lam, wl, u)


def test_status_names_match_the_library(prop2d):
    for code, name in prop2d.STATUS.items():
        assert prop2d.lib.gspn_status_str(code).decode().startswith(name)
