"""The C ABI without a GPU: the library builds and loads, exports every
function that include/gspn.h declares, and rejects bad arguments on the host
before touching CUDA."""
import ctypes
import os
import re

import pytest

from spatial_propagation_vision_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    path = build.build_library()
    return ctypes.CDLL(path)


def declared_functions():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s*(gspn_[a-z0-9_]+)\s*\(",
                                src, flags=re.M)
    return names


def test_header_declares_entry_points():
    names = declared_functions()
    assert "gspn_prop2d_fwd" in names and "gspn_status_str" in names, names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"


def _fwd(lib):
    f = lib.gspn_prop2d_fwd
    f.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int] * 7 + [ctypes.c_void_p] * 2
    f.restype = ctypes.c_int
    return f


P = 0x10000  # fake, 16-byte aligned "device" address: never dereferenced on these paths


@pytest.mark.parametrize("args,status", [
    ((P, P, P, P, -1, 4, 8, 8, 15, 0, 0, P), 2),          # negative B
    ((P, P, P, P, 1, 4, 8, -8, 15, 0, 0, P), 2),          # negative W
    ((P, P, P, P, 1, 4, 8, 8, 0, 0, 0, P), 3),            # empty direction mask
    ((P, P, P, P, 1, 4, 8, 8, 16, 0, 0, P), 3),           # mask beyond the 4 directions
    ((P, P, P, P, 1, 4, 8, 8, 15, 2, 0, P), 3),           # share_w not 0/1
    ((P, P, P, P, 1, 4, 8, 8, 15, 0, 7, P), 4),           # unknown dtype
    ((None, P, P, P, 1, 4, 8, 8, 15, 0, 0, P), 1),        # NULL input
    ((P, P, P, P, 1, 4, 8, 8, 15, 0, 1, None), 1),        # NULL output
    ((P + 2, P, P, P, 1, 4, 8, 8, 15, 0, 1, P), 5),       # misaligned input
    ((P, P, P, P, 1, 4, 8, 8, 15, 0, 0, P + 4), 5),       # misaligned output
    ((None, None, None, None, 0, 4, 8, 8, 15, 0, 0, None), 0),   # empty batch: nothing to do
    ((None, None, None, None, 1, 4, 0, 8, 15, 0, 1, None), 0),   # empty grid
    ((P, P, P, P, 1, 4, 8, 5000, 15, 0, 0, P), 2),        # line longer than any kernel takes
])
def test_argument_checks(lib, args, status):
    assert _fwd(lib)(*args, None) == status


def test_status_strings(lib):
    lib.gspn_status_str.argtypes = [ctypes.c_int]
    lib.gspn_status_str.restype = ctypes.c_char_p
    for s in range(12):
        assert lib.gspn_status_str(s).decode().startswith("GSPN_")
    assert lib.gspn_status_str(99) is not None


def _fwd_ws(lib):
    f = lib.gspn_prop2d_fwd_ws
    f.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int] * 7 + [ctypes.c_void_p] * 2 + \
                 [ctypes.c_size_t, ctypes.c_void_p]
    f.restype = ctypes.c_int
    return f


def test_workspace_bytes(lib):
    f = lib.gspn_prop2d_workspace_bytes
    f.argtypes = [ctypes.c_int] * 7
    f.restype = ctypes.c_size_t
    # [B][4][3][H][W] fp32 (fp32 inputs) or fp16 (bf16 inputs), compact mode only
    assert f(8, 64, 148, 148, 15, 1, 1) == 8 * 4 * 3 * 148 * 148 * 2
    assert f(2, 3, 5, 7, 15, 1, 0) == 2 * 4 * 3 * 5 * 7 * 4
    assert f(8, 64, 148, 148, 15, 0, 1) == 0      # per-channel logits: none
    assert f(8, 64, 148, 148, 0, 1, 1) == 0       # invalid mask
    assert f(8, 64, 148, 148, 15, 1, 9) == 0      # invalid dtype
    assert f(0, 64, 148, 148, 15, 1, 1) == 0      # empty


N = 2 * 4 * 3 * 8 * 8 * 4   # workspace bytes of B=2, 8x8, fp32


@pytest.mark.parametrize("ws,size,status", [
    (None, N, 1),          # compact mode without a workspace
    (P, N - 4, 8),         # too small
    (P + 8, N, 5),         # misaligned
])
def test_workspace_checks(lib, ws, size, status):
    assert _fwd_ws(lib)(P, P, P, P, 2, 4, 8, 8, 15, 1, 0, P, ws, size, None) == status


def test_workspace_ignored_without_share_w(lib):
    # per-channel logits: the workspace is not looked at, the other checks still apply
    assert _fwd_ws(lib)(None, P, P, P, 2, 4, 8, 8, 15, 0, 0, P, None, 0, None) == 1
    assert _fwd_ws(lib)(P, P, P, P, 2, 4, 8, 8, 16, 0, 0, P, None, 0, None) == 3
    assert _fwd_ws(lib)(None, None, None, None, 0, 4, 8, 8, 15, 1, 0, None, None, 0, None) == 0


def _fwd_ex(lib):
    f = lib.gspn_prop2d_fwd_ex
    f.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int] * 8 + [ctypes.c_void_p] * 2
    f.restype = ctypes.c_int
    return f


@pytest.mark.parametrize("args,status", [
    ((P, P, P, P, 1, 4, 8, 8, 15, 2, 4, 0, P), 10),       # gate_dirs neither 1 nor 4
    ((P, P, P, P, 1, 4, 8, 8, 15, 4, 3, 0, P), 10),       # w_groups does not divide Cc
    ((P, P, P, P, 1, 4, 8, 8, 15, 4, 0, 0, P), 10),       # no logit field
    ((P, P, P, P, 1, 4, 8, 8, 0, 4, 4, 0, P), 3),         # empty direction mask
    ((P, P, P, P, -1, 4, 8, 8, 15, 1, 2, 0, P), 2),       # negative B
    ((None, None, None, None, 0, 4, 8, 8, 15, 1, 2, 0, None), 0),   # empty batch
])
def test_ex_argument_checks(lib, args, status):
    assert _fwd_ex(lib)(*args, None) == status


def _fwd_algo(lib):
    f = lib.gspn_prop2d_fwd_algo
    f.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int] * 9 + [ctypes.c_void_p] * 2
    f.restype = ctypes.c_int
    return f


@pytest.mark.parametrize("args,status", [
    ((P, P, P, P, 1, 4, 8, 8, 15, 4, 4, 0, 5, P), 11),     # unknown algorithm
    ((P, P, P, P, 1, 4, 8, 8, 15, 4, 4, 0, -1, P), 11),
    ((P, P, P, P, 1, 4, 8, 8, 15, 2, 4, 0, 3, P), 10),     # sharing checked first
    ((P, P, P, P, 1, 4, 8, 8, 16, 4, 4, 0, 3, P), 3),      # then the direction mask
    ((P, P, P, P, -1, 4, 8, 8, 15, 4, 4, 0, 1, P), 2),     # negative B
    ((None, None, None, None, 0, 4, 8, 8, 15, 4, 4, 0, 2, None), 0),   # empty batch
])
def test_algo_argument_checks(lib, args, status):
    """gspn_prop2d_fwd_algo rejects bad arguments before it touches a device."""
    assert _fwd_algo(lib)(*args, None) == status


def _bwd_ex(lib):
    f = lib.gspn_prop2d_bwd_ex
    f.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 8 + [ctypes.c_void_p] * 5
    f.restype = ctypes.c_int
    return f


@pytest.mark.parametrize("args,status", [
    ((P, P, P, P, P, 1, 4, 8, 8, 15, 2, 4, 0, P, P, P, P), 10),    # gate_dirs neither 1 nor 4
    ((P, P, P, P, P, 1, 4, 8, 8, 15, 1, 3, 0, P, P, P, P), 10),    # w_groups does not divide Cc
    ((P, P, P, P, P, 1, 4, 8, 8, 0, 1, 2, 0, P, P, P, P), 3),      # empty direction mask
    ((P, P, P, P, P, -1, 4, 8, 8, 15, 1, 2, 0, P, P, P, P), 2),    # negative B
    ((None,) * 5 + (0, 4, 8, 8, 15, 1, 2, 0) + (None,) * 4, 0),     # empty batch
])
def test_bwd_ex_argument_checks(lib, args, status):
    """gspn_prop2d_bwd_ex rejects bad arguments before it touches a device."""
    assert _bwd_ex(lib)(*args, None) == status
