"""Prop2D CPU oracle (fp64, single-threaded C) and its ctypes wrapper.

TEST INFRASTRUCTURE ONLY.  The oracle is the correctness reference for the
CUDA library.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import it.  It shares no code with the CUDA
path; the two meet only through the seeded input generators.

The arithmetic lives in ``prop2d_oracle.c`` (its header lists the passages of
"Scaling Parallel Sequence Models to Foundation-Scale Vision Encoders" it
follows and the readings taken where they are silent).  This module only
compiles it with gcc and marshals numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "prop2d_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_prop2d.so")


def compile_oracle(src: str, lib: str) -> str:
    """gcc -O2, strict IEEE (no fast-math, no FMA contraction)."""
    tmp = lib + f".tmp{os.getpid()}"
    subprocess.check_call(
        ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
         "-ffp-contract=off", src, "-o", tmp, "-lm"])
    os.replace(tmp, lib)
    return lib


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/liboracle_prop2d.so`` if it is stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(SOURCE):
        compile_oracle(SOURCE, _LIB)
    return _LIB


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


class Oracle:
    """Bound view of one compiled oracle library."""

    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        dp = ctypes.POINTER(ctypes.c_double)
        lib.oracle_prop2d_f64.argtypes = [dp, dp, dp, dp] + [ctypes.c_int] * 6 + [dp]
        lib.oracle_prop2d_f64.restype = ctypes.c_int
        lib.oracle_prop2d_weights_f64.argtypes = [dp] + [ctypes.c_int] * 5 + [dp]
        lib.oracle_prop2d_weights_f64.restype = ctypes.c_int
        lib.oracle_prop2d_bwd_f64.argtypes = [dp] * 5 + [ctypes.c_int] * 6 + [dp] * 4
        lib.oracle_prop2d_bwd_f64.restype = ctypes.c_int
        lib.oracle_prop2d_ex_f64.argtypes = [dp, dp, dp, dp] + [ctypes.c_int] * 7 + [dp]
        lib.oracle_prop2d_ex_f64.restype = ctypes.c_int
        lib.oracle_prop2d_bwd_ex_f64.argtypes = [dp] * 5 + [ctypes.c_int] * 7 + [dp] * 4
        lib.oracle_prop2d_bwd_ex_f64.restype = ctypes.c_int
        self._lib = lib

    def prop2d(self, x, lam, wlogit, u, dirs: int = 15, share_w: int = 0) -> np.ndarray:
        """y = Prop2D(x; u, lambda, w) in fp64.

        x [B,Cc,H,W]; lam, u [B,4,Cc,H,W]; wlogit [B,4,Cw,3,H,W] with
        Cw = 1 if share_w else Cc.  Inputs are widened to fp64 (bf16 and fp32
        values are represented exactly).
        """
        x, lam, wlogit, u = (_f64(t) for t in (x, lam, wlogit, u))
        B, Cc, H, W = x.shape
        Cw = 1 if share_w else Cc
        assert lam.shape == (B, 4, Cc, H, W) and u.shape == lam.shape, (lam.shape, u.shape)
        assert wlogit.shape == (B, 4, Cw, 3, H, W), wlogit.shape
        out = np.zeros((B, Cc, H, W), dtype=np.float64)
        rc = self._lib.oracle_prop2d_f64(_ptr(x), _ptr(lam), _ptr(wlogit), _ptr(u),
                                         B, Cc, H, W, int(dirs), int(bool(share_w)), _ptr(out))
        if rc != 0:
            raise ValueError("oracle_prop2d_f64 rejected its arguments")
        return out

    def prop2d_ex(self, x, lam, wlogit, u, dirs: int = 15, gate_dirs: int = 4,
                  w_groups: int | None = None) -> np.ndarray:
        """Forward with shared gates / grouped logits: lam, u [B,gate_dirs,Cc,H,W]
        (gate_dirs 4 or 1); wlogit [B,4,G,3,H,W], channel c using field
        c // (Cc // G) (G = w_groups, default Cc)."""
        x, lam, wlogit, u = (_f64(t) for t in (x, lam, wlogit, u))
        B, Cc, H, W = x.shape
        G = Cc if w_groups is None else int(w_groups)
        assert lam.shape == (B, gate_dirs, Cc, H, W) and u.shape == lam.shape, lam.shape
        assert wlogit.shape == (B, 4, G, 3, H, W), wlogit.shape
        out = np.zeros((B, Cc, H, W), dtype=np.float64)
        rc = self._lib.oracle_prop2d_ex_f64(_ptr(x), _ptr(lam), _ptr(wlogit), _ptr(u), B, Cc, H,
                                            W, int(dirs), int(gate_dirs), G, _ptr(out))
        if rc != 0:
            raise ValueError("oracle_prop2d_ex_f64 rejected its arguments")
        return out

    def prop2d_bwd(self, x, lam, wlogit, u, gy, dirs: int = 15, share_w: int = 0) -> dict:
        """Backward of Prop2D in fp64: given gy = dL/dy, the gradients
        {"x", "lam", "wlogit", "u"} of L, in the input layouts."""
        x, lam, wlogit, u, gy = (_f64(t) for t in (x, lam, wlogit, u, gy))
        B, Cc, H, W = x.shape
        Cw = 1 if share_w else Cc
        assert lam.shape == (B, 4, Cc, H, W) and u.shape == lam.shape, (lam.shape, u.shape)
        assert wlogit.shape == (B, 4, Cw, 3, H, W), wlogit.shape
        assert gy.shape == x.shape, gy.shape
        g = {"x": np.zeros_like(x), "lam": np.zeros_like(lam), "wlogit": np.zeros_like(wlogit),
             "u": np.zeros_like(u)}
        rc = self._lib.oracle_prop2d_bwd_f64(
            _ptr(x), _ptr(lam), _ptr(wlogit), _ptr(u), _ptr(gy), B, Cc, H, W, int(dirs),
            int(bool(share_w)), _ptr(g["x"]), _ptr(g["lam"]), _ptr(g["wlogit"]), _ptr(g["u"]))
        if rc != 0:
            raise ValueError("oracle_prop2d_bwd_f64 rejected its arguments")
        return g

    def prop2d_bwd_ex(self, x, lam, wlogit, u, gy, dirs: int = 15, gate_dirs: int = 4,
                      w_groups=None) -> dict:
        """Backward of the sharing variants in fp64 (layouts of prop2d_ex): the
        gradients {"x", "lam", "wlogit", "u"}; a shared input's gradient sums
        the gradients of its uses."""
        x, lam, wlogit, u, gy = (_f64(t) for t in (x, lam, wlogit, u, gy))
        B, Cc, H, W = x.shape
        G = Cc if w_groups is None else int(w_groups)
        assert lam.shape == (B, gate_dirs, Cc, H, W) and u.shape == lam.shape, (lam.shape, u.shape)
        assert wlogit.shape == (B, 4, G, 3, H, W), wlogit.shape
        assert gy.shape == x.shape, gy.shape
        g = {"x": np.zeros_like(x), "lam": np.zeros_like(lam), "wlogit": np.zeros_like(wlogit),
             "u": np.zeros_like(u)}
        rc = self._lib.oracle_prop2d_bwd_ex_f64(
            _ptr(x), _ptr(lam), _ptr(wlogit), _ptr(u), _ptr(gy), B, Cc, H, W, int(dirs),
            int(gate_dirs), G, _ptr(g["x"]), _ptr(g["lam"]), _ptr(g["wlogit"]), _ptr(g["u"]))
        if rc != 0:
            raise ValueError("oracle_prop2d_bwd_ex_f64 rejected its arguments")
        return g

    def weights(self, wlogit) -> np.ndarray:
        """Normalised tridiagonal weights [B,4,Cw,3,H,W] of a logit field (0 in off-grid slots)."""
        wlogit = _f64(wlogit)
        B, _, Cw, _, H, W = wlogit.shape
        out = np.zeros_like(wlogit)
        rc = self._lib.oracle_prop2d_weights_f64(_ptr(wlogit), B, Cw, H, W, 0, _ptr(out))
        if rc != 0:
            raise ValueError("oracle_prop2d_weights_f64 rejected its arguments")
        return out


_default: Oracle | None = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def prop2d(x, lam, wlogit, u, dirs: int = 15, share_w: int = 0) -> np.ndarray:
    return default().prop2d(x, lam, wlogit, u, dirs=dirs, share_w=share_w)


def weights(wlogit) -> np.ndarray:
    return default().weights(wlogit)


def prop2d_bwd(x, lam, wlogit, u, gy, dirs: int = 15, share_w: int = 0) -> dict:
    return default().prop2d_bwd(x, lam, wlogit, u, gy, dirs=dirs, share_w=share_w)


def prop2d_ex(x, lam, wlogit, u, dirs: int = 15, gate_dirs: int = 4, w_groups=None) -> np.ndarray:
    return default().prop2d_ex(x, lam, wlogit, u, dirs=dirs, gate_dirs=gate_dirs, w_groups=w_groups)


def prop2d_bwd_ex(x, lam, wlogit, u, gy, dirs: int = 15, gate_dirs: int = 4, w_groups=None) -> dict:
    return default().prop2d_bwd_ex(x, lam, wlogit, u, gy, dirs=dirs, gate_dirs=gate_dirs,
                                   w_groups=w_groups)
