"""Thin ctypes binding of libgspn.so (include/gspn.h).

Argument marshalling only: tensors are checked and their device pointers
and the current CUDA stream are handed to the C ABI; every step of Prop2D
runs in the library's kernels.  Importing this module loads the library and
raises if it is missing: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgspn.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m spatial_propagation_vision_b200.build` "
        "(nvcc, sm_100a). There is no non-CUDA fallback.")

lib = ctypes.CDLL(LIB_PATH)

GSPN_F32, GSPN_BF16 = 0, 1
STATUS = {0: "GSPN_OK", 1: "GSPN_ERR_NULL", 2: "GSPN_ERR_SHAPE", 3: "GSPN_ERR_DIRS",
          4: "GSPN_ERR_DTYPE", 5: "GSPN_ERR_ALIGN", 6: "GSPN_ERR_CUDA", 7: "GSPN_ERR_DEVICE",
          8: "GSPN_ERR_WORKSPACE", 9: "GSPN_ERR_NOALLOC_LIMIT", 10: "GSPN_ERR_SHARING",
          11: "GSPN_ERR_ALGO"}

# kernel choices of gspn_prop2d_fwd_algo (gspn_algo)
ALGO = {"auto": 0, "direction": 1, "sweep_pair": 2, "split": 3, "generic": 4}

# bytes of the library's built-in scratch array (GSPN_NOALLOC_WORKSPACE_BYTES)
NOALLOC_WORKSPACE_BYTES = 8 * 1024 * 1024

_vp, _i = ctypes.c_void_p, ctypes.c_int
lib.gspn_prop2d_fwd.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp, _vp]
lib.gspn_prop2d_fwd.restype = _i
lib.gspn_prop2d_fwd_ws.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp, _vp,
                                   ctypes.c_size_t, _vp]
lib.gspn_prop2d_fwd_ws.restype = _i
lib.gspn_prop2d_fwd_ex.argtypes = [_vp, _vp, _vp, _vp] + [_i] * 8 + [_vp, _vp]
lib.gspn_prop2d_fwd_ex.restype = _i
lib.gspn_prop2d_fwd_algo.argtypes = [_vp, _vp, _vp, _vp] + [_i] * 9 + [_vp, _vp]
lib.gspn_prop2d_fwd_algo.restype = _i
lib.gspn_prop2d_bwd.argtypes = [_vp] * 5 + [_i] * 7 + [_vp] * 5
lib.gspn_prop2d_bwd.restype = _i
lib.gspn_prop2d_bwd_ex.argtypes = [_vp] * 5 + [_i] * 8 + [_vp] * 5
lib.gspn_prop2d_bwd_ex.restype = _i
lib.gspn_prop2d_fwd_noalloc.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp, _vp]
lib.gspn_prop2d_fwd_noalloc.restype = _i
lib.gspn_prop2d_workspace_bytes.argtypes = [_i] * 7
lib.gspn_prop2d_workspace_bytes.restype = ctypes.c_size_t
lib.gspn_prop2d_fwd_host.argtypes = [_vp] * 10 + [_i] * 7 + [_vp]
lib.gspn_prop2d_fwd_host.restype = _i
lib.gspn_status_str.argtypes = [_i]
lib.gspn_status_str.restype = ctypes.c_char_p
lib.gspn_last_launch_info.argtypes = [ctypes.POINTER(_i)] * 4 + [ctypes.POINTER(ctypes.c_char_p)]
lib.gspn_last_launch_info.restype = None


class GspnError(RuntimeError):
    def __init__(self, status: int):
        super().__init__(lib.gspn_status_str(status).decode())
        self.status = status


_DT = {torch.float32: GSPN_F32, torch.bfloat16: GSPN_BF16}


def _dims(x: torch.Tensor):
    if x.dim() != 4:
        raise ValueError(f"x must be [B, Cc, H, W], got {tuple(x.shape)}")
    return tuple(int(s) for s in x.shape)


def _check(name, t, shape, dtype, device, cuda=True):
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name}: expected dtype {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if cuda and t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")


def _stream_handle(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def workspace_bytes(B: int, Cc: int, H: int, W: int, dirs: int = 15, share_w: int = 0,
                    dtype: torch.dtype = torch.float32) -> int:
    """Bytes of workspace gspn_prop2d_fwd_ws uses (0 unless share_w)."""
    return int(lib.gspn_prop2d_workspace_bytes(B, Cc, H, W, int(dirs), int(share_w), _DT[dtype]))


def prop2d_fwd(x: torch.Tensor, lam: torch.Tensor, wlogit: torch.Tensor, u: torch.Tensor,
               dirs: int = 15, share_w: int = 0, out: torch.Tensor | None = None,
               stream: torch.cuda.Stream | None = None,
               workspace: torch.Tensor | None = None) -> torch.Tensor:
    """y = Prop2D(x; u, lambda, w) on the GPU (gspn_prop2d_fwd).

    x [B,Cc,H,W]; lam, u [B,4,Cc,H,W]; wlogit [B,4,Cw,3,H,W] (Cw = 1 if share_w
    else Cc); all float32 or all bfloat16, contiguous, on one CUDA device.
    Returns ``out`` ([B,Cc,H,W], same dtype), allocated if not given.
    Asynchronous on ``stream`` (default: the current stream).  With
    ``workspace`` (a contiguous CUDA tensor of at least ``workspace_bytes``
    bytes) the call goes through gspn_prop2d_fwd_ws: in the compact mode the
    shared weights are then normalised once for all channels.
    """
    B, Cc, H, W = _dims(x)
    if x.dtype not in _DT:
        raise ValueError(f"unsupported dtype {x.dtype}")
    if not x.is_cuda:
        raise ValueError("x must be a CUDA tensor")
    Cw = 1 if share_w else Cc
    dev = x.device
    _check("x", x, (B, Cc, H, W), x.dtype, dev)
    _check("lam", lam, (B, 4, Cc, H, W), x.dtype, dev)
    _check("u", u, (B, 4, Cc, H, W), x.dtype, dev)
    _check("wlogit", wlogit, (B, 4, Cw, 3, H, W), x.dtype, dev)
    if out is None:
        out = torch.empty((B, Cc, H, W), dtype=x.dtype, device=dev)
    _check("out", out, (B, Cc, H, W), x.dtype, dev)
    with torch.cuda.device(dev):
        if workspace is None:
            st = lib.gspn_prop2d_fwd(x.data_ptr(), lam.data_ptr(), wlogit.data_ptr(), u.data_ptr(),
                                     B, Cc, H, W, int(dirs), int(share_w), _DT[x.dtype],
                                     out.data_ptr(), _stream_handle(stream))
        else:
            if not workspace.is_contiguous() or workspace.device != dev:
                raise ValueError(f"workspace must be a contiguous tensor on {dev}")
            st = lib.gspn_prop2d_fwd_ws(x.data_ptr(), lam.data_ptr(), wlogit.data_ptr(),
                                        u.data_ptr(), B, Cc, H, W, int(dirs), int(share_w),
                                        _DT[x.dtype], out.data_ptr(), workspace.data_ptr(),
                                        workspace.numel() * workspace.element_size(),
                                        _stream_handle(stream))
    if st != 0:
        raise GspnError(st)
    return out


def prop2d_fwd_ex(x: torch.Tensor, lam: torch.Tensor, wlogit: torch.Tensor, u: torch.Tensor,
                  dirs: int = 15, gate_dirs: int = 4, w_groups: int | None = None,
                  out: torch.Tensor | None = None,
                  stream: torch.cuda.Stream | None = None, algo: str | None = None) -> torch.Tensor:
    """Prop2D with wider sharing (gspn_prop2d_fwd_ex): lam, u are
    [B,gate_dirs,Cc,H,W] (gate_dirs 4, or 1 shared by all directions);
    wlogit is [B,4,G,3,H,W] with G = w_groups (default Cc), channel c using
    logit field c // (Cc // G).  `algo` (a key of ALGO) names the kernel
    (gspn_prop2d_fwd_algo); None is the library's choice."""
    B, Cc, H, W = _dims(x)
    if x.dtype not in _DT:
        raise ValueError(f"unsupported dtype {x.dtype}")
    if not x.is_cuda:
        raise ValueError("x must be a CUDA tensor")
    G = Cc if w_groups is None else int(w_groups)
    dev = x.device
    _check("x", x, (B, Cc, H, W), x.dtype, dev)
    _check("lam", lam, (B, gate_dirs, Cc, H, W), x.dtype, dev)
    _check("u", u, (B, gate_dirs, Cc, H, W), x.dtype, dev)
    _check("wlogit", wlogit, (B, 4, G, 3, H, W), x.dtype, dev)
    if out is None:
        out = torch.empty((B, Cc, H, W), dtype=x.dtype, device=dev)
    _check("out", out, (B, Cc, H, W), x.dtype, dev)
    with torch.cuda.device(dev):
        if algo is None:
            st = lib.gspn_prop2d_fwd_ex(x.data_ptr(), lam.data_ptr(), wlogit.data_ptr(), u.data_ptr(),
                                        B, Cc, H, W, int(dirs), int(gate_dirs), G, _DT[x.dtype],
                                        out.data_ptr(), _stream_handle(stream))
        else:
            st = lib.gspn_prop2d_fwd_algo(x.data_ptr(), lam.data_ptr(), wlogit.data_ptr(),
                                          u.data_ptr(), B, Cc, H, W, int(dirs), int(gate_dirs), G,
                                          _DT[x.dtype], ALGO[algo], out.data_ptr(),
                                          _stream_handle(stream))
    if st != 0:
        raise GspnError(st)
    return out


def prop2d_bwd(x: torch.Tensor, lam: torch.Tensor, wlogit: torch.Tensor, u: torch.Tensor,
               gy: torch.Tensor, dirs: int = 15, share_w: int = 0,
               stream: torch.cuda.Stream | None = None) -> dict:
    """Gradients of Prop2D (gspn_prop2d_bwd) for the upstream gradient gy
    ([B,Cc,H,W], dtype of x): fp32 tensors {"x", "lam", "wlogit", "u"} in the
    input layouts."""
    B, Cc, H, W = _dims(x)
    if x.dtype not in _DT:
        raise ValueError(f"unsupported dtype {x.dtype}")
    if not x.is_cuda:
        raise ValueError("x must be a CUDA tensor")
    Cw = 1 if share_w else Cc
    dev = x.device
    _check("x", x, (B, Cc, H, W), x.dtype, dev)
    _check("gy", gy, (B, Cc, H, W), x.dtype, dev)
    _check("lam", lam, (B, 4, Cc, H, W), x.dtype, dev)
    _check("u", u, (B, 4, Cc, H, W), x.dtype, dev)
    _check("wlogit", wlogit, (B, 4, Cw, 3, H, W), x.dtype, dev)
    g = {"x": torch.empty((B, Cc, H, W), dtype=torch.float32, device=dev),
         "lam": torch.empty((B, 4, Cc, H, W), dtype=torch.float32, device=dev),
         "wlogit": torch.empty((B, 4, Cw, 3, H, W), dtype=torch.float32, device=dev),
         "u": torch.empty((B, 4, Cc, H, W), dtype=torch.float32, device=dev)}
    with torch.cuda.device(dev):
        st = lib.gspn_prop2d_bwd(x.data_ptr(), lam.data_ptr(), wlogit.data_ptr(), u.data_ptr(),
                                 gy.data_ptr(), B, Cc, H, W, int(dirs), int(share_w), _DT[x.dtype],
                                 g["x"].data_ptr(), g["lam"].data_ptr(), g["wlogit"].data_ptr(),
                                 g["u"].data_ptr(), _stream_handle(stream))
    if st != 0:
        raise GspnError(st)
    return g


def prop2d_bwd_ex(x: torch.Tensor, lam: torch.Tensor, wlogit: torch.Tensor, u: torch.Tensor,
                  gy: torch.Tensor, dirs: int = 15, gate_dirs: int = 4, w_groups: int | None = None,
                  stream: torch.cuda.Stream | None = None) -> dict:
    """Gradients of the sharing variants (gspn_prop2d_bwd_ex), layouts of
    prop2d_fwd_ex: fp32 tensors {"x", "lam", "wlogit", "u"}; a shared input's
    gradient sums the gradients of its uses."""
    B, Cc, H, W = _dims(x)
    if x.dtype not in _DT:
        raise ValueError(f"unsupported dtype {x.dtype}")
    if not x.is_cuda:
        raise ValueError("x must be a CUDA tensor")
    G = Cc if w_groups is None else int(w_groups)
    dev = x.device
    _check("x", x, (B, Cc, H, W), x.dtype, dev)
    _check("gy", gy, (B, Cc, H, W), x.dtype, dev)
    _check("lam", lam, (B, gate_dirs, Cc, H, W), x.dtype, dev)
    _check("u", u, (B, gate_dirs, Cc, H, W), x.dtype, dev)
    _check("wlogit", wlogit, (B, 4, G, 3, H, W), x.dtype, dev)
    g = {"x": torch.empty((B, Cc, H, W), dtype=torch.float32, device=dev),
         "lam": torch.empty((B, gate_dirs, Cc, H, W), dtype=torch.float32, device=dev),
         "wlogit": torch.empty((B, 4, G, 3, H, W), dtype=torch.float32, device=dev),
         "u": torch.empty((B, gate_dirs, Cc, H, W), dtype=torch.float32, device=dev)}
    with torch.cuda.device(dev):
        st = lib.gspn_prop2d_bwd_ex(x.data_ptr(), lam.data_ptr(), wlogit.data_ptr(), u.data_ptr(),
                                    gy.data_ptr(), B, Cc, H, W, int(dirs), int(gate_dirs), G,
                                    _DT[x.dtype], g["x"].data_ptr(), g["lam"].data_ptr(),
                                    g["wlogit"].data_ptr(), g["u"].data_ptr(), _stream_handle(stream))
    if st != 0:
        raise GspnError(st)
    return g


def prop2d_fwd_noalloc(x: torch.Tensor, lam: torch.Tensor, wlogit: torch.Tensor,
                       u: torch.Tensor, dirs: int = 15, share_w: int = 0,
                       out: torch.Tensor | None = None,
                       stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """Prop2D through gspn_prop2d_fwd_noalloc: the compact mode without a
    caller workspace (the library's built-in scratch array holds the shared
    weights), for callers that cannot allocate device memory while they run.
    Arguments as ``prop2d_fwd``; only ``out`` may be allocated here, and only
    when it is not given."""
    B, Cc, H, W = _dims(x)
    if x.dtype not in _DT:
        raise ValueError(f"unsupported dtype {x.dtype}")
    if not x.is_cuda:
        raise ValueError("x must be a CUDA tensor")
    Cw = 1 if share_w else Cc
    dev = x.device
    _check("x", x, (B, Cc, H, W), x.dtype, dev)
    _check("lam", lam, (B, 4, Cc, H, W), x.dtype, dev)
    _check("u", u, (B, 4, Cc, H, W), x.dtype, dev)
    _check("wlogit", wlogit, (B, 4, Cw, 3, H, W), x.dtype, dev)
    if out is None:
        out = torch.empty((B, Cc, H, W), dtype=x.dtype, device=dev)
    _check("out", out, (B, Cc, H, W), x.dtype, dev)
    with torch.cuda.device(dev):
        st = lib.gspn_prop2d_fwd_noalloc(x.data_ptr(), lam.data_ptr(), wlogit.data_ptr(),
                                         u.data_ptr(), B, Cc, H, W, int(dirs), int(share_w),
                                         _DT[x.dtype], out.data_ptr(), _stream_handle(stream))
    if st != 0:
        raise GspnError(st)
    return out


def prop2d_fwd_host(h: dict, d: dict, dirs: int = 15, share_w: int = 0,
                    stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """Prop2D on host tensors through gspn_prop2d_fwd_host.

    ``h``: pinned CPU tensors x, lam, wlogit, u, out; ``d``: device tensors of
    the same shapes (the library copies h -> d, runs, copies d["out"] ->
    h["out"] and synchronises the stream).  Returns h["out"].
    """
    x = h["x"]
    B, Cc, H, W = _dims(x)
    Cw = 1 if share_w else Cc
    shapes = {"x": (B, Cc, H, W), "lam": (B, 4, Cc, H, W), "u": (B, 4, Cc, H, W),
              "wlogit": (B, 4, Cw, 3, H, W), "out": (B, Cc, H, W)}
    dev = d["x"].device
    for k, s in shapes.items():
        _check("host " + k, h[k], s, x.dtype, None, cuda=False)
        _check("device " + k, d[k], s, x.dtype, dev)
    with torch.cuda.device(dev):
        st = lib.gspn_prop2d_fwd_host(
            h["x"].data_ptr(), h["lam"].data_ptr(), h["wlogit"].data_ptr(), h["u"].data_ptr(),
            h["out"].data_ptr(), d["x"].data_ptr(), d["lam"].data_ptr(), d["wlogit"].data_ptr(),
            d["u"].data_ptr(), d["out"].data_ptr(), B, Cc, H, W, int(dirs), int(share_w),
            _DT[x.dtype], _stream_handle(stream))
    if st != 0:
        raise GspnError(st)
    return h["out"]


def launch_info() -> dict:
    """Geometry of the launch made by the last successful call on this thread."""
    n, g, b, s = (ctypes.c_int() for _ in range(4))
    path = ctypes.c_char_p()
    lib.gspn_last_launch_info(ctypes.byref(n), ctypes.byref(g), ctypes.byref(b), ctypes.byref(s),
                              ctypes.byref(path))
    return {"launches": n.value, "grid": g.value, "block": b.value, "smem": s.value,
            "path": (path.value or b"").decode()}


class Prop2DFunction(torch.autograd.Function):
    """Prop2D as an autograd function: the forward is gspn_prop2d_fwd_ex, the
    backward gspn_prop2d_bwd_ex (the inputs' gradients are computed in fp32
    and returned in the inputs' dtype)."""

    @staticmethod
    def forward(ctx, x, lam, wlogit, u, dirs: int = 15, gate_dirs: int = 4, w_groups=None):
        ctx.save_for_backward(x, lam, wlogit, u)
        ctx.conf = (int(dirs), int(gate_dirs), w_groups)
        return prop2d_fwd_ex(x, lam, wlogit, u, dirs=dirs, gate_dirs=gate_dirs, w_groups=w_groups)

    @staticmethod
    def backward(ctx, gy):
        x, lam, wlogit, u = ctx.saved_tensors
        dirs, gate_dirs, w_groups = ctx.conf
        g = prop2d_bwd_ex(x, lam, wlogit, u, gy.contiguous().to(x.dtype), dirs=dirs,
                          gate_dirs=gate_dirs, w_groups=w_groups)
        return (g["x"].to(x.dtype), g["lam"].to(lam.dtype), g["wlogit"].to(wlogit.dtype),
                g["u"].to(u.dtype), None, None, None)


def prop2d_autograd(x: torch.Tensor, lam: torch.Tensor, wlogit: torch.Tensor, u: torch.Tensor,
                    dirs: int = 15, gate_dirs: int = 4, w_groups: int | None = None) -> torch.Tensor:
    """y = Prop2D(x; u, lambda, w) with gradients for x, lam, wlogit and u
    (layouts of prop2d_fwd_ex)."""
    return Prop2DFunction.apply(x, lam, wlogit, u, dirs, gate_dirs, w_groups)
