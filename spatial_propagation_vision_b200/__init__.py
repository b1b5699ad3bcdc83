"""B200-native Prop2D: the four-direction GSPN line-scan propagation of C-GSPN.

The compute path is the C-ABI library ``libgspn.so`` (CUDA, sm_100a); the
Python binding in ``prop2d.py`` only marshals torch tensors to it.  Importing
this package does not load the library; ``prop2d`` does, and fails loudly
when it is missing.
"""

__all__ = ["prop2d_fwd", "prop2d_fwd_ex", "prop2d_bwd", "prop2d_bwd_ex", "prop2d_autograd",
           "workloads"]

_LAZY = ("prop2d_fwd", "prop2d_fwd_ex", "prop2d_fwd_noalloc", "prop2d_fwd_host",
         "prop2d_bwd", "prop2d_bwd_ex", "prop2d_autograd", "Prop2DFunction", "launch_info", "lib")


def __getattr__(name):
    if name in _LAZY:
        from . import prop2d
        return getattr(prop2d, name)
    raise AttributeError(name)
