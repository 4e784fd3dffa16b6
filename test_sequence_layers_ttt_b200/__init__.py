"""B200-native (sm_100a) forward scan of the Test-Time-Training (TTT) layer.

The product is the C-ABI library ``libttt_b200.so`` (include/ttt.h) with
hand-written CUDA kernels; this package holds its sources (``csrc/``), the
build step (``build.py``), the thin ctypes binding (``_binding``) and the
seeded synthetic workloads (``inputs``).

``ttt_linear_forward`` and ``ttt_mlp_forward`` are loaded lazily so that the
input generators can be imported on machines where the library is not built;
calling either without the library raises ImportError.
"""

__all__ = ["ttt_linear_forward", "ttt_mlp_forward", "TTTError", "status_string"]


def __getattr__(name):
    if name in __all__:
        from . import _binding
        return getattr(_binding, name)
    raise AttributeError(name)
