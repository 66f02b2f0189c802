"""Training-free block-sparse attention forward for B200 (sm_100a).

The compute path lives in the CUDA library ``libsparseattn.so`` (sources
under ``csrc/``) behind the C ABI declared in ``include/sparse_attn.h``;
``long_context_mean_b200.sa`` is the thin ctypes binding over it and is
loaded lazily, so importing this package (for example to use the seeded
input generators in ``inputs``) never touches the GPU.
"""

import importlib

__all__ = ["sa", "inputs"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
