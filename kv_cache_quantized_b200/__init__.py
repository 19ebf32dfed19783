"""B200-native (sm_100a) AXELRAM decode-time attention from quantized key-cache indices.

The compute lives in libaxr.so (C ABI, include/axr.h): the write path (sign flip + Walsh-Hadamard + Lloyd-Max
indices + fp16 norm, bit-packed), the LUT scorer, the split-T online-softmax . V decode kernel (fp16 or quantized
values), a dense fp16 decode kernel used as the bandwidth reference, and the sign-pattern selector.  This package is
the thin Python binding (``ops``) plus seeded synthetic workloads (``workloads``).  Importing it does not load the
library; the first op call does, and raises if the library is missing.
"""

from ._abi import AxrError  # noqa: F401

__version__ = "0.1.0"


def __getattr__(name):  # lazy: keep `import kv_cache_quantized_b200` free of torch/CUDA work
    if name in ("ops", "workloads", "build"):
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
