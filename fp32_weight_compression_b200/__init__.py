"""B200 (sm_100a) lossless weight compression: exponent-plane rANS.

The codec itself is libwc.so (C ABI in include/wc.h, CUDA kernels in csrc/);
`fp32_weight_compression_b200.wc` is its Python binding.  Importing the
package loads nothing; the binding loads the library on first use.
"""
import importlib

__all__ = ["wc", "build"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f".{name}", __name__)
    raise AttributeError(name)
