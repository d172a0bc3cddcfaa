"""DiG token mixer on B200: chunkwise Gated Linear Attention forward/backward and
the SREM reorient + 3x3 depthwise conv, as sm_100a CUDA kernels behind a C ABI
(include/dig.h, libdig.so).

``gated_linear_attention_fwd_b200.dig`` is the thin ctypes binding (argument
marshalling only); ``gated_linear_attention_fwd_b200.inputs`` holds the seeded
synthetic-input recipe.  Importing the package itself loads nothing.
"""

__all__ = ["dig", "inputs"]


def __getattr__(name):
    if name in __all__:
        import importlib
        return importlib.import_module("." + name, __name__)
    raise AttributeError(name)
