"""B200-native hot path of a Dynamic SplitFuse forward pass: rotary on Q/K,
append into a blocked (paged) KV cache, one ragged causal attention.

The library is ``libfg.so`` (C ABI declared in include/fg.h); ``fg`` is its
Python binding and ``workloads`` the seeded input generator. Importing this
package loads nothing; the binding loads the library on first use.
"""

__all__ = ["fg", "workloads"]


def __getattr__(name):
    if name in __all__:
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
