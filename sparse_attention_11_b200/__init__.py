"""DeepSeek Sparse Attention (DSA) forward path for NVIDIA B200 (sm_100a).

The compute lives in libdsa.so (hand-written CUDA, C ABI in include/dsa.h);
`sparse_attention_11_b200.dsa` is its Python binding and
`sparse_attention_11_b200.workloads` draws the seeded synthetic inputs.
The binding is imported lazily so that the input generators are usable on
hosts where the library has not been built.
"""
__all__ = ["dsa", "workloads", "problem"]


def __getattr__(name):
    if name in ("dsa", "problem"):
        import importlib
        return importlib.import_module(f".{name}", __name__)
    raise AttributeError(name)
