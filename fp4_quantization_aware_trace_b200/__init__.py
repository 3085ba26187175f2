"""B200-native (sm_100a) TRACE rollout-guided NVFP4 rounding.

The hot path -- rollout capture of the compact cache and the guided QAT
fake-quant forward with its masked straight-through backward -- runs in the
hand-written CUDA kernels of ``libtrace_fp4.so`` behind a C ABI
(``include/trace_fp4.h``).  ``ops`` is the thin ctypes binding; ``inputs``
draws the seeded synthetic activations.
"""
__all__ = ["ops", "inputs"]


def __getattr__(name):
    if name in ("ops", "inputs"):
        import importlib
        return importlib.import_module(f".{name}", __name__)
    raise AttributeError(name)
