"""libssmscan: the Mamba selective-scan forward pass, its decode step and the
Mamba-2 scalar-decay chunked scan as hand-written CUDA kernels for B200
(sm_100a), behind a C ABI (include/ssmscan.h).

``api`` holds the torch-tensor binding (imported lazily: it needs torch);
``synth`` the seeded workload generator; ``build`` compiles the library.
"""
__all__ = ["api", "synth", "build"]


def __getattr__(name):
    if name in ("api", "synth", "build", "_abi"):
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
