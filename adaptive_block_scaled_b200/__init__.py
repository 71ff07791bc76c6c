"""IF4 (Int/Float 4) adaptive block-scaled quantization on NVIDIA B200.

``libif4.so`` (hand-written sm_100a CUDA behind a C ABI, see include/if4.h)
does the work; ``binding`` is its ctypes binding.  Attributes of the binding
are resolved on first use, so ``adaptive_block_scaled_b200.workloads`` (the
seeded input generators) can be imported without the built library.
"""

__all__ = ["binding", "workloads"]


def __getattr__(name):
    if name in ("binding", "workloads", "build"):
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    from . import binding
    return getattr(binding, name)
