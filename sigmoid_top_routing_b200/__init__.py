"""B200 (sm_100a) routed mixture-of-experts block: sigmoid top-k routing with a
selection-only expert bias, the grouped expert plan, grouped expert GEMMs
(SwiGLU gate-first or relu^2; bf16 or MLX-style affine 4-bit) and the
weighted combine.  The compute lives in the C-ABI library built from csrc/
(see include/moe.h); ``api`` binds it to torch tensors.

Submodules load lazily, so ``sigmoid_top_routing_b200.inputs`` (the seeded
workload generator) imports without torch or the built library.
"""
import importlib

__all__ = ["api", "abi", "inputs", "build"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f".{name}", __name__)
    api = importlib.import_module(".api", __name__)
    if hasattr(api, name):
        return getattr(api, name)
    raise AttributeError(name)
