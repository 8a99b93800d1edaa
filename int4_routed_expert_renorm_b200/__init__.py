"""B200-native routed-expert MoE step: Route -> Union -> int4 SwiGLU expert FFN -> combine.

The compute path is the C-ABI library ``libcolimoe.so`` (``include/coli_moe.h``,
CUDA kernels for sm_100a in ``csrc/``); ``_lib`` is its ctypes binding and
``layer`` a small holder for one layer's device tensors; ``ep`` runs a layer's
experts spread over several GPUs (expert parallelism); ``tier`` keeps a
layer's routed experts in host memory with a device cache of them.  The library is loaded
on first use of any binding name; if it has not been built
(``python -m int4_routed_expert_renorm_b200.build``) that first use raises
ImportError.  There is no fallback path.
"""
import importlib

_LAZY = {"layer": ("MoELayer", "dims_for"),
         "ep": ("ExpertParallelLayer", "expert_range", "local_tensors", "allreduce_partial"),
         "tier": ("TieredLayer",)}


def __getattr__(name):
    if name.startswith("__"):
        raise AttributeError(name)
    if name in ("_lib", "layer", "build", "ep", "tier"):
        return importlib.import_module(f".{name}", __name__)
    for mod, names in _LAZY.items():
        if name in names:
            return getattr(importlib.import_module(f".{mod}", __name__), name)
    lib = importlib.import_module("._lib", __name__)
    if hasattr(lib, name):
        return getattr(lib, name)
    raise AttributeError(name)
