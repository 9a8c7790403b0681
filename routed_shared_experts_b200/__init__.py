"""B200 (sm_100a) forward pass of a routed + shared-expert MoE layer.

The compute lives in ``libmoe_b200.so`` (hand-written CUDA, C ABI declared in
``include/moe_b200.h``). ``routed_shared_experts_b200.capi`` marshals torch
tensors into that ABI; ``routed_shared_experts_b200.layer`` composes the five
calls into one layer forward (shared expert on a side stream). The library is
loaded on first use, and a missing or unbuilt library is an error: there is no
fallback path.
"""
__all__ = ["configs", "synth", "capi", "layer"]


def __getattr__(name):
    if name in ("capi", "layer"):
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
