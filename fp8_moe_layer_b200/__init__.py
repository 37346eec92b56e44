"""B200-native FP8 (W8A8 e4m3) MoE layer forward: router, top-k, permutation, grouped expert
FFN and weighted combine, as hand-written sm_100a CUDA kernels behind a small C ABI.

``fp8_moe_layer_b200.ops`` is the Python binding of that C ABI (it loads the compiled library
and raises if it is missing); ``fp8_moe_layer_b200.inputs`` draws seeded synthetic layers.
The binding is imported on first use so that the input generator works without a GPU build.
"""

__all__ = ["ops", "inputs"]


def __getattr__(name):
    if name in __all__:
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
