"""Megatron-LM tensor-parallel Transformer layer on one B200 (sm_100a).

The C-ABI library ``libtp.so`` (hand-written CUDA kernels) does the work;
``tensor_transformer_layer_linear_b200.tp`` is its thin ctypes binding and
raises at import when the library has not been built. ``synth`` draws the
seeded synthetic inputs and needs no GPU.
"""
import importlib

__all__ = ["tp", "synth"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
