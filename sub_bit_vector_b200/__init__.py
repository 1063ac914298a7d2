"""LoopVQ decode-path library for NVIDIA B200 (sm_100a).

The compute lives in ``libloopvq.so`` (hand-written CUDA, C ABI declared in
``include/loopvq.h``).  ``sub_bit_vector_b200.loopvq`` is the thin ctypes
binding; ``sub_bit_vector_b200.synth`` holds the seeded synthetic inputs.
Nothing is imported eagerly, so ``synth`` can be used without the library.
"""
__all__ = ["loopvq", "synth"]


def __getattr__(name):
    if name in __all__:
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
