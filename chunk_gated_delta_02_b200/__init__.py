"""B200-native CARVE chunk-parallel recurrent core.

The compute lives in ``libcarve.so`` (hand-written sm_100a CUDA behind a
C ABI declared in ``include/carve.h``); ``carve`` is a thin ctypes binding
that only marshals torch CUDA tensors into that ABI.  There is no CPU
fallback: calling the op without the built library, or with CPU tensors,
raises.

    from chunk_gated_delta_02_b200 import carve
    o, S_T, m_T, ws = carve.chunk_fwd(q, k, v, g, bx, w, u_down, u_up, L=64)
"""

__all__ = ["carve", "inputs"]


def __getattr__(name):
    if name in __all__:
        import importlib
        return importlib.import_module("." + name, __name__)
    raise AttributeError(name)
