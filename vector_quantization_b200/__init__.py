"""B200-native rotation + Lloyd-Max + QJL vector codec (TurboQuant-style).

The compute path is ``libtq.so`` (hand-written sm_100a CUDA kernels behind the
C ABI of ``include/tq.h``); :mod:`vector_quantization_b200.tq` is its ctypes
binding and raises on import if the library is missing.  Attributes of this
package resolve lazily so that ``python -m vector_quantization_b200.build``
can run before the library exists.
"""
_EXPORTS = ("Rotation", "TQError", "alloc_workspace", "decode_attention", "decode_workspace_size",
            "empty_records", "lloyd_max", "quantize_kv", "version", "profile_next_decode",
            "encoder_attention", "quantize_dense", "search_topk", "search_workspace_size")


def __getattr__(name):
    import importlib
    if name == "tq":
        return importlib.import_module(__name__ + ".tq")
    if name in _EXPORTS:
        return getattr(importlib.import_module(__name__ + ".tq"), name)
    raise AttributeError(name)


__all__ = ["tq", *_EXPORTS]
