"""B200-native FlashLoop decode path: cross-loop INT4 KV cache and loop-aware sparse attention.

The compute lives in ``libflashloop_b200.so`` (hand-written sm_100a kernels behind a
C ABI declared in ``include/flashloop.h``).  ``abi`` is the thin ctypes binding with
the same entry-point names; importing it loads the library and raises if it is
missing.  ``bytemodel`` and ``cache`` are host-side helpers that need no GPU.
"""
_ABI_NAMES = None


def __getattr__(name):
    if name.startswith("fl_") or name in ("FlashLoopError", "Dims", "lib"):
        from . import abi
        return getattr(abi, name)
    raise AttributeError(name)
