"""ctypes binding of librpk.so (declared in include/rpk.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels. Loading fails loudly when the library has not been built.
"""

from __future__ import annotations

import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "librpk.so")


class RpkError(RuntimeError):
    """A non-zero status from the C ABI."""


_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RpkError(f"librpk.so is not built ({LIB_PATH}); run "
                           "python -m ragged_paged_kv_rope_b200.build")
        _lib = C.CDLL(LIB_PATH)
    return _lib


def rope_qk_paged_ragged(*args, **kwargs):  # pragma: no cover - filled in with the ABI
    raise RpkError("not built")


def ragged_paged_attention(*args, **kwargs):  # pragma: no cover
    raise RpkError("not built")


def ragged_paged_attention_workspace_size(*args, **kwargs):  # pragma: no cover
    raise RpkError("not built")


def freqs_cis(*args, **kwargs):  # pragma: no cover
    raise RpkError("not built")
