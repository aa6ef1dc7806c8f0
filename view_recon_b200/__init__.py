"""Dynamic tile-sparse global attention for feed-forward 3-D reconstruction on B200.

The compute lives in libsa.so (C-ABI, include/sa.h); `sa` is its thin binding
and `pipeline` strings the four steps together on torch-managed buffers.
"""
from . import sa  # noqa: F401

__all__ = ["sa"]
