"""CPU oracle for the block-quantized projection path.

TEST INFRASTRUCTURE ONLY: imported by the test suite, the smoke check and the
benchmark's CPU-baseline leg, never by the product library.  The arithmetic
lives in plain C (``dsqref.c``); this module builds it with gcc and exposes
numpy-friendly wrappers.
"""
from .dsqref import *  # noqa: F401,F403
from .dsqref import build, lib  # noqa: F401
