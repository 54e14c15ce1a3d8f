"""B200-native (sm_100a) Clebsch-Gordan tensor-product convolution.

The compute lives in libcgtp.so (C ABI in include/cgtp.h); ``api`` is the
torch binding, ``synthetic`` draws the seeded benchmark workloads.  Nothing
here falls back to a CPU implementation: without the built library every
entry point raises.
"""
from ._lib import CGTPError, LIB_PATH, lib  # noqa: F401

__all__ = ["CGTPError", "LIB_PATH", "lib"]
