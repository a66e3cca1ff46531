"""SPTS (Self-Predictive Token Skipping) prefill hot path for NVIDIA B200.

The product is the C-ABI library ``libspts.so`` (declared in
``include/spts.h``) built from ``csrc/`` for sm_100a.  This package holds its
build script and a thin ctypes binding whose functions carry the same names
as the C entry points.  PyTorch is used only for device memory and streams.
"""

from ._lib import *  # noqa: F401,F403
from ._lib import lib, SptsError, version  # noqa: F401
