"""MFA decode attention and the MFA low-rank query projection on B200 (sm_100a).

The compute runs in the hand-written CUDA kernels of ``libmfa.so`` (a C-ABI
library, see ``include/mfa.h``); this package only marshals arguments to it.
"""
from . import inputs  # noqa: F401

__all__ = ["inputs"]
