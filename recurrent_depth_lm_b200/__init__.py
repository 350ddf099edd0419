"""WISE attention hot path on NVIDIA B200 (sm_100a): Python front end of libwise.so.

Importing the package loads the CUDA library; if it is missing the import
fails (there is no CPU fallback).  Build it with `python
recurrent_depth_lm_b200/build.py`.
"""

from ._lib import WiseError, WiseShape, version  # noqa: F401  (loads libwise.so)
from . import ops  # noqa: F401
from .trajectory import WiseTrajectory  # noqa: F401

__all__ = ["ops", "WiseTrajectory", "WiseError", "WiseShape", "version"]
