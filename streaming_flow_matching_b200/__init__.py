"""Performer next-unit flow-matching denoise step on B200: Python binding of libsfm.

Importing this package loads libsfm.so (built in-tree by
``python streaming_flow_matching_b200/build.py``) and fails if it is missing.
"""
from . import _lib
from ._lib import SfmError, lib  # noqa: F401
from .performer import Performer, attention, attention_workspace_bytes, euler_update, linear  # noqa: F401

__all__ = ["Performer", "attention", "attention_workspace_bytes", "euler_update", "linear", "SfmError",
           "lib"]
