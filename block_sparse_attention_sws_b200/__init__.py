"""Sketch&Walk sparse attention for B200 (sm_100a): Python binding of libsws.

The computation lives in ``libsws.so`` (CUDA, built by ``build.build()``);
this package only marshals torch tensors into the C ABI of include/sws.h.
"""
from ._lib import *  # noqa: F401,F403
from ._lib import Handle, SwsConfig, SwsError, load, make_config  # noqa: F401
from .pipeline import DecodePath, PrefillBatch, PrefillPath  # noqa: F401
