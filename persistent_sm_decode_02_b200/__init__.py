"""Batch-1 persistent decode step for B200 (sm_100a): Python binding of the C ABI in include/dec.h.

Argument marshalling only: every step of the decode path runs in the CUDA
kernels of libdec.so.  Importing this package loads the library and fails
loudly if it has not been built (there is no CPU fallback).
"""
from .dec import *  # noqa: F401,F403
from .dec import LIB_PATH, DecError, Decoder, config_from_workload, load_library  # noqa: F401
