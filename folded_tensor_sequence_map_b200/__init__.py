"""Folded Tensor-Sequence-Parallel (TSP) decoder layer on one B200 (sm_100a).

The library ``libtsp.so`` (C ABI in ``include/tsp.h``) holds every kernel;
``tsp`` is its thin ctypes binding and ``layer`` a small convenience wrapper
that allocates the caller-owned buffers with PyTorch.
"""

from .tsp import *  # noqa: F401,F403
from .tsp import EXPORTED, LIB_PATH, Plan, TSPError  # noqa: F401
