"""Folded Tensor-Sequence-Parallel (TSP) decoder layer on one B200 (sm_100a).

The library ``libtsp.so`` (C ABI in ``include/tsp.h``) holds every kernel;
``folded_tensor_sequence_map_b200.tsp`` is its thin ctypes binding, and its
names are re-exported here.  The binding is loaded on first attribute access
(so that ``folded_tensor_sequence_map_b200.build`` can run before the library
exists); a missing or unloadable library raises ImportError there.
"""


import importlib


def __getattr__(name):
    if name.startswith("__"):
        raise AttributeError(name)
    _tsp = importlib.import_module(__name__ + ".tsp")
    try:
        return getattr(_tsp, name)
    except AttributeError:
        raise AttributeError(f"module {__name__!r} has no attribute {name!r}") from None
