"""Plain, slow fp64 CPU oracle of the folded Tensor-Sequence-Parallel layer.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute anything in this package: only ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.
It shares no code with the CUDA library.
"""

from .tsp_oracle import *  # noqa: F401,F403
from .long_sequence import layer_forward_backward_blocked  # noqa: F401
