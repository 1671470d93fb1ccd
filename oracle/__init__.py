"""fp64 CPU oracle (test infrastructure only; see oracle.py)."""
from .oracle import (attention, build, hybrid2_parallel, hybrid2_recurrent, hybrid_parallel,  # noqa: F401
                     hybrid_recurrent, merge, num_threads, ring_model, rope, stream)
