"""fp64 CPU oracle (test infrastructure only; see oracle.py)."""
from .oracle import (attention, build, hybrid_parallel, hybrid_recurrent, num_threads,  # noqa: F401
                     ring_model, rope, stream)
