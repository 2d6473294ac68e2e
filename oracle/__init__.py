"""fp64 CPU oracle (test infrastructure only; see oracle.py)."""
from .oracle import build, forward, chunkwise, max_threads, rel_err, DIRECTIONS  # noqa: F401
