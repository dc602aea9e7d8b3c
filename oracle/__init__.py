"""CPU oracle of the decode step (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this package. The engine (``bandwidth_bound_stream_b200``) never does.
"""
from .oracle import OracleModel, lib  # noqa: F401
