"""fp64 CPU oracle for the routed MoE FFN (test infrastructure only).

Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference
legs may import this package.  It shares no code with expert_decode_b200/.
"""
from .oracle import Oracle, OracleError, load  # noqa: F401
