"""Float64 CPU oracle for the SLA / SLA2 forward pass (test infrastructure only).

Imported only by tests/, __graft_entry__.smoke() and bench.py's CPU-baseline
and reference legs. It shares no code with the CUDA library or its binding.
"""
from .sla_oracle import *  # noqa: F401,F403
