"""CPU oracle of the MoE layer forward.  Test infrastructure only: imported by
tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference legs,
never by the library."""
from . import moe_oracle  # noqa: F401
