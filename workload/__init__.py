"""Seeded synthetic workloads for the LoopKV decode path.

This package only describes shapes and draws random inputs.  It holds none
of the method's arithmetic (no quantisation, no attention), so both the CUDA
path and the CPU oracle may take their inputs from it.
"""

from .configs import WORKLOADS, Workload, get_workload  # noqa: F401
from .gen import (  # noqa: F401
    CELL_KINDS,
    block_table_for,
    cell_kv,
    cell_new_token,
    cell_query,
    make_plan,
    seq_lens_for,
)
