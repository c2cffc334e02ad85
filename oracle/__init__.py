"""Float64 CPU oracle of the Titans memory write-and-read (test infrastructure).

Only tests/, the smoke check and bench.py's CPU-baseline leg may import this
package. The CUDA library never does.
"""
from .oracle import run, run_workload, surprise, use_library, DT_F64, DT_F32, DT_BF16  # noqa: F401
