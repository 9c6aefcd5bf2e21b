"""fp64 CPU oracle of the LoRA linear layer (test infrastructure only).

Only the tests, the package's smoke check and the benchmark's CPU-baseline leg may
import this package.  The product path never does.
"""
from .oracle import (  # noqa: F401
    build,
    lib_path,
    threads,
    set_threads,
    weight,
    xa,
    h,
    g,
    dx,
    db,
    da,
    forward,
    backward,
    h_projections,
    dx_projections,
    merged_weight,
    h_dense,
    dx_dense,
)
