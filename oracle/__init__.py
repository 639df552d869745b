"""mHC CPU oracle (fp64). TEST INFRASTRUCTURE ONLY.

Only tests/, the package smoke check and bench.py's cpu_baseline leg (and its ``--impl reference``
arm) import this package. The CUDA library never does, and the two share no code: the only module
both sides use is the seeded input generator, which holds none of the method's arithmetic.

Two independent restatements live here:

* ``c_oracle``  -- plain C loops (``mhc_oracle.c``), built with ``gcc -O2 -fopenmp`` without
  fast-math; the one the parity tests and the CPU baseline use.
* ``numpy_ref`` -- the same definitions written separately with NumPy, used to cross-check the C
  code on tiny inputs.
"""

from .c_oracle import (  # noqa: F401
    build,
    bf16_bits_to_f64,
    round_bf16,
    norm_project,
    sinkhorn,
    sinkhorn_converge,
    sinkhorn_variant,
    coefficients,
    aggregate,
    pre,
    post,
    threads,
    set_threads,
)
from .big_fuse import big_fuse, big_fuse_with_prenorm, sum_of_squares  # noqa: F401
from . import boundary  # noqa: F401
from . import backward  # noqa: F401
