"""fp64 CPU oracle for R-SWA.  Test infrastructure only (tests, smoke check,
CPU baseline of the benchmark); never imported by the product path."""

from .rswa_oracle import *  # noqa: F401,F403
from .rswa_oracle import decode_step_full  # noqa: F401
