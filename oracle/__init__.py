"""CPU oracle (test infrastructure only): a plain fp64 statement of the sparse
MoE FFN layer forward pass.  Imported only by the tests, the smoke check and
the CPU-baseline leg of the benchmark; never by the product path."""

from .moe_oracle import *  # noqa: F401,F403
from . import moe_oracle  # noqa: F401
