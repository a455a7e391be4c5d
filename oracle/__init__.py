"""CPU fp64 oracle for the Gated DeltaNet chunked-prefill operator.

Test infrastructure only: used by tests/, the smoke check and the benchmark's
CPU-baseline leg, never by the product path. Shares no code with the CUDA
library.
"""
from .gdn_oracle import *  # noqa: F401,F403
