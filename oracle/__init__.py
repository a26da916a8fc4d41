"""fp64 CPU oracle for the NVFP4 GPTQ + Schur Replay layer solve.

Test infrastructure: only the tests, the smoke check and the benchmark's CPU
baseline use it.  It shares no code with the CUDA library."""
from .nvfp4_oracle import *  # noqa: F401,F403
