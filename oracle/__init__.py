"""CPU oracles of the FP8 MoE-layer forward (FP64): moe.py (numpy) and
moe_oracle.cpp (plain C++ loops, E4M3 through a 256-entry table, std::thread
over row chunks; wrapped by cpp.py under the same function names).

TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and bench.py's CPU
baseline (and its --impl reference arm) may import this package. The product
path never imports it, and it shares no code with the CUDA library: no
kernels, headers, helpers, tables or constant generators. The seeded input
generator (gen/) is the one module both sides use, and it holds none of the
layer's forward arithmetic.

Every function of both is pinned by the `-m "not gpu"` tests against closed
forms, brute force or library routines (tests/test_oracle_*.py runs each
pin on both), and the two are checked against each other
(tests/test_oracle_cpp.py); the
final FP32 accumulation order of the kernels is not reproduced, so output
parity beyond the stated tolerance is unpinned.
"""
from . import e4m3, moe  # noqa: F401
