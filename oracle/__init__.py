"""CPU oracle for Jensen-bias-corrected attention over a low-bit KV cache.

TEST INFRASTRUCTURE ONLY. This package is the plain, slow, obviously correct
restatement of the method that the CUDA path is checked against. Only the test
suite, the smoke check of the package entry file and the CPU-baseline /
reference arm of the benchmark may import it. The product path (the C-ABI
library and its Python binding) never imports, calls or links it, and shares no
code with it; the only module both sides use is the seeded input generator,
which holds none of the method's arithmetic.
"""
from .qkv_oracle import *  # noqa: F401,F403
