"""CPU oracle of the Spark-Attn forward pass.

TEST INFRASTRUCTURE ONLY: tests/, __graft_entry__.smoke() and bench.py's
CPU-baseline and reference legs are its only users. The CUDA library and its
Python binding never import it.

spark_oracle  - the step-by-step float64 statement of every stage.
brute_force   - an independent loop-free statement for N <= 256.

Every function is pinned by tests in tests/test_oracle_*.py against closed
forms, textbook routines, invariants the pages fix and brute force. Parity
unpinned: nothing (the pages' PSNR/VBench figures need model weights and are
out of scope, so they are not oracle functions).
"""

from . import brute_force, spark_oracle  # noqa: F401
