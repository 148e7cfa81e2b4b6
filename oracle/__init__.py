"""CPU oracle for the latent-KV decode path: test infrastructure only.

Only the tests, the package smoke check and the CPU-baseline leg of the bench
import this package.  The library itself never does.
"""
from .lk_oracle import *  # noqa: F401,F403
