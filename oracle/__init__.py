"""CPU oracle for the PSA forward path (test infrastructure only).

Only the tests, the smoke check and the benchmark's CPU-baseline legs may
import this package; the product path never does.
"""
from .psa_oracle import *  # noqa: F401,F403
from .psa_oracle import SKIP, LN2  # noqa: F401
