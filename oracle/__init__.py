"""The oracle: a plain float64 CPU restatement of TokenGate's gated prefill.

TEST INFRASTRUCTURE ONLY. The tests, the package's smoke check and the
benchmark's CPU-baseline leg may import it; the CUDA library and its Python
binding never do, and the two share no code.
"""
from .tokengate_oracle import *  # noqa: F401,F403
from . import tokengate_oracle as ref  # noqa: F401
