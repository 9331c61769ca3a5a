"""Plain fp64 CPU oracle for pooled block-sparse video attention.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package smoke check and the
benchmark's CPU-baseline leg may import this package.  The CUDA library never
calls into it and it shares no code with the CUDA library.
"""
from .vsa_oracle import *  # noqa: F401,F403
from .cluster_oracle import *  # noqa: F401,F403
from .rectify_oracle import *  # noqa: F401,F403
