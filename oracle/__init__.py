"""Plain fp64 CPU oracle for the Medusa draft-and-verify step.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check in
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import this
package.  The product path (the CUDA library and its Python binding) never
imports it and has no CPU fallback.
"""
from .medusa_oracle import *  # noqa: F401,F403
