"""The oracle for the GPTQ solver: test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import this
package.  The CUDA library never calls it, links it or falls back to it.
"""
from .gptq_oracle import *  # noqa: F401,F403
