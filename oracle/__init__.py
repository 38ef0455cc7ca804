"""CPU oracle for the Elastic Attention prefill path (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA path.
"""
from .ea_oracle import *  # noqa: F401,F403
from .ea_oracle import __all__  # noqa: F401
