"""Plain fp64 CPU oracle for chunk-causal block-sparse attention (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA library.
"""
from .uf_oracle import *  # noqa: F401,F403
from .uf_oracle import __all__  # noqa: F401
