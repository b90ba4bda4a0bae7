"""CPU oracle for NVFP4 sparse MLA decode -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never imports it and
shares no code with it.
"""
from .oracle import *  # noqa: F401,F403
from . import indexer  # noqa: F401,E402
from . import blhnc  # noqa: F401,E402
