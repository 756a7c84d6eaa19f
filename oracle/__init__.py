"""fp64 CPU oracle for the GALE 1-bit expert path (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  See ``gale_oracle`` for the
definitions and the readings it takes.
"""
from .gale_oracle import *  # noqa: F401,F403
from . import gale_oracle  # noqa: F401
from .w4_oracle import *  # noqa: F401,F403,E402
from . import w4_oracle  # noqa: F401,E402
from . import encoder_oracle  # noqa: F401,E402
