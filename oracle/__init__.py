"""fp64 CPU oracle for the absorbed MLA path — test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference legs of
``bench.py`` import this package.  The library never does, and the oracle imports nothing from
the library: the two share only the seeded input generator (``mla_synth``).
"""
from .mla_oracle import *  # noqa: F401,F403
from .mla_oracle import __all__  # noqa: F401
