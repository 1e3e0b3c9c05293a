"""fp64 CPU oracle of the DSpark draft round -- test infrastructure only.

Imported by ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline leg, never by the library. See ``oracle/dspark.py``.
"""
from . import dspark  # noqa: F401
