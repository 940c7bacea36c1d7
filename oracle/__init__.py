"""Float64 CPU oracle of the GPTQ layer solver — test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference legs may import this package.  It shares no code with the CUDA path.
"""
from . import gptq_ref  # noqa: F401
