"""Float64 CPU oracle for the blocked-Shampoo step (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s cpu_baseline /
reference leg may import this package.  The CUDA path never imports it and it
never imports the CUDA path.  See ``oracle/shampoo_oracle.py`` for the
functions, their citations and the list of readings where the pages are silent.
"""
from .shampoo_oracle import *  # noqa: F401,F403
