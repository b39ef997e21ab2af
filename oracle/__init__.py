"""fp64 CPU oracle of the MSA hot path — test infrastructure only.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline /
reference arm may import this package; the product path never does.
"""
from .msa_oracle import *  # noqa: F401,F403
from .msa_backward import *  # noqa: F401,F403
