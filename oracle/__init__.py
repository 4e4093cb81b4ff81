"""CPU oracle of the CSA / HCA layer (plain C, double precision) with a numpy front end.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may use it; the CUDA product path never does.
See ``csa_oracle.h`` for each definition and the page it follows.
"""
from .oracle import *  # noqa: F401,F403
from .oracle import __all__  # noqa: F401
