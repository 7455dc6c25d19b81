"""CPU oracle of the FLUX.2-klein transformer forward (test infrastructure only).

Only tests, ``__graft_entry__.smoke()`` and the CPU-baseline legs of ``bench.py``
may import this package; the CUDA product path never does.
"""
from . import flux_oracle
