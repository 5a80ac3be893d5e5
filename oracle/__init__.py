"""CPU fp64 oracle for CoWA attention — test infrastructure only.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline and
reference legs may import this package; the library never does.
"""

from .cowa_oracle import *  # noqa: F401,F403
from .cowa_oracle import __all__  # noqa: F401
