"""fp64 CPU oracle for Kascade sparse attention (test infrastructure only).

Only tests/, __graft_entry__.smoke() and the CPU-baseline leg of bench.py may
import this package; the product path never does.
"""
from .kascade_oracle import *  # noqa: F401,F403
from .kascade_oracle import __all__  # noqa: F401
