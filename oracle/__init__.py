"""CPU oracle for the recurrent-state step (test infrastructure only).

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may import this
package.  The product library neither imports nor links it.
"""
from .oracle import *  # noqa: F401,F403
from .oracle import RULES, DTYPES  # noqa: F401
