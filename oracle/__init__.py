"""CPU oracle of the per-frame decode step -- TEST INFRASTRUCTURE.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may
import this package.  The product library never does and shares no code
with it.
"""
