"""B200-native one-forward tree verification (JetSpec's verify step).

The compute lives in ``libjsv.so`` (hand-written CUDA for sm_100a behind a
C ABI, declared in ``include/jsv.h``).  ``tree_verification_jsv_b200.jsv``
is the thin ctypes binding; ``synth`` builds seeded synthetic workloads.
Importing the package loads nothing; the binding loads the library on first
use and raises if it is missing.
"""
__version__ = "0.1.0"
