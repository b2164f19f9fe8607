"""CPU float64 oracle for the differential-attention forward (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline arm of
``bench.py`` may import this package; the library never does.
"""
