"""B200-native ParaRNN hot path: Newton iterations with a parallel scan over time.

The compute lives in ``libpararnn_b200.so`` (hand-written CUDA for sm_100a,
C-ABI declared in ``include/pararnn_b200.h``); :mod:`.binding` is the thin
ctypes layer with the same entry-point names, and :mod:`.workloads` draws the
seeded synthetic inputs.
"""
