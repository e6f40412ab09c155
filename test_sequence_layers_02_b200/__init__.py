"""B200-native TTT-Linear inner-loop scan.

The scan runs in hand-written sm_100a CUDA kernels behind the C-ABI library
``libttt_scan.so`` (declared in ``include/ttt_scan.h``); ``ttt_scan`` is the thin
ctypes binding. Importing the package does not load the library; the first call
into ``ttt_scan`` does, and fails loudly if it is missing.
"""
