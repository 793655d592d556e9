"""B200-native sparse decode step of RTPurbo-style per-head sparse attention.

The compute path is the C-ABI library ``librtp.so`` (hand-written CUDA for
sm_100a, built from ``csrc/``); ``ops`` is its thin Python binding.
"""
