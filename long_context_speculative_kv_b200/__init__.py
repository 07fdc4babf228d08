"""Windowed-MTP decode attention for B200 (sm_100a): a C-ABI CUDA library (libwmtp.so) and its
thin Python binding.

The binding only marshals arguments; every step of the path runs in the library's kernels.
Importing the package does not load the library; the first call does, and fails loudly when the
library is missing.
"""
