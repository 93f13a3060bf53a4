"""B200-native Mamba-3 SISO selective scan: Python binding of ``libm3ssd``.

The binding only marshals arguments (device pointers, sizes, the current CUDA
stream) into the C-ABI of ``libm3ssd.so``; every step of the scan runs in the
library's CUDA kernels.  Importing this package does not load the library; the
first call does, and it raises if the library is missing.
"""
