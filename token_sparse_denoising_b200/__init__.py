"""B200-native hot path of Heterogeneous Step Allocation (HSA) for video DiTs.

`hsa` is the ctypes binding of libhsa.so (include/hsa.h); `synthetic` draws the
seeded inputs.  Importing the package loads nothing; `hsa.load()` does.
"""
