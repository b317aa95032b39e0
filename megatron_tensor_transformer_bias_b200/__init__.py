"""libtpblock: the Megatron column->row tensor-parallel transformer block on one B200.

The compute path is the C-ABI shared library ``libtpblock.so`` (hand-written
CUDA for sm_100a) declared in ``include/tpblock.h``; ``tpblock`` is its thin
ctypes binding.  Importing this package does not load the library; the
binding loads it on first use and raises if it is missing.
"""
