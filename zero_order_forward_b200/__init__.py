"""zero_order_forward_b200: the 1SPSA / 1.5-SPSA zero-order training hot path on B200.

The product is libzo.so (hand-written sm_100a CUDA kernels behind the C ABI declared in
include/zo.h).  This package is its thin Python binding: same names, argument
marshalling only.  Importing it fails loudly if libzo.so has not been built.
"""
from ._lib import *  # noqa: F401,F403
from ._lib import Ctx, ZoError, lib, LIB_PATH  # noqa: F401
