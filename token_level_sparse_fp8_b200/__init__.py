"""B200-native (sm_100a) Joint Subspace Sparse Attention decode: CUDA kernels behind the C ABI
of ``libjssa.so`` (``include/jssa.h``) and a thin PyTorch binding (``api``).

Importing the package does not load the library; the first call does, and fails loudly if the
library has not been built (``python -m token_level_sparse_fp8_b200.build``).
"""

from . import _lib  # noqa: F401
from .api import *  # noqa: F401,F403
from .api import __all__  # noqa: F401

LIB_PATH = _lib.LIB_PATH
