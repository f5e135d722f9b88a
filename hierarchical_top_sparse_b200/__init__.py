"""Log-linear Sparse Attention (LLSA) on B200 (sm_100a).

The product is libllsa.so, a C-ABI library of hand-written CUDA kernels
(include/llsa.h); ``llsa`` is its thin Python binding.  Importing this
package does not load the library; the first call does, and fails loudly if
it has not been built.
"""
from . import llsa  # noqa: F401
from .llsa import BF16, FP32, LLSAError, Pipeline, Problem  # noqa: F401
