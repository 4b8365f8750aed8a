"""B200 (sm_100a) implementation of the SpectralQuant compressed-KV hot path.

The work runs in libsq (CUDA, C ABI in include/sq.h); ``sq`` is its Python
binding under the same names. Build the library with ``build.build()``.
"""

from . import sq  # noqa: F401
