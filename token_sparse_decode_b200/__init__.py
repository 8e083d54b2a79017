"""B200-native token-sparse decode step (sm_100a CUDA kernels behind a C ABI).

The compute path lives in ``libaoh.so`` (built from ``csrc/`` by ``build.py``);
``binding`` marshals torch tensors into its C entry points and ``step`` composes
them into whole decode steps.  Importing ``binding`` or ``step`` does not load
the library; the first call does, and fails if it has not been built.
"""

from . import binding  # noqa: F401
from .binding import AohError, ROLE_DENSE, ROLE_SPARSE, ROLE_STREAM  # noqa: F401
