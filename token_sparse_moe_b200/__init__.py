"""B200-native TokenMixer-Large forward: a C-ABI CUDA library (libtm.so) and its Python binding.

The library itself lives in libtm.so (include/tm.h); `api` marshals torch tensors
into it.  Importing the package loads the library and fails loudly if it is missing.
"""
from . import _abi
from ._abi import TMError, load

load()

from . import api  # noqa: E402

__all__ = ["api", "load", "TMError"]
