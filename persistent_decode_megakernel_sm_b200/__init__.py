"""B200 persistent decode megakernel: a C-ABI CUDA library (libmk.so) and its
thin Python binding.  See include/mk.h for the ABI."""
from . import mk  # noqa: F401  (fails loudly if libmk.so is missing)
from .runtime import Megakernel, KVCache, desc_from  # noqa: F401
