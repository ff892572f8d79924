"""TurboQuant KV-cache compression and decode attention for NVIDIA B200 (sm_100a).

The compute path is the CUDA library ``libtq.so`` (C ABI in include/tq.h);
``binding`` marshals torch tensors into it. Importing the package requires
the built library: there is no CPU fallback.
"""
from .binding import *  # noqa: F401,F403
from .binding import (Cache, Context, TQError, attend_host, new_cache, new_workspace,  # noqa: F401
                      EXPORTS, LIB_PATH)
