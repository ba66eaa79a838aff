"""B200-native heterogeneous-batch LoRA adapter branch.

The compute lives in liblora.so (CUDA, sm_100a) behind the C ABI of
include/lora.h; this package only marshals torch tensors into those calls.
"""
from . import _binding
from ._binding import *  # noqa: F401,F403
from .layer import AdapterCache, AdapterLayer, AdapterPrefetcher, PrefetchTicket, apply_multi  # noqa: F401
from . import tp  # noqa: F401
