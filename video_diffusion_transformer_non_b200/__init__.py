"""vidattn: segment-masked, non-causal multi-head attention forward for video
diffusion transformers, as hand-written sm_100a CUDA behind a C ABI.

The Python layer only marshals arguments to the shared library
``csrc/libvidattn.so``; every step of the computation runs in its kernels.
"""
from .binding import (  # noqa: F401
    VIDATTN_OK, status_string, vidattn_fwd, vidattn_fwd_host, attention, library_path,
    load_library, exported_symbols,
)
