"""LSCD SpMM for B200: Tiled-CSL encoder and C = A x B on sm_100a tensor cores.

Thin Python binding over the C-ABI library ``libflashspmm.so`` (declared in
``include/flashspmm.h``).  Every step of the path runs in the library's CUDA
kernels; this package only marshals torch tensors (device memory) and CUDA
streams into the C calls.  There is no CPU fallback: if the library or a CUDA
device is missing, the calls raise.
"""
from .binding import (TCSL, FlashSpmmError, check_device_status, launch_count, load_library,  # noqa: F401
                      partition_host, partition_pieces, predict_us, prefer_sparse, spmm_lscd, spmm_lscd_host,
                      spmm_lscd_noalloc, spmm_workspace_bytes, tcsl_encode, tcsl_validate)
