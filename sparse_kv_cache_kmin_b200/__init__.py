"""Query-aware sparse decode attention over a paged KV cache, for NVIDIA B200 (sm_100a).

The CUDA library libekv.so (C ABI in include/ekv.h) does all of the work; this package is
its thin ctypes binding (``ekv``), a convenience decoder that strings the four calls of one
decode step together (``decoder``), seeded synthetic workloads (``workloads``) and the build
script (``build``). Nothing falls back to a CPU path: without the library, calls raise.
"""
from .ekv import (ALPHA, EKV_BF16, EKV_DEV_BAD_BLOCK, EKV_DEV_BAD_LEN, EKV_DEV_BAD_RANGE,
                  EKV_DEV_BAD_SEL, EKV_DEV_SEL_OVERFLOW, EKV_ENTMAX15, EKV_ERR_CUDA,
                  EKV_ERR_DEVICE, EKV_ERR_INVALID_ARG, EKV_ERR_UNSUPPORTED, EKV_ERR_WORKSPACE,
                  EKV_F32, EKV_OK, EKV_SEL_GAUSS, EKV_SEL_GAUSS_MAX, EKV_SEL_TOPK, EKV_SOFTMAX, EKV_SPARSEMAX,
                  EkvError, PagedKVCache, ekv_clear_device_status, ekv_decode_workspace_bytes,
                  ekv_device_status, ekv_page_meta_update, ekv_score_pages, ekv_select_pages,
                  ekv_sparse_decode, load_library)
from .decoder import SparseDecoder

__all__ = [n for n in dir() if not n.startswith("_")]
