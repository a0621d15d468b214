"""Thin Python binding of libekv (include/ekv.h): argument marshalling only.

Every function here has the name of the C entry point it calls and does nothing but check
tensor placement, build the plain-data ``ekv_cache`` struct and pass raw device pointers and
the current CUDA stream. All of the work runs in the CUDA kernels of libekv.so; if the
library is missing, loading it raises.

Tensors (all on one CUDA device, contiguous):
  k_cache, v_cache  [num_blocks, H_kv, P, d]   float32 or bfloat16
  meta_bbox         [num_blocks, H_kv, 2, d]   same dtype (row 0 kmin, row 1 kmax)
  meta_mom          [num_blocks, H_kv, 2, d]   float32 (mean, variance) or None
  page_table        [B, max_pages] int32;  seq_lens [B] int32;  dev_status [1] int32
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

from .build import LIB_PATH

EKV_OK, EKV_ERR_INVALID_ARG, EKV_ERR_UNSUPPORTED, EKV_ERR_WORKSPACE, EKV_ERR_CUDA, EKV_ERR_DEVICE = range(6)
EKV_F32, EKV_BF16 = 0, 1
EKV_SOFTMAX, EKV_ENTMAX15, EKV_SPARSEMAX = 0, 1, 2
EKV_SEL_TOPK, EKV_SEL_GAUSS, EKV_SEL_GAUSS_MAX = 0, 1, 2
EKV_DEV_BAD_BLOCK, EKV_DEV_BAD_LEN, EKV_DEV_BAD_SEL, EKV_DEV_SEL_OVERFLOW, EKV_DEV_BAD_RANGE = \
    0x1, 0x2, 0x4, 0x8, 0x10
EKV_DEV_TIMEOUT = 0x20
ALPHA = {EKV_SOFTMAX: 1.0, EKV_ENTMAX15: 1.5, EKV_SPARSEMAX: 2.0}

EXPORTED = ["ekv_page_meta_update", "ekv_score_pages", "ekv_select_pages", "ekv_sparse_decode",
            "ekv_decode_workspace_bytes", "ekv_device_status", "ekv_clear_device_status",
            "ekv_status_str"]


class EkvError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s failed: %s" % (where, status_str(status)))


class EkvCacheStruct(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("num_blocks", ctypes.c_int32), ("batch", ctypes.c_int32),
                ("max_pages", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("k_cache", ctypes.c_void_p), ("v_cache", ctypes.c_void_p),
                ("meta_bbox", ctypes.c_void_p), ("meta_mom", ctypes.c_void_p),
                ("page_table", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p),
                ("dev_status", ctypes.c_void_p)]


_lib = None


def load_library(path: Optional[str] = None):
    """Load libekv.so (raises if it has not been built)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise RuntimeError("libekv.so not found at %s; build it with "
                           "`python -m sparse_kv_cache_kmin_b200.build`" % path)
    lib = ctypes.CDLL(path)
    P, I32, U64, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t, ctypes.c_float
    cp = ctypes.POINTER(EkvCacheStruct)
    sig = {
        "ekv_page_meta_update": ([cp, P, P, I32, P], ctypes.c_int),
        "ekv_score_pages": ([cp, P, I32, F, I32, P, P], ctypes.c_int),
        "ekv_select_pages": ([cp, I32, I32, I32, F, F, P, P, P, I32, P, P], ctypes.c_int),
        "ekv_sparse_decode": ([cp, P, I32, F, I32, P, P, I32, P, P, P, U64, P], ctypes.c_int),
        "ekv_decode_workspace_bytes": ([cp, I32, I32], U64),
        "ekv_device_status": ([cp, ctypes.POINTER(ctypes.c_uint32), P], ctypes.c_int),
        "ekv_clear_device_status": ([cp, P], ctypes.c_int),
        "ekv_status_str": ([ctypes.c_int], ctypes.c_char_p),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes, fn.restype = args, res
    if path == LIB_PATH:
        _lib = lib
    return lib


def status_str(status: int) -> str:
    try:
        return load_library().ekv_status_str(status).decode()
    except Exception:
        return "status %d" % status


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(status: int, where: str):
    if status != EKV_OK:
        raise EkvError(status, where)


@dataclass
class PagedKVCache:
    """Caller-owned device buffers of a paged KV cache and its page metadata."""
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    meta_bbox: torch.Tensor
    meta_mom: Optional[torch.Tensor]
    page_table: torch.Tensor
    seq_lens: torch.Tensor
    dev_status: torch.Tensor

    @staticmethod
    def allocate(num_blocks: int, num_kv_heads: int, page_size: int, head_dim: int,
                 batch: int, max_pages: int, dtype=torch.bfloat16, device="cuda",
                 gaussian: bool = True) -> "PagedKVCache":
        shape = (num_blocks, num_kv_heads, page_size, head_dim)
        mshape = (num_blocks, num_kv_heads, 2, head_dim)
        return PagedKVCache(
            k_cache=torch.zeros(shape, dtype=dtype, device=device),
            v_cache=torch.zeros(shape, dtype=dtype, device=device),
            meta_bbox=torch.zeros(mshape, dtype=dtype, device=device),
            meta_mom=torch.zeros(mshape, dtype=torch.float32, device=device) if gaussian else None,
            page_table=torch.zeros((batch, max_pages), dtype=torch.int32, device=device),
            seq_lens=torch.zeros((batch,), dtype=torch.int32, device=device),
            dev_status=torch.zeros((1,), dtype=torch.int32, device=device))

    @property
    def num_kv_heads(self) -> int:
        return self.k_cache.shape[1]

    @property
    def page_size(self) -> int:
        return self.k_cache.shape[2]

    @property
    def head_dim(self) -> int:
        return self.k_cache.shape[3]

    @property
    def batch(self) -> int:
        return self.page_table.shape[0]

    @property
    def max_pages(self) -> int:
        return self.page_table.shape[1]

    def struct(self) -> EkvCacheStruct:
        """The C view of the cache; rebuilt only when a tensor of it is replaced."""
        key = tuple((t.data_ptr(), tuple(t.shape), t.dtype) if t is not None else None
                    for t in (self.k_cache, self.v_cache, self.meta_bbox, self.meta_mom,
                              self.page_table, self.seq_lens, self.dev_status))
        cached = self.__dict__.get("_struct_cache")
        if cached is not None and cached[0] == key:
            return cached[1]
        s = self._build_struct()
        self.__dict__["_struct_cache"] = (key, s)
        return s

    def _build_struct(self) -> EkvCacheStruct:
        if self.k_cache.dtype == torch.float32:
            dt = EKV_F32
        elif self.k_cache.dtype == torch.bfloat16:
            dt = EKV_BF16
        else:
            raise ValueError("K/V cache dtype must be float32 or bfloat16")
        for name in ("v_cache", "meta_bbox"):
            if getattr(self, name).dtype != self.k_cache.dtype:
                raise ValueError("%s must have the K cache dtype" % name)
        if self.meta_mom is not None and self.meta_mom.dtype != torch.float32:
            raise ValueError("meta_mom must be float32")
        for name in ("page_table", "seq_lens", "dev_status"):
            if getattr(self, name).dtype != torch.int32:
                raise ValueError("%s must be int32" % name)
        s = EkvCacheStruct()
        s.dtype = dt
        s.num_blocks, s.num_kv_heads, s.page_size, s.head_dim = self.k_cache.shape
        s.batch, s.max_pages = self.page_table.shape
        s.reserved = 0
        s.k_cache = _ptr(self.k_cache)
        s.v_cache = _ptr(self.v_cache)
        s.meta_bbox = _ptr(self.meta_bbox)
        s.meta_mom = _ptr(self.meta_mom)
        s.page_table = _ptr(self.page_table)
        s.seq_lens = _ptr(self.seq_lens)
        s.dev_status = _ptr(self.dev_status)
        return s


def ekv_page_meta_update(cache: PagedKVCache, new_start: torch.Tensor, new_count: torch.Tensor,
                         max_new: int, stream=None):
    c = cache.struct()
    _check(load_library().ekv_page_meta_update(ctypes.byref(c), _ptr(new_start), _ptr(new_count),
                                               int(max_new), _stream(stream)),
           "ekv_page_meta_update")


def ekv_score_pages(cache: PagedKVCache, q: torch.Tensor, num_q_heads: int, scale: float,
                    policy: int, scores: torch.Tensor, stream=None):
    c = cache.struct()
    _check(load_library().ekv_score_pages(ctypes.byref(c), _ptr(q), int(num_q_heads),
                                          float(scale), int(policy), _ptr(scores),
                                          _stream(stream)), "ekv_score_pages")


def ekv_refresh_score_pages(cache: PagedKVCache, new_start: torch.Tensor, new_count: torch.Tensor,
                            max_new: int, q: torch.Tensor, num_q_heads: int, scale: float,
                            policy: int, scores: torch.Tensor, stream=None):
    """ekv_page_meta_update followed by ekv_score_pages, in one call (one kernel for a short
    top-k append over few (sequence, KV head) pairs), with the two calls' results bit for bit."""
    P, I32, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float
    fn = _moment_fn("ekv_refresh_score_pages", [ctypes.POINTER(EkvCacheStruct), P, P, I32, P, I32,
                                                F, I32, P, P])
    c = cache.struct()
    _check(fn(ctypes.byref(c), _ptr(new_start), _ptr(new_count), int(max_new), _ptr(q),
              int(num_q_heads), float(scale), int(policy), _ptr(scores), _stream(stream)),
           "ekv_refresh_score_pages")


def ekv_select_pages(cache: PagedKVCache, num_q_heads: int, policy: int, topk: int, alpha: float,
                     delta: float, scores: torch.Tensor, sel_idx: torch.Tensor,
                     sel_count: torch.Tensor, max_sel: int, tau_hat: Optional[torch.Tensor],
                     stream=None):
    c = cache.struct()
    _check(load_library().ekv_select_pages(ctypes.byref(c), int(num_q_heads), int(policy),
                                           int(topk), float(alpha), float(delta), _ptr(scores),
                                           _ptr(sel_idx), _ptr(sel_count), int(max_sel),
                                           _ptr(tau_hat), _stream(stream)), "ekv_select_pages")


def ekv_sparse_decode(cache: PagedKVCache, q: torch.Tensor, num_q_heads: int, scale: float,
                      attn: int, sel_idx: torch.Tensor, sel_count: torch.Tensor, max_sel: int,
                      out: torch.Tensor, stat: torch.Tensor, ws: torch.Tensor, stream=None):
    c = cache.struct()
    _check(load_library().ekv_sparse_decode(ctypes.byref(c), _ptr(q), int(num_q_heads),
                                            float(scale), int(attn), _ptr(sel_idx),
                                            _ptr(sel_count), int(max_sel), _ptr(out), _ptr(stat),
                                            _ptr(ws), ws.numel() * ws.element_size(),
                                            _stream(stream)), "ekv_sparse_decode")


def ekv_select_decode(cache: PagedKVCache, q: torch.Tensor, num_q_heads: int, scale: float,
                      attn: int, topk: int, scores: torch.Tensor, sel_idx: torch.Tensor,
                      sel_count: torch.Tensor, max_sel: int, out: torch.Tensor, stat: torch.Tensor,
                      ws: torch.Tensor, stream=None):
    """Top-k selection and sparse decode in one call: the results of ekv_select_pages (top-k
    policy) followed by ekv_sparse_decode."""
    P, I32, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float
    fn = _moment_fn("ekv_select_decode", [ctypes.POINTER(EkvCacheStruct), P, I32, F, I32, I32, P,
                                          P, P, I32, P, P, P, ctypes.c_size_t, P])
    c = cache.struct()
    _check(fn(ctypes.byref(c), _ptr(q), int(num_q_heads), float(scale), int(attn), int(topk),
              _ptr(scores), _ptr(sel_idx), _ptr(sel_count), int(max_sel), _ptr(out), _ptr(stat),
              _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)), "ekv_select_decode")


def ekv_wait_selftest(cache: PagedKVCache, limit_ns: int, stream=None):
    """One thread waits on a barrier nothing completes, bounded by limit_ns, then sets
    EKV_DEV_TIMEOUT in the cache's status word (the device-side timeout path on its own)."""
    fn = _moment_fn("ekv_wait_selftest", [ctypes.POINTER(EkvCacheStruct), ctypes.c_uint64,
                                          ctypes.c_void_p])
    c = cache.struct()
    _check(fn(ctypes.byref(c), int(limit_ns), _stream(stream)), "ekv_wait_selftest")


def ekv_decode_workspace_bytes(cache: PagedKVCache, num_q_heads: int, max_sel: int) -> int:
    c = cache.struct()
    return int(load_library().ekv_decode_workspace_bytes(ctypes.byref(c), int(num_q_heads),
                                                         int(max_sel)))


def ekv_device_status(cache: PagedKVCache, stream=None):
    """Synchronise and return (status, bits): EKV_OK or EKV_ERR_DEVICE with the EKV_DEV_* bits."""
    c = cache.struct()
    bits = ctypes.c_uint32(0)
    st = load_library().ekv_device_status(ctypes.byref(c), ctypes.byref(bits), _stream(stream))
    if st not in (EKV_OK, EKV_ERR_DEVICE):
        raise EkvError(st, "ekv_device_status")
    return st, bits.value


def ekv_clear_device_status(cache: PagedKVCache, stream=None):
    c = cache.struct()
    _check(load_library().ekv_clear_device_status(ctypes.byref(c), _stream(stream)),
           "ekv_clear_device_status")


def ekv_sparse_decode_noalloc(cache: PagedKVCache, q: torch.Tensor, num_q_heads: int,
                              scale: float, attn: int, sel_idx: torch.Tensor,
                              sel_count: torch.Tensor, max_sel: int, out: torch.Tensor,
                              stat: torch.Tensor, stream=None):
    """ekv_sparse_decode with the library's fixed scratch (no workspace argument): for callers
    that cannot allocate device memory. Its first call on a device should precede any stream
    capture; calls that overlap on the GPU share the scratch and must be serialised."""
    lib = load_library()
    fn = lib.ekv_sparse_decode_noalloc
    if fn.restype is not ctypes.c_int or fn.argtypes is None:
        P, I32, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float
        fn.argtypes = [ctypes.POINTER(EkvCacheStruct), P, I32, F, I32, P, P, I32, P, P, P]
        fn.restype = ctypes.c_int
    c = cache.struct()
    _check(fn(ctypes.byref(c), _ptr(q), int(num_q_heads), float(scale), int(attn), _ptr(sel_idx),
              _ptr(sel_count), int(max_sel), _ptr(out), _ptr(stat), _stream(stream)),
           "ekv_sparse_decode_noalloc")


def _moment_fn(name, args, res=ctypes.c_int):
    """An entry point beyond the four calls, its signature set on first use."""
    fn = getattr(load_library(), name)
    if fn.argtypes is None:
        fn.argtypes, fn.restype = args, res
    return fn


def ekv_moment_bytes(cache: PagedKVCache) -> int:
    """Bytes of the running-moment records [batch][H_kv][EKV_MOMENT_FLOATS(d)] fp32."""
    fn = _moment_fn("ekv_moment_bytes", [ctypes.POINTER(EkvCacheStruct)], ctypes.c_size_t)
    c = cache.struct()
    return int(fn(ctypes.byref(c)))


def ekv_moment_update(cache: PagedKVCache, moments: torch.Tensor, new_start: torch.Tensor,
                      new_count: torch.Tensor, max_new: int, stream=None):
    """Add the token ranges [new_start[b], new_start[b] + new_count[b]) to the running moments
    (a zero-filled float32 tensor of ekv_moment_bytes bytes before the first update)."""
    P, I32 = ctypes.c_void_p, ctypes.c_int32
    fn = _moment_fn("ekv_moment_update", [ctypes.POINTER(EkvCacheStruct), P, P, P, I32, P])
    c = cache.struct()
    _check(fn(ctypes.byref(c), _ptr(moments), _ptr(new_start), _ptr(new_count), int(max_new),
              _stream(stream)), "ekv_moment_update")


def ekv_moment_decode_workspace_bytes(cache: PagedKVCache, num_q_heads: int, max_sel: int) -> int:
    fn = _moment_fn("ekv_moment_decode_workspace_bytes",
                    [ctypes.POINTER(EkvCacheStruct), ctypes.c_int32, ctypes.c_int32],
                    ctypes.c_size_t)
    c = cache.struct()
    return int(fn(ctypes.byref(c), int(num_q_heads), int(max_sel)))


def ekv_sparse_decode_moment(cache: PagedKVCache, moments: torch.Tensor, q: torch.Tensor,
                             num_q_heads: int, scale: float, sel_idx: torch.Tensor,
                             sel_count: torch.Tensor, max_sel: int, out: torch.Tensor,
                             stat: torch.Tensor, ws: torch.Tensor, stream=None):
    """Softmax over the selected pages, corrected for the skipped tokens from the running
    moments (see include/ekv.h)."""
    P, I32, F, U64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    fn = _moment_fn("ekv_sparse_decode_moment",
                    [ctypes.POINTER(EkvCacheStruct), P, P, I32, F, P, P, I32, P, P, P, U64, P])
    c = cache.struct()
    _check(fn(ctypes.byref(c), _ptr(moments), _ptr(q), int(num_q_heads), float(scale),
              _ptr(sel_idx), _ptr(sel_count), int(max_sel), _ptr(out), _ptr(stat), _ptr(ws),
              ws.numel() * ws.element_size(), _stream(stream)), "ekv_sparse_decode_moment")


def ekv_token_workspace_bytes(cache: PagedKVCache, max_sel: int) -> int:
    fn = _moment_fn("ekv_token_workspace_bytes", [ctypes.POINTER(EkvCacheStruct), ctypes.c_int32],
                    ctypes.c_size_t)
    c = cache.struct()
    return int(fn(ctypes.byref(c), int(max_sel)))


def ekv_select_tokens(cache: PagedKVCache, q: torch.Tensor, num_q_heads: int, scale: float,
                      sel_idx: torch.Tensor, sel_count: torch.Tensor, max_sel: int, T: int,
                      tok_page: torch.Tensor, tok_pos: torch.Tensor, tok_count: torch.Tensor,
                      ws: torch.Tensor, stream=None):
    """Token-level top-T inside the selected pages, per KV head (see include/ekv.h)."""
    P, I32, F, U64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    fn = _moment_fn("ekv_select_tokens", [ctypes.POINTER(EkvCacheStruct), P, I32, F, P, P, I32,
                                          I32, P, P, P, P, U64, P])
    c = cache.struct()
    _check(fn(ctypes.byref(c), _ptr(q), int(num_q_heads), float(scale), _ptr(sel_idx),
              _ptr(sel_count), int(max_sel), int(T), _ptr(tok_page), _ptr(tok_pos),
              _ptr(tok_count), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "ekv_select_tokens")


def ekv_sparse_decode_tokens(cache: PagedKVCache, q: torch.Tensor, num_q_heads: int,
                             scale: float, attn: int, tok_page: torch.Tensor,
                             tok_pos: torch.Tensor, tok_count: torch.Tensor, T: int,
                             out: torch.Tensor, stat: torch.Tensor, stream=None):
    """Attention over the kept tokens, read in place through the page table."""
    P, I32, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float
    fn = _moment_fn("ekv_sparse_decode_tokens", [ctypes.POINTER(EkvCacheStruct), P, I32, F, I32,
                                                 P, P, P, I32, P, P, P])
    c = cache.struct()
    _check(fn(ctypes.byref(c), _ptr(q), int(num_q_heads), float(scale), int(attn),
              _ptr(tok_page), _ptr(tok_pos), _ptr(tok_count), int(T), _ptr(out), _ptr(stat),
              _stream(stream)), "ekv_sparse_decode_tokens")


def ekv_selection_quality(cache: PagedKVCache, q: torch.Tensor, num_q_heads: int, scale: float,
                          attn: int, stat_full: torch.Tensor, sel_idx: torch.Tensor,
                          sel_count: torch.Tensor, max_sel: int, dropped: torch.Tensor,
                          support: torch.Tensor, stream=None):
    """Full-cache weight outside the selected pages (dropped [B, H_q] float64) and the support
    counts (support [B, H_q, 2] int32: size, inside the selection) for the full-cache statistic
    stat_full [B, H_q] (see include/ekv.h)."""
    P, I32, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float
    fn = _moment_fn("ekv_selection_quality", [ctypes.POINTER(EkvCacheStruct), P, I32, F, I32, P,
                                              P, P, I32, P, P, P])
    c = cache.struct()
    _check(fn(ctypes.byref(c), _ptr(q), int(num_q_heads), float(scale), int(attn),
              _ptr(stat_full), _ptr(sel_idx), _ptr(sel_count), int(max_sel), _ptr(dropped),
              _ptr(support), _stream(stream)), "ekv_selection_quality")


def ekv_score_select_pages(cache: PagedKVCache, q: torch.Tensor, num_q_heads: int, scale: float,
                           topk: int, scores: Optional[torch.Tensor], sel_idx: torch.Tensor,
                           sel_count: torch.Tensor, max_sel: int, stream=None):
    """Top-k page scores and selection in one call (one cluster per sequence and KV head);
    the results of ekv_score_pages + ekv_select_pages with the top-k policy, bit for bit."""
    P, I32, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float
    fn = _moment_fn("ekv_score_select_pages", [ctypes.POINTER(EkvCacheStruct), P, I32, F, I32, P,
                                               P, P, I32, P])
    c = cache.struct()
    _check(fn(ctypes.byref(c), _ptr(q), int(num_q_heads), float(scale), int(topk), _ptr(scores),
              _ptr(sel_idx), _ptr(sel_count), int(max_sel), _stream(stream)),
           "ekv_score_select_pages")
