"""ekv_sparse_decode_noalloc: the decode entry point for callers that cannot allocate device
memory (an engine whose allocator already holds all of HBM, a latency-critical loop that must
not risk a synchronising cudaMalloc, a plug-in handed only its inputs and outputs). It uses
the library's fixed scratch array instead of a caller workspace; its results must equal
ekv_sparse_decode's bit for bit (same kernels, same inputs), call after call.

This file is collected last on purpose, and it works both alone in a fresh process (where its
first call also performs the one-time per-device look-up of the scratch address) and after
the rest of the suite."""
import ctypes

import pytest
import torch

from sparse_kv_cache_kmin_b200 import ekv
from sparse_kv_cache_kmin_b200.decoder import SparseDecoder
from sparse_kv_cache_kmin_b200.workloads import make_random

pytestmark = pytest.mark.gpu


def c_noalloc():
    fn = ekv.load_library().ekv_sparse_decode_noalloc
    P, I32, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float
    fn.argtypes = [ctypes.POINTER(ekv.EkvCacheStruct), P, I32, F, I32, P, P, I32, P, P, P]
    fn.restype = ctypes.c_int
    return fn


def ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def setup(seed, attn):
    wl = make_random(B=3, H_kv=2, G=4, d=128, P=16, lens=(3000, 1234, 17), dtype=torch.bfloat16,
                     device="cuda", seed=seed, topk=40)
    nb, H, P, d = wl.k_cache.shape
    cache = ekv.PagedKVCache(
        k_cache=wl.k_cache, v_cache=wl.v_cache,
        meta_bbox=torch.empty((nb, H, 2, d), dtype=wl.k_cache.dtype, device="cuda"),
        meta_mom=None, page_table=wl.page_table, seq_lens=wl.seq_lens,
        dev_status=torch.zeros(1, dtype=torch.int32, device="cuda"))
    ekv.ekv_page_meta_update(cache, torch.zeros(3, dtype=torch.int32, device="cuda"), wl.seq_lens,
                             int(wl.seq_lens.max()))
    dec = SparseDecoder(cache, wl.num_q_heads, ekv.EKV_SEL_TOPK, attn, topk=wl.topk)
    dec.step(wl.q)  # the existing entry point: scores, selection, and its decode into dec.out
    return wl, cache, dec


@pytest.mark.parametrize("attn", [ekv.EKV_ENTMAX15, ekv.EKV_SOFTMAX, ekv.EKV_SPARSEMAX])
def test_noalloc_matches_workspace_decode_on_consecutive_calls(cuda_device, attn):
    fn = c_noalloc()
    for seed in (21, 22):  # two calls in a row, on different inputs, sharing the scratch
        wl, cache, dec = setup(seed, attn)
        out = torch.full_like(dec.out, float("nan"))
        stat = torch.full_like(dec.stat, float("nan"))
        c = cache.struct()
        st = fn(ctypes.byref(c), ptr(wl.q), wl.num_q_heads, 1.0, attn, ptr(dec.sel_idx),
                ptr(dec.sel_count), dec.max_sel, ptr(out), ptr(stat),
                ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == ekv.EKV_OK, ekv.status_str(st)
        torch.cuda.synchronize()
        assert ekv.ekv_device_status(cache)[0] == ekv.EKV_OK
        # the same kernels on the same inputs and selection: identical bit for bit (a scratch
        # that aliased or kept stale words would show here, not hide inside a tolerance)
        assert torch.equal(out, dec.out)
        assert torch.equal(stat.isnan(), dec.stat.isnan()) and not bool(stat.isnan().any())
        assert torch.equal(stat, dec.stat)


def test_noalloc_refuses_geometry_beyond_its_scratch(cuda_device):
    wl, cache, dec = setup(23, ekv.EKV_ENTMAX15)
    big = ekv.PagedKVCache(cache.k_cache, cache.v_cache, cache.meta_bbox, None,
                           torch.zeros((64, 4096), dtype=torch.int32, device="cuda"),
                           torch.zeros(64, dtype=torch.int32, device="cuda"), cache.dev_status)
    assert ekv.ekv_decode_workspace_bytes(big, wl.num_q_heads, 4096) > (16 << 20)
    out = torch.empty((64, wl.num_q_heads, 128), device="cuda")
    stat = torch.empty((64, wl.num_q_heads), device="cuda")
    sel = torch.zeros((64, 2, 4096), dtype=torch.int32, device="cuda")
    cnt = torch.zeros((64, 2), dtype=torch.int32, device="cuda")
    c = big.struct()
    st = c_noalloc()(ctypes.byref(c), ptr(wl.q), wl.num_q_heads, 1.0, ekv.EKV_ENTMAX15, ptr(sel),
                     ptr(cnt), 4096, ptr(out), ptr(stat), None)
    assert st == ekv.EKV_ERR_WORKSPACE
