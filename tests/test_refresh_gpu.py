"""GPU parity of ekv_refresh_score_pages (the metadata refresh of an append and the page scores in
one call): its metadata, scores and device status equal those of ekv_page_meta_update followed by
ekv_score_pages bit for bit, and both match the oracle. Cases: an append of one whole page
(one refresh group per pair), ranges that straddle a page and an 8-page group boundary, 2 P
tokens over three pages, sequences without an append, a cache with Gaussian statistics, fp32 and
d = 64, and the paths that run the two kernels (a Gaussian policy; many (sequence, head) pairs);
a range past the sequence's end and a bad page-table entry raise the same flags as the two
calls."""
import numpy as np
import pytest
import torch

import oracle as O
from sparse_kv_cache_kmin_b200 import ekv
from sparse_kv_cache_kmin_b200.workloads import GAUSS, TOPK, make_random
from parity_utils import HostCopy, check_meta, make_cache, prefill_metadata, topk_score_tol

pytestmark = pytest.mark.gpu


def bits(t):
    return t.view(torch.int16 if t.element_size() == 2 else torch.int32)


def run_both(wl, counts, gaussian, policy, max_new=None, starts=None, break_block=None):
    """Prefill at the shorter lengths, append `counts` tokens with fresh keys, then refresh and
    score both ways on caches with the same metadata."""
    B, P = wl.batch, wl.page_size
    L = wl.seq_lens.clone()
    counts_t = torch.tensor(counts, dtype=torch.int32, device="cuda")
    wl.seq_lens.copy_(L - counts_t)
    a = make_cache(wl, gaussian)
    prefill_metadata(a, wl)
    wl.seq_lens.copy_(L)
    gen = torch.Generator(device="cuda").manual_seed(int(L.sum().item()))
    H = wl.num_kv_heads
    for b in range(B):
        for t in range(int(L[b]) - counts[b], int(L[b])):
            blk = int(wl.page_table[b, t // P])
            wl.k_cache[blk, :, t % P] = torch.randn((H, wl.head_dim), generator=gen,
                                                    device="cuda").to(wl.k_cache.dtype)
    if break_block is not None:
        b, j = break_block
        wl.page_table[b, j] = wl.k_cache.shape[0] + 3
    b_cache = ekv.PagedKVCache(
        k_cache=wl.k_cache, v_cache=wl.v_cache, meta_bbox=a.meta_bbox.clone(),
        meta_mom=a.meta_mom.clone() if a.meta_mom is not None else None,
        page_table=wl.page_table, seq_lens=wl.seq_lens,
        dev_status=torch.zeros(1, dtype=torch.int32, device="cuda"))
    stale = a.meta_bbox.clone()
    start = (L - counts_t) if starts is None else torch.tensor(starts, dtype=torch.int32,
                                                              device="cuda")
    mn = max(counts) if max_new is None else max_new
    if policy == TOPK:
        shape = (B, H, a.max_pages)
    else:
        shape = (B, wl.num_q_heads, 3, a.max_pages)
    sa = torch.full(shape, 12345.0, device="cuda")
    sb = sa.clone()
    ekv.ekv_page_meta_update(a, start, counts_t, mn)
    ekv.ekv_score_pages(a, wl.q, wl.num_q_heads, wl.scale, policy, sa)
    ekv.ekv_refresh_score_pages(b_cache, start, counts_t, mn, wl.q, wl.num_q_heads, wl.scale,
                                policy, sb)
    torch.cuda.synchronize()
    assert torch.equal(bits(a.meta_bbox), bits(b_cache.meta_bbox))
    if gaussian:
        assert torch.equal(bits(a.meta_mom), bits(b_cache.meta_mom))
    assert torch.equal(bits(sa), bits(sb))
    assert ekv.ekv_device_status(a) == ekv.ekv_device_status(b_cache)
    return b_cache, sb, stale


def check_oracle(wl, cache, scores):
    for b in range(wl.batch):
        hc = HostCopy(wl, b)
        for h in range(wl.num_kv_heads):
            meta = O.page_meta_head(hc.k, hc.pt, hc.L, h)
            check_meta(cache, hc, h, meta)
            qg = hc.q[h]
            _, S = O.score_head(qg, wl.scale, meta[0], meta[1])
            tol = topk_score_tol(qg, meta[0], meta[1], wl.scale)
            got = scores[b, h, :hc.np].double().cpu().numpy()
            assert np.all(np.abs(got - S) <= tol)


CASES = [  # B, H_kv, G, d, P, dtype, final lengths, appended tokens per sequence, gaussian
    (1, 8, 8, 128, 64, torch.bfloat16, (64 * 300,), (64,), False),           # one whole page
    (2, 2, 4, 128, 16, torch.bfloat16, (16 * 8 * 5 + 7, 16 * 40 + 1), (10, 1), False),
    (1, 4, 2, 128, 16, torch.bfloat16, (16 * 20 + 1,), (32,), False),         # 3 pages, 1 group
    (1, 4, 2, 128, 16, torch.bfloat16, (16 * 24 + 1,), (32,), False),         # 3 pages, 2 groups
    (3, 2, 4, 128, 32, torch.bfloat16, (32 * 30, 32 * 9 + 5, 700), (16, 0, 5), False),
    (2, 2, 4, 128, 16, torch.bfloat16, (16 * 33 + 3, 16 * 16), (9, 16), True),  # with mean/var
    (2, 2, 1, 64, 32, torch.float32, (32 * 17 + 2, 32 * 9), (40, 32), False),
    (2, 2, 4, 128, 16, torch.bfloat16, (20, 16 * 30), (20, 5), False),  # first tokens of a sequence
]


@pytest.mark.parametrize("B,H,G,d,P,dtype,lens,counts,gaussian", CASES,
                         ids=["c%d" % i for i in range(len(CASES))])
def test_refresh_score_equals_the_two_calls_and_the_oracle(cuda_device, B, H, G, d, P, dtype,
                                                           lens, counts, gaussian):
    wl = make_random(B=B, H_kv=H, G=G, d=d, P=P, lens=lens, dtype=dtype, device="cuda",
                     seed=sum(lens) + G, kv_scale=1.5)
    cache, scores, stale = run_both(wl, list(counts), gaussian, TOPK)
    assert ekv.ekv_device_status(cache)[0] == ekv.EKV_OK
    # the appended pages' boxes did change, so the refresh is what made them right
    changed = 0
    for b in range(B):
        if counts[b]:
            last = int(wl.page_table[b, (lens[b] - 1) // P])
            changed += int(not torch.equal(bits(stale[last]), bits(cache.meta_bbox[last])))
    assert changed == sum(1 for n in counts if n)
    check_oracle(wl, cache, scores)


def test_refresh_score_gaussian_policy_runs_the_two_kernels(cuda_device):
    wl = make_random(B=2, H_kv=2, G=4, d=128, P=16, lens=(16 * 30 + 5, 300), device="cuda",
                     seed=91, policy=GAUSS)
    run_both(wl, [21, 16], True, GAUSS)


def test_refresh_score_many_pairs_runs_the_two_kernels(cuda_device):
    lens = tuple(16 * (20 + 3 * i) + i for i in range(16))
    wl = make_random(B=16, H_kv=8, G=4, d=128, P=16, lens=lens, device="cuda", seed=92)
    cache, scores, _ = run_both(wl, [17] * 16, False, TOPK)
    assert ekv.ekv_device_status(cache)[0] == ekv.EKV_OK


def test_refresh_score_range_past_the_end_is_flagged_alike(cuda_device):
    wl = make_random(B=2, H_kv=2, G=4, d=128, P=16, lens=(16 * 9, 16 * 12 + 3), device="cuda",
                     seed=93)
    # sequence 1 asks for 9 tokens from 3 before its end: clamped to the last 3, flagged
    starts = [16 * 9 - 8, 16 * 12]
    cache, _, _ = run_both(wl, [8, 9], False, TOPK, starts=starts)
    st, bits_ = ekv.ekv_device_status(cache)
    assert st == ekv.EKV_ERR_DEVICE and bits_ & ekv.EKV_DEV_BAD_RANGE


def test_refresh_score_bad_page_table_entry_is_flagged_alike(cuda_device):
    wl = make_random(B=1, H_kv=4, G=2, d=128, P=16, lens=(16 * 20 + 4,), device="cuda", seed=94)
    cache, scores, _ = run_both(wl, [4], False, TOPK, break_block=(0, 20))
    st, bits_ = ekv.ekv_device_status(cache)
    assert st == ekv.EKV_ERR_DEVICE and bits_ & ekv.EKV_DEV_BAD_BLOCK
    assert torch.all(scores[0, :, 20] == float("-inf"))


def test_refresh_score_with_no_append_in_any_sequence(cuda_device):
    # max_new > 0 but every count 0: the one-kernel path runs and refreshes nothing
    wl = make_random(B=2, H_kv=2, G=4, d=128, P=16, lens=(16 * 12 + 3, 16 * 9), device="cuda",
                     seed=95)
    cache, scores, stale = run_both(wl, [0, 0], False, TOPK, max_new=16)
    assert ekv.ekv_device_status(cache)[0] == ekv.EKV_OK
    assert torch.equal(bits(stale), bits(cache.meta_bbox))
    check_oracle(wl, cache, scores)
