"""GPU parity of the fused top-k scan and selection (ekv_score_select_pages: one thread-block
cluster per sequence and KV head) with the two standalone calls ekv_score_pages +
ekv_select_pages, which the oracle parity tests pin: the scores and the selection must be
identical bit for bit, at every cluster size the launch picks (1 to 16 CTAs per pair), on
ragged lengths, heavy ties, k >= n, empty sequences and bad page-table entries."""
import itertools

import numpy as np
import pytest
import torch

from sparse_kv_cache_kmin_b200 import ekv
from sparse_kv_cache_kmin_b200.workloads import TOPK, make, make_random
from parity_utils import make_cache, prefill_metadata

pytestmark = pytest.mark.gpu


def both_paths(wl, cache, topk, max_sel=None, scores_out=True):
    B, H, mp = wl.batch, wl.num_kv_heads, wl.max_pages
    max_sel = max_sel or max(1, min(topk, mp))
    dev = wl.k_cache.device
    res = []
    for fused in (False, True):
        scores = torch.full((B, H, mp), float("nan"), device=dev)
        sel = torch.full((B, H, max_sel), -7, dtype=torch.int32, device=dev)
        cnt = torch.full((B, H), -7, dtype=torch.int32, device=dev)
        if fused:
            ekv.ekv_score_select_pages(cache, wl.q, wl.num_q_heads, wl.scale, topk,
                                       scores if scores_out else None, sel, cnt, max_sel)
        else:
            ekv.ekv_score_pages(cache, wl.q, wl.num_q_heads, wl.scale, TOPK, scores)
            ekv.ekv_select_pages(cache, wl.num_q_heads, TOPK, topk, 1.5, 0.0, scores, sel, cnt,
                                 max_sel, None)
        torch.cuda.synchronize()
        res.append((scores, sel, cnt))
    return res


def assert_same(wl, res, check_scores=True):
    (s0, i0, c0), (s1, i1, c1) = res
    P = wl.page_size
    n_pages = ((wl.seq_lens.long() + P - 1) // P).tolist()
    assert torch.equal(c0, c1), (c0, c1)
    assert torch.equal(i0, i1)
    if check_scores:
        for b, n in enumerate(n_pages):
            # bit for bit (NaN-free: every existing page is written)
            assert torch.equal(s0[b, :, :n].view(torch.int32), s1[b, :, :n].view(torch.int32))


SHAPES = list(itertools.product([64, 128], [16, 32, 64], [1, 2, 4, 8]))


@pytest.mark.parametrize("d,P,G", SHAPES, ids=["d%d-P%d-G%d" % s for s in SHAPES])
def test_fused_score_select_matches_the_two_calls(cuda_device, d, P, G):
    lens = (1000 + 7 * P, 517, 33, 2 * P, 0, 1)
    for topk in (1, 9, 40, 10_000):
        wl = make_random(B=6, H_kv=2, G=G, d=d, P=P, lens=lens, dtype=torch.bfloat16,
                         device="cuda", seed=d + P + G + topk, kv_scale=2.0, topk=topk)
        cache = make_cache(wl)
        prefill_metadata(cache, wl)
        assert_same(wl, both_paths(wl, cache, topk))
        assert ekv.ekv_device_status(cache)[0] == ekv.EKV_OK


@pytest.mark.parametrize("B", [1, 2, 4, 8, 20])
def test_fused_score_select_every_cluster_size(cuda_device, B):
    # 8 KV heads: 8, 16, 32, 64 and 160 pairs give clusters of 16, 8, 4, 2 and 1 CTAs
    lens = tuple(int(x) for x in np.random.default_rng(B).integers(1, 20000, size=B))
    wl = make_random(B=B, H_kv=8, G=4, d=128, P=16, lens=lens, dtype=torch.bfloat16,
                     device="cuda", seed=50 + B, topk=256)
    cache = make_cache(wl)
    prefill_metadata(cache, wl)
    res = both_paths(wl, cache, 256)
    assert_same(wl, res)
    # without a scores output the selection is the same
    res2 = both_paths(wl, cache, 256, scores_out=False)
    assert torch.equal(res2[1][1], res[0][1]) and torch.equal(res2[1][2], res[0][2])


def test_fused_score_select_heavy_ties(cuda_device):
    # every page of a sequence has the same bound: the lowest page indices are kept, across the
    # cluster's CTAs in rank order; half-equal scores exercise the tie quota at the boundary
    wl = make_random(B=4, H_kv=2, G=4, d=128, P=16, lens=(20000, 7777, 3000, 16 * 300),
                     dtype=torch.bfloat16, device="cuda", seed=61, topk=300)
    wl.k_cache.fill_(0.5)
    cache = make_cache(wl)
    prefill_metadata(cache, wl)
    res = both_paths(wl, cache, 300)
    assert_same(wl, res)
    assert torch.equal(res[1][1][0, 0], torch.arange(300, dtype=torch.int32, device="cuda"))
    # two score levels: pages with a bigger key block take precedence, ties broken by index
    k = wl.k_cache.view(wl.k_cache.shape[0], -1)
    k[::3] = 0.75
    cache = make_cache(wl)
    prefill_metadata(cache, wl)
    assert_same(wl, both_paths(wl, cache, 300))


def test_fused_score_select_bad_page_table_entry(cuda_device):
    wl = make_random(B=2, H_kv=2, G=2, d=64, P=16, lens=(3000, 200), dtype=torch.bfloat16,
                     device="cuda", seed=62, topk=8)
    cache = make_cache(wl)
    prefill_metadata(cache, wl)
    wl.page_table[1, 3] = wl.k_cache.shape[0] + 5
    res = both_paths(wl, cache, 8)
    assert_same(wl, res)
    st, bits = ekv.ekv_device_status(cache)
    assert st == ekv.EKV_ERR_DEVICE and bits & ekv.EKV_DEV_BAD_BLOCK


def test_fused_score_select_needle_workload(cuda_device):
    wl = make("needle128k", device="cuda")
    cache = make_cache(wl)
    prefill_metadata(cache, wl)
    assert_same(wl, both_paths(wl, cache, wl.topk))


def test_fused_score_select_long_context_workload(cuda_device):
    wl = make("long1m", device="cuda")
    cache = make_cache(wl)
    prefill_metadata(cache, wl)
    assert_same(wl, both_paths(wl, cache, wl.topk))
