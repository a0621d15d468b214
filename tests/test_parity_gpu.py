"""GPU parity: the CUDA path, called through the C ABI, against the CPU oracle on the same
seeded inputs -- every stage (metadata, scores, selection, attention) of every (sequence, KV
head) on small ragged cases that span several tiles, and sampled heads of the full-size
workloads in the launch configuration the benchmark times."""
import itertools

import numpy as np
import pytest
import torch

import oracle as O
from sparse_kv_cache_kmin_b200 import ekv
from sparse_kv_cache_kmin_b200.workloads import GAUSS, GAUSS_MAX, TOPK, make, make_random
from parity_utils import HostCopy, check_head, close, make_cache, prefill_metadata, run_gpu, widen

pytestmark = pytest.mark.gpu

ATTN = [ekv.EKV_SOFTMAX, ekv.EKV_ENTMAX15, ekv.EKV_SPARSEMAX]


def assert_status_ok(cache):
    st, bits = ekv.ekv_device_status(cache)
    assert st == ekv.EKV_OK, hex(bits)


TOPK_CASES = list(itertools.product([torch.float32, torch.bfloat16], [64, 128], [16, 32, 64],
                                    [1, 2, 4, 8]))


@pytest.mark.parametrize("dtype,d,P,G", TOPK_CASES,
                         ids=["%s-d%d-P%d-G%d" % (str(t)[6:], d, P, G) for t, d, P, G in TOPK_CASES])
def test_topk_small_ragged(cuda_device, dtype, d, P, G):
    lens = (1000 + 7 * P, 517, 33, 2 * P)
    wl = make_random(B=4, H_kv=2, G=G, d=d, P=P, lens=lens, dtype=dtype, device="cuda",
                     seed=d + P + G, kv_scale=2.0, topk=9)
    for attn in ATTN:
        cache, dec = run_gpu(wl, attn)
        assert_status_ok(cache)
        for b in range(wl.batch):
            for h in range(wl.num_kv_heads):
                check_head(wl, cache, dec, b, h, attn)


GAUSS_CASES = list(itertools.product([torch.float32, torch.bfloat16], [64, 128], [16, 32],
                                     [1, 4, 8], [ekv.EKV_ENTMAX15, ekv.EKV_SPARSEMAX]))


@pytest.mark.parametrize("dtype,d,P,G,attn", GAUSS_CASES,
                         ids=["%s-d%d-P%d-G%d-a%d" % (str(t)[6:], d, P, G, a) for t, d, P, G, a in GAUSS_CASES])
def test_gauss_small_ragged(cuda_device, dtype, d, P, G, attn):
    lens = (3000 + 5, 700, 64 * 3 + 1)
    alpha = 1.5 if attn == ekv.EKV_ENTMAX15 else 2.0
    wl = make_random(B=3, H_kv=2, G=G, d=d, P=P, lens=lens, dtype=dtype, device="cuda",
                     seed=100 + d + P + G, kv_scale=1.0, q_scale=0.6, policy=GAUSS, alpha=alpha,
                     delta=0.1)
    cache, dec = run_gpu(wl, attn)
    assert_status_ok(cache)
    for b in range(wl.batch):
        for h in range(wl.num_kv_heads):
            check_head(wl, cache, dec, b, h, attn)


GAUSS_MAX_CASES = list(itertools.product([torch.float32, torch.bfloat16], [128], [16, 32], [1, 4],
                                         [ekv.EKV_ENTMAX15, ekv.EKV_SPARSEMAX]))


@pytest.mark.parametrize("dtype,d,P,G,attn", GAUSS_MAX_CASES,
                         ids=["%s-d%d-P%d-G%d-a%d" % (str(t)[6:], d, P, G, a) for t, d, P, G, a in GAUSS_MAX_CASES])
def test_gauss_estimated_max_small_ragged(cuda_device, dtype, d, P, G, attn):
    # the second reading of the estimated page maximum: min(UB, m + sqrt(2 ln n) sqrt(v))
    lens = (3000 + 5, 700, 64 * 3 + 1)
    alpha = 1.5 if attn == ekv.EKV_ENTMAX15 else 2.0
    wl = make_random(B=3, H_kv=2, G=G, d=d, P=P, lens=lens, dtype=dtype, device="cuda",
                     seed=200 + d + P + G, kv_scale=1.0, q_scale=0.6, policy=GAUSS_MAX,
                     alpha=alpha, delta=0.1)
    cache, dec = run_gpu(wl, attn)
    assert_status_ok(cache)
    for b in range(wl.batch):
        for h in range(wl.num_kv_heads):
            check_head(wl, cache, dec, b, h, attn)


def test_gauss_estimated_max_on_the_gauss_workload(cuda_device):
    wl = make("gauss", device="cuda")
    wl.policy = GAUSS_MAX
    cache = make_cache(wl)
    prefill_metadata(cache, wl)
    _, dec = run_gpu(wl, ekv.EKV_ENTMAX15, cache=cache)
    assert_status_ok(cache)
    for b, h in [(0, 0), (9, 4), (15, 7)]:
        check_head(wl, cache, dec, b, h, ekv.EKV_ENTMAX15)


@pytest.mark.parametrize("policy", [GAUSS, GAUSS_MAX], ids=["gauss", "gauss_max"])
@pytest.mark.parametrize("attn", [ekv.EKV_ENTMAX15, ekv.EKV_SPARSEMAX])
def test_gauss_two_query_groups(cuda_device, policy, attn):
    # G = 2: clusters of two CTAs (one per query) for the selection
    alpha = 1.5 if attn == ekv.EKV_ENTMAX15 else 2.0
    wl = make_random(B=3, H_kv=2, G=2, d=128, P=16, lens=(2500, 600, 17), dtype=torch.bfloat16,
                     device="cuda", seed=31, kv_scale=1.0, q_scale=0.6, policy=policy,
                     alpha=alpha, delta=0.1)
    cache, dec = run_gpu(wl, attn)
    assert_status_ok(cache)
    for b in range(wl.batch):
        for h in range(wl.num_kv_heads):
            check_head(wl, cache, dec, b, h, attn)


def test_gauss_long_sequence_beyond_the_staged_slices(cuda_device):
    # 20000 pages: a warp's slice exceeds its shared-memory capacity, so the model is read from
    # global memory for the maximum and, where the survivors overflow, on every Newton step
    wl = make_random(B=1, H_kv=1, G=4, d=64, P=16, lens=(20000 * 16 - 9,), dtype=torch.bfloat16,
                     device="cuda", seed=32, kv_scale=0.2, q_scale=0.3, policy=GAUSS_MAX,
                     alpha=1.5, delta=0.1)
    cache, dec = run_gpu(wl, ekv.EKV_ENTMAX15)
    assert_status_ok(cache)
    check_head(wl, cache, dec, 0, 0, ekv.EKV_ENTMAX15)


def test_multi_chunk_pages(cuda_device):
    # enough selected pages that each (sequence, head) spans several multi-page chunks
    wl = make_random(B=4, H_kv=8, G=4, d=128, P=16, lens=(8000, 8000 - 3, 4100, 8000),
                     dtype=torch.bfloat16, device="cuda", seed=7, topk=200)
    for attn in ATTN:
        cache, dec = run_gpu(wl, attn)
        assert_status_ok(cache)
        for b, h in [(0, 0), (1, 7), (2, 3), (3, 5)]:
            check_head(wl, cache, dec, b, h, attn)


LARGE_CASES = [(torch.bfloat16, 2e-3), (torch.float32, 2e-3), (torch.bfloat16, 0.05),
               (torch.bfloat16, 0.0)]


@pytest.mark.parametrize("dtype,q_scale", LARGE_CASES,
                         ids=["%s-q%g" % (str(t)[6:], s) for t, s in LARGE_CASES])
def test_entmax_large_candidate_sets(cuda_device, dtype, q_scale):
    # nearly flat logits put thousands of tokens within 1 of the maximum: the per-warp lists
    # overflow, the threshold bracket descends several histogram levels, and q = 0 makes every
    # logit equal (ties in the last bin)
    wl = make_random(B=2, H_kv=2, G=4, d=128, P=16, lens=(20000, 7777), dtype=dtype,
                     device="cuda", seed=11, q_scale=q_scale, topk=1250)
    for attn in [ekv.EKV_ENTMAX15, ekv.EKV_SPARSEMAX]:
        wl.alpha = 1.5 if attn == ekv.EKV_ENTMAX15 else 2.0
        cache, dec = run_gpu(wl, attn)
        assert_status_ok(cache)
        for b, h in [(0, 0), (0, 1), (1, 1)]:
            check_head(wl, cache, dec, b, h, attn)


# ------------------------------------------------------------------ the five named workloads
def test_tiny_full_and_support_invariant(cuda_device):
    wl = make("tiny", device="cuda")
    for attn in [ekv.EKV_SOFTMAX, ekv.EKV_ENTMAX15]:
        cache, dec = run_gpu(wl, attn)
        assert_status_ok(cache)
        check_head(wl, cache, dec, 0, 0, attn)
    # full-cache 1.5-entmax on the GPU (every page selected) against the oracle
    n_pages = wl.max_pages
    wl.topk = n_pages
    cache, full = run_gpu(wl, ekv.EKV_ENTMAX15)
    hc = HostCopy(wl, 0)
    out_o, stat_o, w = O.attend_head(hc.k, hc.v, hc.pt, hc.L, 0, hc.q[0], 1.0, O.ENTMAX15,
                                     np.arange(n_pages), want_weights=True)
    close(full.out[0].double().cpu().numpy(), out_o, False)
    # support invariant: a selection containing the full-cache support gives the same output
    support = sorted(set((np.nonzero(w[0] > 0)[0] // wl.page_size).tolist()))
    wl.topk = 32
    _, sparse = run_gpu(wl, ekv.EKV_ENTMAX15)
    sel = set(sparse.sel_idx[0, 0, :int(sparse.sel_count[0, 0])].cpu().numpy().tolist())
    if set(support) <= sel:
        close(sparse.out[0].double().cpu().numpy(), out_o, False)
    # and by construction: select support pages plus others directly
    keep = sorted(set(support) | set(range(0, n_pages, 11)))
    sel_idx = torch.full((1, 1, len(keep)), -1, dtype=torch.int32, device="cuda")
    sel_idx[0, 0] = torch.tensor(keep, dtype=torch.int32)
    cnt = torch.tensor([[len(keep)]], dtype=torch.int32, device="cuda")
    out = torch.empty((1, 1, 64), device="cuda")
    stat = torch.empty((1, 1), device="cuda")
    ws = torch.empty(ekv.ekv_decode_workspace_bytes(cache, 1, len(keep)), dtype=torch.uint8, device="cuda")
    ekv.ekv_sparse_decode(cache, wl.q, 1, 1.0, ekv.EKV_ENTMAX15, sel_idx, cnt, len(keep), out, stat, ws)
    torch.cuda.synchronize()
    close(out[0].double().cpu().numpy(), out_o, False)


@pytest.mark.parametrize("name,heads", [
    ("gqa32k", [(0, 0), (3, 7)]),
    ("needle128k", [(0, 0), (5, 3), (7, 7)]),
    ("gauss", [(0, 0), (9, 4), (15, 7)]),
    ("long1m", [(0, 0), (0, 5)]),
])
def test_named_workload_sampled_heads(cuda_device, name, heads):
    wl = make(name, device="cuda")
    cache = make_cache(wl)
    prefill_metadata(cache, wl)
    if wl.append is not None:  # the decode step appends the last page and refreshes its metadata
        start, count = wl.append
        st = torch.full((wl.batch,), start, dtype=torch.int32, device="cuda")
        ct = torch.full((wl.batch,), count, dtype=torch.int32, device="cuda")
        ekv.ekv_page_meta_update(cache, st, ct, count)
    for attn in wl.attn_modes:
        _, dec = run_gpu(wl, attn, cache=cache)
        assert_status_ok(cache)
        hcs = {}
        for b, h in heads:
            hc = hcs.setdefault(b, HostCopy(wl, b))
            check_head(wl, cache, dec, b, h, attn, hc=hc)


def test_host_to_host_graph_matches_the_eager_step(cuda_device):
    # the end-to-end path: one graph copies the query in, runs the step, copies outputs out
    wl = make_random(B=2, H_kv=2, G=4, d=128, P=16, lens=(3000, 1111), dtype=torch.bfloat16,
                     device="cuda", seed=31, topk=40)
    cache, dec = run_gpu(wl, ekv.EKV_ENTMAX15)
    out_ref, stat_ref = dec.out.clone(), dec.stat.clone()
    q_dev = torch.empty_like(wl.q)
    q_host = wl.q.cpu().pin_memory()
    out_host = torch.empty(dec.out.shape, dtype=dec.out.dtype).pin_memory()
    stat_host = torch.empty(dec.stat.shape, dtype=dec.stat.dtype).pin_memory()
    g = dec.capture_host(q_dev, q_host, out_host, stat_host)
    for _ in range(2):
        g.replay()
        torch.cuda.synchronize()
    assert_status_ok(cache)
    assert torch.equal(out_host, out_ref.cpu()) and torch.equal(stat_host, stat_ref.cpu())


# ------------------------------------------------------------------ edge cases
def test_edge_lengths_and_budgets(cuda_device):
    # empty sequence, one token, exactly one page, k >= n_pages
    wl = make_random(B=4, H_kv=2, G=2, d=64, P=16, lens=(0, 1, 16, 40), dtype=torch.float32,
                     device="cuda", seed=11, topk=3)
    for attn in ATTN:
        cache, dec = run_gpu(wl, attn)
        assert_status_ok(cache)
        assert dec.sel_count[0].tolist() == [0, 0]
        assert torch.all(dec.out[0] == 0) and torch.all(torch.isinf(dec.stat[0]))
        for b in (1, 2, 3):
            for h in range(2):
                check_head(wl, cache, dec, b, h, attn)


@pytest.mark.parametrize("dtype,d", [(torch.float32, 64), (torch.bfloat16, 128)], ids=["f32", "bf16"])
def test_every_sequence_empty(cuda_device, dtype, d):
    # a batch whose sequences all hold no token: every step kernel runs with nothing to do
    wl = make_random(B=3, H_kv=2, G=4, d=d, P=16, lens=(0, 0, 0), dtype=dtype, device="cuda",
                     seed=14, topk=8)
    for attn in ATTN:
        cache, dec = run_gpu(wl, attn)
        assert_status_ok(cache)
        assert torch.all(dec.sel_count == 0)
        assert torch.all(dec.out == 0) and torch.all(torch.isinf(dec.stat)) and torch.all(dec.stat < 0)


def test_tie_storm_prefers_lower_pages(cuda_device):
    wl = make_random(B=2, H_kv=2, G=4, d=128, P=16, lens=(4096, 3000), dtype=torch.bfloat16,
                     device="cuda", seed=12, topk=37)
    wl.k_cache.fill_(0.5)  # every page has the same bound
    cache, dec = run_gpu(wl, ekv.EKV_ENTMAX15)
    assert_status_ok(cache)
    for b in range(2):
        for h in range(2):
            np.testing.assert_array_equal(dec.sel_idx[b, h, :37].cpu().numpy(), np.arange(37))
            check_head(wl, cache, dec, b, h, ekv.EKV_ENTMAX15)


# Page counts on each side of the selection kernels' size classes: keys held in registers, 8
# or 16 per thread (up to 8192 and 16384 pages), and keys staged in shared memory or read
# from L2 beyond that.
SEL_SIZES = [8192, 8193, 12000, 16384, 20000]


@pytest.mark.parametrize("pages", SEL_SIZES, ids=["pages%d" % n for n in SEL_SIZES])
def test_topk_selection_at_each_key_count(cuda_device, pages):
    P = 16
    lens = (pages * P - 3, pages * P // 3 + 5)
    wl = make_random(B=2, H_kv=1, G=2, d=64, P=P, lens=lens, dtype=torch.bfloat16,
                     device="cuda", seed=pages, topk=333)
    cache, dec = run_gpu(wl, ekv.EKV_ENTMAX15)
    assert_status_ok(cache)
    for b in range(2):
        check_head(wl, cache, dec, b, 0, ekv.EKV_ENTMAX15)


@pytest.mark.parametrize("pages", [512, 12000, 20000], ids=["pages512", "pages12000", "pages20000"])
def test_tie_storm_heavy_boundary(cuda_device, pages):
    # every page has the same bound, so the boundary holds more ties than the exact ranking
    # takes: the radix path decides, keeping the lowest pages
    P = 16
    wl = make_random(B=1, H_kv=1, G=2, d=64, P=P, lens=(pages * P,), dtype=torch.bfloat16,
                     device="cuda", seed=7, topk=301)
    wl.k_cache.fill_(0.5)
    cache, dec = run_gpu(wl, ekv.EKV_SOFTMAX)
    assert_status_ok(cache)
    np.testing.assert_array_equal(dec.sel_idx[0, 0, :301].cpu().numpy(), np.arange(301))
    check_head(wl, cache, dec, 0, 0, ekv.EKV_SOFTMAX)


def test_bad_page_table_entry_is_flagged_not_trapped(cuda_device):
    wl = make_random(B=2, H_kv=2, G=2, d=64, P=16, lens=(300, 200), dtype=torch.float32,
                     device="cuda", seed=13, topk=4)
    cache = make_cache(wl)
    prefill_metadata(cache, wl)
    assert_status_ok(cache)
    wl.page_table[1, 3] = wl.k_cache.shape[0] + 5  # out of range
    _, dec = run_gpu(wl, ekv.EKV_SOFTMAX, cache=cache)
    st, bits = ekv.ekv_device_status(cache)
    assert st == ekv.EKV_ERR_DEVICE and bits & ekv.EKV_DEV_BAD_BLOCK
    ekv.ekv_clear_device_status(cache)
    assert ekv.ekv_device_status(cache)[0] == ekv.EKV_OK
    # sequence 0 is untouched by the bad entry
    check_head(wl, cache, dec, 0, 1, ekv.EKV_SOFTMAX)


def test_bounded_wait_gives_up_and_reports_a_timeout(cuda_device):
    # the device-side timeout path on its own: a wait on a barrier nothing completes gives up
    # after 1 ms, sets EKV_DEV_TIMEOUT and returns; the context stays usable
    wl = make_random(B=2, H_kv=2, G=4, d=128, P=16, lens=(700, 300), dtype=torch.bfloat16,
                     device="cuda", seed=14, topk=8)
    cache = make_cache(wl)
    prefill_metadata(cache, wl)
    ekv.ekv_clear_device_status(cache)
    ekv.ekv_wait_selftest(cache, 1_000_000)
    st, bits = ekv.ekv_device_status(cache)
    assert st == ekv.EKV_ERR_DEVICE and bits == ekv.EKV_DEV_TIMEOUT
    ekv.ekv_clear_device_status(cache)
    _, dec = run_gpu(wl, ekv.EKV_ENTMAX15, cache=cache)
    assert_status_ok(cache)
    check_head(wl, cache, dec, 1, 1, ekv.EKV_ENTMAX15)


def test_bad_selection_is_flagged(cuda_device):
    wl = make_random(B=1, H_kv=1, G=1, d=64, P=16, lens=(100,), dtype=torch.float32,
                     device="cuda", seed=14)
    cache = make_cache(wl)
    prefill_metadata(cache, wl)
    sel = torch.tensor([[[0, 99]]], dtype=torch.int32, device="cuda")
    cnt = torch.tensor([[2]], dtype=torch.int32, device="cuda")
    out = torch.empty((1, 1, 64), device="cuda")
    stat = torch.empty((1, 1), device="cuda")
    ws = torch.empty(ekv.ekv_decode_workspace_bytes(cache, 1, 2), dtype=torch.uint8, device="cuda")
    ekv.ekv_sparse_decode(cache, wl.q, 1, 1.0, ekv.EKV_SOFTMAX, sel, cnt, 2, out, stat, ws)
    st, bits = ekv.ekv_device_status(cache)
    assert st == ekv.EKV_ERR_DEVICE and bits & ekv.EKV_DEV_BAD_SEL
    hc = HostCopy(wl, 0)
    ref, _, _ = O.attend_head(hc.k, hc.v, hc.pt, hc.L, 0, hc.q[0], 1.0, O.SOFTMAX, [0])
    close(out[0].double().cpu().numpy(), ref, False)


def test_small_workspace_and_unsupported_shapes_are_refused(cuda_device):
    wl = make_random(B=1, H_kv=1, G=1, d=64, P=16, lens=(64,), dtype=torch.float32,
                     device="cuda", seed=15)
    cache = make_cache(wl)
    sel = torch.zeros((1, 1, 4), dtype=torch.int32, device="cuda")
    cnt = torch.zeros((1, 1), dtype=torch.int32, device="cuda")
    out = torch.empty((1, 1, 64), device="cuda")
    stat = torch.empty((1, 1), device="cuda")
    need = ekv.ekv_decode_workspace_bytes(cache, 1, 4)
    ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(ekv.EkvError) as e:
        ekv.ekv_sparse_decode(cache, wl.q, 1, 1.0, ekv.EKV_SOFTMAX, sel, cnt, 4, out, stat, ws)
    assert e.value.status == ekv.EKV_ERR_WORKSPACE
    with pytest.raises(ekv.EkvError) as e:  # group size 3 is not a supported shape
        ekv.ekv_score_pages(cache, wl.q, 3, 1.0, ekv.EKV_SEL_TOPK,
                            torch.empty(64, device="cuda"))
    assert e.value.status == ekv.EKV_ERR_UNSUPPORTED
    wl2 = make_random(B=1, H_kv=2, G=1, d=64, P=16, lens=(64,), dtype=torch.float32,
                      device="cuda", seed=15)
    with pytest.raises(ekv.EkvError) as e:  # 3 query heads do not split over 2 KV heads
        ekv.ekv_score_pages(make_cache(wl2), wl2.q, 3, 1.0, ekv.EKV_SEL_TOPK,
                            torch.empty(64, device="cuda"))
    assert e.value.status == ekv.EKV_ERR_INVALID_ARG


def test_meta_update_append_equals_from_scratch(cuda_device):
    # grow sequences token by token in uneven increments; incremental upkeep must equal a
    # from-scratch build (and the oracle)
    wl = make_random(B=3, H_kv=2, G=2, d=128, P=16, lens=(150, 77, 16), dtype=torch.bfloat16,
                     device="cuda", seed=16, policy=GAUSS)
    full = wl.seq_lens.clone()
    cache = make_cache(wl)
    cur = torch.zeros_like(full)
    rng = np.random.default_rng(0)
    while bool((cur < full).any()):
        inc = torch.as_tensor(rng.integers(0, 23, size=3), dtype=torch.int32, device="cuda")
        new = torch.minimum(cur + inc, full)
        wl.seq_lens.copy_(new)
        ekv.ekv_page_meta_update(cache, cur, new - cur, 22)
        cur = new
    assert_status_ok(cache)
    ref = make_cache(wl)
    prefill_metadata(ref, wl)
    torch.cuda.synchronize()
    for b in range(3):
        n = (int(full[b]) + 15) // 16
        blocks = wl.page_table[b, :n].long()
        assert torch.equal(cache.meta_bbox[blocks], ref.meta_bbox[blocks])
        assert torch.allclose(cache.meta_mom[blocks], ref.meta_mom[blocks], rtol=1e-6, atol=1e-6)
    from parity_utils import check_meta
    for b in range(3):
        hc = HostCopy(wl, b)
        for h in range(2):
            check_meta(cache, hc, h, O.page_meta_head(hc.k, hc.pt, hc.L, h))
