"""GPU parity of ekv_select_decode (top-k selection and sparse attention in one call): its
selection equals ekv_select_pages on the same scores bit for bit, and its outputs match the
oracle fed that selection, on ragged cases (sequences shorter than k, heavy ties, the
selection's size classes, cluster sizes) and on the geometries the decode serves with its
chunk kernels (fp32, softmax)."""
import pytest
import torch

from sparse_kv_cache_kmin_b200 import ekv
from sparse_kv_cache_kmin_b200.decoder import SparseDecoder
from sparse_kv_cache_kmin_b200.workloads import TOPK, make, make_random
from parity_utils import check_head, make_cache, prefill_metadata

pytestmark = pytest.mark.gpu


def select_decode_step(wl, attn, cache=None):
    if cache is None:
        cache = make_cache(wl)
        prefill_metadata(cache, wl)
    dec = SparseDecoder(cache, wl.num_q_heads, TOPK, attn, topk=wl.topk, alpha=wl.alpha,
                        scale=wl.scale)
    ekv.ekv_score_pages(cache, wl.q, wl.num_q_heads, wl.scale, TOPK, dec.scores)
    ekv.ekv_select_decode(cache, wl.q, wl.num_q_heads, wl.scale, attn, wl.topk, dec.scores,
                          dec.sel_idx, dec.sel_count, dec.max_sel, dec.out, dec.stat, dec.ws)
    torch.cuda.synchronize()
    return cache, dec


def standalone_selection(cache, wl, dec):
    sel = torch.full_like(dec.sel_idx, 7777)
    cnt = torch.full_like(dec.sel_count, 7777)
    ekv.ekv_select_pages(cache, wl.num_q_heads, TOPK, wl.topk, 1.5, 0.0, dec.scores, sel, cnt,
                         dec.max_sel, dec.tau_hat)
    torch.cuda.synchronize()
    return sel, cnt


def check_all(wl, cache, dec, attn, heads=None):
    st, bits = ekv.ekv_device_status(cache)
    assert st == ekv.EKV_OK, hex(bits)
    sel, cnt = standalone_selection(cache, wl, dec)
    assert torch.equal(dec.sel_count, cnt)
    assert torch.equal(dec.sel_idx, sel)
    pairs = heads or [(b, h) for b in range(wl.batch) for h in range(wl.num_kv_heads)]
    for b, h in pairs:
        check_head(wl, cache, dec, b, h, attn)


CASES = [  # d, P, G, lens, topk
    (128, 16, 4, (1000 * 16 + 7, 200 * 16, 33, 16), 37),
    (64, 32, 8, (3000, 517, 1), 9),
    (128, 64, 1, (64 * 70 + 3, 64 * 3), 5),
    (64, 16, 2, (4096 * 16, 16 * 300 + 5), 256),
]


@pytest.mark.parametrize("attn", [ekv.EKV_ENTMAX15, ekv.EKV_SPARSEMAX])
@pytest.mark.parametrize("d,P,G,lens,topk", CASES, ids=["d%d-P%d-G%d" % c[:3] for c in CASES])
def test_select_decode_matches_selection_and_oracle(cuda_device, d, P, G, lens, topk, attn):
    wl = make_random(B=len(lens), H_kv=2, G=G, d=d, P=P, lens=lens, dtype=torch.bfloat16,
                     device="cuda", seed=d + P + G + topk, kv_scale=1.5, topk=topk)
    cache, dec = select_decode_step(wl, attn)
    check_all(wl, cache, dec, attn)


@pytest.mark.parametrize("B", [1, 3, 20])
def test_select_decode_every_cluster_size(cuda_device, B):
    lens = tuple(16 * (40 + 37 * i) + i for i in range(B))
    wl = make_random(B=B, H_kv=2, G=4, d=128, P=16, lens=lens, dtype=torch.bfloat16,
                     device="cuda", seed=50 + B, topk=24)
    cache, dec = select_decode_step(wl, ekv.EKV_ENTMAX15)
    check_all(wl, cache, dec, ekv.EKV_ENTMAX15, heads=[(0, 0), (B - 1, 1), (B // 2, 0)])


@pytest.mark.parametrize("pages", [8192, 8193], ids=["pages8192", "pages8193"])
def test_select_decode_page_count_limit(cuda_device, pages):
    P = 16
    wl = make_random(B=2, H_kv=1, G=4, d=128, P=P, lens=(pages * P - 5, 1000), dtype=torch.bfloat16,
                     device="cuda", seed=pages, topk=256)
    cache, dec = select_decode_step(wl, ekv.EKV_ENTMAX15)
    check_all(wl, cache, dec, ekv.EKV_ENTMAX15)


def test_select_decode_heavy_ties(cuda_device):
    # every page has the same bound: the kept pages are the lowest ones
    wl = make_random(B=2, H_kv=2, G=4, d=128, P=16, lens=(16 * 3000, 16 * 700 + 3),
                     dtype=torch.bfloat16, device="cuda", seed=61, topk=301)
    wl.k_cache.fill_(0.5)
    cache, dec = select_decode_step(wl, ekv.EKV_ENTMAX15)
    check_all(wl, cache, dec, ekv.EKV_ENTMAX15)
    assert dec.sel_idx[0, 0, :301].tolist() == list(range(301))


@pytest.mark.parametrize("dtype,attn", [(torch.float32, ekv.EKV_ENTMAX15),
                                        (torch.bfloat16, ekv.EKV_SOFTMAX),
                                        (torch.float32, ekv.EKV_SOFTMAX)],
                         ids=["f32-entmax", "bf16-softmax", "f32-softmax"])
def test_select_decode_chunk_kernel_geometries(cuda_device, dtype, attn):
    wl = make_random(B=3, H_kv=2, G=4, d=64, P=16, lens=(5000, 700, 16), dtype=dtype,
                     device="cuda", seed=71, topk=20)
    cache, dec = select_decode_step(wl, attn)
    check_all(wl, cache, dec, attn)


def test_select_decode_bad_page_table_entry_is_flagged(cuda_device):
    wl = make_random(B=2, H_kv=2, G=4, d=128, P=16, lens=(300, 200), dtype=torch.bfloat16,
                     device="cuda", seed=81, topk=40)
    cache = make_cache(wl)
    prefill_metadata(cache, wl)
    wl.page_table[1, 3] = wl.k_cache.shape[0] + 9  # out of range; every page of both is kept
    _, dec = select_decode_step(wl, ekv.EKV_ENTMAX15, cache=cache)
    st, bits = ekv.ekv_device_status(cache)
    assert st == ekv.EKV_ERR_DEVICE and bits & ekv.EKV_DEV_BAD_BLOCK
    ekv.ekv_clear_device_status(cache)
    for h in range(2):
        check_head(wl, cache, dec, 0, h, ekv.EKV_ENTMAX15)


def test_select_decode_needle_workload_sampled_heads(cuda_device):
    wl = make("needle128k", device="cuda")
    cache, dec = select_decode_step(wl, ekv.EKV_ENTMAX15)
    check_all(wl, cache, dec, ekv.EKV_ENTMAX15, heads=[(0, 0), (3, 5), (7, 7)])


def test_select_decode_many_pairs(cuda_device):
    # 72 x 8 (sequence, KV head) pairs, two chunk slots each: one selection CTA per pair and
    # about a quarter of the logits kernel's warps busy
    B = 72
    lens = tuple(16 * (30 + i % 7) + i % 5 for i in range(B))
    wl = make_random(B=B, H_kv=8, G=4, d=128, P=16, lens=lens, dtype=torch.bfloat16,
                     device="cuda", seed=97, topk=16)
    cache, dec = select_decode_step(wl, ekv.EKV_ENTMAX15)
    check_all(wl, cache, dec, ekv.EKV_ENTMAX15, heads=[(0, 0), (B - 1, 7), (35, 3), (50, 6)])
