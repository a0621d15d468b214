"""GPU parity of token-level selection inside the selected pages and of the attention indexed
through the page table (after the JSSA abstract): the kept tokens against the oracle's top-T
(equal except near-ties, and in candidate order), and the outputs against the oracle fed the
GPU's own token list, in all three attention modes."""
import itertools

import numpy as np
import pytest
import torch

import oracle as O
from sparse_kv_cache_kmin_b200 import ekv
from sparse_kv_cache_kmin_b200.workloads import make_random
from parity_utils import HostCopy, MODE, close, run_gpu

pytestmark = pytest.mark.gpu

CASES = list(itertools.product([torch.float32, torch.bfloat16], [64, 128], [16, 32], [1, 4, 8],
                               [ekv.EKV_SOFTMAX, ekv.EKV_ENTMAX15, ekv.EKV_SPARSEMAX]))


@pytest.mark.parametrize("dtype,d,P,G,attn", CASES)
def test_token_selection_and_attention_small_ragged(cuda_device, dtype, d, P, G, attn):
    check_tokens(dtype, d, P, G, attn, T=40, lens=(900, 333, 5))


SPLIT = [(torch.bfloat16, 128, 16, 4, ekv.EKV_ENTMAX15), (torch.float32, 64, 32, 8, ekv.EKV_SOFTMAX),
         (torch.bfloat16, 64, 16, 1, ekv.EKV_SPARSEMAX)]


@pytest.mark.parametrize("dtype,d,P,G,attn", SPLIT)
def test_token_row_counts_that_split_a_warp(cuda_device, dtype, d, P, G, attn):
    # 35 and 3 kept tokens: the two halves of a warp stream different numbers of rows (4 at a
    # time, 8 per warp), so their reductions must not wait on each other
    check_tokens(dtype, d, P, G, attn, T=35, lens=(900, 3, 333))


@pytest.mark.parametrize("B,topk", [(16, 128), (32, 128)], ids=["pages32_per_cta", "pages64_per_cta"])
def test_token_scores_with_long_per_cta_runs(cuda_device, B, topk):
    # B x 8 (sequence, KV head) pairs with 128 selected pages: the token scores take 32 or 64
    # selected pages per CTA (the most that leave 3 CTAs per SM), not the 8 of the small cases
    lens = tuple(16 * (140 + 5 * i) + i % 7 for i in range(B))
    check_tokens(torch.bfloat16, 128, 16, 4, ekv.EKV_ENTMAX15, T=512, lens=lens, H=8, topk=topk,
                 heads=[(0, 0), (B // 2, 5), (B - 1, 7)])


def check_tokens(dtype, d, P, G, attn, T, lens, H=2, topk=12, heads=None):
    wl = make_random(B=len(lens), H_kv=H, G=G, d=d, P=P, lens=lens, dtype=dtype, device="cuda",
                     seed=9, topk=topk)
    cache, dec = run_gpu(wl, attn)
    B, H = wl.batch, wl.num_kv_heads
    ws = torch.zeros(ekv.ekv_token_workspace_bytes(cache, dec.max_sel), dtype=torch.uint8, device="cuda")
    tp = torch.empty((B, H, T), dtype=torch.int32, device="cuda")
    tt = torch.empty_like(tp)
    tc = torch.empty((B, H), dtype=torch.int32, device="cuda")
    ekv.ekv_select_tokens(cache, wl.q, wl.num_q_heads, wl.scale, dec.sel_idx, dec.sel_count,
                          dec.max_sel, T, tp, tt, tc, ws)
    out = torch.empty_like(dec.out)
    stat = torch.empty_like(dec.stat)
    ekv.ekv_sparse_decode_tokens(cache, wl.q, wl.num_q_heads, wl.scale, attn, tp, tt, tc, T, out, stat)
    torch.cuda.synchronize()
    st, bits = ekv.ekv_device_status(cache)
    assert st == ekv.EKV_OK, hex(bits)
    bf16 = dtype == torch.bfloat16
    heads = heads or [(b, h) for b in range(B) for h in range(H)]
    for b in sorted({b for b, _ in heads}):
        hc = HostCopy(wl, b)
        for h in [h for bb, h in heads if bb == b]:
            ns = int(dec.sel_count[b, h].item())
            sel = dec.sel_idx[b, h, :ns].cpu().numpy()
            pages, pos = O.token_topk_head(hc.k, hc.pt, hc.L, h, hc.q[h], wl.scale, sel, T)
            n = int(tc[b, h].item())
            assert n == len(pages)
            got = list(zip(tp[b, h, :n].tolist(), tt[b, h, :n].tolist()))
            want = list(zip(pages.tolist(), pos.tolist()))
            assert got == sorted(got, key=lambda x: (list(sel).index(x[0]), x[1]))  # candidate order
            if got != want:
                # only near-ties may differ: every token in the symmetric difference scores
                # within 1e-6 (relative) of the T-th best oracle score
                rows = {}
                for j in sel:
                    for t in range(min(wl.page_size, hc.L - int(j) * wl.page_size)):
                        kv = hc.k[hc.pt[j], h, t]
                        kv = kv.astype(np.float64) if kv.dtype == np.float32 else \
                            (kv.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
                        rows[(int(j), t)] = wl.scale * float(hc.q[h].sum(axis=0) @ kv)
                kth = sorted(rows.values(), reverse=True)[len(want) - 1]
                for x in set(got) ^ set(want):
                    assert abs(rows[x] - kth) <= 1e-6 * max(1.0, abs(kth)), (x, rows[x], kth)
            gp = np.array([p for p, _ in got], np.int32)
            gt = np.array([t for _, t in got], np.int32)
            ref, rstat = O.attend_tokens_head(hc.k, hc.v, hc.pt, hc.L, h, hc.q[h], wl.scale,
                                              MODE[attn], gp, gt)
            close(out[b, h * G:(h + 1) * G].double().cpu().numpy(), ref, bf16)
            close(stat[b, h * G:(h + 1) * G].double().cpu().numpy(), rstat, bf16)


def test_bad_page_table_entry_is_flagged_by_token_selection(cuda_device):
    # a selected page whose page-table entry is out of range: its tokens score -inf (never
    # kept) and EKV_DEV_BAD_BLOCK is raised; a selected page outside the sequence raises
    # EKV_DEV_BAD_SEL
    wl = make_random(B=1, H_kv=2, G=2, d=64, P=16, lens=(200,), dtype=torch.float32,
                     device="cuda", seed=31, topk=4)
    cache, dec = run_gpu(wl, ekv.EKV_SOFTMAX)
    assert ekv.ekv_device_status(cache)[0] == ekv.EKV_OK
    wl.page_table[0, 3] = wl.k_cache.shape[0] + 5
    sel = torch.tensor([[[0, 3, 5, -1], [1, 2, 3, -1]]], dtype=torch.int32, device="cuda")
    cnt = torch.tensor([[3, 3]], dtype=torch.int32, device="cuda")
    T = 48
    ws = torch.empty(ekv.ekv_token_workspace_bytes(cache, 4), dtype=torch.uint8, device="cuda")
    tp = torch.empty((1, 2, T), dtype=torch.int32, device="cuda")
    tt = torch.empty_like(tp)
    tc = torch.empty((1, 2), dtype=torch.int32, device="cuda")
    ekv.ekv_select_tokens(cache, wl.q, wl.num_q_heads, wl.scale, sel, cnt, 4, T, tp, tt, tc, ws)
    st, bits = ekv.ekv_device_status(cache)
    assert st == ekv.EKV_ERR_DEVICE and bits & ekv.EKV_DEV_BAD_BLOCK, hex(bits)
    # only the two good pages' 32 tokens are candidates, and page 3 is never kept
    assert tc.tolist() == [[32, 32]]
    assert 3 not in tp[0, :, :32].unique().tolist()
    ekv.ekv_clear_device_status(cache)
    bad = torch.tensor([[[0, 99, -1, -1], [1, -1, -1, -1]]], dtype=torch.int32, device="cuda")
    ekv.ekv_select_tokens(cache, wl.q, wl.num_q_heads, wl.scale, bad,
                          torch.tensor([[2, 1]], dtype=torch.int32, device="cuda"), 4, T, tp, tt,
                          tc, ws)
    st, bits = ekv.ekv_device_status(cache)
    assert st == ekv.EKV_ERR_DEVICE and bits & ekv.EKV_DEV_BAD_SEL, hex(bits)
