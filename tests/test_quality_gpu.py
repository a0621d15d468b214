"""GPU parity of the selection-quality diagnostics (EntmaxKV summary §3-§4): the full-cache
weight outside the selected pages (delta) and the support counts, against the oracle's
``selection_quality_head`` fed the same full-cache statistic, on small ragged cases and on
sampled heads of the needle workload at full size.

Tolerances come from the fp32 logits: s = scale q.k carries at most
eps_s = 2 (d + 2) u scale sum_c |q_c k_c| (u = 2^-24), so z = (alpha-1) s carries
eps_z = (alpha-1) eps_s, and each weight moves by at most
  softmax      p (eps_s + 2^-21)                 (exp of a perturbed exponent)
  sparsemax    eps_z + u |r|                     (p = r, r = z - tau)
  1.5-entmax   2 |r| eps_z + eps_z^2 + 2 u r^2   (p = r^2)
for tokens with r > -eps_z (the rest weigh zero on both sides). The counts may differ only by
tokens within eps_z of the threshold."""
import itertools

import numpy as np
import pytest
import torch

import oracle as O
from sparse_kv_cache_kmin_b200 import ekv
from sparse_kv_cache_kmin_b200.workloads import make, make_random
from parity_utils import HostCopy, MODE, U, make_cache, prefill_metadata, run_gpu

pytestmark = pytest.mark.gpu


def full_cache_stat(wl, cache, attn):
    """The full-cache statistic: ekv_sparse_decode with every page of every sequence selected."""
    B, H, P = wl.batch, wl.num_kv_heads, wl.page_size
    mp = int(wl.page_table.shape[1])
    n_pages = ((wl.seq_lens.long() + P - 1) // P).to(torch.int32)
    sel = torch.arange(mp, dtype=torch.int32, device="cuda").expand(B, H, mp).contiguous()
    sel = torch.where(sel < n_pages.view(B, 1, 1), sel, torch.full_like(sel, -1))
    cnt = n_pages.view(B, 1).expand(B, H).contiguous()
    out = torch.empty((B, wl.num_q_heads, wl.head_dim), device="cuda")
    stat = torch.empty((B, wl.num_q_heads), device="cuda")
    ws = torch.empty(ekv.ekv_decode_workspace_bytes(cache, wl.num_q_heads, mp), dtype=torch.uint8,
                     device="cuda")
    ekv.ekv_sparse_decode(cache, wl.q, wl.num_q_heads, wl.scale, attn, sel, cnt, mp, out, stat, ws)
    return stat


def gpu_quality(wl, cache, dec, attn, stat_full):
    B, Hq = wl.batch, wl.num_q_heads
    dropped = torch.full((B, Hq), float("nan"), dtype=torch.float64, device="cuda")
    support = torch.full((B, Hq, 2), -1, dtype=torch.int32, device="cuda")
    ekv.ekv_selection_quality(cache, wl.q, Hq, wl.scale, attn, stat_full, dec.sel_idx,
                              dec.sel_count, dec.max_sel, dropped, support)
    torch.cuda.synchronize()
    return dropped.cpu().numpy(), support.cpu().numpy()


def dense_keys(hc, h):
    k = hc.k[:, h]  # [np, P, d] in page order (the host copy renumbers the blocks)
    k = k.astype(np.float64) if k.dtype == np.float32 else \
        (k.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return k.reshape(-1, k.shape[-1])[:hc.L]


def check_quality_head(wl, hc, h, attn, sel, stat_g, dropped_g, support_g):
    G, P = hc.G, wl.page_size
    alpha = O.ALPHA_OF_MODE[MODE[attn]]
    d_o, ns_o, nk_o = O.selection_quality_head(hc.k, hc.v, hc.pt, hc.L, h, hc.q[h], wl.scale,
                                               MODE[attn], sel, stat=stat_g)
    K = dense_keys(hc, h)
    in_sel = np.isin(np.arange(hc.L) // P, sel)
    d = K.shape[1]
    for g in range(G):
        q = hc.q[h][g]
        s = wl.scale * K @ q
        eps_s = 2 * (d + 2) * U * wl.scale * (np.abs(K) @ np.abs(q)) + 1e-30
        if attn == ekv.EKV_SOFTMAX:
            p = np.exp(s - stat_g[g])
            bound = p * (eps_s + 2.0 ** -21)
            ambiguous = np.zeros(len(s), bool)
        else:
            eps_z = (alpha - 1) * eps_s
            r = (alpha - 1) * s - stat_g[g]
            live = r > -eps_z
            if attn == ekv.EKV_SPARSEMAX:
                bound = np.where(live, eps_z + U * np.abs(r), 0.0)
            else:
                bound = np.where(live, 2 * np.abs(r) * eps_z + eps_z ** 2 + 2 * U * r * r, 0.0)
            ambiguous = np.abs(r) <= eps_z
        tol = bound[~in_sel].sum() + 1e-12
        assert abs(dropped_g[g] - d_o[g]) <= tol, (g, dropped_g[g], d_o[g], tol)
        amb, amb_in = int(ambiguous.sum()), int((ambiguous & in_sel).sum())
        assert abs(int(support_g[g, 0]) - int(ns_o[g])) <= amb, (support_g[g], ns_o[g], amb)
        assert abs(int(support_g[g, 1]) - int(nk_o[g])) <= amb_in, (support_g[g], nk_o[g], amb_in)
    return d_o, ns_o, nk_o


CASES = list(itertools.product([torch.float32, torch.bfloat16], [64, 128], [16, 32], [1, 4, 8],
                               [ekv.EKV_SOFTMAX, ekv.EKV_ENTMAX15, ekv.EKV_SPARSEMAX]))


@pytest.mark.parametrize("dtype,d,P,G,attn", CASES,
                         ids=["%s-d%d-P%d-G%d-a%d" % (str(t)[6:], d, P, G, a) for t, d, P, G, a in CASES])
def test_selection_quality_small_ragged(cuda_device, dtype, d, P, G, attn):
    # lengths that span several CTA slices (256 pages) and end on partial pages
    lens = (256 * P + 3 * P + 5, 700, 1)
    wl = make_random(B=3, H_kv=2, G=G, d=d, P=P, lens=lens, dtype=dtype, device="cuda",
                     seed=300 + d + P + G, kv_scale=1.5, topk=40)
    cache, dec = run_gpu(wl, attn)
    stat_full = full_cache_stat(wl, cache, attn)
    dropped, support = gpu_quality(wl, cache, dec, attn, stat_full)
    st, bits = ekv.ekv_device_status(cache)
    assert st == ekv.EKV_OK, hex(bits)
    for b in range(wl.batch):
        hc = HostCopy(wl, b)
        for h in range(wl.num_kv_heads):
            sel = dec.sel_idx[b, h, :int(dec.sel_count[b, h])].cpu().numpy()
            sl = slice(h * G, (h + 1) * G)
            check_quality_head(wl, hc, h, attn, sel, stat_full[b, sl].double().cpu().numpy(),
                               dropped[b, sl], support[b, sl])


def test_selection_quality_all_and_no_pages(cuda_device):
    # every page selected: nothing dropped and every support token kept; nothing selected:
    # everything dropped (the weights sum to one)
    wl = make_random(B=2, H_kv=2, G=4, d=128, P=16, lens=(3000, 999), dtype=torch.bfloat16,
                     device="cuda", seed=310, kv_scale=1.5, topk=10_000)
    for attn in [ekv.EKV_SOFTMAX, ekv.EKV_ENTMAX15, ekv.EKV_SPARSEMAX]:
        cache, dec = run_gpu(wl, attn)
        stat_full = full_cache_stat(wl, cache, attn)
        dropped, support = gpu_quality(wl, cache, dec, attn, stat_full)
        assert np.all(dropped == 0) and np.array_equal(support[..., 0], support[..., 1])
        dec.sel_count.zero_()
        dropped0, support0 = gpu_quality(wl, cache, dec, attn, stat_full)
        assert np.all(support0[..., 1] == 0) and np.array_equal(support0[..., 0], support[..., 0])
        G = wl.num_q_heads // wl.num_kv_heads
        for b in range(wl.batch):
            hc = HostCopy(wl, b)
            for h in range(wl.num_kv_heads):
                sl = slice(h * G, (h + 1) * G)
                d_o, _, _ = check_quality_head(wl, hc, h, attn, np.zeros(0, np.int32),
                                               stat_full[b, sl].double().cpu().numpy(),
                                               dropped0[b, sl], support0[b, sl])
                # the weights the full-cache statistic defines sum to one, up to that
                # statistic's own rounding (the decode's bf16 tolerance)
                np.testing.assert_allclose(d_o, 1.0, atol=2e-2)


def test_selection_quality_needle_workload_sampled_heads(cuda_device):
    # the full-size 128K needle workload in the benchmark's configuration: every query head of
    # three sampled (sequence, KV head) pairs
    wl = make("needle128k", device="cuda")
    cache = make_cache(wl)
    prefill_metadata(cache, wl)
    _, dec = run_gpu(wl, ekv.EKV_ENTMAX15, cache=cache)
    stat_full = full_cache_stat(wl, cache, ekv.EKV_ENTMAX15)
    dropped, support = gpu_quality(wl, cache, dec, ekv.EKV_ENTMAX15, stat_full)
    G = wl.num_q_heads // wl.num_kv_heads
    for b, h in [(0, 0), (3, 5), (7, 7)]:
        hc = HostCopy(wl, b)
        sel = dec.sel_idx[b, h, :int(dec.sel_count[b, h])].cpu().numpy()
        sl = slice(h * G, (h + 1) * G)
        check_quality_head(wl, hc, h, ekv.EKV_ENTMAX15, sel,
                           stat_full[b, sl].double().cpu().numpy(), dropped[b, sl], support[b, sl])
