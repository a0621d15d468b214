"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI, move the
inputs to the host, run the oracle on the same inputs, and compare.

Tolerances (derived from the arithmetic; u = 2^-24 is the fp32 unit roundoff):
  kmin/kmax                  bit-exact (min/max of stored values)
  mean, variance (fp32, two-pass over n tokens)
                             |err| <= 4 n u max|x|   and   4 n u max|x - mean|^2 (+ mean's error)
  top-k group bound          S = scale (Q+ . kmax + Q- . kmin) in fp32 with Q+- summed over G:
                             |err| <= 2 (2d + G + 1) u T,  T = scale sum_c |Q+_c||kmax_c| + |Q-_c||kmin_c|
  Gaussian UB, m, v          |err| <= 2 (2d + 2) u times the sum of the magnitudes of the terms
  top-k selection            bit-exact on the GPU's own scores; against the oracle's float64
                             scores, pages in the symmetric difference must be ties within 1e-6
                             of the k-th score (relative)
  Gaussian tau-hat           on the GPU's own m, v: within 1e-6 max(1, |tau|) of the oracle's
                             tau-hat on those statistics (the solver). On the oracle's own m, v:
                             that, plus twice the first-order propagation of the m, v bounds
                             above: |d tau| <= sum_j n_j (E_a |da_j| + E_b |db_j|) / sum_j n_j E_a,
                             E_a, E_b the derivatives of the truncated moment in a and b
  Gaussian selection         bit-exact on the GPU's own statistics and tau-hat; against the
                             oracle's, a page in the symmetric difference must lie within
                             (alpha-1) |d stat| + |d tau| + 1e-6 max(1, |tau|) of the threshold
  attention output / stat    fp32 inputs: 1e-5 absolute; bf16 inputs: 2e-2 relative + 5e-3 absolute
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle as O
from sparse_kv_cache_kmin_b200 import ekv
from sparse_kv_cache_kmin_b200.decoder import SparseDecoder
from sparse_kv_cache_kmin_b200.workloads import GAUSS, GAUSS_MAX, TOPK

U = 2.0 ** -24
MODE = {ekv.EKV_SOFTMAX: O.SOFTMAX, ekv.EKV_ENTMAX15: O.ENTMAX15, ekv.EKV_SPARSEMAX: O.SPARSEMAX}


def to_host(t: torch.Tensor) -> np.ndarray:
    """Cache tensor -> numpy float32, or uint16 bf16 bit patterns (exact)."""
    t = t.detach()
    if t.dtype == torch.bfloat16:
        return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    return t.contiguous().cpu().numpy()


def widen(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().double().cpu().numpy()


def make_cache(wl, gaussian=None):
    gaussian = wl.policy in (GAUSS, GAUSS_MAX) if gaussian is None else gaussian
    nb, H, P, d = wl.k_cache.shape
    dev = wl.k_cache.device
    return ekv.PagedKVCache(
        k_cache=wl.k_cache, v_cache=wl.v_cache,
        meta_bbox=torch.full((nb, H, 2, d), float("nan"), dtype=wl.k_cache.dtype, device=dev),
        meta_mom=torch.full((nb, H, 2, d), float("nan"), dtype=torch.float32, device=dev) if gaussian else None,
        page_table=wl.page_table, seq_lens=wl.seq_lens,
        dev_status=torch.zeros(1, dtype=torch.int32, device=dev))


def prefill_metadata(cache, wl):
    B = wl.batch
    zeros = torch.zeros(B, dtype=torch.int32, device=wl.k_cache.device)
    max_new = int(wl.seq_lens.max().item()) if B else 0
    ekv.ekv_page_meta_update(cache, zeros, wl.seq_lens, max_new)


def run_gpu(wl, attn, cache=None, max_sel=None):
    """One decode step through the C ABI; a new cache gets its metadata built first."""
    if cache is None:
        cache = make_cache(wl)
        prefill_metadata(cache, wl)
    dec = SparseDecoder(cache, wl.num_q_heads, wl.policy, attn, topk=wl.topk, alpha=wl.alpha,
                        delta=wl.delta, scale=wl.scale, max_sel=max_sel)
    dec.step(wl.q)
    torch.cuda.synchronize()
    return cache, dec


class HostCopy:
    """Host copies of one sequence's blocks (all heads), with the page table renumbered."""

    def __init__(self, wl, b):
        P = wl.page_size
        self.L = int(wl.seq_lens[b].item())
        self.np = (self.L + P - 1) // P
        blocks = wl.page_table[b, :self.np].long()
        self.blocks = blocks
        self.k = to_host(wl.k_cache[blocks])
        self.v = to_host(wl.v_cache[blocks])
        self.pt = np.arange(self.np, dtype=np.int32)
        G = wl.num_q_heads // wl.num_kv_heads
        self.G = G
        self.q = widen(wl.q[b]).reshape(wl.num_kv_heads, G, -1)


def gpu_meta(cache, hc, h):
    bbox = cache.meta_bbox[hc.blocks, h].float().double().cpu().numpy()
    mom = cache.meta_mom[hc.blocks, h].double().cpu().numpy() if cache.meta_mom is not None else None
    return bbox, mom


def check_meta(cache, hc, h, meta):
    kmin, kmax, mean, var = meta
    bbox, mom = gpu_meta(cache, hc, h)
    np.testing.assert_array_equal(bbox[:, 0], kmin)
    np.testing.assert_array_equal(bbox[:, 1], kmax)
    if mom is not None:
        P = hc.k.shape[2]
        kv = hc.k if hc.k.dtype == np.float32 else (hc.k.astype(np.uint32) << 16).view(np.float32)
        rows = kv[:, h].astype(np.float64)  # [np, P, d]
        n = np.array([min(P, hc.L - j * P) for j in range(hc.np)])
        mask = np.arange(P)[None, :] < n[:, None]
        amax = np.where(mask[..., None], np.abs(rows), 0).max(1)
        dev = np.where(mask[..., None], np.abs(rows - mean[:, None, :]), 0).max(1)
        tol_m = 4 * n[:, None] * U * amax + 1e-30
        tol_v = 4 * n[:, None] * U * dev * dev + 2 * dev * tol_m + 1e-30
        assert np.all(np.abs(mom[:, 0] - mean) <= tol_m)
        assert np.all(np.abs(mom[:, 1] - var) <= tol_v)


def topk_score_tol(q_group, kmin, kmax, scale):
    d = q_group.shape[1]
    G = q_group.shape[0]
    Qp = np.maximum(q_group, 0).sum(0)
    Qm = np.minimum(q_group, 0).sum(0)
    T = scale * (np.abs(kmax) @ np.abs(Qp) + np.abs(kmin) @ np.abs(Qm))
    return 2 * (2 * d + G + 1) * U * T + 1e-30


def check_topk_selection(sel_gpu, scores_gpu, S_oracle, k):
    """Bit-exact against the oracle's rule on the GPU's scores; tie-tolerant against the
    oracle's float64 scores."""
    ref_same_inputs = O.topk(scores_gpu.astype(np.float64), k)
    np.testing.assert_array_equal(sel_gpu, ref_same_inputs)
    ref = O.topk(S_oracle, k)
    diff = np.setxor1d(sel_gpu, ref)
    if len(diff):
        kth = np.sort(S_oracle)[::-1][min(k, len(S_oracle)) - 1]
        gap = np.abs(S_oracle[diff] - kth)
        assert np.all(gap <= 1e-6 * abs(kth)), (diff, gap, kth)
    return len(diff)


def tau_sensitivity(m, v, cnt, alpha, tau, dm, dv):
    """First-order bound on how far the root of sum_j n_j E_j(tau) = 1 moves when each page's
    m, v move by at most dm, dv: E_j(tau) = E[(X - tau)_+^p], X ~ N(a, b^2), a = (alpha-1) m,
    b = (alpha-1) sqrt(v). Derivatives (u = (a - tau) / b):
      p = 1: dE/da = Phi(u),              dE/db = phi(u)
      p = 2: dE/da = 2 (r Phi + b phi),   dE/db = 2 b Phi(u)     (r = a - tau)
    and dE/dtau = -dE/da, so |d tau| <= sum n (E_a |da| + E_b |db|) / sum n E_a."""
    from scipy import special
    am1 = alpha - 1.0
    a = am1 * m
    b = am1 * np.sqrt(np.maximum(v, 0.0))
    r = a - tau
    with np.errstate(divide="ignore", invalid="ignore"):
        u = np.where(b > 0, r / np.where(b > 0, b, 1.0), np.sign(r) * np.inf)
    Phi = special.ndtr(u)
    phi = np.where(np.isfinite(u), np.exp(-0.5 * np.where(np.isfinite(u), u, 0.0) ** 2), 0.0) \
        / math.sqrt(2 * math.pi)
    if alpha == 2.0:
        Ea, Eb = Phi, phi
    else:
        Ea, Eb = 2 * (np.maximum(r, 0) * (b == 0) + (r * Phi + b * phi) * (b > 0)), 2 * b * Phi
    da = am1 * dm
    with np.errstate(divide="ignore", invalid="ignore"):
        db = am1 * np.minimum(np.sqrt(dv), np.where(v > 0, dv / (2 * np.sqrt(np.maximum(v, 1e-300))), np.inf))
    den = np.sum(cnt * Ea)
    return np.sum(cnt * (Ea * da + Eb * db)) / den if den > 0 else np.inf


def close(a, b, dtype_bf16):
    if dtype_bf16:
        np.testing.assert_allclose(a, b, rtol=2e-2, atol=5e-3)
    else:
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-5)


def check_head(wl, cache, dec, b, h, attn, hc=None, check_scores=True):
    """Compare every stage for one (sequence, KV head) against the oracle. Returns details."""
    hc = hc or HostCopy(wl, b)
    bf16 = wl.k_cache.dtype == torch.bfloat16
    G = hc.G
    meta = O.page_meta_head(hc.k, hc.pt, hc.L, h)
    check_meta(cache, hc, h, meta)
    kmin, kmax, mean, var = meta
    qg = hc.q[h]
    ub, S = O.score_head(qg, wl.scale, kmin, kmax)
    n_sel = int(dec.sel_count[b, h].item())
    sel_gpu = dec.sel_idx[b, h, :n_sel].cpu().numpy()
    assert np.all(dec.sel_idx[b, h, n_sel:].cpu().numpy() == -1)
    info = {}
    if wl.policy == TOPK:
        sg = dec.scores[b, h, :hc.np].double().cpu().numpy()
        if check_scores:
            tol = topk_score_tol(qg, kmin, kmax, wl.scale)
            assert np.all(np.abs(sg - S) <= tol), np.max(np.abs(sg - S) - tol)
        info["sel_diff"] = check_topk_selection(sel_gpu, sg, S, wl.topk)
    else:
        m, v = O.gauss_stats_head(qg, wl.scale, mean, var)
        sc = dec.scores[b, h * G:(h + 1) * G, :, :hc.np].double().cpu().numpy()  # [G, 3, np]
        d = qg.shape[1]
        Tu = wl.scale * (np.abs(qg) @ np.maximum(np.abs(kmin), np.abs(kmax)).T)
        Tm = wl.scale * (np.abs(qg) @ np.abs(mean).T)
        Tv = wl.scale ** 2 * ((qg * qg) @ np.abs(var).T)
        f = 2 * (2 * d + 2) * U
        # m and v also carry the fp32 rounding of the page mean / variance they read
        P = wl.page_size
        kabs = np.maximum(np.abs(kmin), np.abs(kmax))
        Tk2 = wl.scale ** 2 * ((qg * qg) @ (kabs * kabs).T)
        tol_u = f * Tu + 1e-30
        tol_m = f * Tm + 4 * P * U * Tu + 1e-30
        tol_v = f * Tv + 24 * P * U * Tk2 + 1e-30
        if check_scores:
            assert np.all(np.abs(sc[:, 0] - ub) <= tol_u)
            assert np.all(np.abs(sc[:, 1] - m) <= tol_m)
            assert np.all(np.abs(sc[:, 2] - v) <= tol_v)
        cnt = O.page_counts(hc.L, wl.page_size)
        tau_o = np.array([O.gauss_tau(m[g], v[g], cnt, wl.alpha) for g in range(G)])
        tau_g = dec.tau_hat[b, h * G:(h + 1) * G].double().cpu().numpy()
        # the solver: the oracle's tau-hat on the GPU's own statistics (float64 of its floats)
        tau_same = np.array([O.gauss_tau(sc[g, 1], sc[g, 2], cnt, wl.alpha) for g in range(G)])
        assert np.all(np.abs(tau_g - tau_same) <= 1e-6 * np.maximum(1, np.abs(tau_same))), \
            (tau_g, tau_same)
        # end to end: plus the propagated error of the GPU's fp32 statistics
        tol_tau = np.array([1e-6 * max(1.0, abs(tau_o[g])) +
                            2 * tau_sensitivity(m[g], v[g], cnt, wl.alpha, tau_o[g], tol_m[g], tol_v[g])
                            for g in range(G)])
        assert np.all(np.abs(tau_g - tau_o) <= tol_tau), (tau_g, tau_o, tol_tau)
        # the GPU's decision on its own statistics and tau-hat is the oracle's rule, exactly
        tau_gf = tau_g.astype(np.float32).astype(np.float64)
        if wl.policy == GAUSS_MAX:
            same = O.gauss_select_est(sc[:, 0], sc[:, 1], sc[:, 2], cnt, tau_gf, wl.alpha, wl.delta)
            ref = O.gauss_select_est(ub, m, v, cnt, tau_o, wl.alpha, wl.delta)
            stat_o = np.array([[O.est_max(ub[g, j], m[g, j], v[g, j], cnt[j]) for j in range(ub.shape[1])]
                               for g in range(G)])
            zn = np.sqrt(2 * np.log(np.maximum(cnt, 1)))
            tol_stat = np.maximum(tol_u, tol_m + zn[None, :] * np.sqrt(tol_v))
        else:
            same = O.gauss_select(sc[:, 0], tau_gf, wl.alpha, wl.delta)
            ref = O.gauss_select(ub, tau_o, wl.alpha, wl.delta)
            stat_o = ub
            tol_stat = tol_u
        np.testing.assert_array_equal(sel_gpu, same)
        diff = np.setxor1d(sel_gpu, ref)
        if len(diff):
            # a page decided differently must lie, for the query whose decision flips, within the
            # statistic's and tau-hat's error of the threshold
            margin = (wl.alpha - 1) * stat_o[:, diff] - (tau_o[:, None] - wl.delta)
            tol = (wl.alpha - 1) * tol_stat[:, diff] + tol_tau[:, None] + \
                1e-6 * np.maximum(1, np.abs(tau_o))[:, None]
            assert np.all((np.abs(margin) <= tol).any(0)), (diff, margin, tol)
        info["sel_diff"] = len(diff)
        info["kept"] = n_sel
    out_o, stat_o, _ = O.attend_head(hc.k, hc.v, hc.pt, hc.L, h, qg, wl.scale, MODE[attn], sel_gpu)
    out_g = dec.out[b, h * G:(h + 1) * G].double().cpu().numpy()
    stat_g = dec.stat[b, h * G:(h + 1) * G].double().cpu().numpy()
    close(out_g, out_o, bf16)
    fin = np.isfinite(stat_o)
    assert np.array_equal(fin, np.isfinite(stat_g))
    close(stat_g[fin], stat_o[fin], bf16)
    info["n_sel"] = n_sel
    return info
