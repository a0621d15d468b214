"""CPU oracle for query-aware sparse decode over a paged KV cache (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this package. It wraps ``ekv_oracle.c`` -- plain float64 loops that follow the EntmaxKV
technical summary (gist.science), §2.A-§2.C -- with numpy marshalling. It shares nothing with
the CUDA library and never imports it.

Host data conventions (mirroring the paged layout the pages describe in §2):
  k_cache, v_cache  numpy [num_blocks, H_kv, P, d], float32, or uint16 holding bf16 bit patterns
  page_table        int32 [B, max_pages]   logical page j of sequence b lives in block page_table[b, j]
  seq_lens          int32 [B]
  q                 float64 [B, H_q, d]     (bf16/fp32 values widened exactly by the caller)
"""
from __future__ import annotations

import ctypes
import os
import time

import numpy as np

from .build import build_oracle, library_path

SOFTMAX, ENTMAX15, SPARSEMAX = 0, 1, 2
ALPHA_OF_MODE = {SOFTMAX: 1.0, ENTMAX15: 1.5, SPARSEMAX: 2.0}

_lib = None
_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int32)


def _load():
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        build_oracle()
    lib = ctypes.CDLL(path)
    c_int, c_double, vp = ctypes.c_int, ctypes.c_double, ctypes.c_void_p
    lib.ora_page_meta_head.argtypes = [vp, c_int, c_int, c_int, c_int, c_int, _ip, c_int, c_int,
                                       _dp, _dp, _dp, _dp]
    lib.ora_page_meta_head.restype = c_int
    lib.ora_score_head.argtypes = [_dp, c_int, c_int, c_double, _dp, _dp, c_int, _dp, _dp]
    lib.ora_score_head.restype = None
    lib.ora_gauss_stats_head.argtypes = [_dp, c_int, c_int, c_double, _dp, _dp, c_int, _dp, _dp]
    lib.ora_gauss_stats_head.restype = None
    lib.ora_topk.argtypes = [_dp, c_int, c_int, _ip]
    lib.ora_topk.restype = c_int
    lib.ora_trunc_moment.argtypes = [c_double, c_double, c_double, c_double]
    lib.ora_trunc_moment.restype = c_double
    lib.ora_gauss_F.argtypes = [_dp, _dp, _ip, c_int, c_double, c_double]
    lib.ora_gauss_F.restype = c_double
    lib.ora_gauss_tau.argtypes = [_dp, _dp, _ip, c_int, c_double]
    lib.ora_gauss_tau.restype = c_double
    lib.ora_gauss_select.argtypes = [_dp, _dp, c_int, c_int, c_double, c_double, _ip]
    lib.ora_gauss_select.restype = c_int
    lib.ora_est_max.argtypes = [c_double, c_double, c_double, c_int]
    lib.ora_est_max.restype = c_double
    lib.ora_gauss_select_est.argtypes = [_dp, _dp, _dp, _ip, _dp, c_int, c_int, c_double, c_double, _ip]
    lib.ora_gauss_select_est.restype = c_int
    lib.ora_entmax_tau.argtypes = [_dp, c_int, c_double]
    lib.ora_entmax_tau.restype = c_double
    lib.ora_attend_head.argtypes = [vp, vp, c_int, c_int, c_int, c_int, c_int, _ip, c_int, c_int,
                                    _dp, c_int, c_double, c_int, _ip, c_int, _dp, _dp, _dp]
    lib.ora_attend_head.restype = c_int
    lib.ora_moment_corrected_head.argtypes = [vp, vp, c_int, c_int, c_int, c_int, c_int, _ip, c_int,
                                              c_int, _dp, c_int, c_double, _ip, c_int, _dp, _dp]
    lib.ora_moment_corrected_head.restype = c_int
    lib.ora_moment_sums_head.argtypes = [vp, vp, c_int, c_int, c_int, c_int, c_int, _ip, c_int,
                                         c_int, _ip, c_int, _dp, _dp, _dp]
    lib.ora_moment_sums_head.restype = c_int
    lib.ora_token_topk_head.argtypes = [vp, c_int, c_int, c_int, c_int, c_int, _ip, c_int, c_int,
                                        _dp, c_int, c_double, _ip, c_int, c_int, _ip, _ip]
    lib.ora_token_topk_head.restype = c_int
    lib.ora_attend_tokens_head.argtypes = [vp, vp, c_int, c_int, c_int, c_int, c_int, _ip, c_int,
                                           c_int, _dp, c_int, c_double, c_int, _ip, _ip, c_int,
                                           _dp, _dp]
    lib.ora_attend_tokens_head.restype = c_int
    lib.ora_selection_quality_head.argtypes = [vp, vp, c_int, c_int, c_int, c_int, c_int, _ip,
                                               c_int, c_int, _dp, c_int, c_double, c_int, _dp,
                                               _ip, c_int, _dp, _ip, _ip]
    lib.ora_selection_quality_head.restype = c_int
    _lib = lib
    return lib


def _d(a):
    a = np.ascontiguousarray(a, dtype=np.float64)
    return a, a.ctypes.data_as(_dp)


def _i(a):
    a = np.ascontiguousarray(a, dtype=np.int32)
    return a, a.ctypes.data_as(_ip)


def _cache_dtype(arr: np.ndarray) -> int:
    if arr.dtype == np.float32:
        return 0
    if arr.dtype == np.uint16:
        return 1
    raise TypeError("cache must be float32 or uint16 (bf16 bits), got %s" % arr.dtype)


def pages_of(seq_len: int, P: int) -> int:
    return (int(seq_len) + P - 1) // P


# ----------------------------------------------------------------------------- §2.A metadata
def page_meta_head(k_cache: np.ndarray, pt_row, seq_len: int, h: int):
    """kmin, kmax, mean, var ([N_p, d] float64) of every page of one sequence, one KV head."""
    nb, H_kv, P, d = k_cache.shape
    k_cache = np.ascontiguousarray(k_cache)
    n = pages_of(seq_len, P)
    outs = [np.zeros((max(n, 1), d)) for _ in range(4)]
    pt, ptp = _i(pt_row)
    rc = _load().ora_page_meta_head(k_cache.ctypes.data, _cache_dtype(k_cache), nb, H_kv, P, d,
                                    ptp, int(seq_len), int(h),
                                    *[o.ctypes.data_as(_dp) for o in outs])
    if rc < 0:
        raise ValueError("page table entry out of range")
    return tuple(o[:n] for o in outs)


# ----------------------------------------------------------------------------- §2.A scores
def score_head(q, scale: float, kmin, kmax):
    """Per-query bounds UB [G, N_p] and group sums S [N_p]."""
    q, qp = _d(np.atleast_2d(q))
    kmin, kp = _d(kmin)
    kmax, kxp = _d(kmax)
    G, d = q.shape
    n = kmin.shape[0]
    ub = np.zeros((G, max(n, 1)))
    S = np.zeros(max(n, 1))
    _load().ora_score_head(qp, G, d, float(scale), kp, kxp, n, ub.ctypes.data_as(_dp),
                           S.ctypes.data_as(_dp))
    return ub[:, :n], S[:n]


def gauss_stats_head(q, scale: float, mean, var):
    """Gaussian score model per query and page: m, v [G, N_p]."""
    q, qp = _d(np.atleast_2d(q))
    mean, mp = _d(mean)
    var, vp_ = _d(var)
    G, d = q.shape
    n = mean.shape[0]
    m = np.zeros((G, max(n, 1)))
    v = np.zeros((G, max(n, 1)))
    _load().ora_gauss_stats_head(qp, G, d, float(scale), mp, vp_, n, m.ctypes.data_as(_dp),
                                 v.ctypes.data_as(_dp))
    return m[:, :n], v[:, :n]


# ----------------------------------------------------------------------------- §2.B selection
def topk(S, k: int) -> np.ndarray:
    S, sp = _d(S)
    out = np.zeros(max(len(S), 1), dtype=np.int32)
    cnt = _load().ora_topk(sp, len(S), int(k), out.ctypes.data_as(_ip))
    return out[:cnt].copy()


def trunc_moment(a: float, b: float, tau: float, alpha: float) -> float:
    return _load().ora_trunc_moment(float(a), float(b), float(tau), float(alpha))


def gauss_F(m, v, cnt, alpha: float, tau: float) -> float:
    m, mp = _d(m)
    v, vp_ = _d(v)
    cnt, cp = _i(cnt)
    return _load().ora_gauss_F(mp, vp_, cp, len(m), float(alpha), float(tau))


def gauss_tau(m, v, cnt, alpha: float) -> float:
    m, mp = _d(m)
    v, vp_ = _d(v)
    cnt, cp = _i(cnt)
    return _load().ora_gauss_tau(mp, vp_, cp, len(m), float(alpha))


def gauss_select(ub, tau_hat, alpha: float, delta: float) -> np.ndarray:
    ub, up = _d(np.atleast_2d(ub))
    tau_hat, tp = _d(np.atleast_1d(tau_hat))
    G, n = ub.shape
    out = np.zeros(max(n, 1), dtype=np.int32)
    cnt = _load().ora_gauss_select(up, tp, G, n, float(alpha), float(delta),
                                   out.ctypes.data_as(_ip))
    return out[:cnt].copy()


def est_max(ub: float, m: float, v: float, n: int) -> float:
    return _load().ora_est_max(float(ub), float(m), float(v), int(n))


def gauss_select_est(ub, m, v, cnt, tau_hat, alpha: float, delta: float) -> np.ndarray:
    """The Gaussian rule with the capped Gaussian estimate of each page's maximum."""
    ub, up = _d(np.atleast_2d(ub))
    m, mp = _d(np.atleast_2d(m))
    v, vp_ = _d(np.atleast_2d(v))
    cnt, cp = _i(cnt)
    tau_hat, tp = _d(np.atleast_1d(tau_hat))
    G, n = ub.shape
    out = np.zeros(max(n, 1), dtype=np.int32)
    k = _load().ora_gauss_select_est(up, mp, vp_, cp, tp, G, n, float(alpha), float(delta),
                                     out.ctypes.data_as(_ip))
    return out[:k].copy()


# ----------------------------------------------------------------------------- §2.C attention
def entmax_tau(z, alpha: float) -> float:
    z, zp = _d(np.atleast_1d(z))
    return _load().ora_entmax_tau(zp, len(z), float(alpha))


def entmax(z, alpha: float) -> np.ndarray:
    """alpha-entmax probabilities in the z domain: p = [z - tau]_+^(1/(alpha-1))."""
    z = np.asarray(z, dtype=np.float64)
    tau = entmax_tau(z, alpha)
    r = np.maximum(z - tau, 0.0)
    return r if alpha == 2.0 else r * r


def attend_head(k_cache, v_cache, pt_row, seq_len: int, h: int, q, scale: float, mode: int,
                sel, want_weights: bool = False):
    """Attention of the G queries `q` [G, d] of KV head h over the selected logical pages.

    Returns (out [G, d], stat [G], weights [G, n_tok] or None)."""
    nb, H_kv, P, d = k_cache.shape
    k_cache = np.ascontiguousarray(k_cache)
    v_cache = np.ascontiguousarray(v_cache)
    dt = _cache_dtype(k_cache)
    if _cache_dtype(v_cache) != dt:
        raise TypeError("K and V caches must share a dtype")
    q, qp = _d(np.atleast_2d(q))
    G = q.shape[0]
    pt, ptp = _i(pt_row)
    sel, sp = _i(np.asarray(sel, dtype=np.int32).reshape(-1))
    n_tok_max = max(1, len(sel) * P)
    out = np.zeros((G, d))
    stat = np.zeros(G)
    w = np.zeros(G * n_tok_max) if want_weights else None
    rc = _load().ora_attend_head(k_cache.ctypes.data, v_cache.ctypes.data, dt, nb, H_kv, P, d,
                                 ptp, int(seq_len), int(h), qp, G, float(scale), int(mode), sp,
                                 len(sel), out.ctypes.data_as(_dp), stat.ctypes.data_as(_dp),
                                 w.ctypes.data_as(_dp) if w is not None else None)
    if rc < 0:
        raise ValueError("selected page or page-table entry out of range")
    weights = w[:G * rc].reshape(G, rc) if w is not None else None
    return out, stat, weights


def selection_quality_head(k_cache, v_cache, pt_row, seq_len: int, h: int, q, scale: float,
                           mode: int, sel, stat=None):
    """How much of the full-cache attention the selected pages keep, per query of KV head h
    (EntmaxKV summary §3-§4; see ``ora_selection_quality_head``).

    Returns (dropped [G]: full-cache weight outside the selected pages, n_sup [G]: support size
    (entmax) or valid tokens (softmax), n_kept [G]: those inside the selected pages). With
    ``stat`` ([G] full-cache log-partition or tau) the weights are the ones it defines;
    without, the oracle's own full-cache attention."""
    nb, H_kv, P, d = k_cache.shape
    k_cache = np.ascontiguousarray(k_cache)
    v_cache = np.ascontiguousarray(v_cache)
    dt = _cache_dtype(k_cache)
    q, qp = _d(np.atleast_2d(q))
    G = q.shape[0]
    pt, ptp = _i(pt_row)
    sel, sp = _i(np.asarray(sel, dtype=np.int32).reshape(-1))
    st, stp = (None, None) if stat is None else _d(np.asarray(stat, dtype=np.float64).reshape(G))
    dropped = np.zeros(G)
    n_sup = np.zeros(G, np.int32)
    n_kept = np.zeros(G, np.int32)
    rc = _load().ora_selection_quality_head(k_cache.ctypes.data, v_cache.ctypes.data, dt, nb, H_kv,
                                            P, d, ptp, int(seq_len), int(h), qp, G, float(scale),
                                            int(mode), stp, sp, len(sel),
                                            dropped.ctypes.data_as(_dp),
                                            n_sup.ctypes.data_as(_ip), n_kept.ctypes.data_as(_ip))
    if rc < 0:
        raise ValueError("selected page or page-table entry out of range")
    return dropped, n_sup, n_kept


def moment_corrected_head(k_cache, v_cache, pt_row, seq_len: int, h: int, q, scale: float, sel):
    """Softmax over the selected pages, corrected for the skipped ones from their moments
    (MomentKV technical summary, Methodology §1, §2, §4; see ``ora_moment_corrected_head``).

    Returns (out [G, d], stat [G] = log of the estimated partition sum, n_e evicted tokens)."""
    nb, H_kv, P, d = k_cache.shape
    k_cache = np.ascontiguousarray(k_cache)
    v_cache = np.ascontiguousarray(v_cache)
    dt = _cache_dtype(k_cache)
    if _cache_dtype(v_cache) != dt:
        raise TypeError("K and V caches must share a dtype")
    q, qp = _d(np.atleast_2d(q))
    G = q.shape[0]
    pt, ptp = _i(pt_row)
    sel, sp = _i(np.asarray(sel, dtype=np.int32).reshape(-1))
    out = np.zeros((G, d))
    stat = np.zeros(G)
    rc = _load().ora_moment_corrected_head(k_cache.ctypes.data, v_cache.ctypes.data, dt, nb, H_kv,
                                           P, d, ptp, int(seq_len), int(h), qp, G, float(scale),
                                           sp, len(sel), out.ctypes.data_as(_dp),
                                           stat.ctypes.data_as(_dp))
    if rc < 0:
        raise ValueError("selected page or page-table entry out of range")
    return out, stat, rc


def moment_sums_head(k_cache, v_cache, pt_row, seq_len: int, h: int, pages=None):
    """Count, key sum, value sum and value-key outer-product sum S[a][c] = sum v_a k_c over the
    valid tokens of the listed logical pages (all pages when None) of one (sequence, KV head)
    (MomentKV technical summary, Methodology §1). Returns (n, sk [d], sv [d], S [d, d])."""
    nb, H_kv, P, d = k_cache.shape
    k_cache = np.ascontiguousarray(k_cache)
    v_cache = np.ascontiguousarray(v_cache)
    dt = _cache_dtype(k_cache)
    if _cache_dtype(v_cache) != dt:
        raise TypeError("K and V caches must share a dtype")
    if pages is None:
        pages = np.arange(pages_of(seq_len, P))
    pt, ptp = _i(pt_row)
    pg, pgp = _i(np.asarray(pages, dtype=np.int32).reshape(-1))
    sk, sv, S = np.zeros(d), np.zeros(d), np.zeros((d, d))
    n = _load().ora_moment_sums_head(k_cache.ctypes.data, v_cache.ctypes.data, dt, nb, H_kv, P, d,
                                     ptp, int(seq_len), int(h), pgp, len(pg),
                                     sk.ctypes.data_as(_dp), sv.ctypes.data_as(_dp),
                                     S.ctypes.data_as(_dp))
    if n < 0:
        raise ValueError("page or page-table entry out of range")
    return n, sk, sv, S


def token_topk_head(k_cache, pt_row, seq_len: int, h: int, q, scale: float, sel, T: int):
    """Token-level selection inside the selected pages for one KV head (JSSA abstract; see
    ``ora_token_topk_head``): the T candidate tokens with the largest group score
    sum_g scale * q_g . k, ties to the earlier candidate, in candidate order.

    Returns (pages [n] int32, positions [n] int32)."""
    nb, H_kv, P, d = k_cache.shape
    k_cache = np.ascontiguousarray(k_cache)
    q, qp = _d(np.atleast_2d(q))
    pt, ptp = _i(pt_row)
    sel, sp = _i(np.asarray(sel, dtype=np.int32).reshape(-1))
    cap = max(1, len(sel) * P)
    pages = np.zeros(cap, dtype=np.int32)
    pos = np.zeros(cap, dtype=np.int32)
    rc = _load().ora_token_topk_head(k_cache.ctypes.data, _cache_dtype(k_cache), nb, H_kv, P, d,
                                     ptp, int(seq_len), int(h), qp, q.shape[0], float(scale), sp,
                                     len(sel), int(T), pages.ctypes.data_as(_ip),
                                     pos.ctypes.data_as(_ip))
    if rc < 0:
        raise ValueError("selected page or page-table entry out of range")
    return pages[:rc].copy(), pos[:rc].copy()


def attend_tokens_head(k_cache, v_cache, pt_row, seq_len: int, h: int, q, scale: float,
                       mode: int, tok_pages, tok_pos):
    """Attention of the G queries over an explicit (logical page, position) token list, read
    through the page table. Returns (out [G, d], stat [G])."""
    nb, H_kv, P, d = k_cache.shape
    k_cache = np.ascontiguousarray(k_cache)
    v_cache = np.ascontiguousarray(v_cache)
    dt = _cache_dtype(k_cache)
    if _cache_dtype(v_cache) != dt:
        raise TypeError("K and V caches must share a dtype")
    q, qp = _d(np.atleast_2d(q))
    G = q.shape[0]
    pt, ptp = _i(pt_row)
    tp, tpp = _i(np.asarray(tok_pages, dtype=np.int32).reshape(-1))
    tt, ttp = _i(np.asarray(tok_pos, dtype=np.int32).reshape(-1))
    if len(tp) != len(tt):
        raise ValueError("token pages and positions differ in length")
    out = np.zeros((G, d))
    stat = np.zeros(G)
    rc = _load().ora_attend_tokens_head(k_cache.ctypes.data, v_cache.ctypes.data, dt, nb, H_kv, P,
                                        d, ptp, int(seq_len), int(h), qp, G, float(scale),
                                        int(mode), tpp, ttp, len(tp), out.ctypes.data_as(_dp),
                                        stat.ctypes.data_as(_dp))
    if rc < 0:
        raise ValueError("token page, position or page-table entry out of range")
    return out, stat


def page_counts(seq_len: int, P: int) -> np.ndarray:
    """Valid tokens per page of a sequence (the last page may be partial)."""
    n = pages_of(seq_len, P)
    return np.array([min(P, int(seq_len) - j * P) for j in range(n)], dtype=np.int32)


# ----------------------------------------------------------------------------- one decode step
def decode_step_head(k_cache, v_cache, pt_row, seq_len, h, q_group, scale, mode, policy,
                     topk_k=0, alpha=1.5, delta=0.0, meta=None):
    """One full decode step (score -> select -> attend) for one (sequence, KV head).

    policy: "topk", "gauss" or "gauss_max". `meta` is (kmin, kmax, mean, var) for this (sequence, head);
    computed from scratch here when None. Returns a dict with every intermediate."""
    if meta is None:
        meta = page_meta_head(k_cache, pt_row, seq_len, h)
    kmin, kmax, mean, var = meta
    ub, S = score_head(q_group, scale, kmin, kmax)
    res = {"ub": ub, "S": S}
    if policy == "topk":
        sel = topk(S, topk_k)
    else:
        m, v = gauss_stats_head(q_group, scale, mean, var)
        cnt = page_counts(seq_len, k_cache.shape[2])
        tau_hat = np.array([gauss_tau(m[g], v[g], cnt, alpha) for g in range(m.shape[0])])
        if policy == "gauss_max":
            sel = gauss_select_est(ub, m, v, cnt, tau_hat, alpha, delta)
        else:
            sel = gauss_select(ub, tau_hat, alpha, delta)
        res.update(m=m, v=v, tau_hat=tau_hat)
    out, stat, _ = attend_head(k_cache, v_cache, pt_row, seq_len, h, q_group, scale, mode, sel)
    res.update(sel=sel, out=out, stat=stat)
    return res


def time_decode_heads(k_cache, v_cache, page_table, seq_lens, q, heads, scale, mode, policy,
                      topk_k=0, alpha=1.5, delta=0.0, metas=None):
    """Wall time (s) of the oracle decode step over the listed (b, h_kv) pairs, single thread.

    Metadata is taken from `metas[(b, h)]` when given (it is built before a decode step, so it
    is not part of the step), else computed untimed first."""
    H_kv = k_cache.shape[1]
    G = q.shape[1] // H_kv
    metas = dict(metas or {})
    for (b, h) in heads:
        if (b, h) not in metas:
            metas[(b, h)] = page_meta_head(k_cache, page_table[b], seq_lens[b], h)
    t0 = time.perf_counter()
    for (b, h) in heads:
        decode_step_head(k_cache, v_cache, page_table[b], seq_lens[b], h,
                         q[b, h * G:(h + 1) * G], scale, mode, policy, topk_k, alpha, delta,
                         meta=metas[(b, h)])
    return time.perf_counter() - t0
