#!/usr/bin/env python
"""Benchmark of one sparse decode step (page scores -> page selection -> sparse attention,
plus the page-metadata refresh when the workload appends a page) on B200.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload needle128k]
                  [--variant pages|tokens|moment] [--impl ours|reference]

One process per GPU (torchrun for N > 1). Every rank decodes its own seeded batch (weak
scaling, no collective on the data path); the timed region is bracketed by a barrier and a
device synchronise, and the whole-job rate uses the slowest rank's device time. L2 is flushed
(a 256 MiB write, outside the timed events) before every timed step. Rank 0 prints one JSON
line. `--impl reference` times the CPU oracle on the same workload.

Variants (what one step runs after scoring and top-k page selection):
  pages    exact attention over the selected pages (the method's decode)
  tokens   the T best tokens of the selected pages per KV head, then attention over those
  moment   softmax over the selected pages corrected for the skipped ones from running moments
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import hashlib
import json
import os
import platform
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse decode steps/s at 128K ctx; achieved HBM GB/s vs ~8 TB/s peak"
ATTN_NAME = {0: "softmax", 1: "entmax1.5", 2: "sparsemax"}
POLICY_NAME = {0: "topk", 1: "gauss", 2: "gauss_max"}
FALLBACK_HBM_GBS = 6650.0
TARGET_FRAC = 0.70  # the 128K step's required bytes at >= 70% of the HBM roofline


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="needle128k",
                    choices=["tiny", "gqa32k", "needle128k", "gauss", "long1m"])
    ap.add_argument("--variant", default="pages", choices=["pages", "tokens", "moment"])
    ap.add_argument("--tokens", type=int, default=None,
                    help="tokens kept per KV head by the tokens variant (default: a quarter of "
                         "the selected pages' tokens)")
    ap.add_argument("--attn", type=int, default=None, help="attention mode (default: workload's first)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-sample-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (smaller cases for profiler captures)")
    ap.add_argument("--no-full-cache", action="store_true",
                    help="skip the full-cache decode (every page selected) timed for comparison")
    ap.add_argument("--fused-select", action="store_true",
                    help="top-k scores and selection through the one-launch cluster kernel "
                         "(ekv_score_select_pages) instead of the two calls")
    ap.add_argument("--split-select", action="store_true",
                    help="top-k: ekv_select_pages and ekv_sparse_decode as two calls (timed "
                         "apart) instead of the one ekv_select_decode call")
    ap.add_argument("--split-refresh", action="store_true",
                    help="appending workloads: ekv_page_meta_update and ekv_score_pages as two "
                         "calls instead of the one ekv_refresh_score_pages call")
    ap.add_argument("--policy", default=None, choices=["topk", "gauss", "gauss_max"],
                    help="selection policy (default: the workload's); gauss_max is the estimated-"
                         "maximum reading of the Gaussian rule")
    return ap.parse_args()


def setup_workload(args, make, rank, device):
    from sparse_kv_cache_kmin_b200 import replicas
    kw = {"B": args.batch} if args.batch else {}
    wl = make(args.workload, device=device, seed=replicas.workload_seed(args.workload, rank), **kw)
    attn = wl.attn_modes[0] if args.attn is None else args.attn
    if args.variant == "moment":
        attn = 0  # the moment correction is a softmax remedy
    if args.policy is not None:
        wl.policy = {v: k for k, v in POLICY_NAME.items()}[args.policy]
        if wl.policy == 0 and not wl.topk:
            raise SystemExit("--policy topk needs a workload with a top-k budget")
    if args.variant != "pages" and wl.policy != 0:
        raise SystemExit("the tokens and moment variants run after top-k page selection")
    T = None
    if args.variant == "tokens":
        T = args.tokens or max(1, wl.topk * wl.page_size // 4)
    return wl, attn, T


def config_of(wl, attn, variant, T, world):
    """The workload a line measures; the same dict in both arms."""
    cfg = {"workload": wl.name, "batch_per_gpu": wl.batch, "ctx": int(wl.seq_lens.max()),
           "q_heads": wl.num_q_heads, "kv_heads": wl.num_kv_heads, "head_dim": wl.head_dim,
           "page": wl.page_size,
           "policy": "top-k %d" % wl.topk if wl.policy == 0 else "%s delta %g" % (POLICY_NAME[wl.policy], wl.delta),
           "attn": ATTN_NAME[attn], "variant": variant,
           "l2": "flushed before every step (256 MiB write, outside the timed events)",
           "parallelism": "replicas x%d, no collective" % world}
    if T is not None:
        cfg["tokens_per_kv_head"] = T
    return cfg


# ----------------------------------------------------------------------------- byte accounting
def selected_tokens(wl, dec):
    P = wl.page_size
    lens = wl.seq_lens.long().cpu()
    sel = dec.sel_idx.long().cpu()
    cnt = dec.sel_count.long().cpu()
    n = 0
    for b in range(wl.batch):
        L = int(lens[b])
        for h in range(wl.num_kv_heads):
            j = sel[b, h, :int(cnt[b, h])]
            n += int(torch.clamp(L - j * P, 0, P).sum())
    return n


def step_bytes(wl, dec, attn, variant, extra):
    """Required bytes of one step and of each call (what the computation must touch once).

    Every variant: the metadata rows of every existing page (bbox, plus moments for the
    Gaussian policy), the page-table rows, q and the outputs; the appended page when the
    workload appends one. Then
      pages    the K rows of the selected pages' valid tokens and the V rows that carry weight
               (softmax: all of them; entmax: the tokens in the support of some query of the
               group -- the rest provably have zero weight and are not read);
      tokens   the K rows of the selected pages' valid tokens (token scores) and the K and V
               rows of the kept tokens;
      moment   the K and V rows of the selected pages' valid tokens and the running-moment
               records."""
    P, d, H = wl.page_size, wl.head_dim, wl.num_kv_heads
    esz = wl.k_cache.element_size()
    lens = wl.seq_lens.long().cpu()
    total_pages = int(((lens + P - 1) // P).sum())
    meta_row = 2 * d * esz + (2 * d * 4 if wl.policy != 0 else 0)
    meta = total_pages * H * meta_row
    ptab = total_pages * 4
    qb = wl.q.numel() * wl.q.element_size()
    scores_out = total_pages * H * 4 if wl.policy == 0 else total_pages * wl.num_q_heads * 12
    sel_tok = selected_tokens(wl, dec)
    row = d * esz
    out_b = wl.batch * wl.num_q_heads * (d + 1) * 4
    append_b = 0
    if wl.append is not None:
        append_b = wl.batch * H * wl.append[1] * d * esz + wl.batch * H * meta_row
    sel_out = dec.sel_idx.numel() * 4
    by = {"score": meta + ptab + qb + scores_out, "select": scores_out + sel_out,
          "refresh_score": meta + ptab + qb + scores_out + append_b,
          "score_select": meta + ptab + qb + scores_out + sel_out,
          "selected_tokens": sel_tok, "meta_bytes": meta}
    if variant == "pages":
        v_rows = sel_tok if attn == 0 else support_rows(wl, dec, attn)
        by["decode"] = sel_tok * row + v_rows * row + qb + out_b + ptab
        by["select_decode"] = scores_out + sel_out + by["decode"]
        body, body_all_v = sel_tok * row + v_rows * row, 2 * sel_tok * row
        by["support_rows"] = v_rows
    elif variant == "tokens":
        kept = int(extra["tok_count"].long().sum())
        by["select_tokens"] = sel_tok * row + qb + kept * 8
        by["decode_tokens"] = 2 * kept * row + qb + out_b + kept * 8
        body = body_all_v = sel_tok * row + 2 * kept * row
        by["kept_tokens"] = kept
    else:
        mom = extra["moments"].numel() * 4
        by["decode_moment"] = 2 * sel_tok * row + mom + qb + out_b + ptab
        body = body_all_v = 2 * sel_tok * row + mom
    by["required_step"] = meta + ptab + qb + body + out_b + append_b
    by["required_step_all_v"] = meta + ptab + qb + body_all_v + out_b + append_b
    return by


def support_rows(wl, dec, attn):
    """V rows with non-zero weight for some query of the group: z > tau, recomputed on the
    device from the stored threshold (stat) with torch -- accounting only."""
    P, H = wl.page_size, wl.num_kv_heads
    G = wl.num_q_heads // H
    alpha = 1.5 if attn == 1 else 2.0
    rows = 0
    for b in range(wl.batch):
        L = int(wl.seq_lens[b])
        for h in range(H):
            n = int(dec.sel_count[b, h])
            if n == 0:
                continue
            j = dec.sel_idx[b, h, :n].long()
            blk = wl.page_table[b].long()[j]
            t = torch.arange(P, device=j.device)
            valid = (j[:, None] * P + t[None, :]) < L
            kk = wl.k_cache[blk, h].float()  # [n, P, d]
            q = wl.q[b, h * G:(h + 1) * G].float()  # [G, d]
            z = (alpha - 1.0) * wl.scale * torch.einsum("npd,gd->gnp", kk, q)
            tau = dec.stat[b, h * G:(h + 1) * G].float()
            live = (z > tau[:, None, None]).any(0) & valid
            rows += int(live.sum())
    return rows


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), "ekv_clocks_rank%d_%d.csv" % (index, os.getpid()))

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.QUERY,
                 "--format=csv,noheader,nounits", "-lms", "50"], stdout=self.f,
                stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            p = [x.strip() for x in line.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                smax = float(p[2])
            except ValueError:
                continue
            for n, v in zip(names, p[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- roofline inputs
def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        v = json.load(open(p))["hbm_gbs"]
        return float(v), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def ncu_traffic(kernel_file, summary_name, units):
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken on the current
    source of the kernel (its sha256 is recorded there) -- else None. The summary gives the
    bytes of its captured launch and the units it processed; scale to `units`."""
    path = os.path.join(ROOT, "profiles", summary_name)
    try:
        text = open(path).read()
    except OSError:
        return None
    kv = {}
    for line in text.splitlines():
        if line.startswith("- ") and ":" in line:
            k, v = line[2:].split(":", 1)
            kv[k.strip()] = v.strip().strip("`")
    src = os.path.join(ROOT, "sparse_kv_cache_kmin_b200", "csrc", kernel_file)
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()
    if kv.get("source_sha256") != sha:
        return None
    try:
        return float(kv["dram_bytes_per_launch"]) * units / float(kv["units_per_launch"])
    except (KeyError, ValueError):
        return None


def launch_duration_us(step, name, nbytes, call_us, flush, stream, dev, n=16, reps=5):
    """Average device duration of one launch of the step's call `name`. When the call's bytes
    exceed the L2, n launches run back to back between two events (each re-reads its inputs
    from HBM, so no flush is needed between them) and the median over `reps` such runs, divided
    by n, is the launch duration: the per-call event timing also counts the gap before a lone
    call starts. Otherwise the per-call time behind an L2 flush stands."""
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    if nbytes <= l2:
        return call_us, "one call per event pair, behind an L2 flush (inputs fit the L2)"
    fn = dict(step.calls)[name]
    runs = []
    for _ in range(reps):
        flush.fill_(1)  # keeps the GPU busy while the host queues the launches
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        runs.append(a.elapsed_time(b) * 1e3 / n)
    return (statistics.median(runs),
            "%d launches back to back per event pair (%.0f MB per launch > %.0f MB L2), median "
            "of %d" % (n, nbytes / 1e6, l2 / 1e6, reps))


# ----------------------------------------------------------------------------- oracle timing
def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


class OracleStep:
    """The CPU oracle's decode step, one (sequence, KV head) problem at a time, on host copies
    of the workload (taken once, outside every timed region). Problems are independent, and
    the oracle's C routines release the GIL, so a thread pool runs them on all host cores."""

    def __init__(self, wl, attn, variant, T):
        import numpy as np
        import oracle as O
        sys.path.insert(0, os.path.join(ROOT, "tests"))
        from parity_utils import HostCopy
        self.O, self.np = O, np
        self.wl, self.variant, self.T = wl, variant, T
        self.mode = {0: O.SOFTMAX, 1: O.ENTMAX15, 2: O.SPARSEMAX}[attn]
        self.H = wl.num_kv_heads
        self.problems = [(b, h) for b in range(wl.batch) for h in range(self.H)]
        self.hc = {b: HostCopy(wl, b) for b in range(wl.batch)}
        # page metadata is built at prefill, not in a step
        self.meta = {(b, h): O.page_meta_head(self.hc[b].k, self.hc[b].pt, self.hc[b].L, h)
                     for (b, h) in self.problems}

    def run(self, b, h):
        O, wl, hc = self.O, self.wl, self.hc[b]
        meta = self.meta[(b, h)]
        q = hc.q[h]
        if self.variant == "pages":
            O.decode_step_head(hc.k, hc.v, hc.pt, hc.L, h, q, wl.scale, self.mode,
                               POLICY_NAME[wl.policy], wl.topk, wl.alpha, wl.delta, meta=meta)
        else:
            _, S = O.score_head(q, wl.scale, meta[0], meta[1])
            sel = O.topk(S, wl.topk)
            if self.variant == "tokens":
                pages, pos = O.token_topk_head(hc.k, hc.pt, hc.L, h, q, wl.scale, sel, self.T)
                O.attend_tokens_head(hc.k, hc.v, hc.pt, hc.L, h, q, wl.scale, self.mode, pages, pos)
            else:
                O.moment_corrected_head(hc.k, hc.v, hc.pt, hc.L, h, q, wl.scale, sel)
        if wl.append is not None:  # the step also rebuilds the appended page's metadata
            O.page_meta_head(hc.k[-1:], self.np.zeros(1, self.np.int32),
                             hc.L - (hc.np - 1) * wl.page_size, h)

    def single_thread(self, budget_s, seed=0):
        """Seconds per full step, single-threaded, from as many problems as `budget_s` allows."""
        order = list(self.problems)
        self.np.random.default_rng(seed).shuffle(order)
        spent, done = 0.0, 0
        for b, h in order:
            t0 = time.perf_counter()
            self.run(b, h)
            spent += time.perf_counter() - t0
            done += 1
            if spent >= budget_s:
                break
        return spent / done * len(self.problems), done

    def all_cores(self, threads, budget_s, per_problem_s):
        """Seconds per full step with every problem on a pool of `threads` threads (wall time);
        when the whole step would overrun `budget_s`, a whole number of rounds of `threads`
        problems is timed and scaled."""
        n = len(self.problems)
        rounds_fit = max(1, int(budget_s / max(per_problem_s, 1e-9)))
        m = min(n, threads * rounds_fit)
        work = self.problems[:m]
        with cf.ThreadPoolExecutor(max_workers=threads) as ex:
            t0 = time.perf_counter()
            list(ex.map(lambda p: self.run(*p), work))
            wall = time.perf_counter() - t0
        return wall * n / m, m


def cpu_baseline(wl, attn, variant, T, budget_s):
    st = OracleStep(wl, attn, variant, T)
    n = len(st.problems)
    single, done1 = st.single_thread(budget_s / 2)
    threads = os.cpu_count() or 1
    per_problem = single / n
    multi, done_m = st.all_cores(threads, budget_s / 2, per_problem)
    return {"value": 1.0 / multi, "unit": "steps/s", "cores": threads, "kind": "oracle",
            "cpu_model": cpu_model(), "nproc": threads,
            "sample": "%d of %d (sequence, KV head) decode problems of the step on a pool of %d "
                      "threads (the oracle's C routines release the GIL), wall time scaled to "
                      "the full step" % (done_m, n, threads),
            "single_thread": {"value": 1.0 / single, "unit": "steps/s", "cores": 1,
                              "sample": "%d of %d problems, scaled to the full step" % (done1, n)}}


# ----------------------------------------------------------------------------- the step on the GPU
class Step:
    """The public calls of one decode step of a variant, as (name, fn) pairs, with the buffers
    they write. Every call goes through the C ABI binding; nothing here computes."""

    def __init__(self, ekv, SparseDecoder, cache, wl, attn, variant, T, fused_select=False,
                 split_select=False, split_refresh=False):
        self.wl, self.variant, self.T = wl, variant, T
        dev = wl.k_cache.device
        B, H = wl.batch, wl.num_kv_heads
        self.dec = dec = SparseDecoder(cache, wl.num_q_heads, wl.policy, attn, topk=wl.topk,
                                       alpha=wl.alpha, delta=wl.delta, scale=wl.scale)
        self.extra = {}
        calls = []
        q = wl.q
        # top-k pages: the selection and the attention in one call
        joint = wl.policy == 0 and variant == "pages" and not fused_select and not split_select
        refresh = wl.append is not None and joint and not split_refresh
        if wl.append is not None:
            ap_start = torch.full((B,), wl.append[0], dtype=torch.int32, device=dev)
            ap_count = torch.full((B,), wl.append[1], dtype=torch.int32, device=dev)
            if refresh:
                # the appended page's metadata rebuilt inside the scan (one call)
                calls.append(("refresh_score", lambda: ekv.ekv_refresh_score_pages(
                    cache, ap_start, ap_count, wl.append[1], q, wl.num_q_heads, wl.scale,
                    wl.policy, dec.scores)))
            else:
                calls.append(("meta", lambda: ekv.ekv_page_meta_update(cache, ap_start, ap_count,
                                                                       wl.append[1])))
        if joint:
            if not refresh:
                calls.append(("score", lambda: ekv.ekv_score_pages(
                    cache, q, wl.num_q_heads, wl.scale, wl.policy, dec.scores)))
        elif wl.policy == 0 and fused_select:
            # top-k scores and selection in one launch (one cluster per sequence and KV head)
            calls.append(("score_select", lambda: ekv.ekv_score_select_pages(
                cache, q, wl.num_q_heads, wl.scale, wl.topk, dec.scores, dec.sel_idx,
                dec.sel_count, dec.max_sel)))
        else:
            calls.append(("score", lambda: ekv.ekv_score_pages(cache, q, wl.num_q_heads, wl.scale,
                                                               wl.policy, dec.scores)))
            calls.append(("select", lambda: ekv.ekv_select_pages(
                cache, wl.num_q_heads, wl.policy, wl.topk, wl.alpha, wl.delta, dec.scores,
                dec.sel_idx, dec.sel_count, dec.max_sel, dec.tau_hat)))
        self.out, self.stat = dec.out, dec.stat
        if joint:
            calls.append(("select_decode", lambda: ekv.ekv_select_decode(
                cache, q, wl.num_q_heads, wl.scale, attn, wl.topk, dec.scores, dec.sel_idx,
                dec.sel_count, dec.max_sel, dec.out, dec.stat, dec.ws)))
            self.kernels = {"meta": 1, "refresh_score": 1, "score": 1, "select_decode": 1}
        elif variant == "pages":
            calls.append(("decode", lambda: ekv.ekv_sparse_decode(
                cache, q, wl.num_q_heads, wl.scale, attn, dec.sel_idx, dec.sel_count,
                dec.max_sel, dec.out, dec.stat, dec.ws)))
            self.kernels = {"meta": 1, "score_select": 1, "score": 1, "select": 1, "decode": 2}
        elif variant == "tokens":
            tws = torch.empty(ekv.ekv_token_workspace_bytes(cache, dec.max_sel), dtype=torch.uint8,
                              device=dev)
            tp = torch.empty((B, H, T), dtype=torch.int32, device=dev)
            tt = torch.empty_like(tp)
            tc = torch.empty((B, H), dtype=torch.int32, device=dev)
            self.extra.update(tok_page=tp, tok_pos=tt, tok_count=tc)
            calls.append(("select_tokens", lambda: ekv.ekv_select_tokens(
                cache, q, wl.num_q_heads, wl.scale, dec.sel_idx, dec.sel_count, dec.max_sel, T,
                tp, tt, tc, tws)))
            calls.append(("decode_tokens", lambda: ekv.ekv_sparse_decode_tokens(
                cache, q, wl.num_q_heads, wl.scale, attn, tp, tt, tc, T, dec.out, dec.stat)))
            self.kernels = {"score_select": 1, "score": 1, "select": 1, "select_tokens": 2,
                            "decode_tokens": 1}
        else:
            moments = torch.zeros(ekv.ekv_moment_bytes(cache) // 4, dtype=torch.float32, device=dev)
            ekv.ekv_moment_update(cache, moments, torch.zeros(B, dtype=torch.int32, device=dev),
                                  wl.seq_lens, int(wl.seq_lens.max()))
            mws = torch.empty(ekv.ekv_moment_decode_workspace_bytes(cache, wl.num_q_heads,
                                                                    dec.max_sel),
                              dtype=torch.uint8, device=dev)
            self.extra.update(moments=moments)
            calls.append(("decode_moment", lambda: ekv.ekv_sparse_decode_moment(
                cache, moments, q, wl.num_q_heads, wl.scale, dec.sel_idx, dec.sel_count,
                dec.max_sel, dec.out, dec.stat, mws)))
            self.kernels = {"score_select": 1, "score": 1, "select": 1, "decode_moment": 4}
        self.calls = calls

    def launches(self):
        return sum(self.kernels.get(name, 1) for name, _ in self.calls)

    def run(self):
        for _, fn in self.calls:
            fn()

    def graph(self):
        g = torch.cuda.CUDAGraph(keep_graph=True)
        with torch.cuda.graph(g):
            self.run()
        return g

    def graph_host(self, q_host, out_host, stat_host, host_pre=None):
        """A whole host-to-host step: the query copied in from pinned host memory, the calls,
        the outputs copied back to pinned host buffers."""
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            if host_pre is not None:
                host_pre()
            self.wl.q.copy_(q_host, non_blocking=True)
            self.run()
            out_host.copy_(self.out, non_blocking=True)
            stat_host.copy_(self.stat, non_blocking=True)
        return g


def graph_kernel_nodes(g):
    """Kernel nodes of a captured step graph: every kernel one step launches (the captured
    calls are the library's own, so every kernel node is one of its kernels)."""
    from cuda.bindings import runtime as rt
    h = rt.cudaGraph_t(init_value=int(g.raw_cuda_graph()))
    err, _, n = rt.cudaGraphGetNodes(h, 0)
    if err != rt.cudaError_t.cudaSuccess:
        raise RuntimeError(str(err))
    err, nodes, n = rt.cudaGraphGetNodes(h, n)
    if err != rt.cudaError_t.cudaSuccess:
        raise RuntimeError(str(err))
    kinds = [rt.cudaGraphNodeGetType(x)[1] for x in nodes[:n]]
    return sum(1 for k in kinds if k == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel)


def full_cache_time(ekv, cache, wl, attn, steps, flush, stream):
    """The same attention over every page of every sequence (no scoring, no selection): one
    ekv_sparse_decode call with the identity selection, captured in a graph and timed like the
    sparse step. Returns (ms per step, out, stat)."""
    B, H, P = wl.batch, wl.num_kv_heads, wl.page_size
    dev = wl.k_cache.device
    n_pages = ((wl.seq_lens.long() + P - 1) // P).to(torch.int32)
    mp = int(wl.page_table.shape[1])
    sel = torch.arange(mp, dtype=torch.int32, device=dev).expand(B, H, mp).contiguous()
    sel = torch.where(sel < n_pages.view(B, 1, 1), sel, torch.full_like(sel, -1))
    cnt = n_pages.view(B, 1).expand(B, H).contiguous()
    out = torch.empty((B, wl.num_q_heads, wl.head_dim), dtype=torch.float32, device=dev)
    stat = torch.empty((B, wl.num_q_heads), dtype=torch.float32, device=dev)
    ws = torch.empty(ekv.ekv_decode_workspace_bytes(cache, wl.num_q_heads, mp), dtype=torch.uint8,
                     device=dev)

    def call():
        ekv.ekv_sparse_decode(cache, wl.q, wl.num_q_heads, wl.scale, attn, sel, cnt, mp, out,
                              stat, ws)
    call()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    for _ in range(3):
        flush.fill_(1)
        g.replay()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for i in range(steps):
        flush.fill_(i & 0xff)
        ev[i][0].record(stream)
        g.replay()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    del g
    return statistics.median(a.elapsed_time(b) for a, b in ev), out, stat


def selection_quality(ekv, cache, wl, dec, attn, stat_full):
    """How much of the full-cache attention the page selection keeps, per query, from the
    library's ekv_selection_quality kernel (outside every timed region): the dropped mass delta
    (the quantity of the 2 B delta error bound) and, for entmax, the recall of the full-cache
    support."""
    dev = wl.k_cache.device
    dropped = torch.empty((wl.batch, wl.num_q_heads), dtype=torch.float64, device=dev)
    support = torch.empty((wl.batch, wl.num_q_heads, 2), dtype=torch.int32, device=dev)
    ekv.ekv_selection_quality(cache, wl.q, wl.num_q_heads, wl.scale, attn, stat_full, dec.sel_idx,
                              dec.sel_count, dec.max_sel, dropped, support)
    torch.cuda.synchronize()
    dl = dropped.flatten().tolist()
    P = wl.page_size
    out = {"dropped_mass_mean": statistics.mean(dl), "dropped_mass_max": max(dl),
           "kept_pages_mean": float(dec.sel_count.float().mean()),
           "pages_mean": float(((wl.seq_lens.float() + P - 1) // P).mean()),
           "how": "ekv_selection_quality on the full-cache stat of this GPU"}
    if attn != 0:
        sup = support.double()
        rec = (sup[..., 1] / sup[..., 0].clamp(min=1)).flatten().tolist()
        out["support_recall_mean"] = statistics.mean(rec)
        out["support_recall_min"] = min(rec)
        out["support_size_mean"] = float(sup[..., 0].mean())
    return out


# ----------------------------------------------------------------------------- main
def main():
    args = parse()
    from sparse_kv_cache_kmin_b200 import replicas
    from sparse_kv_cache_kmin_b200.workloads import make

    rank, world, local = replicas.rank_info()

    if args.impl == "reference":
        return reference_arm(args, rank, world, make)

    from sparse_kv_cache_kmin_b200 import ekv
    from sparse_kv_cache_kmin_b200.decoder import SparseDecoder

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist

    wl, attn, T = setup_workload(args, make, rank, dev)
    nb, H, P, d = wl.k_cache.shape
    cache = ekv.PagedKVCache(
        k_cache=wl.k_cache, v_cache=wl.v_cache,
        meta_bbox=torch.empty((nb, H, 2, d), dtype=wl.k_cache.dtype, device=dev),
        meta_mom=torch.empty((nb, H, 2, d), dtype=torch.float32, device=dev) if wl.policy != 0 else None,
        page_table=wl.page_table, seq_lens=wl.seq_lens,
        dev_status=torch.zeros(1, dtype=torch.int32, device=dev))
    B = wl.batch
    ekv.ekv_page_meta_update(cache, torch.zeros(B, dtype=torch.int32, device=dev), wl.seq_lens,
                             int(wl.seq_lens.max()))
    step = Step(ekv, SparseDecoder, cache, wl, attn, args.variant, T, args.fused_select,
                args.split_select, args.split_refresh)
    dec = step.dec
    stream = torch.cuda.current_stream()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    # eager steps first: one-time set-up (kernel attributes, occupancy queries) stays outside
    # the graph captures
    for _ in range(2):
        flush.fill_(1)
        step.run()
    torch.cuda.synchronize()
    # the step as one graph launch (the timed loop)
    graph = step.graph()
    try:
        launches_per_step, launches_src = graph_kernel_nodes(graph), "kernel nodes of the step graph"
    except Exception as exc:  # the count then comes from the calls' known kernel counts
        launches_per_step, launches_src = step.launches(), "per-call table (%s)" % type(exc).__name__

    for _ in range(max(args.warmup, 3)):
        flush.fill_(1)
        graph.replay()
    torch.cuda.synchronize()
    st, bits = ekv.ekv_device_status(cache)
    if st != ekv.EKV_OK:
        raise RuntimeError("device status 0x%x after warm-up" % bits)

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    with ClockSampler(local) as clocks:
        # The timed steps last milliseconds, shorter than the clock sampling period; the same
        # flush-and-step loop runs for about half a second before them (untimed; no collective
        # inside) so that the samples see the GPU under this load, then the timed steps follow,
        # bracketed by a barrier and a device synchronisation.
        rounds, t_end = 0, time.time() + 0.5
        while time.time() < t_end and rounds < 1000:
            for i in range(20):
                flush.fill_(i & 0xff)
                graph.replay()
            torch.cuda.synchronize()
            rounds += 1
        if pg:
            pg.barrier()
        torch.cuda.synchronize()
        for i in range(args.steps):
            flush.fill_(i & 0xff)
            ev[i][0].record(stream)
            graph.replay()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        if pg:
            pg.barrier()
        step_ms = [a.elapsed_time(b) for a, b in ev]
        # per-call durations: each call launched on its own K more times, bracketed by events on
        # the launching stream, behind an L2 flush that keeps the GPU busy while the host queues
        # the call (so the events time the call's kernels, not the host)
        names = [n for n, _ in step.calls]
        part_ms = {n: [] for n in names}
        for n, fn in step.calls:
            pev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.steps)]
            for i in range(args.steps):
                flush.fill_(i & 0xff)
                pev[i][0].record(stream)
                fn()
                pev[i][1].record(stream)
            torch.cuda.synchronize()
            part_ms[n] = [a.elapsed_time(b) for a, b in pev]
    total_s = replicas.max_over_ranks(sum(step_ms) / 1e3, device=dev)
    median_ms = replicas.max_over_ranks(statistics.median(step_ms), device=dev)
    st, bits = ekv.ekv_device_status(cache)
    if st != ekv.EKV_OK:
        raise RuntimeError("device status 0x%x after timing" % bits)

    # ---- end to end through the public API with host buffers (pinned), copies inside
    q_host = wl.q.cpu().pin_memory()
    out_host = torch.empty(step.out.shape, dtype=step.out.dtype).pin_memory()
    stat_host = torch.empty(step.stat.shape, dtype=step.stat.dtype).pin_memory()
    h2d = q_host.numel() * q_host.element_size()
    app_host = None
    if wl.append is not None:
        last = int(wl.page_table[0, wl.append[0] // P])  # a host index: no sync in the graph
        app_host = (wl.k_cache[last].cpu().pin_memory(), wl.v_cache[last].cpu().pin_memory(), last)
        h2d += 2 * app_host[0].numel() * app_host[0].element_size()

    def host_pre():
        # the appended page's K and V rows arrive from the host (its metadata refresh is the
        # step's first call)
        if app_host is not None:
            wl.k_cache[app_host[2]].copy_(app_host[0], non_blocking=True)
            wl.v_cache[app_host[2]].copy_(app_host[1], non_blocking=True)
    graph_e2e = step.graph_host(q_host, out_host, stat_host, host_pre=host_pre)
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
    for i in range(args.steps + 3):
        flush.fill_(1)
        if i >= 3:
            e2e_ev[i - 3][0].record(stream)
        graph_e2e.replay()
        if i >= 3:
            e2e_ev[i - 3][1].record(stream)
        stream.synchronize()
    e2e_s = replicas.max_over_ranks(sum(a.elapsed_time(b) for a, b in e2e_ev) / 1e3, device=dev)
    d2h = out_host.numel() * 4 + stat_host.numel() * 4

    full_ms, quality = None, None
    if not args.no_full_cache and world == 1:
        full_ms, _, stat_full = full_cache_time(ekv, cache, wl, attn, min(args.steps, 20), flush,
                                                stream)
        quality = selection_quality(ekv, cache, wl, dec, attn, stat_full)
        st, bits = ekv.ekv_device_status(cache)
        if st != ekv.EKV_OK:
            raise RuntimeError("device status 0x%x after the full-cache decode" % bits)

    if rank != 0:
        if pg:
            pg.barrier()
            pg.destroy_process_group()
        return

    by = step_bytes(wl, dec, attn, args.variant, step.extra)
    peak, peak_kind = measured_peak()
    call_us = {k: statistics.median(v) * 1e3 for k, v in part_ms.items()}
    value = replicas.job_rate(args.steps, world, total_s)
    ms = total_s / args.steps * 1e3
    dom = max((n for n in call_us if n in by), key=lambda n: call_us[n])
    traffic = None
    if dom == "score" and args.workload == "needle128k":
        total_pages = int(((wl.seq_lens.long() + P - 1) // P).sum())
        traffic = ncu_traffic("score.cu", "score_pages_needle128k.md", total_pages * H)
    dom_us, dom_timing = launch_duration_us(step, dom, by[dom], call_us[dom], flush, stream, dev)
    achieved = by[dom] / (dom_us / 1e6) / 1e9
    frac_step = by["required_step"] / (ms / 1e3) / 1e9 / peak
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        cpu = cpu_baseline(wl, attn, args.variant, T, args.cpu_sample_seconds)
    line = {
        "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": ms,
        "ms_per_step_median": median_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype":
            "bf16" if wl.k_cache.dtype == torch.bfloat16 else "f32",
        "data": "synthetic (seeded; rank r decodes its own batch)",
        "config": config_of(wl, attn, args.variant, T, world),
        "hbm": {"required_bytes_per_step": by["required_step"],
                "achieved_GBps": by["required_step"] / (ms / 1e3) / 1e9,
                "frac_of_8TBps": by["required_step"] / (ms / 1e3) / 8e12,
                "frac_of_measured": frac_step,
                "required_bytes_if_all_v": by["required_step_all_v"],
                "selected_tokens": by["selected_tokens"],
                **({"v_rows_read": by["support_rows"]} if "support_rows" in by else {}),
                **({"kept_tokens": by["kept_tokens"]} if "kept_tokens" in by else {})},
        "target": {"what": "the step's required bytes at >= %.2f of the measured HBM copy "
                           "bandwidth" % TARGET_FRAC,
                   "frac": frac_step, "met": frac_step >= TARGET_FRAC},
        "per_call_us": call_us,
        "roofline": {"kernel": {"score": "score_pages", "score_select": "step_score_select"}.get(dom, dom),
                     "bound": "hbm",
                     "achieved": achieved, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "algorithmic_bytes_per_launch": by[dom], "launch_us": dom_us,
                     "timing": dom_timing},
        "call_fracs": {n: by[n] / (call_us[n] / 1e6) / 1e9 / peak for n in call_us if n in by},
        "full_cache": None if full_ms is None else {
            "what": "the same attention over every page (no scoring, no selection) on this GPU",
            "ms_per_step": full_ms, "steps_per_s": 1e3 / full_ms,
            "sparse_speedup": full_ms / median_ms},
        "selection_quality": quality,
        "e2e": {"value": replicas.job_rate(args.steps, world, e2e_s), "unit": "steps/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step * args.steps,
        "gpu_launches_source": launches_src,
        "launch": "one CUDA graph per step (programmatic dependent launch between its kernels)",
        "clocks": clocks.summary(),
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


def reference_arm(args, rank, world, make):
    """The CPU oracle as it stands, on all host cores, same workload/metric/unit; rank 0 only."""
    if rank != 0:
        return
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    wl, attn, T = setup_workload(args, make, 0, dev)
    st = OracleStep(wl, attn, args.variant, T)
    threads = os.cpu_count() or 1
    single, _ = st.single_thread(2.0)
    n_steps = max(args.warmup, 3) + args.steps
    budget = max(1.0, 150.0 / n_steps)  # the whole run stays within a few minutes
    times, done = [], 0
    for i in range(n_steps):
        per_step, done = st.all_cores(threads, budget, single / len(st.problems))
        if i >= max(args.warmup, 3):
            times.append(per_step)
    value = 1.0 / statistics.mean(times)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(args.warmup, 3),
        "ms_per_step": statistics.mean(times) * 1e3,
        "ms_per_step_median": statistics.median(times) * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded)",
        "config": config_of(wl, attn, args.variant, T, world),
        "cpu_baseline": {"value": value, "unit": "steps/s", "cores": threads, "kind": "oracle",
                         "cpu_model": cpu_model(), "nproc": threads,
                         "sample": "%d of %d (sequence, KV head) problems per step on a pool of "
                                   "%d threads, wall time scaled to the full step; each step a "
                                   "fresh timing" % (done, len(st.problems), threads),
                         "single_thread": {"value": 1.0 / single, "unit": "steps/s", "cores": 1}},
        "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
