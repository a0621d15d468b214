#!/usr/bin/env python
"""Benchmark of one sparse decode step (page scores -> page selection -> sparse attention,
plus the page-metadata refresh when the workload appends a page) on B200.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload needle128k] [--impl ours|reference]

One process per GPU (torchrun for N > 1). Every rank decodes its own seeded batch (weak
scaling, no collective on the data path); the timed region is bracketed by a barrier and a
device synchronise, and the whole-job rate uses the slowest rank's device time. L2 is flushed
(a 256 MiB write, outside the timed events) before every timed step. Rank 0 prints one JSON
line. `--impl reference` times the CPU oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
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


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="needle128k",
                    choices=["tiny", "gqa32k", "needle128k", "gauss", "long1m"])
    ap.add_argument("--attn", type=int, default=None, help="attention mode (default: workload's first)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-sample-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (smaller cases for profiler captures)")
    ap.add_argument("--no-full-cache", action="store_true",
                    help="skip the full-cache decode (every page selected) timed for comparison")
    ap.add_argument("--policy", default=None, choices=["topk", "gauss", "gauss_max"],
                    help="selection policy (default: the workload's); gauss_max is the estimated-"
                         "maximum reading of the Gaussian rule")
    return ap.parse_args()


# ----------------------------------------------------------------------------- byte accounting
def step_bytes(wl, dec, attn):
    """Required bytes of one step and of each call (what the computation must touch once).

    metadata rows of every existing page (bbox, plus moments for the Gaussian policy), the
    page-table rows, q, the K rows of the selected pages' valid tokens, the V rows that carry
    weight (softmax: all selected tokens; entmax: the tokens in the support of some query of
    the group -- the rest provably have zero weight and are not read), the outputs; the
    appended page when the workload appends one."""
    P, d, H = wl.page_size, wl.head_dim, wl.num_kv_heads
    esz = wl.k_cache.element_size()
    lens = wl.seq_lens.long().cpu()
    n_pages = (lens + P - 1) // P
    total_pages = int(n_pages.sum())
    meta_row = 2 * d * esz + (2 * d * 4 if wl.policy != 0 else 0)
    meta = total_pages * H * meta_row
    ptab = total_pages * 4
    qb = wl.q.numel() * wl.q.element_size()
    scores_out = total_pages * H * 4 if wl.policy == 0 else total_pages * wl.num_q_heads * 12
    # selected tokens (valid ones) from the device selection
    sel = dec.sel_idx.long().cpu()
    cnt = dec.sel_count.long().cpu()
    sel_tok = 0
    for b in range(wl.batch):
        L = int(lens[b])
        for h in range(H):
            j = sel[b, h, :int(cnt[b, h])]
            sel_tok += int(torch.clamp(L - j * P, 0, P).sum())
    k_bytes = sel_tok * d * esz
    if attn == 0:
        v_rows = sel_tok
    else:
        v_rows = support_rows(wl, dec, attn)
    v_bytes = v_rows * d * esz
    out_b = dec.out.numel() * 4 + dec.stat.numel() * 4
    append_b = 0
    if wl.append is not None:
        append_b = wl.batch * H * wl.append[1] * d * esz + wl.batch * H * meta_row
    return {
        "score": meta + ptab + qb + scores_out,
        "select": scores_out + dec.sel_idx.numel() * 4,
        "decode": k_bytes + v_bytes + qb + out_b + ptab,
        "required_step": meta + ptab + qb + k_bytes + v_bytes + out_b + append_b,
        "required_step_all_v": meta + ptab + qb + 2 * k_bytes + out_b + append_b,
        "selected_tokens": sel_tok, "support_rows": v_rows, "meta_bytes": meta,
    }


def support_rows(wl, dec, attn):
    """V rows with non-zero weight for some query of the group: z > tau, recomputed on the
    device from the stored threshold (stat) with torch -- accounting only."""
    P, d, H = wl.page_size, wl.head_dim, wl.num_kv_heads
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
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f,
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


# ----------------------------------------------------------------------------- oracle timing
def oracle_sample(wl, attn, budget_s, max_heads=None):
    """Time the CPU oracle's decode step on (sequence, KV head) problems of the workload until
    `budget_s` of CPU time is spent; returns (seconds per full step, description)."""
    import numpy as np
    import oracle as O
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from parity_utils import HostCopy
    H = wl.num_kv_heads
    G = wl.num_q_heads // H
    mode = {0: O.SOFTMAX, 1: O.ENTMAX15, 2: O.SPARSEMAX}[attn]
    order = [(b, h) for b in range(wl.batch) for h in range(H)]
    rng = np.random.default_rng(0)
    rng.shuffle(order)
    if max_heads:
        order = order[:max_heads]
    spent, done, hcs = 0.0, 0, {}
    for b, h in order:
        hc = hcs.get(b) or HostCopy(wl, b)
        hcs = {b: hc}
        meta = O.page_meta_head(hc.k, hc.pt, hc.L, h)  # built at prefill, not part of a step
        t0 = time.perf_counter()
        O.decode_step_head(hc.k, hc.v, hc.pt, hc.L, h, hc.q[h], wl.scale, mode,
                           POLICY_NAME[wl.policy], wl.topk, wl.alpha, wl.delta, meta=meta)
        if wl.append is not None:  # the step also rebuilds the appended page's metadata
            O.page_meta_head(hc.k[-1:], np.zeros(1, np.int32), hc.L - (hc.np - 1) * wl.page_size, h)
        spent += time.perf_counter() - t0
        done += 1
        if spent >= budget_s:
            break
    per_step = spent / done * len([(b, h) for b in range(wl.batch) for h in range(H)])
    desc = ("%d of %d (sequence, KV head) decode problems (score all pages, select, attend), "
            "timed single-threaded and scaled to the full step" % (done, wl.batch * H))
    return per_step, desc



# ----------------------------------------------------------------------------- full-cache decode
def full_cache_time(ekv, cache, wl, attn, steps, flush, stream):
    """The same attention over every page of every sequence (no scoring, no selection): one
    ekv_sparse_decode call with the identity selection, captured in a graph and timed like the
    sparse step. Returns ms per step."""
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
    return statistics.mean(a.elapsed_time(b) for a, b in ev), out, stat


def selection_quality(wl, dec, attn, stat_full):
    """How much of the full-cache attention the selection keeps, per query: the dropped mass
    delta = sum of full-cache weights on tokens outside the selected pages (the quantity of the
    2 B delta error bound) and, for entmax, the recall of the full-cache support. Computed with
    torch on the GPU from the cache and the full-cache stat, outside every timed region."""
    P, H = wl.page_size, wl.num_kv_heads
    G = wl.num_q_heads // H
    alpha = {1: 1.5, 2: 2.0}.get(attn)
    deltas, recalls = [], []
    for b in range(wl.batch):
        L = int(wl.seq_lens[b])
        n = (L + P - 1) // P
        blk = wl.page_table[b, :n].long()
        valid = (torch.arange(n, device=blk.device)[:, None] * P
                 + torch.arange(P, device=blk.device)[None, :]) < L
        for h in range(H):
            kk = wl.k_cache[blk, h].float()                          # [n, P, d]
            q = wl.q[b, h * G:(h + 1) * G].float()                   # [G, d]
            s = wl.scale * torch.einsum("npd,gd->gnp", kk, q)
            st = stat_full[b, h * G:(h + 1) * G].float()[:, None, None]
            if alpha is None:
                p = torch.exp(s - st)
            else:
                p = torch.clamp((alpha - 1.0) * s - st, min=0.0) ** (1.0 / (alpha - 1.0))
            p = p * valid
            kept = torch.zeros(n, dtype=torch.bool, device=p.device)
            cnt = int(dec.sel_count[b, h])
            kept[dec.sel_idx[b, h, :cnt].long()] = True
            deltas += (p * (~kept)[None, :, None]).sum((1, 2)).tolist()
            if alpha is not None:
                sup = p > 0
                recalls += ((sup & kept[None, :, None]).sum((1, 2)).float()
                            / sup.sum((1, 2)).clamp(min=1).float()).tolist()
    out = {"dropped_mass_mean": statistics.mean(deltas), "dropped_mass_max": max(deltas),
           "kept_pages_mean": float(dec.sel_count.float().mean()),
           "pages_mean": float(((wl.seq_lens.float() + P - 1) // P).mean())}
    if recalls:
        out["support_recall_mean"] = statistics.mean(recalls)
        out["support_recall_min"] = min(recalls)
    return out

# ----------------------------------------------------------------------------- main
def main():
    args = parse()
    from sparse_kv_cache_kmin_b200 import replicas
    from sparse_kv_cache_kmin_b200.workloads import make

    rank, world, local = replicas.rank_info()

    if args.impl == "reference":
        return reference_arm(args, rank, world, make)

    import sparse_kv_cache_kmin_b200 as ekvpkg
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

    kw = {"B": args.batch} if args.batch else {}
    wl = make(args.workload, device=dev, seed=replicas.workload_seed(args.workload, rank), **kw)
    attn = wl.attn_modes[0] if args.attn is None else args.attn
    if args.policy is not None:
        wl.policy = {v: k for k, v in POLICY_NAME.items()}[args.policy]
        if wl.policy == 0 and not wl.topk:
            raise SystemExit("--policy topk needs a workload with a top-k budget")
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
    dec = SparseDecoder(cache, wl.num_q_heads, wl.policy, attn, topk=wl.topk, alpha=wl.alpha,
                        delta=wl.delta, scale=wl.scale)
    if wl.append is not None:
        ap_start = torch.full((B,), wl.append[0], dtype=torch.int32, device=dev)
        ap_count = torch.full((B,), wl.append[1], dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    def step(q):
        if wl.append is not None:
            ekv.ekv_page_meta_update(cache, ap_start, ap_count, wl.append[1])
        return dec.step(q)

    launches_per_step = 4 + (1 if wl.append is not None else 0)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    pre = None
    if wl.append is not None:
        def pre():
            ekv.ekv_page_meta_update(cache, ap_start, ap_count, wl.append[1])

    # eager steps first: one-time set-up (kernel attributes, occupancy queries) stays outside
    # the graph captures
    for _ in range(2):
        flush.fill_(1)
        step(wl.q)
    torch.cuda.synchronize()
    # graph A: the step as one launch (the timed loop); graph B: the same calls with an
    # event node between them (per-call durations)
    graph = dec.capture(wl.q, pre_step=pre)
    evb = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(5)]
    graph_b = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_b):
        evb[0].record()
        if pre is not None:
            pre()
        evb[1].record()
        ekv.ekv_score_pages(cache, wl.q, wl.num_q_heads, wl.scale, wl.policy, dec.scores)
        evb[2].record()
        ekv.ekv_select_pages(cache, wl.num_q_heads, wl.policy, wl.topk, wl.alpha, wl.delta,
                             dec.scores, dec.sel_idx, dec.sel_count, dec.max_sel, dec.tau_hat)
        evb[3].record()
        ekv.ekv_sparse_decode(cache, wl.q, wl.num_q_heads, wl.scale, attn, dec.sel_idx,
                              dec.sel_count, dec.max_sel, dec.out, dec.stat, dec.ws)
        evb[4].record()

    for _ in range(max(args.warmup, 3)):
        flush.fill_(1)
        graph.replay()
    torch.cuda.synchronize()
    st, bits = ekv.ekv_device_status(cache)
    if st != ekv.EKV_OK:
        raise RuntimeError("device status 0x%x after warm-up" % bits)

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        for i in range(args.steps):
            flush.fill_(i & 0xff)
            ev[i][0].record(stream)
            graph.replay()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        if pg:
            pg.barrier()
        step_ms = [a.elapsed_time(b) for a, b in ev]
        # per-call durations over K more steps of graph B (same work, event nodes between calls)
        part_ms = {"meta": [], "score": [], "select": [], "decode": []}
        for i in range(args.steps):
            flush.fill_(i & 0xff)
            graph_b.replay()
            torch.cuda.synchronize()
            for k, j in [("meta", 0), ("score", 1), ("select", 2), ("decode", 3)]:
                part_ms[k].append(evb[j].elapsed_time(evb[j + 1]))
    total_s = replicas.max_over_ranks(sum(step_ms) / 1e3, device=dev)
    st, bits = ekv.ekv_device_status(cache)
    if st != ekv.EKV_OK:
        raise RuntimeError("device status 0x%x after timing" % bits)

    # ---- end to end through the public API with host buffers (pinned), copies inside
    q_host = wl.q.cpu().pin_memory()
    out_host = torch.empty(dec.out.shape, dtype=dec.out.dtype).pin_memory()
    stat_host = torch.empty(dec.stat.shape, dtype=dec.stat.dtype).pin_memory()
    h2d = q_host.numel() * q_host.element_size()
    app_host = None
    if wl.append is not None:
        last = int(wl.page_table[0, wl.append[0] // P])  # a host index: no sync in the graph
        app_host = (wl.k_cache[last].cpu().pin_memory(), wl.v_cache[last].cpu().pin_memory(), last)
        h2d += 2 * app_host[0].numel() * app_host[0].element_size()
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]

    def host_pre():
        # the appended page's K and V rows arrive from the host, then its metadata is refreshed
        if app_host is not None:
            wl.k_cache[app_host[2]].copy_(app_host[0], non_blocking=True)
            wl.v_cache[app_host[2]].copy_(app_host[1], non_blocking=True)
        if pre is not None:
            pre()
    # one graph per host-to-host step: query in, step, outputs out
    graph_e2e = dec.capture_host(wl.q, q_host, out_host, stat_host, pre_step=host_pre)
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
        quality = selection_quality(wl, dec, attn, stat_full)
        st, bits = ekv.ekv_device_status(cache)
        if st != ekv.EKV_OK:
            raise RuntimeError("device status 0x%x after the full-cache decode" % bits)

    if rank != 0:
        if pg:
            pg.barrier()
            pg.destroy_process_group()
        return

    by = step_bytes(wl, dec, attn)
    peak, peak_kind = measured_peak()
    score_s = statistics.mean(part_ms["score"]) / 1e3
    decode_s = statistics.mean(part_ms["decode"]) / 1e3
    total_pages = int(((wl.seq_lens.long() + P - 1) // P).sum())
    traffic = ncu_traffic("score.cu", "score_pages_needle128k.md", total_pages * H) \
        if args.workload == "needle128k" else None
    achieved = by["score"] / score_s / 1e9
    value = replicas.job_rate(args.steps, world, total_s)
    ms = total_s / args.steps * 1e3
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        per_step, desc = oracle_sample(wl, attn, args.cpu_sample_seconds)
        cpu = {"value": 1.0 / per_step, "unit": "steps/s", "cores": 1, "kind": "oracle",
               "sample": desc}
    line = {
        "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype":
            "bf16" if wl.k_cache.dtype == torch.bfloat16 else "f32",
        "data": "synthetic (seeded; rank r decodes its own batch)",
        "config": {"workload": wl.name, "batch_per_gpu": B, "ctx": int(wl.seq_lens.max()),
                   "q_heads": wl.num_q_heads, "kv_heads": H, "head_dim": d, "page": P,
                   "policy": "top-k %d" % wl.topk if wl.policy == 0 else "%s delta %g" % (POLICY_NAME[wl.policy], wl.delta),
                   "attn": ATTN_NAME[attn], "l2": "flushed before every step (256 MiB write, outside the timed events)",
                   "parallelism": "replicas x%d, no collective" % world},
        "hbm": {"required_bytes_per_step": by["required_step"],
                "achieved_GBps": by["required_step"] / (ms / 1e3) / 1e9,
                "frac_of_8TBps": by["required_step"] / (ms / 1e3) / 8e12,
                "frac_of_measured": by["required_step"] / (ms / 1e3) / 1e9 / peak,
                "required_bytes_if_all_v": by["required_step_all_v"],
                "selected_tokens": by["selected_tokens"], "v_rows_read": by["support_rows"]},
        "per_call_us": {k: statistics.mean(v) * 1e3 for k, v in part_ms.items()},
        "roofline": {"kernel": "score_pages", "bound": "hbm", "achieved": achieved,
                     "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "algorithmic_bytes_per_launch": by["score"]},
        "decode_kernel": {"achieved_GBps": by["decode"] / decode_s / 1e9,
                          "frac": by["decode"] / decode_s / 1e9 / peak},
        "full_cache": None if full_ms is None else {
            "what": "the same attention over every page (no scoring, no selection) on this GPU",
            "ms_per_step": full_ms, "steps_per_s": 1e3 / full_ms,
            "sparse_speedup": full_ms / ms},
        "selection_quality": quality,
        "e2e": {"value": replicas.job_rate(args.steps, world, e2e_s), "unit": "steps/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step * args.steps,
        "launch": "one CUDA graph per step (programmatic dependent launch between its kernels)",
        "clocks": clocks.summary(),
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


def reference_arm(args, rank, world, make):
    """The CPU oracle as it stands, on the host cores, same workload/metric/unit; rank 0 only."""
    if rank != 0:
        return
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    from sparse_kv_cache_kmin_b200 import replicas
    wl = make(args.workload, device=dev, seed=replicas.workload_seed(args.workload, 0))
    attn = wl.attn_modes[0] if args.attn is None else args.attn
    if args.policy is not None:
        wl.policy = {v: k for k, v in POLICY_NAME.items()}[args.policy]
    n_steps = max(args.warmup, 3) + args.steps
    budget = max(2.0, 150.0 / n_steps)  # the whole run stays within a few minutes
    times = []
    desc = ""
    for i in range(n_steps):
        per_step, desc = oracle_sample(wl, attn, budget, max_heads=None)
        if i >= max(args.warmup, 3):
            times.append(per_step)
    value = 1.0 / statistics.mean(times)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(args.warmup, 3),
        "ms_per_step": statistics.mean(times) * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded)",
        "config": {"workload": wl.name, "batch_per_gpu": wl.batch, "ctx": int(wl.seq_lens.max()),
                   "q_heads": wl.num_q_heads, "kv_heads": wl.num_kv_heads,
                   "head_dim": wl.head_dim, "page": wl.page_size, "attn": ATTN_NAME[attn]},
        "cpu_baseline": {"value": value, "unit": "steps/s", "cores": 1, "kind": "oracle",
                         "sample": desc + "; each step a fresh bounded sample"},
        "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
