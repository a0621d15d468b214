"""Seeded synthetic decode workloads: paged K/V caches, page tables, lengths and queries.

Input generation only -- nothing here computes any part of the method. The same tensors feed
the CUDA library and, copied to the host, the CPU oracle. Every draw comes from a generator
seeded by the workload's seed: large tensors from a torch.Generator on the target device,
small host-side choices (positions, run lengths, cluster ids) from numpy's default_rng.

Named workloads (the decode shapes the method is evaluated on; scale = 1 throughout, the
query distribution fixes the logit scale):
  tiny     B1, 1 q / 1 KV head, d64, 4096 tokens, P16, fp32, K/V/q iid N(0,1), top-k 32
  gqa32k   B4, 32 q / 8 KV heads, d128, 32768 tokens, P16, bf16, K/V N(0,1) with the same 4
           seeded channels per KV head scaled x8 (on K and V), q N(0,1)/sqrt(128), top-k 256
  needle128k  B8, 32/8, d128, 131072 tokens, P16, bf16, K/V N(0,1) plus 64 needle keys per
           KV head at distinct seeded positions, needle n aligned with query g = n % 4:
           k = sqrt(d) (0.9 q_hat_g + sqrt(0.19) u_perp); q N(0,1)/sqrt(128); top-k 256, 1.5-entmax
  gauss    B16, lengths uniform in [8192, 65536] (token granularity), 32/8, d128, P32, bf16;
           per KV head 8 cluster centres mu_c ~ N(0, I); keys mu_c + 0.5 N(0, I) in contiguous
           runs of Geometric(mean 512) tokens with a uniform cluster per run; query head g:
           (mu_{c*} + N(0, I)) / sqrt(128) for a uniform c*; V N(0,1); 1.5-entmax, Delta 0.1
  long1m   B1, 64 q / 8 KV heads, d128, 1048576 tokens, P64, bf16, K/V N(0,1), q N(0,1)/sqrt(128);
           the last 4096 keys of KV head h get + 4 * unit(mean of its 8 queries); top-k 164
           (1% of 16384 pages), sparsemax and softmax; every decode step appends the final
           64-token page (its metadata is recomputed in the step)
Physical blocks are a seeded permutation, so consecutive logical pages are scattered as in a
paged allocator; page-table entries past a sequence's last page are -1.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

SOFTMAX, ENTMAX15, SPARSEMAX = 0, 1, 2  # attention modes (values of ekv_attn)
TOPK, GAUSS, GAUSS_MAX = 0, 1, 2        # selection policies (values of ekv_policy)


@dataclass
class Workload:
    name: str
    k_cache: torch.Tensor          # [num_blocks, H_kv, P, d]
    v_cache: torch.Tensor
    page_table: torch.Tensor       # [B, max_pages] int32
    seq_lens: torch.Tensor         # [B] int32
    q: torch.Tensor                # [B, H_q, d], cache dtype
    num_q_heads: int
    policy: int
    attn_modes: list
    topk: int = 0
    alpha: float = 1.5
    delta: float = 0.0
    scale: float = 1.0
    append: Optional[tuple] = None  # (start, count): tokens each decode step appends
    notes: dict = field(default_factory=dict)

    @property
    def batch(self):
        return self.page_table.shape[0]

    @property
    def num_kv_heads(self):
        return self.k_cache.shape[1]

    @property
    def page_size(self):
        return self.k_cache.shape[2]

    @property
    def head_dim(self):
        return self.k_cache.shape[3]

    @property
    def max_pages(self):
        return self.page_table.shape[1]

    def max_sel(self) -> int:
        return min(self.topk, self.max_pages) if self.policy == TOPK else self.max_pages


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _layout(lens, P, rng, device):
    """Scattered block assignment: page j of sequence b -> block page_table[b, j]."""
    pages = [(int(L) + P - 1) // P for L in lens]
    nb = max(1, sum(pages))
    perm = rng.permutation(nb).astype(np.int32)
    max_pages = max(1, max(pages))
    pt = np.full((len(lens), max_pages), -1, np.int32)
    off = 0
    for b, n in enumerate(pages):
        pt[b, :n] = perm[off:off + n]
        off += n
    return nb, torch.from_numpy(pt).to(device), torch.tensor(lens, dtype=torch.int32, device=device)


def token_rows(page_table: torch.Tensor, b: int, h: int, H_kv: int, P: int, tokens) -> torch.Tensor:
    """Row indices into k_cache.view(-1, d) of logical tokens `tokens` of (sequence b, head h)."""
    t = torch.as_tensor(tokens, device=page_table.device, dtype=torch.long)
    blk = page_table[b].long()[t // P]
    return (blk * H_kv + h) * P + t % P


def make_random(B=2, H_kv=2, G=4, d=128, P=16, lens=(100, 37), dtype=torch.bfloat16,
                device="cpu", seed=0, kv_scale=1.0, q_scale=None, policy=TOPK, topk=4,
                attn_modes=(SOFTMAX, ENTMAX15, SPARSEMAX), alpha=1.5, delta=0.1, scale=1.0,
                name="random"):
    """iid N(0, kv_scale^2) keys/values and N(0, q_scale^2) queries on a scattered layout."""
    rng = np.random.default_rng(seed)
    g = _gen(device, seed)
    nb, pt, sl = _layout(list(lens)[:B], P, rng, device)
    k = torch.randn((nb, H_kv, P, d), generator=g, device=device) * kv_scale
    v = torch.randn((nb, H_kv, P, d), generator=g, device=device)
    qs = 1.0 / math.sqrt(d) if q_scale is None else q_scale
    q = torch.randn((B, H_kv * G, d), generator=g, device=device) * qs
    return Workload(name, k.to(dtype), v.to(dtype), pt, sl, q.to(dtype), H_kv * G, policy,
                    list(attn_modes), topk=topk, alpha=alpha, delta=delta, scale=scale)


def make_tiny(device="cpu", seed=1):
    rng = np.random.default_rng(seed)
    g = _gen(device, seed)
    B, H, d, P, L = 1, 1, 64, 16, 4096
    nb, pt, sl = _layout([L], P, rng, device)
    k = torch.randn((nb, H, P, d), generator=g, device=device)
    v = torch.randn((nb, H, P, d), generator=g, device=device)
    q = torch.randn((B, 1, d), generator=g, device=device)
    return Workload("tiny", k, v, pt, sl, q, 1, TOPK, [SOFTMAX, ENTMAX15], topk=32)


def make_gqa32k(device="cuda", seed=2, B=4, L=32768):
    rng = np.random.default_rng(seed)
    g = _gen(device, seed)
    H, G, d, P = 8, 4, 128, 16
    nb, pt, sl = _layout([L] * B, P, rng, device)
    k = torch.randn((nb, H, P, d), generator=g, device=device)
    v = torch.randn((nb, H, P, d), generator=g, device=device)
    for h in range(H):
        ch = torch.as_tensor(rng.choice(d, size=4, replace=False), device=device)
        k[:, h, :, ch] *= 8.0
        v[:, h, :, ch] *= 8.0
    q = torch.randn((B, H * G, d), generator=g, device=device) / math.sqrt(d)
    return Workload("gqa32k", k.to(torch.bfloat16), v.to(torch.bfloat16), pt, sl,
                    q.to(torch.bfloat16), H * G, TOPK, [SOFTMAX, ENTMAX15], topk=256)


def make_needle128k(device="cuda", seed=3, B=8, L=131072, n_needles=64):
    rng = np.random.default_rng(seed)
    g = _gen(device, seed)
    H, G, d, P = 8, 4, 128, 16
    nb, pt, sl = _layout([L] * B, P, rng, device)
    k = torch.randn((nb, H, P, d), generator=g, device=device)
    v = torch.randn((nb, H, P, d), generator=g, device=device)
    q = (torch.randn((B, H * G, d), generator=g, device=device) / math.sqrt(d)).to(torch.bfloat16)
    qf = q.float()
    kflat = k.view(-1, d)
    for b in range(B):
        for h in range(H):
            pos = rng.choice(L, size=n_needles, replace=False)
            qh = qf[b, h * G:(h + 1) * G]
            qh = qh / qh.norm(dim=1, keepdim=True)
            gi = torch.arange(n_needles, device=device) % G
            qhat = qh[gi]
            u = torch.randn((n_needles, d), generator=g, device=device)
            u = u - (u * qhat).sum(1, keepdim=True) * qhat
            u = u / u.norm(dim=1, keepdim=True)
            kflat[token_rows(pt, b, h, H, P, pos)] = math.sqrt(d) * (0.9 * qhat + math.sqrt(0.19) * u)
    return Workload("needle128k", k.to(torch.bfloat16), v.to(torch.bfloat16), pt, sl, q, H * G,
                    TOPK, [ENTMAX15], topk=256, alpha=1.5)


def make_gauss(device="cuda", seed=4, B=16, lo=8192, hi=65536, n_clusters=8, run_mean=512):
    rng = np.random.default_rng(seed)
    g = _gen(device, seed)
    H, G, d, P = 8, 4, 128, 32
    lens = [int(x) for x in rng.integers(lo, hi + 1, size=B)]
    nb, pt, sl = _layout(lens, P, rng, device)
    k = torch.zeros((nb, H, P, d), device=device)
    v = torch.randn((nb, H, P, d), generator=g, device=device)
    q = torch.empty((B, H * G, d), device=device)
    kflat = k.view(-1, d)
    for b in range(B):
        L = lens[b]
        for h in range(H):
            mu = torch.randn((n_clusters, d), generator=g, device=device)
            ids = np.empty(L, np.int64)
            t = 0
            while t < L:
                run = int(rng.geometric(1.0 / run_mean))
                ids[t:t + run] = rng.integers(n_clusters)
                t += run
            idt = torch.from_numpy(ids).to(device)
            rows = token_rows(pt, b, h, H, P, np.arange(L))
            kflat[rows] = mu[idt] + 0.5 * torch.randn((L, d), generator=g, device=device)
            cstar = torch.as_tensor(rng.integers(n_clusters, size=G), device=device)
            q[b, h * G:(h + 1) * G] = (mu[cstar] + torch.randn((G, d), generator=g, device=device)) / math.sqrt(d)
    return Workload("gauss", k.to(torch.bfloat16), v.to(torch.bfloat16), pt, sl,
                    q.to(torch.bfloat16), H * G, GAUSS, [ENTMAX15], alpha=1.5, delta=0.1)


def make_long1m(device="cuda", seed=5, L=1048576, recent=4096, shift=4.0):
    rng = np.random.default_rng(seed)
    g = _gen(device, seed)
    B, H, G, d, P = 1, 8, 8, 128, 64
    nb, pt, sl = _layout([L], P, rng, device)
    k = torch.randn((nb, H, P, d), generator=g, device=device)
    v = torch.randn((nb, H, P, d), generator=g, device=device)
    q = (torch.randn((B, H * G, d), generator=g, device=device) / math.sqrt(d)).to(torch.bfloat16)
    kflat = k.view(-1, d)
    for h in range(H):
        qm = q[0, h * G:(h + 1) * G].float().mean(0)
        rows = token_rows(pt, 0, h, H, P, np.arange(L - recent, L))
        kflat[rows] += shift * qm / qm.norm()
    n_pages = (L + P - 1) // P
    return Workload("long1m", k.to(torch.bfloat16), v.to(torch.bfloat16), pt, sl, q, H * G, TOPK,
                    [SPARSEMAX, SOFTMAX], topk=int(math.ceil(0.01 * n_pages)), alpha=2.0,
                    append=(L - P, P))


NAMED = {"tiny": make_tiny, "gqa32k": make_gqa32k, "needle128k": make_needle128k,
         "gauss": make_gauss, "long1m": make_long1m}


def make(name: str, device="cuda", **kw) -> Workload:
    return NAMED[name](device=device, **kw)
