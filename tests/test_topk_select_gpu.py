"""GPU parity of the top-k page selection on crafted score rows, against the oracle's stable sort
(key descending, lower page first): distributions that drive every branch of the selection --
one histogram pass, refinement of a crowded boundary bin (a tight cluster with far outliers),
a boundary bin that is a single repeated value (ties kept in page order), rows with -inf
entries, lengths below, at and just above k -- at each of the kernel's size classes (keys in
registers up to 8192 and 16384 pages, staged beyond)."""
import numpy as np
import pytest
import torch

import oracle as O
from sparse_kv_cache_kmin_b200 import ekv

pytestmark = pytest.mark.gpu

P = 16


def crafted(kind, n, rng):
    if kind == "normal":
        return rng.standard_normal(n)
    if kind == "cluster":  # nearly all keys within 1e-4 of 1, a few far above and below
        x = 1.0 + 1e-4 * rng.random(n)
        far = rng.choice(n, size=min(12, n), replace=False)
        x[far[:6]] = 1e3 + rng.random(6)
        x[far[6:]] = -1e3 - rng.random(len(far) - 6)
        return x
    if kind == "two_values":
        return np.where(rng.random(n) < 0.5, 1.0, 2.0)
    if kind == "ints":  # many exact ties at several levels
        return rng.integers(0, 40, n).astype(np.float64)
    if kind == "neg_inf":
        x = rng.standard_normal(n)
        x[rng.random(n) < 0.3] = -np.inf
        return x
    raise ValueError(kind)


def run_select(rows, lens, k, max_pages):
    B, H = len(lens), rows.shape[1]
    cache = ekv.PagedKVCache.allocate(num_blocks=4, num_kv_heads=H, page_size=P, head_dim=64,
                                      batch=B, max_pages=max_pages, gaussian=False)
    cache.seq_lens.copy_(torch.tensor([n * P for n in lens], dtype=torch.int32))
    scores = torch.from_numpy(rows.astype(np.float32)).cuda()
    max_sel = min(k, max_pages)
    sel = torch.full((B, H, max_sel), 7777, dtype=torch.int32, device="cuda")
    cnt = torch.full((B, H), 7777, dtype=torch.int32, device="cuda")
    tau = torch.empty((B, H), dtype=torch.float32, device="cuda")
    ekv.ekv_select_pages(cache, H, ekv.EKV_SEL_TOPK, k, 1.5, 0.0, scores, sel, cnt, max_sel, tau)
    st, bits = ekv.ekv_device_status(cache)
    assert st == ekv.EKV_OK, hex(bits)
    return sel.cpu().numpy(), cnt.cpu().numpy()


SIZES = [4096, 8192, 12000, 16384, 20000]
KINDS = ["normal", "cluster", "two_values", "ints", "neg_inf"]


@pytest.mark.parametrize("max_pages", SIZES, ids=["pages%d" % n for n in SIZES])
@pytest.mark.parametrize("kind", KINDS)
def test_topk_selection_matches_the_oracle_sort(cuda_device, kind, max_pages):
    rng = np.random.default_rng(max_pages + len(kind))
    k = 300
    lens = [max_pages, max_pages - 3, k + 1, k, 77]
    H = 2
    rows = np.full((len(lens), H, max_pages), np.nan)  # past a sequence's pages: never read
    for b, n in enumerate(lens):
        for h in range(H):
            rows[b, h, :n] = crafted(kind, n, rng)
    rows = np.nan_to_num(rows, nan=0.0, posinf=np.inf, neginf=-np.inf)
    sel, cnt = run_select(rows, lens, k, max_pages)
    for b, n in enumerate(lens):
        for h in range(H):
            want = O.topk(rows[b, h, :n].astype(np.float32).astype(np.float64), k)
            assert cnt[b, h] == len(want)
            np.testing.assert_array_equal(sel[b, h, :cnt[b, h]], want)
            assert np.all(sel[b, h, cnt[b, h]:] == -1)
