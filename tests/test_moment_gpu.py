"""GPU parity of the moment-corrected softmax (MomentKV technical summary, Methodology §1, §2,
§4): the running sums against the oracle's sums, and the corrected output against the oracle fed
the GPU's own selection, on small ragged cases over every dtype, head size, page size and group
size (one sequence of a single token has nothing skipped)."""
import itertools

import numpy as np
import pytest
import torch

import oracle as O
from sparse_kv_cache_kmin_b200 import ekv
from sparse_kv_cache_kmin_b200.workloads import make_random
from parity_utils import HostCopy, close, run_gpu

pytestmark = pytest.mark.gpu

CASES = list(itertools.product([torch.float32, torch.bfloat16], [64, 128], [16, 64], [1, 4, 8]))


def prefill_moments(cache, wl):
    mom = torch.zeros(ekv.ekv_moment_bytes(cache) // 4, dtype=torch.float32, device="cuda")
    zeros = torch.zeros(wl.batch, dtype=torch.int32, device="cuda")
    ekv.ekv_moment_update(cache, mom, zeros, wl.seq_lens, int(wl.seq_lens.max().item()))
    return mom


@pytest.mark.parametrize("dtype,d,P,G", CASES,
                         ids=["%s-d%d-P%d-G%d" % (str(t)[6:], d, P, G) for t, d, P, G in CASES])
def test_moment_corrected_softmax_small_ragged(cuda_device, dtype, d, P, G):
    wl = make_random(B=3, H_kv=2, G=G, d=d, P=P, lens=(1000, 517, 1),
                     dtype=dtype, device="cuda", seed=5, topk=6)
    check_moment(wl)


@pytest.mark.parametrize("topk", [128, 64], ids=["pages64_per_cta", "pages32_per_cta"])
def test_moment_many_pairs_long_retained_loops(cuda_device, topk):
    # 16 x 8 (sequence, KV head) pairs: the retained sums take 64 or 32 selected pages per CTA
    # (the most that leave 1.5 CTAs per SM), not the 8 of the small cases
    lens = tuple(16 * (150 + 7 * i) + i % 5 for i in range(16))
    wl = make_random(B=16, H_kv=8, G=4, d=128, P=16, lens=lens, dtype=torch.bfloat16,
                     device="cuda", seed=17 + topk, topk=topk)
    check_moment(wl, pairs=[(0, 0), (7, 3), (15, 7)])


def check_moment(wl, pairs=None):
    dtype, d, G = wl.k_cache.dtype, wl.head_dim, wl.num_q_heads // wl.num_kv_heads
    cache, dec = run_gpu(wl, ekv.EKV_SOFTMAX)
    mom = prefill_moments(cache, wl)
    need = ekv.ekv_moment_decode_workspace_bytes(cache, wl.num_q_heads, dec.max_sel)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    out = torch.empty_like(dec.out)
    stat = torch.empty_like(dec.stat)
    ekv.ekv_sparse_decode_moment(cache, mom, wl.q, wl.num_q_heads, wl.scale, dec.sel_idx,
                                 dec.sel_count, dec.max_sel, out, stat, ws)
    torch.cuda.synchronize()
    st, bits = ekv.ekv_device_status(cache)
    assert st == ekv.EKV_OK, hex(bits)
    rec = mom.view(wl.batch, wl.num_kv_heads, -1).double().cpu().numpy()
    bf16 = dtype == torch.bfloat16
    pairs = pairs or [(b, h) for b in range(wl.batch) for h in range(wl.num_kv_heads)]
    for b in sorted({b for b, _ in pairs}):
        hc = HostCopy(wl, b)
        for h in [h for bb, h in pairs if bb == b]:
            n, sk, sv, S = O.moment_sums_head(hc.k, hc.v, hc.pt, hc.L, h)
            assert rec[b, h, 0] == n
            np.testing.assert_allclose(rec[b, h, 4:4 + d], sk, rtol=1e-5, atol=1e-5 * n)
            np.testing.assert_allclose(rec[b, h, 4 + d:4 + 2 * d], sv, rtol=1e-5, atol=1e-5 * n)
            np.testing.assert_allclose(rec[b, h, 4 + 2 * d:].reshape(d, d), S, rtol=1e-5,
                                       atol=1e-5 * n * 10)
            ns = int(dec.sel_count[b, h].item())
            sel = dec.sel_idx[b, h, :ns].cpu().numpy()
            ref, rstat, _ = O.moment_corrected_head(hc.k, hc.v, hc.pt, hc.L, h, hc.q[h], wl.scale, sel)
            close(out[b, h * G:(h + 1) * G].double().cpu().numpy(), ref, bf16)
            close(stat[b, h * G:(h + 1) * G].double().cpu().numpy(), rstat, bf16)
