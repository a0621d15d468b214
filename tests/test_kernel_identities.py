"""CPU checks of the exact identities the CUDA kernels rely on but the oracle does not use.

- The group bound: sum_g max(q_g kmin, q_g kmax) = Q+ . kmax + Q- . kmin with Q+- the group sums
  of the queries' positive and negative parts (kmin <= kmax).
- MomentKV correction: the skipped tokens' count, means and centred cross moment applied to q
  follow from running totals less the selected tokens' sums:
  sum_E (v - vbar)(k - kbar)^T q = [(sum v k^T) q - sum_R v (k.q)] - n_e vbar (kbar . q).
- Token-level attention: the entmax threshold from bisection on [max z - 1, max z] followed by
  the closed form over the support it brackets is the exact sort-based threshold.
Each is evaluated in float64 and compared with the oracle."""
import numpy as np
import pytest

import oracle as O
from test_oracle_pins import make_seq


def test_group_bound_sign_split_identity():
    rng = np.random.default_rng(61)
    for _ in range(20):
        d, G = 16, 4
        a, b = rng.standard_normal((2, d))
        kmin, kmax = np.minimum(a, b), np.maximum(a, b)
        q = rng.standard_normal((G, d))
        lhs = sum(np.maximum(q[g] * kmin, q[g] * kmax).sum() for g in range(G))
        rhs = np.maximum(q, 0).sum(0) @ kmax + np.minimum(q, 0).sum(0) @ kmin
        assert abs(lhs - rhs) <= 1e-12 * (1 + abs(lhs))


@pytest.mark.parametrize("sel", [[0, 5, 9, 17], [38], []])
def test_moment_correction_from_running_sums(sel):
    rng = np.random.default_rng(62)
    L, P, d, h, G, scale = 613, 16, 32, 1, 4, 0.6
    k, v, pt = make_seq(rng, P=P, d=d, L=L, nb=60, H_kv=2)
    q = rng.standard_normal((G, d)) / np.sqrt(d)
    n, sk, sv, S = O.moment_sums_head(k, v, pt, L, h)          # running totals
    nR, skR, svR, _ = O.moment_sums_head(k, v, pt, L, h, sel)  # selected tokens
    fR, statR, _ = O.attend_head(k, v, pt, L, h, q, scale, O.SOFTMAX, sel)
    ref, rstat, n_e = O.moment_corrected_head(k, v, pt, L, h, q, scale, sel)
    rows = [(pt[j], t) for j in sel for t in range(min(P, L - j * P))]
    KR = np.array([k[b_, h, t] for b_, t in rows], np.float64).reshape(-1, d)
    VR = np.array([v[b_, h, t] for b_, t in rows], np.float64).reshape(-1, d)
    assert n - nR == n_e
    for g in range(G):
        u = VR.T @ (KR @ q[g])                     # sum_R v (k . q)
        kbar, vbar = (sk - skR) / n_e, (sv - svR) / n_e
        qk = kbar @ q[g]
        stq = (S @ q[g] - u) - n_e * vbar * qk
        fe = vbar + scale / n_e * stq
        lzr, lze = statR[g], np.log(n_e) + scale * qk
        m = max(lzr, lze)
        zr, ze = np.exp(lzr - m), np.exp(lze - m)
        out = zr / (zr + ze) * fR[g] + ze / (zr + ze) * fe
        np.testing.assert_allclose(out, ref[g], rtol=0, atol=1e-12)
        assert abs(m + np.log(zr + ze) - rstat[g]) < 1e-12


@pytest.mark.parametrize("alpha", [1.5, 2.0])
def test_bisection_then_closed_form_threshold(alpha):
    rng = np.random.default_rng(63)
    for _ in range(60):
        n = int(rng.integers(1, 2000))
        z = (rng.standard_normal(n) * rng.choice([0.01, 0.3, 2.0, 8.0])).astype(np.float32).astype(np.float64)
        lo, hi = z.max() - 1.0, z.max()
        for _ in range(60):
            mid = 0.5 * (lo + hi)
            r = z - mid
            f = r[r > 0].sum() if alpha == 2.0 else (r[r > 0] ** 2).sum()
            lo, hi = (mid, hi) if f >= 1.0 else (lo, mid)
        S = z[z > lo]
        if alpha == 2.0:
            tau = (S.sum() - 1.0) / len(S)
        else:
            # the kernel's route: raw sums, then mean and the squared deviations from them
            k_, s1, s2 = len(S), S.sum(), (S * S).sum()
            mean = s1 / k_
            tau = mean - np.sqrt(max((1.0 - (s2 - k_ * mean * mean)) / k_, 0.0))
        ref = O.entmax_tau(z, alpha)
        assert abs(tau - ref) <= 1e-12 * max(1.0, abs(ref))
