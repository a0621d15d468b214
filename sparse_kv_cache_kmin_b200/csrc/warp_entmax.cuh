// warp_entmax.cuh -- the exact alpha-entmax threshold of a small candidate set held by one
// warp (sparsemax: Martins & Astudillo 2016; 1.5-entmax: Peters, Niculae & Martins 2019), and
// the closed forms of a support's threshold, shared by the decode kernels.
#pragma once

#include "ekv_device.cuh"

namespace ekv {

// Bitonic sort, descending, of 32*R values held R per lane (element e = r*32 + lane).
template <int R>
__device__ __forceinline__ void warp_sort_desc(float (&v)[R])
{
    const int lane = threadIdx.x & 31;
    constexpr int N = 32 * R;
#pragma unroll
    for (int k = 2; k <= N; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            if (j >= 32) {
                const int rj = j / 32;
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    if (r & rj) continue;
                    const int e = r * 32 + lane;
                    const bool up = (e & k) == 0;
                    const float hi = fmaxf(v[r], v[r | rj]), lo = fminf(v[r], v[r | rj]);
                    v[r] = up ? hi : lo;
                    v[r | rj] = up ? lo : hi;
                }
            } else {
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const int e = r * 32 + lane;
                    const float o = __shfl_xor_sync(kFull, v[r], j);
                    const bool up = (e & k) == 0, lower = (lane & j) == 0;
                    v[r] = (lower == up) ? fmaxf(v[r], o) : fminf(v[r], o);
                }
            }
        }
    }
}

// Exact threshold of at most 32*R candidates held R per lane (x = z - zmax in [-1, 0], -inf
// padding): sort descending, prefix sums of x and x^2 in sorted order, then the largest k whose
// closed-form tau(k) satisfies tau(k) <= x_(k) (1.5-entmax also needs a real root). fp32
// throughout: with x in [-1, 0] and at most 128 terms the sums carry ~1e-5 absolute error, far
// inside the output tolerances, and fp32 keeps the dependent chain short.
template <int R>
__device__ __forceinline__ double warp_exact_tau(float (&v)[R], int cnt, bool sparsemax)
{
    const int lane = threadIdx.x & 31;
    warp_sort_desc<R>(v);
    float carry1 = 0.f, carry2 = 0.f, best_t = 0.f;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int e = r * 32 + lane;
        const bool in = e < cnt;
        const float xd = in ? v[r] : 0.f;
        float s1 = xd, s2 = xd * xd;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float t1 = __shfl_up_sync(kFull, s1, o), t2 = __shfl_up_sync(kFull, s2, o);
            if (lane >= o) { s1 += t1; s2 += t2; }
        }
        s1 += carry1;
        s2 += carry2;
        carry1 = __shfl_sync(kFull, s1, 31);
        carry2 = __shfl_sync(kFull, s2, 31);
        const float kk = (float)(e + 1);
        float tk;
        bool ok = in;
        if (sparsemax) {
            tk = (s1 - 1.0f) / kk;
        } else {
            const float mean = s1 / kk;
            const float m2 = fmaxf(s2 - s1 * mean, 0.f);  // sum of squared deviations of the top k
            const float disc = (1.0f - m2) / kk;
            ok = ok && disc >= 0.f;
            tk = mean - sqrtf(fmaxf(disc, 0.f));
        }
        ok = ok && tk <= v[r];
        const unsigned bal = __ballot_sync(kFull, ok);
        if (bal) best_t = __shfl_sync(kFull, tk, 31 - __clz(bal));  // later rows win
    }
    return (double)best_t;  // element 0 is always valid: tau(1) = x_(1) - 1
}

// Whether the closed-form threshold of a support with n members, sum s1 and sum of squares s2
// is real and at most x (the support's smallest member), without a division or a square root:
// sparsemax: (s1 - 1) / n <= x  <=>  s1 - 1 <= n x; 1.5-entmax: with n^2 disc = n - n s2 + s1^2,
// s1 / n - sqrt(disc) <= x  <=>  s1 - n x <= 0 or (s1 - n x)^2 <= n^2 disc.
__device__ __forceinline__ bool closed_form_ok(double n, double s1, double s2, double x, bool sparsemax)
{
    if (sparsemax) return s1 - 1.0 <= n * x;
    const double d2 = n - n * s2 + s1 * s1;
    if (d2 < 0.0) return false;
    const double u = s1 - n * x;
    return u <= 0.0 || u * u <= d2;
}

// Closed-form threshold of a support with n members, sum s1 and sum of squares s2 (x space):
// sparsemax sum (x - tau) = 1; 1.5-entmax sum (x - tau)^2 = 1 (smaller root). Returns false when
// the quadratic has no real root (the support is too wide).
__device__ __forceinline__ bool closed_form_tau(double n, double s1, double s2, bool sparsemax,
                                                double &tau)
{
    if (sparsemax) {
        tau = (s1 - 1.0) / n;
        return true;
    }
    const double mean = s1 / n;
    const double disc = (1.0 - fmax(s2 - s1 * mean, 0.0)) / n;
    tau = mean - sqrt(fmax(disc, 0.0));
    return disc >= 0.0;
}

}  // namespace ekv
