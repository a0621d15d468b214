// topk_cta.cuh -- exact top-k of one (sequence, KV head) by one thread block, each thread
// holding R consecutive keys in registers (EntmaxKV technical summary, §2.B.1: the k pages of
// largest upper-bound score, ties to the lower page index).
//
// Keys are the order-preserving uint32 images of the fp32 scores (NaN lowest, -0 == +0).
// Thread t owns pages [t R, t R + R). The k-th largest key is located by histograms over a
// shrinking key range [lo, hi]: a bin is a run of 2^s consecutive keys, s the fewest bits
// that leave at most 2048 bins (a subtraction and a shift per key, and each bin an exact key
// interval); the bin holding the k-th largest key becomes the next range. Once that bin holds
// at most kTopkRank keys they are ranked exactly (key descending, page ascending) -- or all
// kept, when the bin holds exactly the keys still needed; once the range is a single key value,
// the remaining ties are kept in page order by a block scan.
// Every key above the final range is kept. Three refinements always reach a single value; on
// scores from a continuous distribution one suffices.
#pragma once
#include "ekv_device.cuh"

namespace ekv {

constexpr int kTopkBins = 2048;
constexpr int kTopkRank = 256;  // boundary keys ranked exactly

__device__ __forceinline__ uint32_t topk_order_key(float x)
{
    if (x != x) return 0u;                  // NaN sorts below everything
    uint32_t u = __float_as_uint(x + 0.0f);  // -0 -> +0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct __align__(16) TopkShared {
    int hist[kTopkBins];
    int warp_tot[32];
    uint32_t rk_u[kTopkRank];
    int rk_j[kTopkRank];
    uint32_t lo, hi, bin_lo, bin_hi;
    int bin, above, cnt, mode;  // mode: 0 rank the boundary bin, 1 ties in page order, 2 keep it
};

// Bin width 2^s for the range [lo, hi]: (hi - lo) >> s < 2048.
__device__ __forceinline__ int topk_shift(uint32_t lo, uint32_t hi)
{
    const int bits = 32 - __clz(hi - lo);  // bits of the largest offset
    return bits > 11 ? bits - 11 : 0;
}

// Selects the kk largest of n keys (kk < n, n <= R * NT). u[r] is the key of page t R + r
// (ignored where t R + r >= n). On return keep[r] marks the kept pages and the function returns
// the thread's number of kept pages; every thread of the block must call it.
template <int NT, int R>
__device__ int cta_topk(const uint32_t (&u)[R], int n, int kk, TopkShared &s, bool (&keep)[R])
{
    const int tid = threadIdx.x, lane = tid & 31;
    const int j0 = tid * R;
    uint32_t mn = 0xffffffffu, mx = 0u;
#pragma unroll
    for (int r = 0; r < R; ++r)
        if (j0 + r < n) { mn = min(mn, u[r]); mx = max(mx, u[r]); }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        mn = min(mn, __shfl_xor_sync(kFull, mn, o));
        mx = max(mx, __shfl_xor_sync(kFull, mx, o));
    }
    if (tid == 0) { s.lo = 0xffffffffu; s.hi = 0u; }
    for (int i = tid; i < kTopkBins; i += NT) s.hist[i] = 0;  // the first pass's histogram
    __syncthreads();
    if (lane == 0) { atomicMin(&s.lo, mn); atomicMax(&s.hi, mx); }
    __syncthreads();
    uint32_t lo = s.lo, hi = s.hi;
    int need = kk;
    // refine [lo, hi] until the boundary bin is small or a single value
    for (int pass = 0; pass < 4; ++pass) {
        if (lo == hi) {
            if (tid == 0) s.mode = 1;
            break;
        }
        const int sh = topk_shift(lo, hi);
        if (pass > 0) {
            for (int i = tid; i < kTopkBins; i += NT) s.hist[i] = 0;
            __syncthreads();
        }
#pragma unroll
        for (int r = 0; r < R; ++r)
            if (j0 + r < n && u[r] >= lo && u[r] <= hi) atomicAdd(&s.hist[(u[r] - lo) >> sh], 1);
        __syncthreads();
        // the bin holding the need-th largest key in the range: thread t owns bins from the top
        constexpr int BPT = kTopkBins / NT;
        int cnt[BPT], sum = 0;
#pragma unroll
        for (int q = 0; q < BPT; ++q) {
            cnt[q] = s.hist[kTopkBins - 1 - BPT * tid - q];
            sum += cnt[q];
        }
        const int incl = block_incl_scan<NT>(sum, s.warp_tot, nullptr);
        int run = incl - sum;
#pragma unroll
        for (int q = 0; q < BPT; ++q) {
            if (cnt[q] > 0 && run < need && need <= run + cnt[q]) {
                const int B = kTopkBins - 1 - BPT * tid - q;
                s.bin = B;
                s.above = run;
                s.cnt = cnt[q];
                // key interval of bin B: u - lo in [B 2^s, (B + 1) 2^s - 1], within [lo, hi]
                const unsigned long long top = (unsigned long long)lo + ((unsigned long long)(B + 1) << sh) - 1ull;
                s.bin_lo = lo + ((uint32_t)B << sh);
                s.bin_hi = top < (unsigned long long)hi ? (uint32_t)top : hi;
            }
            run += cnt[q];
        }
        __syncthreads();
        need -= s.above;
        lo = s.bin_lo;
        hi = s.bin_hi;
        if (s.cnt == need) {  // the whole boundary bin is kept: nothing to rank
            if (tid == 0) s.mode = 2;
            break;
        }
        if (s.cnt <= kTopkRank) {
            if (tid == 0) s.mode = 0;
            break;
        }
    }
    __syncthreads();
    // keys above the final range are kept; inside it, rank (mode 0) or page order (mode 1)
    int mine = 0;
    if (s.mode == 0) {
        if (tid == 0) s.cnt = 0;
        __syncthreads();
#pragma unroll
        for (int r = 0; r < R; ++r)
            if (j0 + r < n && u[r] >= lo && u[r] <= hi) {
                const int p = atomicAdd(&s.cnt, 1);
                s.rk_u[p] = u[r];
                s.rk_j[p] = j0 + r;
            }
        __syncthreads();
        const int cb = s.cnt;
        // mark the kept boundary pages in the hist array, reused as a bit set over pages
        static_assert(kTopkBins * 32 >= NT * R, "one bit per page");
        for (int i = tid; i < (n + 31) / 32; i += NT) s.hist[i] = 0;
        __syncthreads();
        if (tid < cb) {
            const uint32_t x = s.rk_u[tid];
            const int j = s.rk_j[tid];
            int rank = 0;
            int m = 0;
            for (; m + 4 <= cb; m += 4) {  // four keys and pages per shared-memory load
                const uint4 y = *reinterpret_cast<const uint4 *>(&s.rk_u[m]);
                const int4 q = *reinterpret_cast<const int4 *>(&s.rk_j[m]);
                rank += (y.x > x || (y.x == x && q.x < j)) + (y.y > x || (y.y == x && q.y < j)) +
                        (y.z > x || (y.z == x && q.z < j)) + (y.w > x || (y.w == x && q.w < j));
            }
            for (; m < cb; ++m) rank += s.rk_u[m] > x || (s.rk_u[m] == x && s.rk_j[m] < j);
            if (rank < need) atomicOr(reinterpret_cast<unsigned *>(&s.hist[j >> 5]), 1u << (j & 31));
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int j = j0 + r;
            keep[r] = j < n && (u[r] > hi ||
                                (u[r] >= lo && ((reinterpret_cast<const unsigned *>(s.hist)[j >> 5] >> (j & 31)) & 1u)));
            mine += keep[r];
        }
    } else if (s.mode == 2) {
#pragma unroll
        for (int r = 0; r < R; ++r) {
            keep[r] = j0 + r < n && u[r] >= lo;
            mine += keep[r];
        }
    } else {
        // a single key value lo == hi: its first `need` pages in page order
        int ties = 0;
#pragma unroll
        for (int r = 0; r < R; ++r) ties += j0 + r < n && u[r] == lo;
        int before = block_incl_scan<NT>(ties, s.warp_tot, nullptr) - ties;
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const bool tie = j0 + r < n && u[r] == lo;
            keep[r] = (j0 + r < n && u[r] > lo) || (tie && before < need);
            before += tie;
            mine += keep[r];
        }
    }
    __syncthreads();
    return mine;
}

}  // namespace ekv
