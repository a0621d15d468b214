// decode_tc.cu -- the logits of the selected pages on the 5th-generation tensor cores, for
// bf16 caches and the entmax modes (EntmaxKV technical summary, §2.C).
//
// One chunk = 128 selected tokens (8 pages of 16, 4 of 32 or 2 of 64) of one (sequence, KV
// head). Per chunk, the group's G query rows Q (G x d) and the chunk's key rows K (128 x d) are
// multiplied on the tensor cores: S^T = K Q^T is one tcgen05.mma of M = 128 tokens, N = 16
// (G query columns, the rest zero), K = d in steps of 16, accumulating in fp32 in tensor memory.
//
// Warp roles of a persistent CTA (224 threads):
//   warp 6    resolver: walks the CTA's chunks, skips empty ones and resolves their pages
//             (selection -> page table, validated) for several chunks at once -- lane l takes
//             page l of the batch -- into a ring of records, running ahead of the issuer;
//   warp 0    issuer: for each record, waits for a free stage and issues TMA tile loads
//             (128-byte swizzle) of each page's K rows and of the query rows into a 3-stage
//             shared-memory ring;
//   warp 1    allocates 64 TMEM columns (16 per stage); lane 0 issues the MMAs of a stage once
//             its loads land and commits them to the stage's `mma_done` barrier;
//   warps 2-5 epilogue: each reads its 32-lane quadrant of the stage's accumulator (one token
//             per thread, G logits in registers), scales, masks tokens past the page's end,
//             writes the logits and the chunk maxima, and releases the stage.
// Every wait is bounded by the global timer (EKV_DEV_TIMEOUT on expiry); TMEM is freed on
// every exit path.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "decode.cuh"
#include "sm100_tc.cuh"

namespace ekv {

constexpr int kTcCT = 128;      // tokens per chunk: one M = 128 tile
constexpr int kTcStages = 3;
constexpr int kTcThreads = 224;  // 7 warps
constexpr int kRes = 8;          // resolved-chunk records between the resolver and the issuer
constexpr int kTcCols = 64;     // TMEM columns allocated (16 per stage, power of two >= 32)

template <int D> struct TcLayout {
    static constexpr int KB = D / 64;                 // 64-element (128-byte) column blocks
    static constexpr int Q_BLOCK = 16 * 128;          // N = 16 rows x 128 B
    static constexpr int K_BLOCK = kTcCT * 128;       // 128 rows x 128 B
    static constexpr int Q_BYTES = KB * Q_BLOCK;
    static constexpr int STAGE = Q_BYTES + KB * K_BLOCK;  // a multiple of 1024
    static constexpr int SMEM = kTcStages * STAGE + 1024; // + slack to align to 1024
};

// Resolver warp of the tensor-core chunk kernels: walks this CTA's items (chunk, sequence, KV
// head), skips empty ones and resolves the pages of several chunks at once -- lane l takes page
// l % CP of chunk l / CP of the batch: selection -> page table, validated, and the block is
// recorded for the finish -- into a ring of kRes records (block ids, valid token counts), one
// per chunk, ending with an end mark (item -1). Waits for a free record are bounded.
__device__ void tc_resolver(const DecodeArgs &a, long long items, long long *q_item,
                            uint64_t *bar_rfull, uint64_t *bar_rempty, long long *rec_item,
                            int (*rec_blk)[kMaxCP], int (*rec_nt)[kMaxCP])
{
    const int lane = threadIdx.x & 31;
    const ekv_cache &c = a.c;
    const int H = c.num_kv_heads, P = c.page_size, BH = c.batch * H;
    const int CP = a.CP;
    const int IPB = 32 / CP;  // chunks resolved per batch
    long long cand = blockIdx.x;
    int r = 0;
    bool stop = false;
    while (!stop) {
        // 1. the next IPB non-empty chunks of this CTA (32 candidates examined at a time)
        int nb = 0;
        while (nb < IPB && cand < items) {
            const long long cl = cand + (long long)lane * gridDim.x;
            bool v = false;
            if (cl < items) {
                const int ci = (int)(cl / BH), bh = (int)(cl % BH);
                int nsel = a.sel_count[bh];
                nsel = nsel < 0 ? 0 : (nsel > a.max_sel ? a.max_sel : nsel);
                v = ci * CP < nsel;
            }
            const unsigned bal = __ballot_sync(kFull, v);
            const int need = IPB - nb, have = __popc(bal);
            const int rank = __popc(bal & ((1u << lane) - 1u));
            if (v && rank < need) q_item[nb + rank] = cl;
            if (have > need) {
                unsigned b2 = bal;
                for (int t = 0; t < need - 1; ++t) b2 &= b2 - 1;
                cand += (long long)(__ffs(b2)) * gridDim.x;  // just past the last one taken
                nb += need;
            } else {
                cand += 32ll * gridDim.x;
                nb += have;
            }
        }
        __syncwarp();
        if (nb == 0) stop = true;
        // 2. resolve pages: lane l -> chunk l / CP of the batch, page l % CP
        const int m = lane / CP, pg = lane % CP;
        int blk = 0, nt = 0;
        if (m < nb) {
            const long long it = q_item[m];
            const int ci = (int)(it / BH), bh = (int)(it % BH);
            const int b = bh / H;
            int len;
            const int np = seq_pages(c.seq_lens, b, P, c.max_pages, nullptr, &len);
            int nsel = a.sel_count[bh];
            nsel = nsel < 0 ? 0 : (nsel > a.max_sel ? a.max_sel : nsel);
            const int i = ci * CP + pg;
            if (i < nsel) {
                const int j = a.sel_idx[(size_t)bh * a.max_sel + i];
                if (j < 0 || j >= np) {
                    flag(c.dev_status, EKV_DEV_BAD_SEL);
                } else {
                    const int bk = c.page_table[(size_t)b * c.max_pages + j];
                    if (bk < 0 || bk >= c.num_blocks) {
                        flag(c.dev_status, EKV_DEV_BAD_BLOCK);
                    } else {
                        blk = bk;
                        nt = len - j * P < P ? len - j * P : P;
                    }
                }
                a.sel_blk[(size_t)bh * a.max_sel + i] = nt > 0 ? blk : -1;  // for the finish
            }
        }
        // 3. one record per chunk (an end mark when there are none left)
        for (int mm = 0; mm < (stop ? 1 : nb); ++mm) {
            const int slot = r % kRes;
            const uint32_t ph = (r / kRes) & 1;
            int ok = lane == 0 ? (int)mbar_wait_bounded(&bar_rempty[slot], ph ^ 1) : 0;
            ok = __shfl_sync(kFull, ok, 0);
            if (!ok) {
                if (lane == 0) flag(c.dev_status, EKV_DEV_TIMEOUT);
                stop = true;
                break;
            }
            mbar_try_wait(&bar_rempty[slot], ph ^ 1);
            if (m == mm) {
                rec_blk[slot][pg] = blk;
                rec_nt[slot][pg] = nt;
            }
            if (lane == 0) rec_item[slot] = stop ? -1 : q_item[mm];
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_rfull[slot]);
            ++r;
        }
    }
}

template <int D, int G>
__global__ void __launch_bounds__(kTcThreads)
decode_chunk_tc_kernel(const __grid_constant__ CUtensorMap kmap,
                       const __grid_constant__ CUtensorMap qmap, DecodeArgs a)
{
    using L = TcLayout<D>;
    extern __shared__ unsigned char smem_raw[];
    __shared__ uint64_t bar_full[kTcStages], bar_mma[kTcStages], bar_empty[kTcStages];
    __shared__ long long item_s[kTcStages];
    __shared__ int ntok_s[kTcStages][kMaxCP];
    __shared__ long long q_item[32];
    __shared__ uint64_t bar_rfull[kRes], bar_rempty[kRes];
    __shared__ long long rec_item[kRes];
    __shared__ int rec_blk[kRes][kMaxCP], rec_nt[kRes][kMaxCP];
    __shared__ uint32_t tmem_base_s;
    __shared__ float red[2][4][8];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const ekv_cache &c = a.c;
    const int H = c.num_kv_heads, P = c.page_size, BH = c.batch * H;
    const int CP = a.CP;  // pages per chunk (kTcCT / P)
    const long long items = (long long)BH * a.NC;
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);

    if (warp == 1) tmem_alloc(&tmem_base_s, kTcCols);
    if (tid == 0) {
        for (int s = 0; s < kTcStages; ++s) {
            mbar_init(&bar_full[s], 1);
            mbar_init(&bar_mma[s], 1);
            mbar_init(&bar_empty[s], 128);
        }
        for (int i = 0; i < kRes; ++i) {
            mbar_init(&bar_rfull[i], 1);
            mbar_init(&bar_rempty[i], 1);
        }
        fence_mbar_init();
    }
    // query rows G..15 of every stage stay zero (the loads write rows 0..G-1 only)
    for (int s = 0; s < kTcStages; ++s)
        for (int i = tid; i < L::Q_BYTES / 16; i += kTcThreads)
            reinterpret_cast<uint4 *>(smem + s * L::STAGE)[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = tmem_base_s;
    pdl_wait();

    if (warp == 6) {
        tc_resolver(a, items, q_item, bar_rfull, bar_rempty, rec_item, rec_blk, rec_nt);
    } else if (warp == 0) {
        // ------------------------------------------------------------------ TMA issuer
        prefetch_tensor_map(&kmap);
        prefetch_tensor_map(&qmap);
        for (int k = 0;; ++k) {
            const int slot = k % kRes;
            const uint32_t rph = (k / kRes) & 1;
            int ok = lane == 0 ? (int)mbar_wait_bounded(&bar_rfull[slot], rph) : 0;
            ok = __shfl_sync(kFull, ok, 0);
            if (!ok) {
                if (lane == 0) flag(c.dev_status, EKV_DEV_TIMEOUT);
                break;
            }
            mbar_try_wait(&bar_rfull[slot], rph);
            const long long it = rec_item[slot];
            const int s = k % kTcStages;
            const uint32_t ph = (k / kTcStages) & 1;
            ok = lane == 0 ? (int)mbar_wait_bounded(&bar_empty[s], ph ^ 1) : 0;
            ok = __shfl_sync(kFull, ok, 0);
            if (!ok) {
                if (lane == 0) flag(c.dev_status, EKV_DEV_TIMEOUT);
                break;
            }
            mbar_try_wait(&bar_empty[s], ph ^ 1);
            if (it < 0) {
                if (lane == 0) {
                    item_s[s] = -1;
                    mbar_arrive(&bar_full[s]);
                }
                break;
            }
            int blk = 0, nt = 0;
            if (lane < CP) {
                blk = rec_blk[slot][lane];
                nt = rec_nt[slot][lane];
                ntok_s[s][lane] = nt;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_rempty[slot]);  // record consumed
            const uint32_t bytes = nt > 0 ? (uint32_t)(L::KB * P * 128) : 0u;
            const uint32_t total = (uint32_t)warp_sum((int)bytes) + (uint32_t)(L::KB * G * 128);
            if (lane == 0) item_s[s] = it;
            __syncwarp();
            if (lane == 0) mbar_arrive_expect_tx(&bar_full[s], total);
            __syncwarp();
            unsigned char *st = smem + s * L::STAGE;
            const int bh = (int)(it % BH);
            const int h = bh % H;
            if (lane == 0) {
                const int qrow = (bh / H) * a.H_q + h * G;
#pragma unroll
                for (int kb = 0; kb < L::KB; ++kb)
                    tma_load_2d(st + kb * L::Q_BLOCK, &qmap, kb * 64, qrow, &bar_full[s]);
            }
            if (lane < CP && nt > 0) {
                const int krow = (blk * H + h) * P;
#pragma unroll
                for (int kb = 0; kb < L::KB; ++kb)
                    tma_load_2d(st + L::Q_BYTES + kb * L::K_BLOCK + lane * P * 128, &kmap, kb * 64,
                                krow, &bar_full[s]);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = mma_idesc_bf16_f32(kTcCT, 16);
            for (int k = 0;; ++k) {
                const int s = k % kTcStages;
                const uint32_t ph = (k / kTcStages) & 1;
                if (!mbar_wait_bounded(&bar_full[s], ph)) {
                    flag(c.dev_status, EKV_DEV_TIMEOUT);
                    mbar_wait_bounded(&bar_full[s], ph);  // let any load still in flight land
                    break;
                }
                tc_fence_after_sync();
                if (item_s[s] < 0) {
                    mbar_arrive(&bar_mma[s]);  // pass the end mark to the epilogue
                    break;
                }
                const unsigned char *st = smem + s * L::STAGE;
#pragma unroll
                for (int kb = 0; kb < L::KB; ++kb)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc_mma_bf16(tmem + s * 16, sw128_kmajor_desc(st + L::Q_BYTES + kb * L::K_BLOCK + kk * 32),
                                    sw128_kmajor_desc(st + kb * L::Q_BLOCK + kk * 32), idesc,
                                    kb != 0 || kk != 0);
                tc_commit(&bar_mma[s]);
            }
        }
    } else {
        // ------------------------------------------------------------------ epilogue
        const int quad = warp & 3;  // TMEM lane quadrant this warp may read
        const int slot = quad * 32 + lane;
        for (int k = 0;; ++k) {
            const int s = k % kTcStages;
            const uint32_t ph = (k / kTcStages) & 1;
            int ok = lane == 0 ? (int)mbar_wait_bounded(&bar_mma[s], ph) : 0;
            ok = __shfl_sync(kFull, ok, 0);
            if (!named_sync_and(1, 128, ok)) {  // the four epilogue warps stop together
                if (lane == 0) flag(c.dev_status, EKV_DEV_TIMEOUT);
                break;
            }
            mbar_try_wait(&bar_mma[s], ph);
            mbar_try_wait(&bar_full[s], ph);  // also acquire the producer's stage records
            tc_fence_after_sync();
            const long long it = item_s[s];
            if (it < 0) break;
            const int ci = (int)(it / BH), bh = (int)(it % BH);
            const int b = bh / H, h = bh % H;
            uint32_t r[G];
            tmem_ld_32x32b<G>(tmem + ((uint32_t)(quad * 32) << 16) + s * 16, r);
            tmem_ld_wait();
            const int pi = slot >> a.Pshift, t = slot & (P - 1);
            const bool valid = pi < CP && t < ntok_s[s][pi];
            tc_fence_before_sync();
            mbar_arrive(&bar_empty[s]);  // stage (shared memory and accumulator) released
            const size_t bq0 = (size_t)b * a.H_q + h * G;
            float mx[G];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float z = valid ? a.qscale * __uint_as_float(r[g]) : -INFINITY;
                a.logits[(bq0 + g) * (size_t)a.LS + (size_t)ci * kTcCT + slot] = z;
                mx[g] = warp_max(z);
            }
            if (lane == 0) {
#pragma unroll
                for (int g = 0; g < G; ++g) red[k & 1][quad][g] = mx[g];
            }
            named_sync(1, 128);
            if (warp == 2 && lane < G) {
                const float m = fmaxf(fmaxf(red[k & 1][0][lane], red[k & 1][1][lane]),
                                      fmaxf(red[k & 1][2][lane], red[k & 1][3][lane]));
                a.part_ml[((bq0 + lane) * a.NC + ci) * 2] = m;
            }
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 1) tmem_dealloc(tmem, kTcCols);
    pdl_trigger();
}

// ------------------------------------------------------------------------------ softmax
// The softmax chunk partials of bf16 caches on the tensor cores (flash-decoding split over
// chunks of 128 selected tokens). Per chunk, with the group's queries as N = 16 columns:
//   S^T = K Q^T      tcgen05.mma, M = 128 tokens, K = d (fp32 in TMEM)
//   epilogue         per query g: m = max_t z, p_t = 2^(z_t - m), l = sum p (z = scale log2e s);
//                    P^T is written to shared memory in bf16 (the B operand of the next product)
//   O^T = V^T P^T    tcgen05.mma, M = d, K = 128 tokens, V read MN-major straight from the tile
// and (m, l, O) go to the workspace for the finish, which merges the chunks with log-sum-exp.
// Warp roles as in the logits kernel (resolver, TMA issuer, MMA issuer, four epilogue warps);
// the stage holds the query rows, the K and V tiles and the P buffer. TMEM: S of stage s at
// columns [16 s, 16 s + 16), O at [64 + 16 s, ...).
constexpr int kSmStages = 3;
constexpr int kSmCols = 128;  // TMEM columns allocated

template <int D> struct TcSmLayout {
    static_assert(D == kTcCT, "O^T = V^T P^T uses M = d = 128 rows of TMEM");
    static constexpr int KB = D / 64;
    static constexpr int Q_BLOCK = 16 * 128;
    static constexpr int K_BLOCK = kTcCT * 128;
    static constexpr int P_BLOCK = 16 * 128;                 // 16 query rows x 64 tokens (bf16)
    static constexpr int Q_OFF = 0;
    static constexpr int K_OFF = KB * Q_BLOCK;
    static constexpr int V_OFF = K_OFF + KB * K_BLOCK;
    static constexpr int P_OFF = V_OFF + KB * K_BLOCK;
    static constexpr int STAGE = P_OFF + (kTcCT / 64) * P_BLOCK;  // a multiple of 1024
    static constexpr int SMEM = kSmStages * STAGE + 1024;
};

template <int D, int G>
__global__ void __launch_bounds__(kTcThreads)
decode_softmax_tc_kernel(const __grid_constant__ CUtensorMap kmap,
                         const __grid_constant__ CUtensorMap vmap,
                         const __grid_constant__ CUtensorMap qmap, DecodeArgs a)
{
    using L = TcSmLayout<D>;
    constexpr int S = kSmStages;
    extern __shared__ unsigned char smem_raw[];
    __shared__ uint64_t bar_full[S], bar_sdone[S], bar_pready[S], bar_odone[S], bar_ofree[S],
        bar_empty[S], bar_fin;
    __shared__ long long item_s[S];
    __shared__ int ntok_s[S][kMaxCP];
    __shared__ long long q_item[32];
    __shared__ uint64_t bar_rfull[kRes], bar_rempty[kRes];
    __shared__ long long rec_item[kRes];
    __shared__ int rec_blk[kRes][kMaxCP], rec_nt[kRes][kMaxCP];
    __shared__ uint32_t tmem_base_s;
    __shared__ float red_m[2][4][8], red_l[2][4][8];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const ekv_cache &c = a.c;
    const int H = c.num_kv_heads, P = c.page_size, BH = c.batch * H;
    const int CP = a.CP;
    const long long items = (long long)BH * a.NC;
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);

    if (warp == 1) tmem_alloc(&tmem_base_s, kSmCols);
    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&bar_full[s], 1);
            mbar_init(&bar_sdone[s], 1);
            mbar_init(&bar_pready[s], 128);
            mbar_init(&bar_odone[s], 1);
            mbar_init(&bar_ofree[s], 128);
            mbar_init(&bar_empty[s], 1);
        }
        mbar_init(&bar_fin, 1);
        for (int i = 0; i < kRes; ++i) {
            mbar_init(&bar_rfull[i], 1);
            mbar_init(&bar_rempty[i], 1);
        }
        fence_mbar_init();
    }
    // query rows G..15 and P rows G..15 of every stage stay zero
    for (int s = 0; s < S; ++s) {
        for (int i = tid; i < L::K_OFF / 16; i += kTcThreads)
            reinterpret_cast<uint4 *>(smem + s * L::STAGE + L::Q_OFF)[i] = make_uint4(0, 0, 0, 0);
        for (int i = tid; i < (L::STAGE - L::P_OFF) / 16; i += kTcThreads)
            reinterpret_cast<uint4 *>(smem + s * L::STAGE + L::P_OFF)[i] = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async();
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = tmem_base_s;
    pdl_wait();

    if (warp == 6) {
        tc_resolver(a, items, q_item, bar_rfull, bar_rempty, rec_item, rec_blk, rec_nt);
    } else if (warp == 0) {
        // ------------------------------------------------------------------ TMA issuer
        prefetch_tensor_map(&kmap);
        prefetch_tensor_map(&vmap);
        prefetch_tensor_map(&qmap);
        for (int k = 0;; ++k) {
            const int slot = k % kRes;
            const uint32_t rph = (k / kRes) & 1;
            int ok = lane == 0 ? (int)mbar_wait_bounded(&bar_rfull[slot], rph) : 0;
            ok = __shfl_sync(kFull, ok, 0);
            if (!ok) {
                if (lane == 0) flag(c.dev_status, EKV_DEV_TIMEOUT);
                break;
            }
            mbar_try_wait(&bar_rfull[slot], rph);
            const long long it = rec_item[slot];
            const int s = k % S;
            const uint32_t ph = (k / S) & 1;
            ok = lane == 0 ? (int)mbar_wait_bounded(&bar_empty[s], ph ^ 1) : 0;
            ok = __shfl_sync(kFull, ok, 0);
            if (!ok) {
                if (lane == 0) flag(c.dev_status, EKV_DEV_TIMEOUT);
                break;
            }
            mbar_try_wait(&bar_empty[s], ph ^ 1);
            if (it < 0) {
                if (lane == 0) {
                    item_s[s] = -1;
                    mbar_arrive(&bar_full[s]);
                }
                break;
            }
            int blk = 0, nt = 0;
            if (lane < CP) {
                blk = rec_blk[slot][lane];
                nt = rec_nt[slot][lane];
                ntok_s[s][lane] = nt;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_rempty[slot]);  // record consumed
            const uint32_t bytes = nt > 0 ? (uint32_t)(2 * L::KB * P * 128) : 0u;
            const uint32_t total = (uint32_t)warp_sum((int)bytes) + (uint32_t)(L::KB * G * 128);
            if (lane == 0) item_s[s] = it;
            __syncwarp();
            if (lane == 0) mbar_arrive_expect_tx(&bar_full[s], total);
            __syncwarp();
            unsigned char *st = smem + s * L::STAGE;
            const int bh = (int)(it % BH);
            const int h = bh % H;
            if (lane == 0) {
                const int qrow = (bh / H) * a.H_q + h * G;
#pragma unroll
                for (int kb = 0; kb < L::KB; ++kb)
                    tma_load_2d(st + L::Q_OFF + kb * L::Q_BLOCK, &qmap, kb * 64, qrow, &bar_full[s]);
            }
            if (lane < CP && nt > 0) {
                const int krow = (blk * H + h) * P;
#pragma unroll
                for (int kb = 0; kb < L::KB; ++kb) {
                    tma_load_2d(st + L::K_OFF + kb * L::K_BLOCK + lane * P * 128, &kmap, kb * 64,
                                krow, &bar_full[s]);
                    tma_load_2d(st + L::V_OFF + kb * L::K_BLOCK + lane * P * 128, &vmap, kb * 64,
                                krow, &bar_full[s]);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = mma_idesc_bf16_f32(kTcCT, 16);
            constexpr uint32_t idesc_o = mma_idesc_bf16_f32_amn(D, 16);
            auto mma_s = [&](int s) {  // S^T = K Q^T into columns 16 s
                const unsigned char *st = smem + s * L::STAGE;
#pragma unroll
                for (int kb = 0; kb < L::KB; ++kb)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc_mma_bf16(tmem + s * 16,
                                    sw128_kmajor_desc(st + L::K_OFF + kb * L::K_BLOCK + kk * 32),
                                    sw128_kmajor_desc(st + L::Q_OFF + kb * L::Q_BLOCK + kk * 32),
                                    idesc_s, kb != 0 || kk != 0);
            };
            auto mma_o = [&](int s) {  // O^T = V^T P^T into columns 64 + 16 s
                const unsigned char *st = smem + s * L::STAGE;
#pragma unroll
                for (int kt = 0; kt < kTcCT / 16; ++kt)
                    tc_mma_bf16(tmem + 64 + s * 16,
                                sw128_mnmajor_desc(st + L::V_OFF + kt * 2048, L::K_BLOCK),
                                sw128_kmajor_desc(st + L::P_OFF + (kt >> 2) * L::P_BLOCK + (kt & 3) * 32),
                                idesc_o, kt != 0);
            };
            bool ok = mbar_wait_bounded(&bar_full[0], 0);
            if (ok) {
                tc_fence_after_sync();
                if (item_s[0] < 0) {
                    mbar_arrive(&bar_sdone[0]);  // pass the end mark on
                } else {
                    mma_s(0);
                    tc_commit(&bar_sdone[0]);
                    for (int k = 0;; ++k) {
                        const int s = k % S, s1 = (k + 1) % S;
                        const uint32_t ph = (k / S) & 1, ph1 = ((k + 1) / S) & 1;
                        // two independent issues: the next chunk's scores (once its tiles have
                        // landed) and this chunk's O (once its P is written and the columns are
                        // free), whichever is ready first -- neither waits on the other
                        bool next_done = false, next_end = false, o_done = false;
                        const uint64_t t0 = global_ns();
                        while (!(next_done && o_done)) {
                            if (!next_done && mbar_try_wait(&bar_full[s1], ph1)) {
                                tc_fence_after_sync();
                                next_end = item_s[s1] < 0;
                                if (next_end) {
                                    mbar_arrive(&bar_sdone[s1]);  // pass the end mark on
                                } else {
                                    mma_s(s1);
                                    tc_commit(&bar_sdone[s1]);
                                }
                                next_done = true;
                            }
                            if (!o_done && mbar_try_wait(&bar_pready[s], ph) &&
                                (k < S || mbar_try_wait(&bar_ofree[s], ph ^ 1))) {
                                tc_fence_after_sync();
                                mma_o(s);
                                tc_commit(&bar_odone[s]);
                                tc_commit(&bar_empty[s]);  // K, V and P of this stage are free
                                o_done = true;
                            }
                            if (global_ns() - t0 > 2000000000ull) break;
                        }
                        if (!(next_done && o_done)) { ok = false; break; }
                        if (next_end) break;
                    }
                }
            }
            if (!ok) flag(c.dev_status, EKV_DEV_TIMEOUT);
            // every MMA issued has completed before the columns are freed
            tc_commit(&bar_fin);
            mbar_wait_bounded(&bar_fin, 0);
        }
    } else {
        // ------------------------------------------------------------------ epilogue
        const int quad = warp & 3;  // TMEM lane quadrant this warp may read
        const int t = quad * 32 + lane;  // token of the chunk (S rows), then output row (O rows)
        for (int k = 0;; ++k) {
            const int s = k % S;
            const uint32_t ph = (k / S) & 1;
            int ok = lane == 0 ? (int)mbar_wait_bounded(&bar_sdone[s], ph) : 0;
            ok = __shfl_sync(kFull, ok, 0);
            if (!named_sync_and(1, 128, ok)) {  // the four epilogue warps stop together
                if (lane == 0) flag(c.dev_status, EKV_DEV_TIMEOUT);
                break;
            }
            mbar_try_wait(&bar_sdone[s], ph);
            mbar_try_wait(&bar_full[s], ph);  // also acquire the producer's stage records
            tc_fence_after_sync();
            const long long it = item_s[s];
            if (it < 0) break;
            const int ci = (int)(it / BH), bh = (int)(it % BH);
            const int b = bh / H, h = bh % H;
            uint32_t r[G];
            tmem_ld_32x32b<G>(tmem + ((uint32_t)(quad * 32) << 16) + s * 16, r);
            tmem_ld_wait();
            const int pi = t >> a.Pshift, tt = t & (P - 1);
            const bool valid = pi < CP && tt < ntok_s[s][pi];
            if (!valid) {  // a row past the page's tokens (or of a page not loaded) may hold
                           // anything, NaN included: zero it so that 0 * v stays 0 in O
#pragma unroll
                for (int kb = 0; kb < L::KB; ++kb)
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        reinterpret_cast<uint4 *>(smem + s * L::STAGE + L::V_OFF + kb * L::K_BLOCK + t * 128)[i] =
                            make_uint4(0, 0, 0, 0);
            }
            float z[G], m[G], pv[G], l[G];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                z[g] = valid ? a.qscale * __uint_as_float(r[g]) : -INFINITY;
                const float mw = warp_max(z[g]);
                if (lane == 0) red_m[k & 1][quad][g] = mw;
            }
            named_sync(1, 128);
#pragma unroll
            for (int g = 0; g < G; ++g) {
                m[g] = fmaxf(fmaxf(red_m[k & 1][0][g], red_m[k & 1][1][g]),
                             fmaxf(red_m[k & 1][2][g], red_m[k & 1][3][g]));
                // p as the tensor cores will see it (bf16), so that l and O agree
                pv[g] = valid ? __bfloat162float(__float2bfloat16_rn(exp2f(z[g] - m[g]))) : 0.f;
                const float lw = warp_sum(pv[g]);
                if (lane == 0) red_l[k & 1][quad][g] = lw;
            }
            // P^T (row g, column t) into the 128-byte swizzled K-major B buffer
            unsigned char *pb = smem + s * L::STAGE + L::P_OFF + (t >> 6) * L::P_BLOCK;
            const int chunk16 = (t & 63) >> 3;
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const __nv_bfloat16 pbf = __float2bfloat16_rn(pv[g]);
                *reinterpret_cast<__nv_bfloat16 *>(pb + g * 128 + ((chunk16 ^ (g & 7)) << 4) + (t & 7) * 2) = pbf;
            }
            fence_proxy_async();
            tc_fence_before_sync();
            mbar_arrive(&bar_pready[s]);
            named_sync(1, 128);
#pragma unroll
            for (int g = 0; g < G; ++g)
                l[g] = red_l[k & 1][0][g] + red_l[k & 1][1][g] + red_l[k & 1][2][g] + red_l[k & 1][3][g];
            ok = lane == 0 ? (int)mbar_wait_bounded(&bar_odone[s], ph) : 0;
            ok = __shfl_sync(kFull, ok, 0);
            if (!named_sync_and(1, 128, ok)) {
                if (lane == 0) flag(c.dev_status, EKV_DEV_TIMEOUT);
                break;
            }
            mbar_try_wait(&bar_odone[s], ph);
            tc_fence_after_sync();
            tmem_ld_32x32b<G>(tmem + ((uint32_t)(quad * 32) << 16) + 64 + s * 16, r);
            tmem_ld_wait();
            tc_fence_before_sync();
            mbar_arrive(&bar_ofree[s]);
            const size_t bq0 = (size_t)b * a.H_q + h * G;
#pragma unroll
            for (int g = 0; g < G; ++g) a.part_o[((bq0 + g) * a.NC + ci) * D + t] = __uint_as_float(r[g]);
#pragma unroll
            for (int g = 0; g < G; ++g) {
                if (t == g) {
                    a.part_ml[((bq0 + g) * a.NC + ci) * 2] = m[g];
                    a.part_ml[((bq0 + g) * a.NC + ci) * 2 + 1] = l[g];
                }
            }
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 1) tmem_dealloc(tmem, kSmCols);
    pdl_trigger();
}

// ------------------------------------------------------------------------------ host side
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }();
    return fn;
}

// 2-D bf16 tensor map over `rows` rows of `cols` elements, box = 64 columns x `box_rows`,
// 128-byte swizzle.
static bool make_map(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows, uint32_t box_rows)
{
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Whether a tensor-core chunk kernel serves this call (entmax logits: d = 64 or 128; softmax
// partials: d = 128).
bool tc_chunk_supported(const ekv_cache &c, int H_q, bool softmax)
{
    if (c.dtype != EKV_BF16 || (softmax && c.head_dim != 128)) return false;
    const long long rows = (long long)c.num_blocks * c.num_kv_heads * c.page_size;
    return rows < (1ll << 31) && (long long)c.batch * H_q < (1ll << 31) && kTcCT % c.page_size == 0;
}

template <int D, int G>
static cudaError_t launch_tc_t(const DecodeArgs &a, cudaLaunchConfig_t cfg)
{
    using L = TcLayout<D>;
    CUtensorMap kmap, qmap;
    const ekv_cache &c = a.c;
    if (!make_map(&kmap, c.k_cache, D, (uint64_t)c.num_blocks * c.num_kv_heads * c.page_size, c.page_size) ||
        !make_map(&qmap, a.q, D, (uint64_t)c.batch * a.H_q, G))
        return cudaErrorInvalidValue;
    auto k = decode_chunk_tc_kernel<D, G>;
    static bool attr_set = false;  // per instantiation
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = L::SMEM;
    const long long items = (long long)c.batch * c.num_kv_heads * a.NC;
    // two CTAs per SM fit (2 x (L::SMEM + static + reserved) is below the 228 KiB of an SM);
    // the occupancy query reports one, so size the grid from the SM count directly. CTAs never
    // wait on one another, so an over-full grid would only queue.
    int sms = 148, dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long grid = 2ll * sms;
    cfg.gridDim = dim3((unsigned)(items < grid ? items : grid));
    return cudaLaunchKernelEx(&cfg, k, kmap, qmap, a);
}

template <int G>
static cudaError_t launch_softmax_tc_t(const DecodeArgs &a, cudaLaunchConfig_t cfg)
{
    constexpr int D = 128;
    using L = TcSmLayout<D>;
    CUtensorMap kmap, vmap, qmap;
    const ekv_cache &c = a.c;
    const uint64_t rows = (uint64_t)c.num_blocks * c.num_kv_heads * c.page_size;
    if (!make_map(&kmap, c.k_cache, D, rows, c.page_size) ||
        !make_map(&vmap, c.v_cache, D, rows, c.page_size) ||
        !make_map(&qmap, a.q, D, (uint64_t)c.batch * a.H_q, G))
        return cudaErrorInvalidValue;
    auto k = decode_softmax_tc_kernel<D, G>;
    static bool attr_set = false;  // per instantiation
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = L::SMEM;
    const long long items = (long long)c.batch * c.num_kv_heads * a.NC;
    const long long grid = persistent_grid_size((const void *)k, kTcThreads, L::SMEM);
    cfg.gridDim = dim3((unsigned)(items < grid ? items : grid));
    return cudaLaunchKernelEx(&cfg, k, kmap, vmap, qmap, a);
}

cudaError_t launch_softmax_tc(const DecodeArgs &a, int G, cudaLaunchConfig_t cfg)
{
    switch (G) {
    case 1: return launch_softmax_tc_t<1>(a, cfg);
    case 2: return launch_softmax_tc_t<2>(a, cfg);
    case 4: return launch_softmax_tc_t<4>(a, cfg);
    default: return launch_softmax_tc_t<8>(a, cfg);
    }
}

cudaError_t launch_chunk_tc(const DecodeArgs &a, int G, cudaLaunchConfig_t cfg)
{
    if (a.c.head_dim == 128) {
        switch (G) {
        case 1: return launch_tc_t<128, 1>(a, cfg);
        case 2: return launch_tc_t<128, 2>(a, cfg);
        case 4: return launch_tc_t<128, 4>(a, cfg);
        default: return launch_tc_t<128, 8>(a, cfg);
        }
    }
    switch (G) {
    case 1: return launch_tc_t<64, 1>(a, cfg);
    case 2: return launch_tc_t<64, 2>(a, cfg);
    case 4: return launch_tc_t<64, 4>(a, cfg);
    default: return launch_tc_t<64, 8>(a, cfg);
    }
}

}  // namespace ekv
