// decode_direct.cu -- entmax logits of the selected pages, each warp streaming its own pages
// (EntmaxKV technical summary, §2.C: only the keys of the selected pages are read; the value
// rows wait until the support is known).
//
// Output contract: the one of the chunk kernels (decode.cu, decode_tc.cu) for chunks of
// CT = 128 tokens (CP = 128 / P pages): the logits z = (alpha - 1) * scale * q.k of every slot
// of the chunk (-inf past a page's valid tokens or the selection's end), the chunk maximum of
// each query, and the cache block of every selected page.
//
// Design: no producer warp and no CTA barrier. The (sequence, KV head, chunk) slots are
// interleaved over all warps of a persistent grid. A warp resolves the pages of its next
// 32 / CP chunks at once (one lane per page: selection -> page table, validated), then streams
// its chunks as 16-row tiles through a private ring of R tiles in shared memory with 16-byte
// cp.async copies, keeping R - 1 tiles in flight while it computes one. A tile's logits for
// all G queries of the KV head are D / 16 warp-level bf16 MMAs (m16n8k16, fp32 accumulation)
// of the tile against the queries held as B fragments in registers; the next chunk's queries
// are fetched while the current chunk is computed. Every warp issues its own copies, so the
// copy issue rate grows with the warps instead of being one thread's per CTA.
#include "decode.cuh"
#include "warp_mma.cuh"

namespace ekv {

constexpr int kDirWarps = 8;       // warps per CTA
constexpr int kDirTileRows = 16;   // token rows per tile
constexpr int kDirCT = 128;        // tokens per chunk (the tensor-core chunk kernel's tile)

template <int D, int G, int R>
__global__ void __launch_bounds__(kDirWarps * 32, 2)
decode_logits_direct_kernel(DecodeArgs a)
{
    // Per tile the warp computes S (16 rows x 8 query columns) = K_tile (16 x D) . Q^T (D x 8)
    // with D / 16 warp-level bf16 MMAs (fp32 accumulation), queries G..7 being zero columns.
    // The tile sits in the ring with its 16-byte pieces XOR-swizzled by (row & 7), so the
    // eight row addresses of each 8 x 8 matrix load fall in distinct banks.
    constexpr int RB = D * 2;                // bytes per bf16 token row
    constexpr int W = RB / 16;               // 16-byte pieces per row
    constexpr int TB = kDirTileRows * RB;    // tile bytes
    constexpr int TPL = TB / (32 * 16);      // pieces per lane per tile
    constexpr int KS = D / 16;               // MMA k-steps per tile
    constexpr int TPC = kDirCT / kDirTileRows;  // tiles per chunk
    static_assert(G <= 8, "one n = 8 MMA column block");
    static_assert(TPC >= R, "the look-ahead stays within the next chunk");
    extern __shared__ __align__(128) unsigned char smem[];  // [kDirWarps][R][TB]

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const ekv_cache &c = a.c;
    const int H = c.num_kv_heads, P = c.page_size, BH = c.batch * H, CP = a.CP;
    const int TPP = P / kDirTileRows;  // tiles per page
    const int CPB = 32 / CP;           // chunks resolved per batch
    unsigned char *ring = smem + (size_t)warp * R * TB;
    const char *kc = static_cast<const char *>(c.k_cache);
    // Chunk slots in (sequence, KV head)-major order, dealt out in rounds of nw slots. In round
    // k warp w takes slot k * nw + (w + 61 k) mod nw: the rotation keeps a warp from meeting the
    // same chunk index every round (as it would whenever nw is a multiple of NC), so ragged
    // selection counts spread evenly over the warps.
    const long long slots = (long long)BH * a.NC;
    const long long nw = (long long)gridDim.x * kDirWarps;
    const long long ck0 = (long long)blockIdx.x * kDirWarps + warp;

    // The page-table rows do not depend on the selection: CTAs placed while the selection still
    // runs bring them into L2 before waiting for it, so the resolution below hits L2.
    {
        const size_t lines = ((size_t)c.batch * c.max_pages * sizeof(int32_t) + 127) / 128;
        for (size_t l = (size_t)blockIdx.x * blockDim.x + threadIdx.x; l < lines;
             l += (size_t)gridDim.x * blockDim.x)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<const char *>(c.page_table) + l * 128));
    }
    pdl_wait();
    // Lane l of a batch: chunk l / CP of the batch, page l % CP of that chunk. bh < 0 past the
    // last slot; nt = valid tokens of the page (0: no page); ok: the chunk holds a selected page.
    struct Batch { int bh, ci, blk, nt, ok; };
    auto resolve = [&](long long k0) {
        Batch r = {-1, 0, 0, 0, 0};
        const long long kr = k0 + lane / CP;
        const long long cq = kr * nw + (ck0 + 61 * kr) % nw;
        if (cq >= slots) return r;
        r.bh = (int)(cq / a.NC);
        r.ci = (int)(cq - (long long)r.bh * a.NC);
        const int i = r.ci * CP + lane % CP;
        const int b = r.bh / H;
        int ns = a.sel_count[r.bh];
        const int j = i < a.max_sel ? a.sel_idx[(size_t)r.bh * a.max_sel + i] : -1;
        int len;
        const int np = seq_pages(c.seq_lens, b, P, c.max_pages, nullptr, &len);
        ns = ns < 0 ? 0 : (ns > a.max_sel ? a.max_sel : ns);
        r.ok = r.ci * CP < ns;
        if (i < ns) {
            if (j < 0 || j >= np) {
                flag(c.dev_status, EKV_DEV_BAD_SEL);
            } else {
                const int bk = c.page_table[(size_t)b * c.max_pages + j];
                if (bk < 0 || bk >= c.num_blocks) {
                    flag(c.dev_status, EKV_DEV_BAD_BLOCK);
                } else {
                    r.blk = bk;
                    r.nt = len - j * P < P ? len - j * P : P;
                }
            }
            a.sel_blk[(size_t)r.bh * a.max_sel + i] = r.nt > 0 ? r.blk : -1;
        }
        return r;
    };
    // copies of tile t of chunk m of batch bb into ring slot `slot` (one commit group, empty
    // when the tile holds no valid row)
    auto issue = [&](const Batch &bb, int m, int t, int slot) {
        const int src = m * CP + t / TPP;
        const int blk = __shfl_sync(kFull, bb.blk, src);
        const int nt = __shfl_sync(kFull, bb.nt, src);
        const int bh = __shfl_sync(kFull, bb.bh, m * CP);
        const int sub = t % TPP;
        if (nt > sub * kDirTileRows) {
            const char *g = kc + (((size_t)blk * H + bh % H) * P + sub * kDirTileRows) * RB;
            unsigned char *s = ring + slot * TB;
#pragma unroll
            for (int k = 0; k < TPL; ++k) {
                const int p = k * 32 + lane, row = p / W, pc = p % W;
                cp_async16(s + row * RB + ((pc ^ (row & 7)) << 4), g + p * 16);
            }
        }
        cp_async_commit();
    };
    // B fragments of the queries of (sequence, KV head) bh: column n = lane / 4 is query n
    auto load_q = [&](int bh, uint32_t (&qb)[KS][2]) {
        const int n = lane >> 2;
        const int b = bh / H, h = bh % H;
        const uint32_t *qr = reinterpret_cast<const uint32_t *>(
            static_cast<const char *>(a.q) + (((size_t)b * a.H_q + (size_t)h * G + (n < G ? n : 0)) * D) * 2);
#pragma unroll
        for (int s = 0; s < KS; ++s) {
            qb[s][0] = n < G && bh >= 0 ? __ldg(qr + s * 8 + (lane & 3)) : 0u;
            qb[s][1] = n < G && bh >= 0 ? __ldg(qr + s * 8 + 4 + (lane & 3)) : 0u;
        }
    };

    Batch B0 = resolve(0), B1 = B0;
    if (__shfl_sync(kFull, B0.bh, 0) < 0) {
        pdl_trigger();
        return;
    }
#pragma unroll
    for (int n = 0; n < R - 1; ++n) issue(B0, 0, n, n);
    uint32_t qcur[KS][2], qnxt[KS][2];
    load_q(__shfl_sync(kFull, B0.bh, 0), qcur);

    // ldmatrix row addresses: lanes 0-7 / 8-15 / 16-23 / 24-31 give the rows of the four
    // 8 x 8 matrices a0 (rows 0-7, k 0-7), a1 (rows 8-15, k 0-7), a2 (rows 0-7, k 8-15),
    // a3 (rows 8-15, k 8-15) of each 16 x 16 k-step
    const int lrow = lane & 15, lk = lane >> 4;
    const int r0 = lane >> 2, n0 = (lane & 3) * 2;
    long long gt = 0;  // tiles consumed by this warp: ring position
    for (long long k = 0;; ++k) {
        const int m = (int)(k % CPB);
        const int bh = __shfl_sync(kFull, B0.bh, m * CP);
        if (bh < 0) break;
        const int ci = __shfl_sync(kFull, B0.ci, m * CP);
        const bool ok = __shfl_sync(kFull, B0.ok, m * CP) != 0;
        const bool last_of_batch = m == CPB - 1;
        if (last_of_batch) B1 = resolve(k + 1);
        load_q(last_of_batch ? __shfl_sync(kFull, B1.bh, 0) : __shfl_sync(kFull, B0.bh, (m + 1) * CP), qnxt);
        const int b = bh / H, h = bh % H;
        const size_t bq0 = (size_t)b * a.H_q + (size_t)h * G;
        float *zrow = a.logits + bq0 * (size_t)a.LS + (size_t)ci * kDirCT;
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll 1
        for (int t = 0; t < TPC; ++t, ++gt) {
            __syncwarp();  // every lane is done reading the slot about to be refilled
            const int ta = t + R - 1;
            const int slot_a = (int)((gt + R - 1) % R);
            if (ta < TPC) issue(B0, m, ta, slot_a);
            else if (last_of_batch) issue(B1, 0, ta - TPC, slot_a);
            else issue(B0, m + 1, ta - TPC, slot_a);
            cp_async_wait<R - 1>();  // this lane's pieces of tile gt have landed
            __syncwarp();            // ... and every other lane's
            if (!ok) continue;
            const unsigned char *tile = ring + (int)(gt % R) * TB;
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int s = 0; s < KS; ++s) {
                uint32_t af[4];
                const int pc = s * 2 + lk;
                ldsm_x4(af, tile + lrow * RB + ((pc ^ (lrow & 7)) << 4));
                mma_bf16_16816(acc, af, qcur[s][0], qcur[s][1]);
            }
            const int ntt = __shfl_sync(kFull, B0.nt, m * CP + t / TPP) - (t % TPP) * kDirTileRows;
            const float z00 = r0 < ntt ? a.qscale * acc[0] : -INFINITY;
            const float z01 = r0 < ntt ? a.qscale * acc[1] : -INFINITY;
            const float z10 = r0 + 8 < ntt ? a.qscale * acc[2] : -INFINITY;
            const float z11 = r0 + 8 < ntt ? a.qscale * acc[3] : -INFINITY;
            float *zt = zrow + t * kDirTileRows + r0;
            if (n0 < G) {
                zt[(size_t)n0 * a.LS] = z00;
                zt[(size_t)n0 * a.LS + 8] = z10;
                mx0 = fmaxf(mx0, fmaxf(z00, z10));
            }
            if (n0 + 1 < G) {
                zt[(size_t)(n0 + 1) * a.LS] = z01;
                zt[(size_t)(n0 + 1) * a.LS + 8] = z11;
                mx1 = fmaxf(mx1, fmaxf(z01, z11));
            }
        }
        if (ok) {
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
                mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, o));
                mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, o));
            }
            if (lane < 4 && n0 < G) a.part_ml[((bq0 + n0) * a.NC + ci) * 2] = mx0;
            if (lane < 4 && n0 + 1 < G) a.part_ml[((bq0 + n0 + 1) * a.NC + ci) * 2] = mx1;
        }
#pragma unroll
        for (int s = 0; s < KS; ++s) {
            qcur[s][0] = qnxt[s][0];
            qcur[s][1] = qnxt[s][1];
        }
        if (last_of_batch) B0 = B1;
    }
    cp_async_wait<0>();
    pdl_trigger();
}

template <int D, int G, int R>
static cudaError_t launch_direct_t(const DecodeArgs &a, cudaLaunchConfig_t cfg, bool *launched)
{
    auto k = decode_logits_direct_kernel<D, G, R>;
    const size_t smem = (size_t)kDirWarps * R * kDirTileRows * D * 2;
    static bool attr_set = false;  // per instantiation
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    const int grid = persistent_grid_size((const void *)k, kDirWarps * 32, smem);
    // Short streams only: with more than two chunk slots per warp, the tensor-core chunk kernel
    // (bulk tensor copies issued by a producer warp) moves long selections faster.
    const long long slots = (long long)a.c.batch * a.c.num_kv_heads * a.NC;
    *launched = slots <= 2ll * grid * kDirWarps;
    if (!*launched) return cudaSuccess;
    cfg.blockDim = dim3(kDirWarps * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.gridDim = dim3(grid);
    return cudaLaunchKernelEx(&cfg, k, a);
}

// bf16 keys, G <= 8 queries per KV head, P in {16, 32, 64} (the workspace of 128-token chunks)
bool direct_logits_supported(const ekv_cache &c, int H_q)
{
    const int G = H_q / c.num_kv_heads;
    return c.dtype == EKV_BF16 && G <= 8 && kDirCT % c.page_size == 0;
}

// Launches the logits kernel above when the call's chunk slots are few enough for it
// (*launched = true); otherwise launches nothing and leaves the call to the chunk kernels.
cudaError_t launch_logits_direct(const DecodeArgs &a, int G, cudaLaunchConfig_t cfg, bool *launched)
{
    if (a.c.head_dim == 128) {
        switch (G) {
        case 1: return launch_direct_t<128, 1, 3>(a, cfg, launched);
        case 2: return launch_direct_t<128, 2, 3>(a, cfg, launched);
        case 4: return launch_direct_t<128, 4, 3>(a, cfg, launched);
        default: return launch_direct_t<128, 8, 3>(a, cfg, launched);
        }
    }
    switch (G) {
    case 1: return launch_direct_t<64, 1, 4>(a, cfg, launched);
    case 2: return launch_direct_t<64, 2, 4>(a, cfg, launched);
    case 4: return launch_direct_t<64, 4, 4>(a, cfg, launched);
    default: return launch_direct_t<64, 8, 4>(a, cfg, launched);
    }
}

}  // namespace ekv
