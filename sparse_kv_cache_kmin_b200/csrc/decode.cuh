// decode.cuh -- arguments shared by the sparse-decode kernels (decode.cu, decode_tc.cu).
#pragma once

#include "ekv_device.cuh"

namespace ekv {

struct DecodeArgs {
    ekv_cache c;
    const void *q;
    int H_q;
    float qscale;  // softmax: scale * log2(e); entmax: scale * (alpha - 1)
    float alpha;
    const int32_t *sel_idx;
    const int32_t *sel_count;
    int max_sel;
    int CP;         // pages per chunk
    int NC;         // chunks per (sequence, KV head) at most
    int LS;         // logits row stride: NC * CP * P
    int Pshift;     // log2(P)
    int stages;     // pipeline stages of the chunk kernel (2 or 3)
    float *part_ml; // [B * H_q][NC][2]   softmax (m, l); entmax (max z, unused)
    float *part_o;  // [B * H_q][NC][D]   softmax sum p v
    float *logits;  // [B * H_q][LS]       entmax z
    int32_t *sel_blk;  // [B * H_kv][max_sel] entmax: cache block of selected page i (-1: none)
    float *out;
    float *stat;
};

constexpr int kMaxCP = 16;  // pages per chunk at most

}  // namespace ekv
