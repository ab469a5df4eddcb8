// cq_moe.h -- argument blocks of the MoE kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "cq_internal.h"

namespace cq {

constexpr int kMaxExperts = 256;
constexpr int kMaxTopK = 16;

struct SwigluArgs {
    const float *part_r;   // [slots][R_routed][I][2]
    const float *part_s;   // [slots][R_shared][I_shared][2]
    LutPlan plan_r, plan_s;  // partial-slot counts of the gate/up launches
    int64_t R_routed, R_shared;
    int I, I_shared, Imax;
    int log2b_i, log2b_i_shared;
    const int32_t *perm;   // routed row -> slot
    int topk, T;
    const float *x_scales; // [T]
    int bits;
    uint8_t *hq;           // [R][ldhq bytes]
    int64_t ldhq;
    float *h_scales;       // [R]
    void *h_dbg;           // fp16 [R][Imax] or NULL
    __half *f16_r;         // fp16 copies of the routed h codes [R_routed][I], or NULL
    __half *f16_s;         // fp16 copies of the shared h codes [R_shared][I_shared], or NULL
};

struct CombineArgs {
    const float *part_r;   // [slots][R_routed][H]
    const float *part_s;   // [slots][R_shared][H]
    LutPlan plan_r, plan_s;  // partial-slot counts of the down launches
    int64_t R_routed, R_shared;
    int T, H, topk, n_shared;
    const int32_t *inv_perm;  // slot -> routed row
    const float *w;           // [T][topk]
    const float *h_scales;    // [R]
    float *out;               // [T][H]
    float *y_dbg;             // [R][H] or NULL
};

// Routing: top-k + softmax weights, then the expert grouping.  chist:
// route_scratch_bytes(T, E, k) bytes of device scratch (per-chunk counts).
size_t route_scratch_bytes(int T, int E, int k);
cudaError_t launch_route(const float *logits, int T, int E, int k, int renorm, int tile_rows,
                         int32_t *ids, float *w, int32_t *counts, int32_t *offsets, int32_t *perm,
                         int32_t *inv_perm, int32_t *grp_tiles, int32_t *tile_grp,
                         int max_tiles, int32_t *chist, cudaStream_t st);
cudaError_t launch_swiglu_rq(const SwigluArgs &a, int64_t rows, cudaStream_t st);
cudaError_t launch_combine(const CombineArgs &a, cudaStream_t st);

}  // namespace cq
