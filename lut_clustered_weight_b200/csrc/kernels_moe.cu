// kernels_moe.cu -- routing / expert grouping and combine kernels of the
// CodeQuant MoE linear layer (sm_100a).
#include "cq_common.cuh"
#include "cq_internal.h"
#include "cq_moe.h"

namespace cq {

// ------------------------------------------------------------------ routing
// One CTA (1024 threads).  Top-k per token (one warp per token, descending,
// ties to the lower expert id), softmax weights, per-expert counts and
// offsets, a stable permutation of the slots t*k+j grouped by expert, its
// inverse, and the per-expert prefix of token tiles used by the grouped GEMM.
constexpr int kRouteThreads = 1024;
constexpr int kRouteWarps = kRouteThreads / 32;

__global__ void __launch_bounds__(kRouteThreads)
k_route(const float *__restrict__ logits, int T, int E, int k, int renorm, int tile_rows,
        int32_t *__restrict__ ids, float *__restrict__ w, int32_t *__restrict__ counts,
        int32_t *__restrict__ offsets, int32_t *__restrict__ perm, int32_t *__restrict__ inv_perm,
        int32_t *__restrict__ grp_tiles) {
    __shared__ int32_t hist[kRouteWarps][kMaxExperts];
    __shared__ int32_t s_off[kMaxExperts + 1];
    __shared__ int32_t s_tiles[kMaxExperts + 1];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int S = T * k;

    // ---- top-k, one warp per token
    for (int t = warp; t < T; t += kRouteWarps) {
        const float *l = logits + (int64_t)t * E;
        uint32_t taken[kMaxExperts / 32];
#pragma unroll
        for (int i = 0; i < kMaxExperts / 32; i++) taken[i] = 0;
        float top0 = 0.0f;
        float sel_l[16];
        int sel_e[16];
        for (int j = 0; j < k; j++) {
            float bv = -INFINITY;
            int be = 0x7fffffff;
            for (int i = 0; i * 32 < E; i++) {
                const int e = i * 32 + lane;
                if (e < E && !((taken[i] >> lane) & 1u)) {
                    const float v = l[e];
                    if (be == 0x7fffffff || v > bv) { bv = v; be = e; }
                }
            }
#pragma unroll
            for (int o = 16; o; o >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                const int oe = __shfl_xor_sync(0xffffffffu, be, o);
                if (oe != 0x7fffffff &&
                    (be == 0x7fffffff || ov > bv || (ov == bv && oe < be))) {
                    bv = ov;
                    be = oe;
                }
            }
            if ((be & 31) == lane) taken[be >> 5] |= 1u << lane;
            if (j == 0) top0 = bv;
            sel_l[j] = bv;
            sel_e[j] = be;
        }
        float den;
        if (renorm) {
            den = 0.0f;
            for (int j = 0; j < k; j++) den += expf(sel_l[j] - top0);
        } else {
            float part = 0.0f;
            for (int e = lane; e < E; e += 32) part += expf(l[e] - top0);
            den = warp_sum(part);
        }
        if (lane == 0) {
            for (int j = 0; j < k; j++) {
                ids[t * k + j] = sel_e[j];
                w[t * k + j] = expf(sel_l[j] - top0) / den;
            }
        }
    }
    // ---- per-warp histograms over contiguous slot chunks
    for (int i = tid; i < kRouteWarps * kMaxExperts; i += kRouteThreads)
        (&hist[0][0])[i] = 0;
    __syncthreads();  // also orders the ids writes above (same block)
    const int chunk = (S + kRouteWarps - 1) / kRouteWarps;
    const int c0 = warp * chunk, c1 = min(S, c0 + chunk);
    for (int sl = c0 + lane; sl < c1; sl += 32) atomicAdd(&hist[warp][ids[sl]], 1);
    __syncthreads();
    // ---- counts, offsets (exclusive scan), per-warp bases
    if (tid < E) {
        int c = 0;
        for (int ww = 0; ww < kRouteWarps; ww++) c += hist[ww][tid];
        s_off[tid + 1] = c;
        s_tiles[tid + 1] = (c + tile_rows - 1) / tile_rows;
    }
    if (tid == 0) { s_off[0] = 0; s_tiles[0] = 0; }
    __syncthreads();
    if (tid == 0) {
        for (int e = 0; e < E; e++) {
            s_off[e + 1] += s_off[e];
            s_tiles[e + 1] += s_tiles[e];
        }
    }
    __syncthreads();
    if (tid < E) {
        int base = s_off[tid];
        counts[tid] = s_off[tid + 1] - s_off[tid];
        for (int ww = 0; ww < kRouteWarps; ww++) {
            const int h = hist[ww][tid];
            hist[ww][tid] = base;
            base += h;
        }
    }
    if (tid <= E) {
        offsets[tid] = s_off[tid];
        grp_tiles[tid] = s_tiles[tid];
    }
    __syncthreads();
    // ---- stable placement: each warp walks its chunk in slot order
    for (int sb = c0; sb < c1; sb += 32) {
        const int sl = sb + lane;
        const bool ok = sl < c1;
        const int e = ok ? ids[sl] : -1 - lane;
        const unsigned act = __ballot_sync(0xffffffffu, ok);
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(peers & ((1u << lane) - 1u));
        int pos = 0;
        if (ok) pos = hist[warp][e] + rank;
        __syncwarp();
        if (ok && rank == 0) hist[warp][e] += __popc(peers & act);
        __syncwarp();
        if (ok) {
            perm[pos] = sl;
            inv_perm[sl] = pos;
        }
    }
}

cudaError_t launch_route(const float *logits, int T, int E, int k, int renorm, int tile_rows,
                         int32_t *ids, float *w, int32_t *counts, int32_t *offsets, int32_t *perm,
                         int32_t *inv_perm, int32_t *grp_tiles, cudaStream_t st) {
    count_launch();
    k_route<<<1, kRouteThreads, 0, st>>>(logits, T, E, k, renorm, tile_rows, ids, w, counts,
                                          offsets, perm, inv_perm, grp_tiles);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ combine
// out[t, n] = sum_j w[t,j] * s_h[p] * sum_split part[split][p][n]  (j in order)
//           + sum_s s_h[ps] * sum_split part_s[split][ps][n]
__global__ void __launch_bounds__(256) k_combine(CombineArgs a) {
    // slot counts of the shared-expert down launch, per (shared expert, row tile)
    __shared__ int s_ns[4][256];
    const int t = blockIdx.x;
    const int nrt = a.n_shared ? a.plan_s.n_row_tiles : 0;
    for (int i = threadIdx.x; i < a.n_shared * nrt; i += blockDim.x) {
        const int s = i / nrt, rt = i - s * nrt;
        const int64_t lp = (int64_t)s * a.T + t;
        s_ns[s][rt] = lut_splits_at(a.plan_s, lp, rt * a.plan_s.rows_per_rt);
    }
    __syncthreads();
    for (int n = threadIdx.x; n < a.H; n += blockDim.x) {
        float acc = 0.0f;
        for (int j = 0; j < a.topk; j++) {
            const int p = a.inv_perm[t * a.topk + j];
            float y = 0.0f;
            for (int sp = 0; sp < a.plan_r.splits; sp++)
                y += a.part_r[((int64_t)sp * a.R_routed + p) * a.H + n];
            y *= a.h_scales[p];
            if (a.y_dbg) a.y_dbg[(int64_t)p * a.H + n] = y;
            acc += a.w[t * a.topk + j] * y;
        }
        for (int s = 0; s < a.n_shared; s++) {
            const int64_t lp = (int64_t)s * a.T + t;
            float y = 0.0f;
            const int ns = s_ns[s][n / a.plan_s.rows_per_rt];
            for (int sp = 0; sp < ns; sp++)
                y += a.part_s[((int64_t)sp * a.R_shared + lp) * a.H + n];
            y *= a.h_scales[a.R_routed + lp];
            if (a.y_dbg) a.y_dbg[(a.R_routed + lp) * a.H + n] = y;
            acc += y;
        }
        a.out[(int64_t)t * a.H + n] = acc;
    }
}

cudaError_t launch_combine(const CombineArgs &a, cudaStream_t st) {
    if ((int64_t)a.T * a.H == 0) return cudaSuccess;
    count_launch();
    k_combine<<<(unsigned)a.T, 256, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace cq
