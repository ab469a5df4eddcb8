// kernels_moe.cu -- routing / expert grouping and combine kernels of the
// CodeQuant MoE linear layer (sm_100a).
#include <algorithm>

#include "cq_common.cuh"
#include "cq_internal.h"
#include "cq_moe.h"

namespace cq {

// ------------------------------------------------------------------ routing
// (1) k_topk: one warp per token, the token's logits held in registers:
//     the k largest in descending order, ties to the lower expert id, and the
//     softmax weights.
// (2) k_group_hist + k_group_place: per-expert counts and offsets, a stable
//     permutation of the slots t*k+j grouped by expert, its inverse, and the
//     per-expert prefix of token tiles used by the grouped GEMM (below).
constexpr int kTopkWarps = 8;

__global__ void __launch_bounds__(kTopkWarps * 32)
k_topk(const float *__restrict__ logits, int T, int E, int k, int renorm,
       int32_t *__restrict__ ids, float *__restrict__ w) {
    griddep_wait();
    griddep_launch();
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * kTopkWarps + (threadIdx.x >> 5);
    if (t >= T) return;
    const float *l = logits + (int64_t)t * E;
    constexpr int kPer = kMaxExperts / 32;
    float v[kPer];
    uint32_t taken = 0;  // bit i: expert i*32 + lane taken (or absent)
#pragma unroll
    for (int i = 0; i < kPer; i++) {
        const int e = i * 32 + lane;
        v[i] = e < E ? l[e] : -INFINITY;
        if (e >= E) taken |= 1u << i;
    }
    float top0 = 0.0f, den_all = 0.0f;
    float sel_l = 0.0f;  // lane j keeps the logit of choice j
    int sel_e = 0;
    for (int j = 0; j < k; j++) {
        float bv = -INFINITY;
        int be = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < kPer; i++)
            if (!((taken >> i) & 1u) && (be == 0x7fffffff || v[i] > bv)) {
                bv = v[i];
                be = i * 32 + lane;
            }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            if (oe != 0x7fffffff && (be == 0x7fffffff || ov > bv || (ov == bv && oe < be))) {
                bv = ov;
                be = oe;
            }
        }
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
        if (j == 0) top0 = bv;
        if (lane == j) {
            sel_l = bv;
            sel_e = be;
        }
    }
    if (!renorm) {
        float part = 0.0f;
#pragma unroll
        for (int i = 0; i < kPer; i++)
            if (i * 32 + lane < E) part += expf(v[i] - top0);
        den_all = warp_sum(part);
    }
    const float ex = lane < k ? expf(sel_l - top0) : 0.0f;
    const float den = renorm ? warp_sum(ex) : den_all;
    if (lane < k) {
        ids[t * k + lane] = sel_e;
        w[t * k + lane] = ex / den;
    }
}

// Grouping over many CTAs.  The S = T*k slots are cut into contiguous chunks,
// one CTA each.  k_group_hist: per-chunk expert counts.  k_group_place: the
// chunk's base per expert (counts of the chunks before it), the global
// offsets (all chunks' counts, scanned over experts), and a stable placement
// of the chunk's slots (each warp a contiguous run, in slot order) -- the
// same permutation a single pass in slot order gives.  CTA 0 also writes the
// counts, offsets and tile tables.
constexpr int kGroupThreads = 256;
constexpr int kGroupWarps = kGroupThreads / 32;

__global__ void __launch_bounds__(kGroupThreads)
k_group_hist(const int32_t *__restrict__ ids, int S, int E, int chunk, int32_t *__restrict__ chist) {
    __shared__ int32_t hist[kMaxExperts];
    griddep_wait();
    griddep_launch();
    for (int e = threadIdx.x; e < E; e += kGroupThreads) hist[e] = 0;
    __syncthreads();
    const int c0 = blockIdx.x * chunk, c1 = min(S, c0 + chunk);
    for (int sl = c0 + threadIdx.x; sl < c1; sl += kGroupThreads) atomicAdd(&hist[ids[sl]], 1);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += kGroupThreads) chist[(int64_t)blockIdx.x * E + e] = hist[e];
}

__global__ void __launch_bounds__(kGroupThreads)
k_group_place(const int32_t *__restrict__ ids, int S, int E, int tile_rows, int chunk, int nchunk,
              const int32_t *__restrict__ chist, int32_t *__restrict__ counts,
              int32_t *__restrict__ offsets, int32_t *__restrict__ perm,
              int32_t *__restrict__ inv_perm, int32_t *__restrict__ grp_tiles,
              int32_t *__restrict__ tile_grp, int max_tiles) {
    __shared__ int32_t hist[kGroupWarps][kMaxExperts];
    __shared__ int32_t s_off[kMaxExperts + 1];
    __shared__ int32_t s_tiles[kMaxExperts + 1];
    __shared__ int32_t s_base[kMaxExperts];
    griddep_wait();
    griddep_launch();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cb = blockIdx.x;
    for (int i = tid; i < kGroupWarps * kMaxExperts; i += kGroupThreads) (&hist[0][0])[i] = 0;
    __syncthreads();
    // this chunk's slots: a contiguous run per warp, counted per warp
    const int c0 = cb * chunk, c1 = min(S, c0 + chunk);
    const int sub = (c1 - c0 + kGroupWarps - 1) / kGroupWarps;
    const int w0 = min(c1, c0 + warp * sub), w1 = min(c1, w0 + sub);
    for (int sl = w0 + lane; sl < w1; sl += 32) atomicAdd(&hist[warp][ids[sl]], 1);
    __syncthreads();
    // per expert: slots of the chunks before this one, and of all chunks (one
    // chunk: this CTA's own counts, no histogram launch)
    for (int e = tid; e < E; e += kGroupThreads) {
        int before = 0, total = 0;
        if (nchunk == 1) {
            for (int ww = 0; ww < kGroupWarps; ww++) total += hist[ww][e];
        } else {
            for (int c = 0; c < nchunk; c++) {
                const int v = chist[(int64_t)c * E + e];
                before += c < cb ? v : 0;
                total += v;
            }
        }
        s_base[e] = before;
        s_off[e + 1] = total;
        s_tiles[e + 1] = (total + tile_rows - 1) / tile_rows;
    }
    if (tid == 0) { s_off[0] = 0; s_tiles[0] = 0; }
    __syncthreads();
    if (warp == 0) {  // inclusive scans over E <= 256 entries
        int base_o = 0, base_t = 0;
        for (int e0 = 0; e0 < E; e0 += 32) {
            const int e = e0 + lane + 1;
            int vo = e <= E ? s_off[e] : 0, vt = e <= E ? s_tiles[e] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int uo = __shfl_up_sync(0xffffffffu, vo, o);
                const int ut = __shfl_up_sync(0xffffffffu, vt, o);
                if (lane >= o) { vo += uo; vt += ut; }
            }
            if (e <= E) { s_off[e] = vo + base_o; s_tiles[e] = vt + base_t; }
            base_o += __shfl_sync(0xffffffffu, vo, 31);
            base_t += __shfl_sync(0xffffffffu, vt, 31);
        }
    }
    __syncthreads();
    if (cb == 0) {
        for (int e = tid; e < E; e += kGroupThreads) counts[e] = s_off[e + 1] - s_off[e];
        for (int e = tid; e <= E; e += kGroupThreads) {
            offsets[e] = s_off[e];
            grp_tiles[e] = s_tiles[e];
        }
        // tile -> group, so the LUT kernels find a tile's expert with one load
        for (int e = tid; e < E; e += kGroupThreads)
            for (int tl = s_tiles[e]; tl < s_tiles[e + 1] && tl < max_tiles; tl++) tile_grp[tl] = e;
    }
    // bases of the warps' runs
    for (int e = tid; e < E; e += kGroupThreads) {
        int base = s_off[e] + s_base[e];
        for (int ww = 0; ww < kGroupWarps; ww++) {
            const int h = hist[ww][e];
            hist[ww][e] = base;
            base += h;
        }
    }
    __syncthreads();
    for (int sb = w0; sb < w1; sb += 32) {
        const int sl = sb + lane;
        const bool ok = sl < w1;
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

// Slots per grouping chunk: at least 1024 (decode-sized routings take one
// CTA and no histogram launch), at most 128 chunks.
static int group_chunk(int S) { return std::max(1024, (S + 127) / 128); }

size_t route_scratch_bytes(int T, int E, int k) {
    const int S = T * k;
    const int chunk = group_chunk(S);
    return (size_t)((S + chunk - 1) / chunk) * E * sizeof(int32_t);
}

cudaError_t launch_route(const float *logits, int T, int E, int k, int renorm, int tile_rows,
                         int32_t *ids, float *w, int32_t *counts, int32_t *offsets, int32_t *perm,
                         int32_t *inv_perm, int32_t *grp_tiles, int32_t *tile_grp,
                         int max_tiles, int32_t *chist, cudaStream_t st) {
    TimedScope ts(st, CQ_KERNEL_ROUTE);
    const int S = T * k;
    const int chunk = group_chunk(S);
    const int nchunk = (S + chunk - 1) / chunk;
    count_launch(nchunk > 1 ? 3 : 2);
    cudaError_t e = launch_pdl(k_topk, dim3((T + kTopkWarps - 1) / kTopkWarps),
                               dim3(kTopkWarps * 32), 0, st, 1, logits, T, E, k, renorm, ids, w);
    if (e != cudaSuccess) return e;
    if (nchunk > 1) {
        e = launch_pdl(k_group_hist, dim3(nchunk), dim3(kGroupThreads), 0, st, 1,
                       (const int32_t *)ids, S, E, chunk, chist);
        if (e != cudaSuccess) return e;
    }
    return launch_pdl(k_group_place, dim3(nchunk), dim3(kGroupThreads), 0, st, 1,
                      (const int32_t *)ids, S, E, tile_rows, chunk, nchunk,
                      (const int32_t *)chist, counts, offsets, perm, inv_perm, grp_tiles,
                      tile_grp, max_tiles);
}

// ------------------------------------------------------------------ combine
// out[t, n] = sum_j w[t,j] * s_h[p] * sum_split part[split][p][n]  (j in order)
//           + sum_s s_h[ps] * sum_split part_s[split][ps][n]
// One CTA per token and 4 * kCombThreads columns; each thread 4 consecutive
// columns.  The token's routed and shared rows are one list of sources, and
// the loads of eight sources go out together, so a token with up to eight
// rows costs one memory round trip.
constexpr int kCombThreads = 256;
constexpr int kCombF = 8;  // sources in flight per round

__global__ void __launch_bounds__(kCombThreads, 3) k_combine(CombineArgs a) {
    __shared__ int64_t s_row[kMaxTopK + 4];  // source -> partial row (slot 0)
    __shared__ float s_c[kMaxTopK];          // w[t, j] (scale of row p applied separately)
    __shared__ float s_sh[kMaxTopK + 4];     // h scale of the source's row
    __shared__ int s_ns[4][24];              // slot counts, shared expert x row tile of this block (<= 17)
    griddep_wait();
    griddep_launch();
    const int t = blockIdx.x;
    const int n0 = blockIdx.y * 4 * kCombThreads;
    const int F = a.topk + a.n_shared;
    if (threadIdx.x < a.topk) {
        const int p = a.inv_perm[t * a.topk + threadIdx.x];
        s_row[threadIdx.x] = p;
        s_c[threadIdx.x] = a.w[t * a.topk + threadIdx.x];
        s_sh[threadIdx.x] = a.h_scales[p];
    } else if (threadIdx.x < F) {
        const int64_t lp = (int64_t)(threadIdx.x - a.topk) * a.T + t;
        s_row[threadIdx.x] = lp;
        s_sh[threadIdx.x] = a.h_scales[a.R_routed + lp];
    }
    const int rpt = a.n_shared ? a.plan_s.rows_per_rt : 1;
    const int rt0 = n0 / rpt;
    const int nrt = a.n_shared ? (min(n0 + 4 * kCombThreads - 1, a.H - 1)) / rpt - rt0 + 1 : 0;
    for (int i = threadIdx.x; i < a.n_shared * nrt; i += kCombThreads) {
        const int s = i / nrt, r = i - s * nrt;
        s_ns[s][r] = lut_splits_at(a.plan_s, (int64_t)s * a.T + t, (rt0 + r) * rpt);
    }
    __syncthreads();
    const int n = n0 + 4 * threadIdx.x;
    if (n >= a.H) return;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    const int64_t stride_r = a.R_routed * (int64_t)a.H / 4, stride_s = a.R_shared * (int64_t)a.H / 4;
    const int rti = n / rpt - rt0;  // this thread's row tile among the block's
    for (int f0 = 0; f0 < F; f0 += kCombF) {
        // slot 0 of every source, all loads in flight together
        float4 y[kCombF];
        int nsmax = 0;
#pragma unroll
        for (int u = 0; u < kCombF; u++) {
            const int f = f0 + u;
            y[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (f < F) {
                const bool routed = f < a.topk;
                const int ns = routed ? a.plan_r.splits : s_ns[f - a.topk][rti];
                nsmax = max(nsmax, ns);
                if (ns > 0)
                    y[u] = *reinterpret_cast<const float4 *>((routed ? a.part_r : a.part_s) +
                                                             s_row[f] * a.H + n);
            }
        }
        // further split-K slots (a dense layer's decode-time down projection),
        // source by source with eight slot loads in flight, added in slot order
        if (nsmax > 1) {
#pragma unroll
            for (int u = 0; u < kCombF; u++) {
                const int f = f0 + u;
                if (f >= F) break;
                const bool routed = f < a.topk;
                const int ns = routed ? a.plan_r.splits : s_ns[f - a.topk][rti];
                if (ns < 2) continue;
                const int64_t st4 = routed ? stride_r : stride_s;
                const float4 *p1[1] = {reinterpret_cast<const float4 *>(
                                           (routed ? a.part_r : a.part_s) + s_row[f] * a.H + n) +
                                       st4};
                const int ns1[1] = {ns - 1};
                float4 acc1[1] = {y[u]};
                sum_slots<1, 8>(p1, ns1, st4, acc1);
                y[u] = acc1[0];
            }
        }
#pragma unroll
        for (int u = 0; u < kCombF; u++) {
            const int f = f0 + u;
            if (f >= F) break;
            const float sc = s_sh[f];
            y[u].x *= sc; y[u].y *= sc; y[u].z *= sc; y[u].w *= sc;
            const int64_t dbg_row = f < a.topk ? s_row[f] : a.R_routed + s_row[f];
            if (a.y_dbg) *reinterpret_cast<float4 *>(a.y_dbg + dbg_row * a.H + n) = y[u];
            if (f < a.topk) {
                const float c = s_c[f];
                acc.x += c * y[u].x; acc.y += c * y[u].y; acc.z += c * y[u].z; acc.w += c * y[u].w;
            } else {
                acc.x += y[u].x; acc.y += y[u].y; acc.z += y[u].z; acc.w += y[u].w;
            }
        }
    }
    *reinterpret_cast<float4 *>(a.out + (int64_t)t * a.H + n) = acc;
}

cudaError_t launch_combine(const CombineArgs &a, cudaStream_t st) {
    if ((int64_t)a.T * a.H == 0) return cudaSuccess;
    TimedScope ts(st, CQ_KERNEL_COMBINE);
    count_launch();
    const int cols = 4 * kCombThreads;
    return launch_pdl(k_combine, dim3((unsigned)a.T, (unsigned)((a.H + cols - 1) / cols)),
                      dim3(kCombThreads), 0, st, 1, a);
}

}  // namespace cq
