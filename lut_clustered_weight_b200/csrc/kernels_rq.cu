// kernels_rq.cu -- online rotation + per-token quantization of activation
// rows (x before gate/up, and h = SwiGLU(g, u) before down), sm_100a.
//
// One thread-block cluster per row.  The row is cut into whole rotation
// blocks, shared out over the cluster's CTAs; every CTA rotates its blocks
// exactly in fp64 (shared memory), the absmax of the row is reduced across the
// cluster through distributed shared memory, and every CTA then quantizes and
// stores its own part.  At decode (a handful of rows) the cluster spreads a
// row over up to 8 SMs instead of one.
#include <cooperative_groups.h>

#include <algorithm>
#include <mutex>
#include <tuple>
#include <vector>

#include "cq_common.cuh"
#include "cq_internal.h"
#include "cq_moe.h"
#include "rotate_quantize.cuh"

namespace cg = cooperative_groups;

namespace cq {

constexpr int kRqThreads = 256;
constexpr int kMaxCluster = 8;

// CTA `rank` of `csize` handles units [u0, u1) of ub = max(b, 8) positions.
struct RowPart {
    int e0, n;
};
CQ_DEV RowPart row_part(int K, int log2b, int rank, int csize) {
    const int ub = max(1 << log2b, 8);
    const int nu = K / ub;
    const int u0 = rank * nu / csize, u1 = (rank + 1) * nu / csize;
    return {u0 * ub, (u1 - u0) * ub};
}

// Rotate buf[0, n) (complete blocks), reduce the absmax over the row (across
// the cluster when CLUSTER), quantize and store this CTA's codes (and their
// fp16 copies for row mrow of K positions); rank 0 stores the scale.
template <bool CLUSTER>
CQ_DEV void rq_finish(double *buf, RowPart part, int log2b, int bits, uint8_t *qrow,
                      float *s_out, const RqF16 &f16, int64_t mrow, int K) {
    __shared__ double red[33];
    __shared__ double s_amax;
    block_fwht<kRqThreads>(buf, part.n, log2b);
    double A = block_absmax<kRqThreads>(buf, part.n, red);
    bool rank0 = true;
    if (CLUSTER) {
        cg::cluster_group cluster = cg::this_cluster();
        if (threadIdx.x == 0) s_amax = A;
        cluster.sync();
        A = 0.0;
        const int cs = (int)cluster.num_blocks();
        for (int r = 0; r < cs; r++) A = fmax(A, *cluster.map_shared_rank(&s_amax, r));
        cluster.sync();  // every CTA has read every s_amax
        rank0 = cluster.block_rank() == 0;
    }
    block_quantize_range<kRqThreads>(buf, part.n, part.e0, bits, A, qrow, f16, mrow, K);
    if (rank0 && threadIdx.x == 0) {
        const int qmax = (1 << (bits - 1)) - 1;
        const float sq = A > 0.0 ? quant_scale(A, log2b, qmax) : 0.0f;
        *s_out = sq;
        store_copy_scales(f16, mrow, sq);
    }
}

template <bool CLUSTER>
CQ_DEV void cluster_pos(int &cs, int &rank) {
    if (CLUSTER) {
        cg::cluster_group cluster = cg::this_cluster();
        cs = (int)cluster.num_blocks();
        rank = (int)cluster.block_rank();
    } else {
        cs = 1;
        rank = 0;
    }
}

// Loads elements [e0, e0 + n) of one x row into buf as fp64: plainly, or
// (scale / perm non-NULL) as fp16(x[perm[j]] * scale[perm[j]]) -- the online
// smoothing scale and channel grouping.  fp16 x fp16 is exact in fp32 and
// __float2half_rn rounds it to nearest even.  A permutation value outside
// [0, K) is clamped into range, so no load can leave the row.
CQ_DEV void load_x_part(double *buf, const __half *__restrict__ xr, int e0, int n, int K,
                        const __half *__restrict__ scale, const int32_t *__restrict__ perm,
                        int tid, int nthreads) {
    if (!scale && !perm) {
        for (int i = tid; i < n / 8; i += nthreads) {
            const uint4 v = *reinterpret_cast<const uint4 *>(xr + e0 + 8 * i);
            const __half2 *h = reinterpret_cast<const __half2 *>(&v);
#pragma unroll
            for (int j = 0; j < 4; j++) {
                const float2 f = __half22float2(h[j]);
                buf[8 * i + 2 * j] = (double)f.x;
                buf[8 * i + 2 * j + 1] = (double)f.y;
            }
        }
        return;
    }
    for (int i = tid; i < n; i += nthreads) {
        const int j = e0 + i;
        const int c = perm ? (int)min((unsigned)perm[j], (unsigned)(K - 1)) : j;
        float v = __half2float(xr[c]);
        if (scale) v = __half2float(__float2half_rn(v * __half2float(scale[c])));
        buf[i] = (double)v;
    }
}

// ------------------------------------------------------------------ x rows
template <bool CLUSTER>
__global__ void __launch_bounds__(kRqThreads)
k_rq_x(const __half *__restrict__ x, int64_t ldx, int K, int log2b, int bits,
       uint8_t *__restrict__ q, int64_t ldq, float *__restrict__ s,
       const __half *__restrict__ scale, const int32_t *__restrict__ perm, const RqF16 f16) {
    extern __shared__ __align__(16) double buf[];
    int cs, rank;
    griddep_wait();
    griddep_launch();
    cluster_pos<CLUSTER>(cs, rank);
    const int64_t m = blockIdx.x / cs;
    const RowPart part = row_part(K, log2b, rank, cs);
    load_x_part(buf, x + m * ldx, part.e0, part.n, K, scale, perm, threadIdx.x, kRqThreads);
    __syncthreads();
    rq_finish<CLUSTER>(buf, part, log2b, bits, q + m * ldq, s + m, f16, m, K);
}

// ------------------------------------------------------------------ SwiGLU rows
// Row p of the intermediate: g, u = sum of the split-K partials, scaled by the
// token's s_x; h = fp16(silu(g) * u) (round to nearest even); then as above.
template <bool CLUSTER>
__global__ void __launch_bounds__(kRqThreads) k_rq_swiglu(const SwigluArgs a) {
    extern __shared__ __align__(16) double buf[];
    griddep_wait();
    griddep_launch();
    int cs, rank;
    cluster_pos<CLUSTER>(cs, rank);
    const int64_t p = blockIdx.x / cs;
    const bool routed = p < a.R_routed;
    const int I = routed ? a.I : a.I_shared;
    const int log2b = routed ? a.log2b_i : a.log2b_i_shared;
    const float *part = routed ? a.part_r : a.part_s;
    const LutPlan P = routed ? a.plan_r : a.plan_s;
    const int64_t rows = routed ? a.R_routed : a.R_shared;
    const int64_t lp = routed ? p : p - a.R_routed;
    const int tok = routed ? a.perm[p] / a.topk : (int)(lp % a.T);
    const float sx = a.x_scales[tok];
    const RowPart rp = row_part(I, log2b, rank, cs);
    // slot counts of the gate/up launch for the row tiles of this CTA's columns
    __shared__ int s_ns[kMaxK / 64];
    const int rt0 = rp.e0 / P.rows_per_rt;
    const int nrt = rp.n > 0 ? (rp.e0 + rp.n - 1) / P.rows_per_rt - rt0 + 1 : 0;
    for (int i = threadIdx.x; i < nrt; i += kRqThreads)
        s_ns[i] = lut_splits_at(P, lp, (rt0 + i) * P.rows_per_rt);
    __syncthreads();
    // batches of 4 elements per thread: all partial loads first, then the math
    const int64_t slot_stride = rows * 2 * (int64_t)I;
    const float *rowp = part + lp * (2 * (int64_t)I);
    for (int i0 = 0; i0 < rp.n; i0 += 4 * kRqThreads) {
        float2 acc[4];
        const float2 *pf[4];
        int nsf[4];
#pragma unroll
        for (int f = 0; f < 4; f++) {
            acc[f] = make_float2(0.f, 0.f);
            const int i = i0 + f * kRqThreads + threadIdx.x;
            const int n = rp.e0 + min(i, rp.n - 1);
            pf[f] = reinterpret_cast<const float2 *>(rowp + 2 * n);
            nsf[f] = i < rp.n ? s_ns[n / P.rows_per_rt - rt0] : 0;
        }
        sum_slots<4, 4>(pf, nsf, slot_stride / 2, acc);
#pragma unroll
        for (int f = 0; f < 4; f++) {
            const int i = i0 + f * kRqThreads + threadIdx.x;
            if (i < rp.n) {
                const int n = rp.e0 + i;
                const __half h = __float2half_rn(silu_mul(acc[f].x * sx, acc[f].y * sx));
                if (a.h_dbg) reinterpret_cast<__half *>(a.h_dbg)[p * a.Imax + n] = h;
                buf[i] = (double)__half2float(h);
            }
        }
    }
    __syncthreads();
    RqF16 f16{};
    f16.ident = routed ? a.f16_r : a.f16_s;
    rq_finish<CLUSTER>(buf, rp, log2b, a.bits, a.hq + p * a.ldhq, a.h_scales + p, f16, lp, I);
}

// ------------------------------------------------------------------ one warp per row
// For many short rows with rotation blocks of at most 256: no block barrier,
// kWarpRows rows per CTA, each row in its warp's slice of shared memory.
constexpr int kWarpRows = 4;

__global__ void __launch_bounds__(kWarpRows * 32)
k_rq_x_warp(const __half *__restrict__ x, int64_t ldx, int64_t M, int K, int log2b, int bits,
            uint8_t *__restrict__ q, int64_t ldq, float *__restrict__ s,
            const __half *__restrict__ scale, const int32_t *__restrict__ perm, const RqF16 f16) {
    extern __shared__ __align__(16) double wbuf[];
    griddep_wait();
    griddep_launch();
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int64_t m = (int64_t)blockIdx.x * kWarpRows + w;
    if (m >= M) return;
    double *buf = wbuf + (size_t)w * K;
    load_x_part(buf, x + m * ldx, 0, K, K, scale, perm, lane, 32);
    __syncwarp();
    const double A = warp_fwht_absmax(buf, K, log2b);
    warp_quantize_row(buf, K, log2b, bits, A, q + m * ldq, s + m, f16, m);
}

// ------------------------------------------------------------------ rows in registers
// Thread j of a row holds positions [32 j, 32 j + 32) as fp64 registers.
// Index bits 0-4 of the transform are butterflies inside the thread, bits
// 5-9 pair threads j and j ^ 2^(bit - 5) of the same warp (a block's threads
// are consecutive and aligned, since rows and blocks start at multiples of
// min(b, 1024) / 32 threads), and bits 10 .. log2b - 1 pair threads of
// different warps of the row through shared memory.  The row's absmax is
// reduced through shared memory, then every
// thread quantizes its 32 values and stores their codes as 16- or 32-byte
// vectors.  Same exact fp64 arithmetic as the shared-memory kernels, so the
// codes and scales are identical; no row buffer, so many rows per SM.
constexpr int kRegThreads = 512;

// XWARP: blocks over 1024 (levels across warps); FULL: blocks of at least 32
// (all five in-thread levels, unconditional, so no value needs a merge)
template <bool XWARP, bool FULL>
__global__ void __launch_bounds__(kRegThreads)
k_rq_x_reg(const __half *__restrict__ x, int64_t ldx, int64_t M, int K, int log2b, int bits,
           uint8_t *__restrict__ q, int64_t ldq, float *__restrict__ s,
           const __half *__restrict__ scale, const int32_t *__restrict__ perm, int rows_per_cta,
           int n_groups, const RqF16 f16) {
    // [threads]: max |v| of each thread's 32; then, for blocks over 1024, the
    // exchange area [32][threads] (position i of thread t at i * threads + t)
    extern __shared__ __align__(16) double tmax[];
    griddep_wait();
    griddep_launch();
    const int K32 = K >> 5;
    const int tid = threadIdx.x;
    const int r = tid / K32, j = tid - r * K32;  // row within the group, thread within the row
    const bool plain = !scale && !perm;
    // persistent: row groups blockIdx.x, + gridDim.x, ...; the fp16 inputs of
    // the next group are loaded while this one is rotated and quantized
    uint4 nx[4];
    auto fetch = [&](int grp) {
        const int64_t mm = (int64_t)grp * rows_per_cta + r;
        if (plain && grp < n_groups && r < rows_per_cta && mm < M) {
            const uint4 *src = reinterpret_cast<const uint4 *>(x + mm * ldx + 32 * j);
#pragma unroll
            for (int i = 0; i < 4; i++) nx[i] = __ldcs(src + i);
        }
    };
    fetch(blockIdx.x);
    for (int grp = blockIdx.x; grp < n_groups; grp += gridDim.x) {
        const int64_t m = (int64_t)grp * rows_per_cta + r;
        const bool live = r < rows_per_cta && m < M;
        double v[32];
        if (live) {
            const __half *xr = x + m * ldx;
            const int e0 = 32 * j;
            if (plain) {
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    const __half2 *h = reinterpret_cast<const __half2 *>(&nx[i]);
#pragma unroll
                    for (int t = 0; t < 4; t++) {
                        const float2 f = __half22float2(h[t]);
                        v[8 * i + 2 * t] = (double)f.x;
                        v[8 * i + 2 * t + 1] = (double)f.y;
                    }
                }
            } else {
#pragma unroll
                for (int i = 0; i < 32; i++) {
                    const int c = perm ? (int)min((unsigned)perm[e0 + i], (unsigned)(K - 1)) : e0 + i;
                    float f = __half2float(xr[c]);
                    if (scale) f = __half2float(__float2half_rn(f * __half2float(scale[c])));
                    v[i] = (double)f;
                }
            }
        } else {
#pragma unroll
            for (int i = 0; i < 32; i++) v[i] = 0.0;
        }
        fetch(grp + gridDim.x);
        // index bits 0-4: inside the thread
#pragma unroll
        for (int L = 0; L < 5; L++) {
            if (FULL || L < log2b) {
                const int h = 1 << L;
#pragma unroll
                for (int i = 0; i < 32; i++) {
                    if ((i & h) == 0) {
                        const double a = v[i], c = v[i + h];
                        v[i] = a + c;
                        v[i + h] = a - c;
                    }
                }
            }
        }
        // index bits 5-9: across the block's threads of one warp (lower thread
        // keeps v + p, upper p - v: one correctly rounded fma with an exact +-1
        // product)
        for (int L = 5; L < min(log2b, 10); L++) {
            const int bit = 1 << (L - 5);
            const double sg = (j & bit) ? -1.0 : 1.0;
#pragma unroll
            for (int i = 0; i < 32; i++) {
                const double p = __shfl_xor_sync(0xffffffffu, v[i], bit);
                v[i] = fma(sg, v[i], p);
            }
        }
        // index bits 10..: threads j and j ^ 2^(bit - 5) sit in different warps
        if (XWARP) {
            const int T = blockDim.x;
            double *xch = tmax + T;
            for (int L = 10; L < log2b; L++) {
                const int bit = 1 << (L - 5);
#pragma unroll
                for (int i = 0; i < 32; i++) xch[i * T + tid] = v[i];
                __syncthreads();
                const int pt = tid ^ bit;  // same row: rows start at multiples of b / 32 threads
                const bool upper = j & bit;
#pragma unroll
                for (int i = 0; i < 32; i++) {
                    const double p = xch[i * T + pt];
                    v[i] = upper ? p - v[i] : v[i] + p;
                }
                __syncthreads();
            }
        }
        double mx = 0.0;
#pragma unroll
        for (int i = 0; i < 32; i++) mx = fmax(mx, fabs(v[i]));
        tmax[tid] = mx;
        __syncthreads();
        // the row's first thread reduces its K/32 maxima (four independent
        // chains) and leaves the row's absmax in the row's first entry
        if (live && j == 0) {
            double m4[4] = {0.0, 0.0, 0.0, 0.0};
            const double *row = tmax + r * K32;
            int i = 0;
            for (; i + 4 <= K32; i += 4) {
#pragma unroll
                for (int u = 0; u < 4; u++) m4[u] = fmax(m4[u], row[i + u]);
            }
            for (; i < K32; i++) m4[0] = fmax(m4[0], row[i]);
            tmax[r * K32] = fmax(fmax(m4[0], m4[1]), fmax(m4[2], m4[3]));
        }
        __syncthreads();
        if (live) {
            const double A = tmax[r * K32];
            const int qmax = (1 << (bits - 1)) - 1;
            const long long Ai = __double2ll_rn(A * 16777216.0);
            const double R = Ai > 0 ? __ddiv_rn((double)qmax, A) : 0.0;
            // codes packed as they are made (bits 4: 8 per word, bits 8: 4 per word)
            const int per_word = bits == 4 ? 8 : 4, fbits = bits;
            const uint32_t fmask = bits == 4 ? 15u : 255u;
            uint32_t w[8];
#pragma unroll
            for (int t = 0; t < 8; t++) w[t] = 0;
            uint32_t ties = 0;
            if (Ai > 0) {
#pragma unroll
                for (int i = 0; i < 32; i++) {
                    bool t;
                    const int c = quantize_round(v[i], R, t);
                    ties |= (uint32_t)t << i;
                    if (bits == 4)
                        w[i >> 3] |= ((uint32_t)c & 15u) << (4 * (i & 7));
                    else
                        w[i >> 2] |= ((uint32_t)c & 255u) << (8 * (i & 3));
                }
            }
            if (ties) {
                // rare: the exact rotated value again from the input (the block's
                // signed sum, exact in fp64 in any order) and the exact rational decision
                const __half *xr = x + m * ldx;
                const int b = 1 << log2b;
#pragma unroll 1
                for (int i = 0; i < 32; i++) {
                    if (!((ties >> i) & 1u)) continue;
                    const int p = 32 * j + i, blk0 = p & ~(b - 1), pos = p - blk0;
                    double sum = 0.0;
                    for (int k = 0; k < b; k++) {
                        const int e = blk0 + k;
                        const int c = perm ? (int)min((unsigned)perm[e], (unsigned)(K - 1)) : e;
                        float f = __half2float(xr[c]);
                        if (scale) f = __half2float(__float2half_rn(f * __half2float(scale[c])));
                        sum += (__popc(pos & k) & 1) ? -(double)f : (double)f;
                    }
                    const uint32_t c = (uint32_t)quantize_tie(sum, Ai, qmax) & fmask;
                    const int wi = i / per_word, sh = fbits * (i % per_word);
#pragma unroll
                    for (int t = 0; t < 8; t++)
                        if (t == wi) w[t] = (w[t] & ~(fmask << sh)) | (c << sh);
                }
            }
            uint8_t *qrow = q + m * ldq;
            if (bits == 4) {
                *reinterpret_cast<uint4 *>(qrow + 16 * j) = make_uint4(w[0], w[1], w[2], w[3]);
            } else {
                uint4 *dst = reinterpret_cast<uint4 *>(qrow + 32 * j);
                dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
                dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
            }
            const float sq = Ai > 0 ? quant_scale(A, log2b, qmax) : 0.0f;
            if (j == 0) s[m] = sq;
            if (f16.ncopy > 0 || f16.ident) {
                // the 32 codes as fp16 (small integers: exact), 64 bytes per copy
                uint32_t hw[16];
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    int c0, c1;
                    if (bits == 4) {
                        c0 = (int)(w[i >> 3] << (28 - 4 * (i & 7))) >> 28;
                        c1 = (int)(w[(i + 1) >> 3] << (28 - 4 * ((i + 1) & 7))) >> 28;
                    } else {
                        c0 = (int)(w[i >> 2] << (24 - 8 * (i & 3))) >> 24;
                        c1 = (int)(w[(i + 1) >> 2] << (24 - 8 * ((i + 1) & 3))) >> 24;
                    }
                    const __half2 h2 = __halves2half2(__int2half_rn(c0), __int2half_rn(c1));
                    hw[i >> 1] = *reinterpret_cast<const uint32_t *>(&h2);
                }
                auto put = [&](__half *row) {
                    uint4 *dst = reinterpret_cast<uint4 *>(row + 32 * j);
#pragma unroll
                    for (int t = 0; t < 4; t++)
                        dst[t] = make_uint4(hw[4 * t], hw[4 * t + 1], hw[4 * t + 2], hw[4 * t + 3]);
                };
                for (int d = 0; d < f16.ncopy; d++) {
                    const int64_t row = f16.map ? (int64_t)f16.map[m * f16.ncopy + d] : m;
                    put(f16.rows + row * K);
                    if (f16.row_scales && j == 0) f16.row_scales[row] = sq;
                }
                if (f16.ident) put(f16.ident + m * K);
            }
        }  // live
        __syncthreads();  // tmax (and the exchange area) are reused by the next group
    }  // row groups
}

__global__ void __launch_bounds__(kWarpRows * 32) k_rq_swiglu_warp(const SwigluArgs a, int64_t R) {
    extern __shared__ __align__(16) double wbuf[];
    __shared__ int s_ns[kWarpRows][kMaxK / 64];
    griddep_wait();
    griddep_launch();
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int64_t p = (int64_t)blockIdx.x * kWarpRows + w;
    if (p >= R) return;
    const bool routed = p < a.R_routed;
    const int I = routed ? a.I : a.I_shared;
    const int log2b = routed ? a.log2b_i : a.log2b_i_shared;
    const float *part = routed ? a.part_r : a.part_s;
    const LutPlan P = routed ? a.plan_r : a.plan_s;
    const int64_t rows = routed ? a.R_routed : a.R_shared;
    const int64_t lp = routed ? p : p - a.R_routed;
    const int tok = routed ? a.perm[p] / a.topk : (int)(lp % a.T);
    const float sx = a.x_scales[tok];
    double *buf = wbuf + (size_t)w * a.Imax;
    const int nrt = (I + P.rows_per_rt - 1) / P.rows_per_rt;
    for (int i = lane; i < nrt; i += 32) s_ns[w][i] = lut_splits_at(P, lp, i * P.rows_per_rt);
    __syncwarp();
    const int64_t slot_stride = rows * 2 * (int64_t)I;
    const float *rowp = part + lp * (2 * (int64_t)I);
    // 8 columns per lane per round: the loads of a round are all in flight
    // together, so a row of I columns costs I / 256 memory round trips
    constexpr int F = 8;
    for (int n0 = 0; n0 < I; n0 += F * 32) {
        float2 acc[F];
        const float2 *pf[F];
        int nsf[F];
#pragma unroll
        for (int f = 0; f < F; f++) {
            acc[f] = make_float2(0.f, 0.f);
            const int n = n0 + f * 32 + lane;
            pf[f] = reinterpret_cast<const float2 *>(rowp) + min(n, I - 1);
            nsf[f] = n < I ? s_ns[w][n / P.rows_per_rt] : 0;
        }
        sum_slots<F>(pf, nsf, slot_stride / 2, acc);
#pragma unroll
        for (int f = 0; f < F; f++) {
            const int n = n0 + f * 32 + lane;
            if (n < I) {
                const __half h = __float2half_rn(silu_mul(acc[f].x * sx, acc[f].y * sx));
                if (a.h_dbg) reinterpret_cast<__half *>(a.h_dbg)[p * a.Imax + n] = h;
                buf[n] = (double)__half2float(h);
            }
        }
    }
    __syncwarp();
    const double A = warp_fwht_absmax(buf, I, log2b);
    RqF16 f16{};
    f16.ident = routed ? a.f16_r : a.f16_s;
    warp_quantize_row(buf, I, log2b, a.bits, A, a.hq + p * a.ldhq, a.h_scales + p, f16, lp);
}

static bool use_warp_rows(int64_t rows, int K, int log2b) {
    return log2b <= 8 && K <= 4096 && rows >= 4LL * sm_count();
}

// CTAs of `kern` resident per SM at this block size and dynamic shared
// memory (asked once per combination and device).
static int resident_ctas(const void *kern, int threads, size_t smem) {
    static std::mutex mu;
    static std::vector<std::tuple<const void *, int, size_t, int, int>> memo;
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lk(mu);
    for (const auto &m : memo)
        if (std::get<0>(m) == kern && std::get<1>(m) == threads && std::get<2>(m) == smem &&
            std::get<3>(m) == dev)
            return std::get<4>(m);
    configure_kernel_once(kern);  // the shared-memory limit the launch will have
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, threads, smem) != cudaSuccess)
        n = 1;
    n = std::max(n, 1);
    memo.emplace_back(kern, threads, smem, dev, n);
    return n;
}

// The register kernel: blocks of at most 8192, whole rows of at most 512
// threads, 16-byte aligned rows and code rows, and rows enough for the SMs.
static bool use_reg_rows(int64_t rows, int K, int log2b, int bits, const void *x, int64_t ldx,
                         const void *q, int64_t ldq) {
    const bool aligned = (reinterpret_cast<uintptr_t>(x) % 16 == 0) && (ldx % 8 == 0) &&
                         (reinterpret_cast<uintptr_t>(q) % 16 == 0) && (ldq % 16 == 0);
    return log2b <= 13 && K % 32 == 0 && K / 32 <= kRegThreads && (bits == 4 || bits == 8) &&
           aligned && rows >= 2LL * sm_count();
}

// ------------------------------------------------------------------ launchers
static int cluster_size(int64_t rows, int K, int log2b) {
    const int ub = std::max(1 << log2b, 8);
    const int nu = K / ub;
    const int64_t target = 2LL * sm_count();
    int c = (int)std::min<int64_t>(kMaxCluster, std::max<int64_t>(1, (target + rows - 1) / rows));
    return std::max(1, std::min(c, nu));
}

static size_t part_smem(int K, int log2b, int cs) {
    const int ub = std::max(1 << log2b, 8);
    const int nu = K / ub;
    return (size_t)((nu + cs - 1) / cs) * ub * sizeof(double);
}

template <class Kern, class... Args>
static cudaError_t launch_clustered(Kern kern, int64_t rows, int cs, size_t smem,
                                    cudaStream_t st, Args... args) {
    count_launch();
    return launch_pdl(kern, dim3((unsigned)(rows * cs)), dim3(kRqThreads), smem, st, cs, args...);
}

cudaError_t launch_rotate_quantize(const void *x, int64_t ldx, int64_t M, int K, int log2b,
                                   int bits, void *q, int64_t ldq, float *s, cudaStream_t st,
                                   const void *scale, const int32_t *perm, const RqF16 *f16) {
    const __half *sc = reinterpret_cast<const __half *>(scale);
    if (M == 0) return cudaSuccess;
    TimedScope ts(st, CQ_KERNEL_ROTATE_QUANTIZE);
    if (use_reg_rows(M, K, log2b, bits, x, ldx, q, ldq)) {
        const int K32 = K / 32;
        const int rows_per_cta = std::max(1, kRegThreads / K32);
        const int threads = (rows_per_cta * K32 + 31) / 32 * 32;
        const size_t smem = (size_t)threads * sizeof(double) * (log2b > 10 ? 33 : 1);
        const int64_t n_groups = (M + rows_per_cta - 1) / rows_per_cta;
        auto kern = log2b > 10 ? k_rq_x_reg<true, true>
                  : log2b >= 5 ? k_rq_x_reg<false, true> : k_rq_x_reg<false, false>;
        // persistent: as many CTAs as are resident at once, each looping
        const int grid = (int)std::min<int64_t>(
            n_groups, (int64_t)sm_count() * resident_ctas((const void *)kern, threads, smem));
        count_launch();
        return launch_pdl(kern, dim3((unsigned)grid),
                          dim3(threads), smem, st, 1,
                          reinterpret_cast<const __half *>(x), ldx, M, K, log2b, bits,
                          reinterpret_cast<uint8_t *>(q), ldq, s, sc, perm, rows_per_cta,
                          (int)n_groups, f16 ? *f16 : RqF16{});
    }
    const RqF16 f{f16 ? *f16 : RqF16{}};
    if (use_warp_rows(M, K, log2b)) {
        const size_t smem = (size_t)kWarpRows * K * sizeof(double);
        count_launch();
        return launch_pdl(k_rq_x_warp, dim3((unsigned)((M + kWarpRows - 1) / kWarpRows)),
                          dim3(kWarpRows * 32), smem, st, 1, reinterpret_cast<const __half *>(x),
                          ldx, M, K, log2b, bits, reinterpret_cast<uint8_t *>(q), ldq, s, sc,
                          perm, f);
    }
    const int cs = cluster_size(M, K, log2b);
    auto kern = cs == 1 ? k_rq_x<false> : k_rq_x<true>;
    return launch_clustered(kern, M, cs, part_smem(K, log2b, cs), st,
                            reinterpret_cast<const __half *>(x), ldx, K, log2b, bits,
                            reinterpret_cast<uint8_t *>(q), ldq, s, sc, perm, f);
}

cudaError_t launch_swiglu_rq(const SwigluArgs &a, int64_t rows, cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    TimedScope ts(st, CQ_KERNEL_ROTATE_QUANTIZE);
    const bool warp_r = a.R_routed == 0 || use_warp_rows(rows, a.I, a.log2b_i);
    const bool warp_s = a.R_shared == 0 || use_warp_rows(rows, a.I_shared, a.log2b_i_shared);
    if (warp_r && warp_s) {
        const size_t smem = (size_t)kWarpRows * a.Imax * sizeof(double);
        count_launch();
        return launch_pdl(k_rq_swiglu_warp, dim3((unsigned)((rows + kWarpRows - 1) / kWarpRows)),
                          dim3(kWarpRows * 32), smem, st, 1, a, rows);
    }
    // one cluster size for the launch: the coarser of the two row kinds
    int cs = kMaxCluster;
    size_t smem = 0;
    if (a.R_routed > 0) cs = std::min(cs, cluster_size(rows, a.I, a.log2b_i));
    if (a.R_shared > 0) cs = std::min(cs, cluster_size(rows, a.I_shared, a.log2b_i_shared));
    if (a.R_routed > 0) smem = std::max(smem, part_smem(a.I, a.log2b_i, cs));
    if (a.R_shared > 0) smem = std::max(smem, part_smem(a.I_shared, a.log2b_i_shared, cs));
    auto kern = cs == 1 ? k_rq_swiglu<false> : k_rq_swiglu<true>;
    return launch_clustered(kern, rows, cs, smem, st, a);
}

}  // namespace cq
