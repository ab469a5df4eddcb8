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

// Rotate buf[0, n) (complete blocks), reduce the absmax over the cluster,
// quantize and store this CTA's codes; rank 0 stores the scale.
CQ_DEV void rq_finish(double *buf, RowPart part, int K, int log2b, int bits, uint8_t *qrow,
                      float *s_out) {
    __shared__ double red[33];
    __shared__ double s_amax;
    cg::cluster_group cluster = cg::this_cluster();
    block_fwht<kRqThreads>(buf, part.n, log2b);
    const double a_loc = block_absmax<kRqThreads>(buf, part.n, red);
    if (threadIdx.x == 0) s_amax = a_loc;
    cluster.sync();
    double A = 0.0;
    const int cs = (int)cluster.num_blocks();
    for (int r = 0; r < cs; r++) A = fmax(A, *cluster.map_shared_rank(&s_amax, r));
    cluster.sync();  // every CTA has read every s_amax
    block_quantize_range<kRqThreads>(buf, part.n, part.e0, bits, A, qrow);
    if (cluster.block_rank() == 0 && threadIdx.x == 0) {
        const int qmax = (1 << (bits - 1)) - 1;
        *s_out = A > 0.0 ? quant_scale(A, log2b, qmax) : 0.0f;
    }
    (void)K;
}

// ------------------------------------------------------------------ x rows
__global__ void __launch_bounds__(kRqThreads)
k_rq_x(const __half *__restrict__ x, int64_t ldx, int K, int log2b, int bits,
       uint8_t *__restrict__ q, int64_t ldq, float *__restrict__ s) {
    extern __shared__ __align__(16) double buf[];
    cg::cluster_group cluster = cg::this_cluster();
    const int cs = (int)cluster.num_blocks(), rank = (int)cluster.block_rank();
    const int64_t m = blockIdx.x / cs;
    const RowPart part = row_part(K, log2b, rank, cs);
    const __half *xr = x + m * ldx + part.e0;
    for (int i = threadIdx.x; i < part.n / 8; i += kRqThreads) {
        const uint4 v = *reinterpret_cast<const uint4 *>(xr + 8 * i);
        const __half2 *h = reinterpret_cast<const __half2 *>(&v);
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const float2 f = __half22float2(h[j]);
            buf[8 * i + 2 * j] = (double)f.x;
            buf[8 * i + 2 * j + 1] = (double)f.y;
        }
    }
    __syncthreads();
    rq_finish(buf, part, K, log2b, bits, q + m * ldq, s + m);
}

// ------------------------------------------------------------------ SwiGLU rows
// Row p of the intermediate: g, u = sum of the split-K partials, scaled by the
// token's s_x; h = fp16(silu(g) * u) (round to nearest even); then as above.
__global__ void __launch_bounds__(kRqThreads) k_rq_swiglu(const SwigluArgs a) {
    extern __shared__ __align__(16) double buf[];
    cg::cluster_group cluster = cg::this_cluster();
    const int cs = (int)cluster.num_blocks(), rank = (int)cluster.block_rank();
    const int64_t p = blockIdx.x / cs;
    const bool routed = p < a.R_routed;
    const int I = routed ? a.I : a.I_shared;
    const int log2b = routed ? a.log2b_i : a.log2b_i_shared;
    const float *part = routed ? a.part_r : a.part_s;
    const LutPlan &P = routed ? a.plan_r : a.plan_s;
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
    for (int i = threadIdx.x; i < rp.n; i += kRqThreads) {
        const int n = rp.e0 + i;
        float g = 0.0f, u = 0.0f;
        const int splits = s_ns[n / P.rows_per_rt - rt0];
        for (int sp = 0; sp < splits; sp++) {
            const float2 v = *reinterpret_cast<const float2 *>(
                part + ((int64_t)sp * rows + lp) * (2 * (int64_t)I) + 2 * n);
            g += v.x;
            u += v.y;
        }
        g *= sx;
        u *= sx;
        const __half h = __float2half_rn(silu_mul(g, u));
        if (a.h_dbg) reinterpret_cast<__half *>(a.h_dbg)[p * a.Imax + n] = h;
        buf[i] = (double)__half2float(h);
    }
    __syncthreads();
    rq_finish(buf, rp, I, log2b, a.bits, a.hq + p * a.ldhq, a.h_scales + p);
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
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)(kMaxK * sizeof(double)));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(rows * cs));
    cfg.blockDim = dim3(kRqThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    count_launch();
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

cudaError_t launch_rotate_quantize(const void *x, int64_t ldx, int64_t M, int K, int log2b,
                                   int bits, void *q, int64_t ldq, float *s, cudaStream_t st) {
    if (M == 0) return cudaSuccess;
    const int cs = cluster_size(M, K, log2b);
    return launch_clustered(k_rq_x, M, cs, part_smem(K, log2b, cs), st,
                            reinterpret_cast<const __half *>(x), ldx, K, log2b, bits,
                            reinterpret_cast<uint8_t *>(q), ldq, s);
}

cudaError_t launch_swiglu_rq(const SwigluArgs &a, int64_t rows, cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    // one cluster size for the launch: the coarser of the two row kinds
    int cs = kMaxCluster;
    size_t smem = 0;
    if (a.R_routed > 0) cs = std::min(cs, cluster_size(rows, a.I, a.log2b_i));
    if (a.R_shared > 0) cs = std::min(cs, cluster_size(rows, a.I_shared, a.log2b_i_shared));
    if (a.R_routed > 0) smem = std::max(smem, part_smem(a.I, a.log2b_i, cs));
    if (a.R_shared > 0) smem = std::max(smem, part_smem(a.I_shared, a.log2b_i_shared, cs));
    return launch_clustered(k_rq_swiglu, rows, cs, smem, st, a);
}

}  // namespace cq
