// cq_internal.h -- launchers shared between the .cu files of the library.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/cq.h"

namespace cq {

// ---------------------------------------------------------------- rotate + quantize
constexpr int kMaxK = 16384;

// x fp16 rows with stride ldx (elements); one CTA per row.  scale (fp16 [K])
// and perm (int32 [K]) are optional: row element j is fp16(x[perm[j]] *
// scale[perm[j]]) before the rotation.  f16 (optional): fp16 copies of the
// codes as well (see RqF16); only when rq_writes_f16 holds for the same
// arguments, else the call returns cudaErrorNotSupported.
struct RqF16;
cudaError_t launch_rotate_quantize(const void *x, int64_t ldx, int64_t M, int K, int log2b,
                                   int bits, void *q, int64_t ldq_bytes, float *s,
                                   cudaStream_t st, const void *scale = nullptr,
                                   const int32_t *perm = nullptr, const RqF16 *f16 = nullptr);
// fp16 copies of the code rows (the B operand of the tensor-core GEMMs),
// written by every rotate-quantize kernel itself: copy d (d < ncopy) of row m
// goes to rows[map[m * ncopy + d]] (rows[m] when map is NULL), with the row's
// scale at row_scales[that row] when row_scales is non-NULL; ident, when
// non-NULL, receives one more copy at row m.  Rows of K halves.
struct RqF16 {
    __half *rows = nullptr;
    const int32_t *map = nullptr;
    int ncopy = 0;
    float *row_scales = nullptr;
    __half *ident = nullptr;
};

// ---------------------------------------------------------------- LUT GEMM
// Token-row -> code-row mapping used by the grouped GEMM.
enum MapMode : int { kMapIdentity = 0, kMapPerm = 1, kMapModT = 2 };

struct LutLaunch {
    // activation codes
    const uint8_t *codes;   // row r at codes + r * ld_codes
    int64_t ld_codes;       // bytes
    const float *scales;    // per code row (direct epilogue only)
    int act_bits;
    int K;
    int map_mode;           // MapMode
    const int32_t *perm;    // kMapPerm: code row = perm[p] / topk
    int topk;
    int T;                  // kMapModT: code row = p % T
    // groups of rows (rows are relative to this launch)
    int G;
    int uniform_rows;       // > 0: group g = rows [g*u, (g+1)*u); else device arrays
    const int32_t *grp_rows;   // [G+1]
    const int32_t *grp_tiles;  // [G+1] prefix of ceil(rows_g / (8 * plan.nt))
    const int32_t *tile_grp;   // [max_tiles] group of each token tile (below grp_tiles[G])
    int max_tiles;             // grid.y (upper bound on the tile count)
    // weights: expert g of matrix j at idx[j] + g*w_stride, cb[j] + g*cb_stride
    const uint8_t *idx0;
    const void *cb0;
    const uint8_t *idx1;    // dual (gate/up) launches only
    const void *cb1;
    int64_t w_stride;       // bytes
    int64_t cb_stride;      // fp16 elements
    int N;                  // rows per matrix
    bool dual;
    // output
    float *out;             // plain: [splits][rows][N]; dual: [splits][rows][N][2]
    int64_t out_split_stride;  // floats
    int64_t out_row_stride;    // floats
    bool direct;            // plain, splits == 1: out[r*N+n] = scale * acc
    // dual tensor-core launches with one partial slot only: instead of the
    // partials, h[p, n] = fp16(silu(s * g) * (s * u)) with s = scales[code
    // row of p], written at h_out + p * h_row_stride + n
    __half *h_out;
    int64_t h_row_stride;   // elements
    const float *row_scales;  // fused, kMapPerm: scale of output row p, gathered
};

// How one LUT GEMM launch is cut into work.  A work item is (token tile,
// row tile); its contraction is cut into chunks (128 k for the mma.sync
// kernel, 64 k for the tensor-memory kernel), and the units (work item,
// chunk) are shared out in one of two ways:
//   fixed    every work item is split into `splits` equal chunk ranges.  The
//            mma.sync kernel's grid is (row tiles * splits) x (token tiles);
//            the tensor-memory kernel runs one CTA per SM that strides over
//            the (item, split) pieces.  Used when the token tiles are only
//            known on the device (routed experts), and by the tensor-memory
//            kernel whenever there are many work items.
//   stream-K the W*C units of all work items are dealt out in equal
//            contiguous ranges to `grid` CTAs (one wave), so no SM waits on
//            a tail.  A work item is then covered by a variable number of
//            CTAs; its partial sums occupy slots 0..n-1.
struct LutPlan {
    int nt;             // n8 token tiles per CTA (1 or 2): a token tile has 8*nt rows
    int warps;          // mma.sync kernel: warps per CTA (4 or 8)
    int rows_per_rt;    // plain: weight rows per row tile; dual: output columns
    int n_row_tiles;
    int chunks_total;   // C = ceil(K / chunk)
    int cps_max;        // most chunks one CTA stages at a time (shared memory)
    int streamk;
    int grid;           // CTAs (x dimension)
    int splits;         // fixed: chunk ranges per work item; partial slots allocated
    int chunks_per_split;
    int64_t units;      // stream-K: total units (work items * C)
    int uniform_rows;   // rows per group of a uniform launch (token tiles of a group are consecutive)
    int tc;             // 0: mma.sync kernel; 1: tensor-memory kernel (wide token
                        // tiles); 2: tensor-memory decode kernel (64-k chunks, 128-row tiles)
    size_t smem;
};

// Number of CTAs (partial slots) that cover work item w.
__host__ __device__ inline int lut_item_splits(const LutPlan &P, int64_t w) {
    if (!P.streamk) return P.splits;
    const int64_t C = P.chunks_total, G = P.grid, U = P.units;
    const int64_t cf = ((w * C + 1) * G - 1) / U;
    const int64_t cl = (((w + 1) * C) * G - 1) / U;
    return (int)(cl - cf + 1);
}
// CTA whose unit range contains unit u (stream-K).
__host__ __device__ inline int64_t lut_cta_of_unit(const LutPlan &P, int64_t u) {
    return ((u + 1) * (int64_t)P.grid - 1) / P.units;
}
// Work item holding output row p (relative to the launch) and column n
// (stream-K launches, whose groups are uniform).
__host__ __device__ inline int64_t lut_item_of(const LutPlan &P, int64_t p, int n) {
    const int tt = 8 * P.nt;
    const int64_t tpg = (P.uniform_rows + tt - 1) / tt;
    const int64_t g = p / P.uniform_rows;
    const int64_t tile = g * tpg + (p - g * P.uniform_rows) / tt;
    return tile * P.n_row_tiles + n / P.rows_per_rt;
}
// Partial-slot count for output (row p, column n) of a launch.
__host__ __device__ inline int lut_splits_at(const LutPlan &P, int64_t p, int n) {
    return P.streamk ? lut_item_splits(P, lut_item_of(P, p, n)) : P.splits;
}

// uniform_rows > 0: the launch has n_groups groups of uniform_rows rows each
// (dense / shared experts) and may use stream-K; otherwise the groups come
// from device arrays and est_tiles estimates the token tiles.
LutPlan plan_lut(int N, int K, bool dual, int max_rows_per_group, int64_t est_tiles,
                 int uniform_rows = 0, int n_groups = 1);
cudaError_t launch_lut(const LutLaunch &L, const LutPlan &P, cudaStream_t st);

// The LUT GEMM kernels and which one serves a launch.
enum LutKernel : int { kKernMma = 0, kKernTc = 1, kKernTs = 2 };
constexpr int kTcTileRows = 128;  // weight rows per tensor-memory tile
// tiles_bound: an upper bound on the token tiles of the launch; routed: the
// groups are routed experts (token tiles known on the device only).
LutKernel pick_kernel(int64_t rows, int64_t N, bool dual, int64_t K, int64_t tiles_bound,
                      bool routed);

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// A planned cq_lut_gemm call: the launch plan, the token tiles, the scratch
// it needs (split-K partial sums, then for the wide-tile kernel fp16 codes at
// b_off) and its launches.  Shared by the workspace and no-allocation entry
// points, so both run exactly the same kernels with the same partition.
struct LutGemmPlan {
    LutPlan p;
    int tiles;
    size_t ws;
    size_t b_off;
};
LutGemmPlan plan_gemm(int64_t M, int64_t N, int64_t K);
cudaError_t run_lut_gemm(const LutGemmPlan &g, const void *q, const float *s_x, int64_t M,
                         int64_t K, int act_bits, const uint8_t *w_idx, const void *codebook,
                         int64_t N, float *y, void *scratch, cudaStream_t st);

// Tensor-memory (tcgen05) LUT GEMM.  The activations are read as fp16 rows
// b_f16 [b_rows][K]; the GEMM row p of a token tile maps to B row
// (b_row_mod > 0 ? p % b_row_mod : p).
int tc_ntok_for(int max_rows_per_group);
LutPlan plan_lut_tc(int N, int K, bool dual, int max_rows_per_group, int64_t est_tiles,
                    int uniform_rows = 0, int n_groups = 1);
cudaError_t launch_lut_tc(const LutLaunch &L, const LutPlan &P, const void *b_f16, int64_t b_rows,
                          int b_row_mod, cudaStream_t st);
// Tensor-memory decode kernel (groups of at most 32 rows): thread-per-row pair
// tables, index bytes by TMA.  The activations are read like the wide-tile
// kernel's: fp16 rows b_f16 [b_rows][K], GEMM row p of a token tile at B row
// (b_row_mod > 0 ? p % b_row_mod : p).
int ts_ntok_for(int max_rows_per_group);
LutPlan plan_lut_ts(int N, int K, bool dual, int max_rows_per_group, int64_t est_tiles,
                    int uniform_rows = 0, int n_groups = 1);
cudaError_t launch_lut_ts(const LutLaunch &L, const LutPlan &P, const void *b_f16,
                          int64_t b_rows, int b_row_mod, cudaStream_t st);
// fp16 copies of activation codes (B operand), rows mapped like LutLaunch::map_mode.
// scales_in != nullptr: also writes scales_out[p] = scales_in[code row of p].
cudaError_t launch_codes_to_f16(const void *codes, int64_t ld_codes, int bits, int K,
                                int64_t rows, int map_mode, const int32_t *perm, int topk, int T,
                                void *out, cudaStream_t st, const float *scales_in = nullptr,
                                float *scales_out = nullptr);
// Launches the bounded-wait self-test kernel (sets the device error word).
cudaError_t launch_selftest_wait(cudaStream_t st);
// Reads and clears the device error word (-1 if the read failed).
int read_device_error();
// Which LUT kernel a launch uses: "mma" (mma.sync, register tables), "tc"
// (tcgen05 / tensor memory), or automatic (default).
enum LutPath : int { kPathAuto = 0, kPathMma = 1, kPathTc = 2, kPathTs = 3 };
LutPath lut_path();

// LUT GEMM with 3- or 5-bit indices (8 or 32 centroids per row), uniform
// token rows (identity map): plan and launch; partial sums as launch_lut.
LutPlan plan_lut_vb(int M, int N, int K, int idx_bits);
cudaError_t launch_lut_vb(const LutLaunch &L, const LutPlan &P, int idx_bits, cudaStream_t st);

// y[m, n] = s[m] * sum_{s < n(m, n)} part[s][m][n]
cudaError_t launch_reduce_plain(const float *part, const LutPlan &P, int64_t M, int64_t N,
                                const float *s, float *y, cudaStream_t st);

cudaError_t launch_centroid_sums(const void *q, int64_t M, int64_t K, int bits,
                                 const uint8_t *w_idx, int64_t N, int32_t *S, cudaStream_t st);

// ---------------------------------------------------------------- MoE pieces
int sm_count();

// ---------------------------------------------------------------- measurement aids
void count_launch(int n = 1);
bool timing_on();       // LUT GEMM launches are timed
bool timing_on_all();   // every launch is timed
void timing_begin(cudaStream_t st, int kind);  // kind: CQ_KERNEL_*
void timing_end(cudaStream_t st);
// Brackets the launches of its scope with timing events when every launch is timed.
struct TimedScope {
    cudaStream_t st;
    bool on;
    TimedScope(cudaStream_t s, int kind) : st(s), on(timing_on_all()) {
        if (on) timing_begin(st, kind);
    }
    ~TimedScope() {
        if (on) timing_end(st);
    }
    TimedScope(const TimedScope &) = delete;
    TimedScope &operator=(const TimedScope &) = delete;
};

}  // namespace cq
