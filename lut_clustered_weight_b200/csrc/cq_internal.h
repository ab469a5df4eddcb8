// cq_internal.h -- launchers shared between the .cu files of the library.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace cq {

// ---------------------------------------------------------------- rotate + quantize
constexpr int kMaxK = 16384;

// x fp16 rows with stride ldx (elements); one CTA per row.
cudaError_t launch_rotate_quantize(const void *x, int64_t ldx, int64_t M, int K, int log2b,
                                   int bits, void *q, int64_t ldq_bytes, float *s,
                                   cudaStream_t st);

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
};

struct LutPlan {
    int nt;             // n8 token tiles per CTA (1 or 2)
    int n_row_tiles;    // CTA row tiles
    int chunks_total;   // ceil(K / 128)
    int chunks_per_split;
    int splits;
    size_t smem;
};

LutPlan plan_lut(int N, int K, bool dual, int max_rows_per_group, int64_t est_tiles);
cudaError_t launch_lut(const LutLaunch &L, const LutPlan &P, cudaStream_t st);

// y[m, n] = s[m] * sum_s part[s][m][n]
cudaError_t launch_reduce_plain(const float *part, int splits, int64_t M, int64_t N,
                                const float *s, float *y, cudaStream_t st);

cudaError_t launch_centroid_sums(const void *q, int64_t M, int64_t K, int bits,
                                 const uint8_t *w_idx, int64_t N, int32_t *S, cudaStream_t st);

// ---------------------------------------------------------------- MoE pieces
int sm_count();

// ---------------------------------------------------------------- measurement aids
void count_launch(int n = 1);
bool timing_on();
void timing_begin(cudaStream_t st);
void timing_end(cudaStream_t st);

}  // namespace cq
