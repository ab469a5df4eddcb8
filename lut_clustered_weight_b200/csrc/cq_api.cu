// cq_api.cu -- extern "C" entry points: argument checks, planning, launches.
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "../../include/cq.h"
#include "cq_internal.h"
#include "cq_moe.h"

using namespace cq;

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool is_pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }
int ilog2(int64_t v) {
    int l = 0;
    while ((int64_t(1) << l) < v) l++;
    return l;
}
cq_status cuda_status(cudaError_t e) { return e == cudaSuccess ? CQ_OK : CQ_ERR_CUDA; }
int64_t code_bytes(int64_t K, int bits) { return bits == 4 ? K / 2 : K; }

// ------------------------------------------------------------------ LUT GEMM plan
// (plan_gemm / run_lut_gemm are shared with the no-allocation entry point)

}  // namespace

namespace cq {

// Which LUT GEMM kernel serves groups of `rows` typical rows: the tensor-memory
// kernels need whole 128-row weight tiles (64 output columns for gate||up).
// Measured on B200: uniform launches of at most 16 rows (dense decode) are as
// fast on mma.sync and need no fp16 copy of the activations; routed groups of
// at most 32 rows (MoE decode) are faster on the tensor-memory decode kernel;
// wider groups run on the wide-token-tile kernel.
LutKernel pick_kernel(int64_t rows, int64_t N, bool dual, int64_t K, int64_t tiles_bound,
                      bool routed) {
    if (dual ? N % 64 : N % kTcTileRows) return kKernMma;
    // the tensor-memory kernels count their work in 32 bits
    const int64_t units = tiles_bound * (N / (dual ? 64 : kTcTileRows)) * ((K + 63) / 64);
    if (units * sm_count() >= (int64_t(1) << 31)) return kKernMma;
    switch (lut_path()) {
    case kPathMma: return kKernMma;
    case kPathTc: return kKernTc;
    case kPathTs: return kKernTs;  // groups over 32 rows: several 32-token tiles
    default: break;
    }
    if (rows <= 16 && !routed) return kKernMma;
    return rows <= 32 ? kKernTs : kKernTc;
}

LutGemmPlan plan_gemm(int64_t M, int64_t N, int64_t K) {
    LutGemmPlan g{};
    const LutKernel k = pick_kernel(M, N, false, K, (M + 15) / 16, false);
    if (k == kKernTs) {
        const int ntok = ts_ntok_for((int)M);
        g.tiles = (int)((M + ntok - 1) / ntok);
        g.p = plan_lut_ts((int)N, (int)K, false, (int)M, g.tiles, (int)M, 1);
        g.b_off = align256((size_t)g.p.splits * M * N * sizeof(float));
        g.ws = g.b_off + align256((size_t)M * K * 2);
        return g;
    }
    if (k == kKernTc) {
        const int mr = (int)std::min<int64_t>(M, 256);
        const int ntok = tc_ntok_for(mr);
        g.tiles = (int)((M + ntok - 1) / ntok);
        g.p = plan_lut_tc((int)N, (int)K, false, mr, g.tiles, (int)M, 1);
        g.b_off = align256((size_t)g.p.splits * M * N * sizeof(float));
        g.ws = g.b_off + align256((size_t)M * K * 2);
        return g;
    }
    const int nt = M <= 8 ? 1 : 2;
    g.tiles = (int)((M + 8 * nt - 1) / (8 * nt));
    g.p = plan_lut((int)N, (int)K, false, (int)std::min<int64_t>(M, 16), g.tiles, (int)M, 1);
    g.ws = align256((size_t)g.p.splits * M * N * sizeof(float));
    g.b_off = 0;
    return g;
}

cudaError_t run_lut_gemm(const LutGemmPlan &g, const void *q, const float *s_x, int64_t M,
                         int64_t K, int act_bits, const uint8_t *w_idx, const void *codebook,
                         int64_t N, float *y, void *scratch, cudaStream_t st) {
    LutLaunch L{};
    L.codes = reinterpret_cast<const uint8_t *>(q);
    L.ld_codes = act_bits == 4 ? K / 2 : K;
    L.scales = s_x;
    L.act_bits = act_bits;
    L.K = (int)K;
    L.map_mode = kMapIdentity;
    L.G = 1;
    L.uniform_rows = (int)M;
    L.max_tiles = g.tiles;
    L.idx0 = w_idx;
    L.cb0 = codebook;
    L.w_stride = 0;
    L.cb_stride = 0;
    L.N = (int)N;
    L.dual = false;
    L.out_row_stride = N;
    L.direct = false;
    L.out = reinterpret_cast<float *>(scratch);
    L.out_split_stride = M * N;
    cudaError_t e;
    if (g.p.tc != 0) {
        // tensor-memory kernels read the activations as fp16 rows
        void *b = reinterpret_cast<uint8_t *>(scratch) + g.b_off;
        e = launch_codes_to_f16(q, L.ld_codes, act_bits, (int)K, M, kMapIdentity, nullptr, 1, 1,
                                b, st);
        if (e == cudaSuccess)
            e = g.p.tc == 2 ? launch_lut_ts(L, g.p, b, M, 0, st) : launch_lut_tc(L, g.p, b, M, 0, st);
    } else {
        e = launch_lut(L, g.p, st);
    }
    if (e == cudaSuccess) e = launch_reduce_plain(L.out, g.p, M, N, s_x, y, st);
    return e;
}

}  // namespace cq

namespace {

// ------------------------------------------------------------------ MoE plan
struct MoePlan {
    int64_t T, H, I, E, k, ns, Is, Rr, Rs, R;
    int bits, Imax, nt, tile_rows, max_tiles_r, tiles_s, tile_rows_s;
    LutKernel k_r, k_s;                 // kernel of the routed / shared launches
    bool fused;                         // gate/up launches write h (SwiGLU in their epilogue)
    LutPlan gu_r, gu_s, dn_r, dn_s;
    size_t o_xq, o_sx, o_ids, o_w, o_counts, o_offsets, o_perm, o_inv, o_tiles, o_tgrp, o_chist;
    size_t o_pgu_r, o_pgu_s, o_hq, o_sh, o_pdn_r, o_pdn_s;
    size_t o_bx_r, o_bx_s, o_bh_r, o_bh_s;  // fp16 B operands of tensor-core launches
    size_t o_hf;                            // fused: h fp16 [R][Imax]
    size_t o_rs;                            // fused: x scale per routed row [Rr]
    size_t total;
};

MoePlan plan_moe(const cq_moe_desc *d, int64_t T) {
    MoePlan m{};
    m.T = T;
    m.H = d->H;
    m.I = d->I;
    m.E = d->E;
    m.k = d->E > 0 ? d->top_k : 0;
    m.ns = d->n_shared;
    m.Is = d->n_shared > 0 ? d->I_shared : 0;
    m.Rr = T * m.k;
    m.Rs = m.ns * T;
    m.R = m.Rr + m.Rs;
    m.bits = d->act_bits;
    m.Imax = (int)std::max<int64_t>(m.E > 0 ? m.I : 0, m.Is);
    m.nt = T <= 8 ? 1 : 2;
    // routed experts: typical rows per expert decide the kernel and tile size;
    // gate||up and down share one token tiling per group (the routing tables)
    const int64_t avg_r = m.E > 0 ? (m.Rr + m.E - 1) / m.E : 0;
    const int rows_r = (int)std::min<int64_t>(T, std::max<int64_t>(2 * avg_r, 1));
    if (m.E > 0) {
        const int64_t tb = m.Rr / 16 + m.E;
        m.k_r = pick_kernel(rows_r, m.I, true, m.H, tb, true);
        if (pick_kernel(rows_r, m.H, false, m.I, tb, true) != m.k_r) m.k_r = kKernMma;
    }
    m.tile_rows = m.k_r == kKernTs ? ts_ntok_for(rows_r)
                : m.k_r == kKernTc ? tc_ntok_for(rows_r) : 8 * m.nt;
    const int64_t nonempty = std::min<int64_t>(m.E, m.Rr);
    m.max_tiles_r = (int)(m.Rr / m.tile_rows + nonempty);
    // shared experts: every token
    const int rows_s = (int)std::min<int64_t>(T, 256);
    if (m.ns > 0) {
        const int64_t tb = m.ns * ((T + 15) / 16);
        m.k_s = pick_kernel(rows_s, m.Is, true, m.H, tb, false);
        if (pick_kernel(rows_s, m.H, false, m.Is, tb, false) != m.k_s) m.k_s = kKernMma;
    }
    m.tile_rows_s = m.k_s == kKernTs ? ts_ntok_for(rows_s)
                  : m.k_s == kKernTc ? tc_ntok_for(rows_s) : 8 * m.nt;
    m.tiles_s = (int)(m.ns * ((T + m.tile_rows_s - 1) / m.tile_rows_s));
    const int rows_per_group = (int)std::min<int64_t>(T, 16);
    auto plan_for = [&](LutKernel k, int N, int K, bool dual, int tile_rows, int64_t tiles,
                        int uniform_rows, int n_groups) {
        if (k == kKernTs) return plan_lut_ts(N, K, dual, tile_rows, tiles, uniform_rows, n_groups);
        if (k == kKernTc) return plan_lut_tc(N, K, dual, tile_rows, tiles, uniform_rows, n_groups);
        return plan_lut(N, K, dual, rows_per_group, tiles, uniform_rows, n_groups);
    };
    if (m.E > 0) {
        m.gu_r = plan_for(m.k_r, (int)m.I, (int)m.H, true, m.tile_rows, m.max_tiles_r, 0, 1);
        m.dn_r = plan_for(m.k_r, (int)m.H, (int)m.I, false, m.tile_rows, m.max_tiles_r, 0, 1);
    }
    if (m.ns > 0) {
        m.gu_s = plan_for(m.k_s, (int)m.Is, (int)m.H, true, m.tile_rows_s, m.tiles_s, (int)T,
                          (int)m.ns);
        m.dn_s = plan_for(m.k_s, (int)m.H, (int)m.Is, false, m.tile_rows_s, m.tiles_s, (int)T,
                          (int)m.ns);
    }
    // SwiGLU moves into the gate/up epilogue when every gate/up launch runs on
    // the tensor-core kernel with a single partial slot per output
    m.fused = (m.E == 0 || (m.k_r == kKernTc && !m.gu_r.streamk && m.gu_r.splits == 1)) &&
              (m.ns == 0 || (m.k_s == kKernTc && !m.gu_s.streamk && m.gu_s.splits == 1));
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o += align256(bytes);
        return at;
    };
    m.o_xq = take((size_t)T * code_bytes(m.H, m.bits));
    m.o_sx = take((size_t)T * 4);
    m.o_ids = take((size_t)m.Rr * 4);
    m.o_w = take((size_t)m.Rr * 4);
    m.o_counts = take((size_t)m.E * 4);
    m.o_offsets = take((size_t)(m.E + 1) * 4);
    m.o_perm = take((size_t)m.Rr * 4);
    m.o_inv = take((size_t)m.Rr * 4);
    m.o_tiles = take((size_t)(m.E + 1) * 4);
    m.o_tgrp = take((size_t)m.max_tiles_r * 4);
    m.o_chist = take(m.E > 0 ? route_scratch_bytes((int)T, (int)m.E, (int)m.k) : 0);
    m.o_pgu_r = take(m.E > 0 && !m.fused ? (size_t)m.gu_r.splits * m.Rr * m.I * 2 * 4 : 0);
    m.o_pgu_s = take(m.ns > 0 && !m.fused ? (size_t)m.gu_s.splits * m.Rs * m.Is * 2 * 4 : 0);
    m.o_hf = take(m.fused ? (size_t)m.R * m.Imax * 2 : 0);
    m.o_rs = take(m.fused && m.E > 0 ? (size_t)m.Rr * 4 : 0);
    m.o_hq = take((size_t)m.R * code_bytes(m.Imax, m.bits));
    m.o_sh = take((size_t)m.R * 4);
    m.o_pdn_r = take(m.E > 0 ? (size_t)m.dn_r.splits * m.Rr * m.H * 4 : 0);
    m.o_pdn_s = take(m.ns > 0 ? (size_t)m.dn_s.splits * m.Rs * m.H * 4 : 0);
    const bool wide_r = m.k_r != kKernMma, wide_s = m.k_s != kKernMma;  // fp16 B rows
    m.o_bx_r = take(wide_r ? (size_t)m.Rr * m.H * 2 : 0);
    m.o_bx_s = take(wide_s ? (size_t)T * m.H * 2 : 0);
    m.o_bh_r = take(wide_r ? (size_t)m.Rr * m.I * 2 : 0);
    m.o_bh_s = take(wide_s ? (size_t)m.Rs * m.Is * 2 : 0);
    m.total = o;
    return m;
}

cq_status check_moe_desc(const cq_moe_desc *d, int64_t T) {
    if (!d || T < 0) return CQ_ERR_INVALID_ARGUMENT;
    if (d->act_bits != 4 && d->act_bits != 8) return CQ_ERR_INVALID_ARGUMENT;
    if (d->H <= 0 || d->E < 0 || d->n_shared < 0) return CQ_ERR_INVALID_ARGUMENT;
    if (d->E == 0 && d->n_shared == 0) return CQ_ERR_INVALID_ARGUMENT;
    if (d->E > 0) {
        if (d->I <= 0 || d->top_k < 1 || d->top_k > d->E) return CQ_ERR_INVALID_ARGUMENT;
        if (!is_pow2(d->had_block_i) || d->I % d->had_block_i) return CQ_ERR_INVALID_ARGUMENT;
        if (d->E > kMaxExperts || d->top_k > kMaxTopK) return CQ_ERR_UNSUPPORTED;
        if (d->I % 64 || d->I > kMaxK || d->had_block_i > 8192) return CQ_ERR_UNSUPPORTED;
    } else if (d->top_k != 0) {
        return CQ_ERR_INVALID_ARGUMENT;
    }
    if (d->n_shared > 4) return CQ_ERR_UNSUPPORTED;
    if (d->n_shared > 0) {
        if (d->I_shared <= 0) return CQ_ERR_INVALID_ARGUMENT;
        if (!is_pow2(d->had_block_i_shared) || d->I_shared % d->had_block_i_shared)
            return CQ_ERR_INVALID_ARGUMENT;
        if (d->I_shared % 64 || d->I_shared > kMaxK || d->had_block_i_shared > 8192)
            return CQ_ERR_UNSUPPORTED;
    }
    if (!is_pow2(d->had_block_h) || d->H % d->had_block_h) return CQ_ERR_INVALID_ARGUMENT;
    if (d->H % 64 || d->H > kMaxK || d->had_block_h > 8192) return CQ_ERR_UNSUPPORTED;
    if (d->renormalize != 0 && d->renormalize != 1) return CQ_ERR_INVALID_ARGUMENT;
    if ((int64_t)T * std::max<int64_t>(d->top_k, 1) > (int64_t(1) << 30)) return CQ_ERR_UNSUPPORTED;
    return CQ_OK;
}

}  // namespace

extern "C" {

const char *cq_status_string(cq_status s) {
    switch (s) {
    case CQ_OK: return "CQ_OK";
    case CQ_ERR_INVALID_ARGUMENT: return "CQ_ERR_INVALID_ARGUMENT";
    case CQ_ERR_UNSUPPORTED: return "CQ_ERR_UNSUPPORTED";
    case CQ_ERR_WORKSPACE: return "CQ_ERR_WORKSPACE";
    case CQ_ERR_CUDA: return "CQ_ERR_CUDA";
    }
    return "CQ_ERR_UNKNOWN";
}

const char *cq_version(void) { return "cq-b200 0.1 (sm_100a)"; }

cq_status cq_rotate_quantize(const void *x, int64_t M, int64_t K, int32_t had_block,
                             int32_t act_bits, void *q_out, float *s_out, cq_stream_t stream) {
    if (M < 0 || K <= 0) return CQ_ERR_INVALID_ARGUMENT;
    if (act_bits != 4 && act_bits != 8) return CQ_ERR_INVALID_ARGUMENT;
    if (!is_pow2(had_block) || K % had_block) return CQ_ERR_INVALID_ARGUMENT;
    if (M > 0 && (!x || !q_out || !s_out)) return CQ_ERR_INVALID_ARGUMENT;
    if (!aligned16(x) || !aligned16(q_out) || !aligned16(s_out)) return CQ_ERR_INVALID_ARGUMENT;
    if (had_block > 8192 || K % 8 || K > kMaxK || M > INT32_MAX) return CQ_ERR_UNSUPPORTED;
    if (M == 0) return CQ_OK;
    return cuda_status(launch_rotate_quantize(x, K, M, (int)K, ilog2(had_block), act_bits, q_out,
                                              code_bytes(K, act_bits), s_out,
                                              reinterpret_cast<cudaStream_t>(stream)));
}

cq_status cq_rotate_quantize_ex(const void *x, int64_t M, int64_t K, int32_t had_block,
                                int32_t act_bits, const void *scale, const int32_t *perm,
                                void *q_out, float *s_out, cq_stream_t stream) {
    if (M < 0 || K <= 0) return CQ_ERR_INVALID_ARGUMENT;
    if (act_bits != 4 && act_bits != 8) return CQ_ERR_INVALID_ARGUMENT;
    if (!is_pow2(had_block) || K % had_block) return CQ_ERR_INVALID_ARGUMENT;
    if (M > 0 && (!x || !q_out || !s_out)) return CQ_ERR_INVALID_ARGUMENT;
    if (!aligned16(x) || !aligned16(q_out) || !aligned16(s_out) || !aligned16(scale) ||
        !aligned16(perm))
        return CQ_ERR_INVALID_ARGUMENT;
    if (had_block > 8192 || K % 8 || K > kMaxK || M > INT32_MAX) return CQ_ERR_UNSUPPORTED;
    if (M == 0) return CQ_OK;
    return cuda_status(launch_rotate_quantize(x, K, M, (int)K, ilog2(had_block), act_bits, q_out,
                                              code_bytes(K, act_bits), s_out,
                                              reinterpret_cast<cudaStream_t>(stream), scale,
                                              perm));
}

size_t cq_lut_gemm_workspace_size(int64_t M, int64_t N, int64_t K, int32_t act_bits) {
    (void)act_bits;
    if (M <= 0 || N <= 0 || K <= 0) return 0;
    return plan_gemm(M, N, K).ws;
}

cq_status cq_lut_gemm(const void *q, const float *s_x, int64_t M, int64_t K, int32_t act_bits,
                      const uint8_t *w_idx, const void *codebook, int64_t N, float *y,
                      int32_t *centroid_sums, void *workspace, size_t workspace_bytes,
                      cq_stream_t stream) {
    if (M < 0 || K <= 0 || N <= 0) return CQ_ERR_INVALID_ARGUMENT;
    if (act_bits != 4 && act_bits != 8) return CQ_ERR_INVALID_ARGUMENT;
    if (K % 2) return CQ_ERR_INVALID_ARGUMENT;
    if (!w_idx || !codebook || !y || (M > 0 && (!q || !s_x))) return CQ_ERR_INVALID_ARGUMENT;
    if (!aligned16(q) || !aligned16(s_x) || !aligned16(w_idx) || !aligned16(codebook) ||
        !aligned16(y) || !aligned16(centroid_sums) || !aligned16(workspace))
        return CQ_ERR_INVALID_ARGUMENT;
    if (K % 32 || N % 64 || K > (int64_t(1) << 30) || N > (int64_t(1) << 30) ||
        M > (int64_t(1) << 30))
        return CQ_ERR_UNSUPPORTED;
    if (M == 0) return CQ_OK;
    const LutGemmPlan g = plan_gemm(M, N, K);
    if (g.ws > 0 && (!workspace || workspace_bytes < g.ws)) return CQ_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = run_lut_gemm(g, q, s_x, M, K, act_bits, w_idx, codebook, N, y, workspace, st);
    if (e == cudaSuccess && centroid_sums)
        e = launch_centroid_sums(q, M, K, act_bits, w_idx, N, centroid_sums, st);
    return cuda_status(e);
}

size_t cq_lut_gemm_ex_workspace_size(int64_t M, int64_t N, int64_t K, int32_t act_bits,
                                     int32_t idx_bits) {
    if (idx_bits == 4) return cq_lut_gemm_workspace_size(M, N, K, act_bits);
    if ((idx_bits != 3 && idx_bits != 5) || M <= 0 || N <= 0 || K <= 0 || N % 64 || K % 32 ||
        K > (int64_t(1) << 30) || N > (int64_t(1) << 30) || M > (int64_t(1) << 30))
        return 0;
    const LutPlan P = plan_lut_vb((int)M, (int)N, (int)K, idx_bits);
    return align256((size_t)P.splits * M * N * sizeof(float));
}

cq_status cq_lut_gemm_ex(const void *q, const float *s_x, int64_t M, int64_t K, int32_t act_bits,
                         const uint8_t *w_idx, int32_t idx_bits, const void *codebook, int64_t N,
                         float *y, void *workspace, size_t workspace_bytes, cq_stream_t stream) {
    if (idx_bits == 4)
        return cq_lut_gemm(q, s_x, M, K, act_bits, w_idx, codebook, N, y, nullptr, workspace,
                           workspace_bytes, stream);
    if (idx_bits != 3 && idx_bits != 5) return CQ_ERR_UNSUPPORTED;
    if (M < 0 || K <= 0 || N <= 0) return CQ_ERR_INVALID_ARGUMENT;
    if (act_bits != 4 && act_bits != 8) return CQ_ERR_INVALID_ARGUMENT;
    if (K % 2) return CQ_ERR_INVALID_ARGUMENT;
    if (!w_idx || !codebook || !y || (M > 0 && (!q || !s_x))) return CQ_ERR_INVALID_ARGUMENT;
    if (!aligned16(q) || !aligned16(s_x) || !aligned16(w_idx) || !aligned16(codebook) ||
        !aligned16(y) || !aligned16(workspace))
        return CQ_ERR_INVALID_ARGUMENT;
    if (K % 32 || N % 64 || K > (int64_t(1) << 30) || N > (int64_t(1) << 30) ||
        M > (int64_t(1) << 30))
        return CQ_ERR_UNSUPPORTED;
    if (M == 0) return CQ_OK;
    const LutPlan P = plan_lut_vb((int)M, (int)N, (int)K, idx_bits);
    const size_t ws = align256((size_t)P.splits * M * N * sizeof(float));
    if (!workspace || workspace_bytes < ws) return CQ_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    LutLaunch L{};
    L.codes = reinterpret_cast<const uint8_t *>(q);
    L.ld_codes = code_bytes(K, act_bits);
    L.scales = s_x;
    L.act_bits = act_bits;
    L.K = (int)K;
    L.map_mode = kMapIdentity;
    L.G = 1;
    L.uniform_rows = (int)M;
    L.idx0 = w_idx;
    L.cb0 = codebook;
    L.N = (int)N;
    L.out = reinterpret_cast<float *>(workspace);
    L.out_split_stride = M * N;
    L.out_row_stride = N;
    cudaError_t e = launch_lut_vb(L, P, idx_bits, st);
    if (e == cudaSuccess) e = launch_reduce_plain(L.out, P, M, N, s_x, y, st);
    return cuda_status(e);
}

size_t cq_moe_ffn_workspace_size(const cq_moe_desc *d, int64_t T) {
    if (check_moe_desc(d, T) != CQ_OK) return 0;
    return plan_moe(d, T).total;
}

cq_status cq_moe_ffn(const cq_moe_desc *d, const void *x, const float *router_logits, int64_t T,
                     const cq_moe_weights *w, void *workspace, size_t workspace_bytes,
                     float *out, const cq_moe_debug *dbg, cq_stream_t stream) {
    cq_status cs = check_moe_desc(d, T);
    if (cs != CQ_OK) return cs;
    if (!w || (T > 0 && (!x || !out))) return CQ_ERR_INVALID_ARGUMENT;
    if ((d->E > 0) != (router_logits != nullptr)) return CQ_ERR_INVALID_ARGUMENT;
    if (!aligned16(x) || !aligned16(router_logits) || !aligned16(out) || !aligned16(workspace) ||
        !aligned16(w->x_scale) || !aligned16(w->x_perm))
        return CQ_ERR_INVALID_ARGUMENT;
    if (d->E > 0) {
        const void *ps[] = {w->gate_idx, w->up_idx, w->down_idx, w->gate_cb, w->up_cb, w->down_cb};
        for (const void *p : ps)
            if (!p || !aligned16(p)) return CQ_ERR_INVALID_ARGUMENT;
    }
    if (d->n_shared > 0) {
        const void *ps[] = {w->sh_gate_idx, w->sh_up_idx, w->sh_down_idx,
                            w->sh_gate_cb,  w->sh_up_cb, w->sh_down_cb};
        for (const void *p : ps)
            if (!p || !aligned16(p)) return CQ_ERR_INVALID_ARGUMENT;
    }
    if (dbg) {
        const void *ps[] = {dbg->topk_ids, dbg->topk_w, dbg->counts, dbg->offsets, dbg->perm,
                            dbg->x_codes,  dbg->x_scales, dbg->h, dbg->h_codes, dbg->h_scales,
                            dbg->y_rows};
        for (const void *p : ps)
            if (!aligned16(p)) return CQ_ERR_INVALID_ARGUMENT;
    }
    if (T == 0) return CQ_OK;
    const MoePlan m = plan_moe(d, T);
    if (!workspace || workspace_bytes < m.total) return CQ_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *ws = reinterpret_cast<uint8_t *>(workspace);
    uint8_t *xq = ws + m.o_xq;
    float *sx = reinterpret_cast<float *>(ws + m.o_sx);
    int32_t *ids = reinterpret_cast<int32_t *>(ws + m.o_ids);
    float *tw = reinterpret_cast<float *>(ws + m.o_w);
    int32_t *counts = reinterpret_cast<int32_t *>(ws + m.o_counts);
    int32_t *offsets = reinterpret_cast<int32_t *>(ws + m.o_offsets);
    int32_t *perm = reinterpret_cast<int32_t *>(ws + m.o_perm);
    int32_t *inv = reinterpret_cast<int32_t *>(ws + m.o_inv);
    int32_t *tiles = reinterpret_cast<int32_t *>(ws + m.o_tiles);
    int32_t *tgrp = reinterpret_cast<int32_t *>(ws + m.o_tgrp);
    float *pgu_r = reinterpret_cast<float *>(ws + m.o_pgu_r);
    float *pgu_s = reinterpret_cast<float *>(ws + m.o_pgu_s);
    uint8_t *hq = ws + m.o_hq;
    float *sh = reinterpret_cast<float *>(ws + m.o_sh);
    float *pdn_r = reinterpret_cast<float *>(ws + m.o_pdn_r);
    float *pdn_s = reinterpret_cast<float *>(ws + m.o_pdn_s);
    __half *hf = reinterpret_cast<__half *>(ws + m.o_hf);
    float *rsc = reinterpret_cast<float *>(ws + m.o_rs);
    const int64_t ldx = code_bytes(m.H, m.bits), ldh = code_bytes(m.Imax, m.bits);

    // routing first: the x rotation then writes the tensor-core B rows of the
    // routed slots itself (row inv[t * k + j] for token t's j-th expert)
    cudaError_t e = cudaSuccess;
    if (m.E > 0)
        e = launch_route(router_logits, (int)T, (int)m.E, (int)m.k, d->renormalize, m.tile_rows,
                         ids, tw, counts, offsets, perm, inv, tiles, tgrp, m.max_tiles_r,
                         reinterpret_cast<int32_t *>(ws + m.o_chist), st);
    RqF16 xf{};
    if (m.E > 0 && m.k_r != kKernMma) {
        xf.rows = reinterpret_cast<__half *>(ws + m.o_bx_r);
        xf.map = inv;
        xf.ncopy = (int)m.k;
        xf.row_scales = m.fused ? rsc : nullptr;
    }
    if (m.ns > 0 && m.k_s != kKernMma) xf.ident = reinterpret_cast<__half *>(ws + m.o_bx_s);
    if (e == cudaSuccess)
        e = launch_rotate_quantize(x, m.H, T, (int)m.H, ilog2(d->had_block_h), m.bits, xq, ldx,
                                   sx, st, w->x_scale, w->x_perm, &xf);
    // gate / up (dual) -> partial g, u
    if (e == cudaSuccess && m.E > 0) {
        LutLaunch L{};
        L.codes = xq; L.ld_codes = ldx; L.act_bits = m.bits; L.K = (int)m.H;
        L.map_mode = kMapPerm; L.perm = perm; L.topk = (int)m.k; L.T = (int)T;
        L.G = (int)m.E; L.grp_rows = offsets; L.grp_tiles = tiles; L.tile_grp = tgrp; L.max_tiles = m.max_tiles_r;
        L.idx0 = w->gate_idx; L.cb0 = w->gate_cb; L.idx1 = w->up_idx; L.cb1 = w->up_cb;
        L.w_stride = m.I * (m.H / 2); L.cb_stride = m.I * 16; L.N = (int)m.I; L.dual = true;
        L.out = pgu_r; L.out_split_stride = m.Rr * m.I * 2; L.out_row_stride = m.I * 2;
        if (m.fused) {
            L.scales = sx;
            L.row_scales = rsc;
            L.h_out = hf;
            L.h_row_stride = m.Imax;
        }
        if (m.k_r != kKernMma) {
            const void *b = ws + m.o_bx_r;  // written by the x rotation
            e = m.k_r == kKernTs ? launch_lut_ts(L, m.gu_r, b, m.Rr, 0, st)
                               : launch_lut_tc(L, m.gu_r, b, m.Rr, 0, st);
        } else {
            e = launch_lut(L, m.gu_r, st);
        }
    }
    if (e == cudaSuccess && m.ns > 0) {
        LutLaunch L{};
        L.codes = xq; L.ld_codes = ldx; L.act_bits = m.bits; L.K = (int)m.H;
        L.map_mode = kMapModT; L.T = (int)T;
        L.G = (int)m.ns; L.uniform_rows = (int)T; L.max_tiles = m.tiles_s;
        L.idx0 = w->sh_gate_idx; L.cb0 = w->sh_gate_cb; L.idx1 = w->sh_up_idx; L.cb1 = w->sh_up_cb;
        L.w_stride = m.Is * (m.H / 2); L.cb_stride = m.Is * 16; L.N = (int)m.Is; L.dual = true;
        L.out = pgu_s; L.out_split_stride = m.Rs * m.Is * 2; L.out_row_stride = m.Is * 2;
        if (m.fused) {
            L.scales = sx;
            L.h_out = hf + m.Rr * m.Imax;
            L.h_row_stride = m.Imax;
        }
        if (m.k_s != kKernMma) {
            const void *b = ws + m.o_bx_s;  // written by the x rotation
            e = m.k_s == kKernTs ? launch_lut_ts(L, m.gu_s, b, T, (int)T, st)
                               : launch_lut_tc(L, m.gu_s, b, T, (int)T, st);
        } else {
            e = launch_lut(L, m.gu_s, st);
        }
    }
    // SwiGLU + rotate + quantize of h; the rotation also writes the down
    // projections' tensor-core B rows
    __half *bh_r = m.E > 0 && m.k_r != kKernMma ? reinterpret_cast<__half *>(ws + m.o_bh_r) : nullptr;
    __half *bh_s = m.ns > 0 && m.k_s != kKernMma ? reinterpret_cast<__half *>(ws + m.o_bh_s) : nullptr;
    if (e == cudaSuccess && m.fused) {
        // h was written by the gate/up epilogues: rotate + quantize its rows
        // ... and write the down projections' tensor-core B rows as they go
        if (m.E > 0) {
            RqF16 hf16{};
            hf16.ident = bh_r;
            e = launch_rotate_quantize(hf, m.Imax, m.Rr, (int)m.I, ilog2(d->had_block_i), m.bits,
                                       hq, ldh, sh, st, nullptr, nullptr, &hf16);
        }
        if (e == cudaSuccess && m.ns > 0) {
            RqF16 hf16{};
            hf16.ident = bh_s;
            e = launch_rotate_quantize(hf + m.Rr * m.Imax, m.Imax, m.Rs, (int)m.Is,
                                       ilog2(d->had_block_i_shared), m.bits, hq + m.Rr * ldh, ldh,
                                       sh + m.Rr, st, nullptr, nullptr, &hf16);
        }
        if (e == cudaSuccess && dbg && dbg->h)
            e = cudaMemcpyAsync(dbg->h, hf, (size_t)m.R * m.Imax * 2, cudaMemcpyDeviceToDevice, st);
    } else if (e == cudaSuccess) {
        SwigluArgs a{};
        a.part_r = pgu_r; a.part_s = pgu_s;
        a.plan_r = m.gu_r; a.plan_s = m.gu_s;
        a.R_routed = m.Rr; a.R_shared = m.Rs;
        a.I = (int)m.I; a.I_shared = (int)m.Is; a.Imax = m.Imax;
        a.log2b_i = m.E > 0 ? ilog2(d->had_block_i) : 0;
        a.log2b_i_shared = m.ns > 0 ? ilog2(d->had_block_i_shared) : 0;
        a.perm = perm; a.topk = (int)std::max<int64_t>(m.k, 1); a.T = (int)T;
        a.x_scales = sx; a.bits = m.bits; a.hq = hq; a.ldhq = ldh; a.h_scales = sh;
        a.h_dbg = dbg ? dbg->h : nullptr;
        a.f16_r = bh_r;
        a.f16_s = bh_s;
        e = launch_swiglu_rq(a, m.R, st);
    }
    // down -> partial y
    if (e == cudaSuccess && m.E > 0) {
        LutLaunch L{};
        L.codes = hq; L.ld_codes = ldh; L.act_bits = m.bits; L.K = (int)m.I;
        L.map_mode = kMapIdentity;
        L.G = (int)m.E; L.grp_rows = offsets; L.grp_tiles = tiles; L.tile_grp = tgrp; L.max_tiles = m.max_tiles_r;
        L.idx0 = w->down_idx; L.cb0 = w->down_cb;
        L.w_stride = m.H * (m.I / 2); L.cb_stride = m.H * 16; L.N = (int)m.H; L.dual = false;
        L.out = pdn_r; L.out_split_stride = m.Rr * m.H; L.out_row_stride = m.H;
        if (m.k_r != kKernMma) {
            const void *b = bh_r;  // written by the h rotation
            e = m.k_r == kKernTs ? launch_lut_ts(L, m.dn_r, b, m.Rr, 0, st)
                               : launch_lut_tc(L, m.dn_r, b, m.Rr, 0, st);
        } else {
            e = launch_lut(L, m.dn_r, st);
        }
    }
    if (e == cudaSuccess && m.ns > 0) {
        LutLaunch L{};
        L.codes = hq + m.Rr * ldh; L.ld_codes = ldh; L.act_bits = m.bits; L.K = (int)m.Is;
        L.map_mode = kMapIdentity;
        L.G = (int)m.ns; L.uniform_rows = (int)T; L.max_tiles = m.tiles_s;
        L.idx0 = w->sh_down_idx; L.cb0 = w->sh_down_cb;
        L.w_stride = m.H * (m.Is / 2); L.cb_stride = m.H * 16; L.N = (int)m.H; L.dual = false;
        L.out = pdn_s; L.out_split_stride = m.Rs * m.H; L.out_row_stride = m.H;
        if (m.k_s != kKernMma) {
            const void *b = bh_s;  // written by the h rotation
            e = m.k_s == kKernTs ? launch_lut_ts(L, m.dn_s, b, m.Rs, 0, st)
                               : launch_lut_tc(L, m.dn_s, b, m.Rs, 0, st);
        } else {
            e = launch_lut(L, m.dn_s, st);
        }
    }
    if (e == cudaSuccess) {
        CombineArgs c{};
        c.part_r = pdn_r; c.part_s = pdn_s;
        c.plan_r = m.dn_r; c.plan_s = m.dn_s;
        c.R_routed = m.Rr; c.R_shared = m.Rs;
        c.T = (int)T; c.H = (int)m.H; c.topk = (int)m.k; c.n_shared = (int)m.ns;
        c.inv_perm = inv; c.w = tw; c.h_scales = sh; c.out = out;
        c.y_dbg = dbg ? dbg->y_rows : nullptr;
        e = launch_combine(c, st);
    }
    if (e == cudaSuccess && dbg) {
        auto cp = [&](void *dst, const void *src, size_t bytes) {
            if (dst && bytes && e == cudaSuccess)
                e = cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, st);
        };
        cp(dbg->topk_ids, ids, (size_t)m.Rr * 4);
        cp(dbg->topk_w, tw, (size_t)m.Rr * 4);
        cp(dbg->counts, counts, (size_t)m.E * 4);
        cp(dbg->offsets, offsets, (size_t)(m.E > 0 ? m.E + 1 : 0) * 4);
        cp(dbg->perm, perm, (size_t)m.Rr * 4);
        cp(dbg->x_codes, xq, (size_t)T * ldx);
        cp(dbg->x_scales, sx, (size_t)T * 4);
        cp(dbg->h_codes, hq, (size_t)m.R * ldh);
        cp(dbg->h_scales, sh, (size_t)m.R * 4);
    }
    return cuda_status(e);
}

}  // extern "C"
