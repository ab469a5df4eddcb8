// kernels_lut_vb.cu -- LUT GEMM with 8 or 32 centroids per row (3- or 5-bit
// indices): the adaptive codebook size of CodeQuant2 (abstract: codebook sizes
// adapted to each layer's quantization difficulty; Figure 3: adaptive cluster
// allocation).  16 centroids (4 bits) run on the kernels of cq_lut_gemm.
//
//   y[m, n] = s_x[m] * sum_k C[n, I[n,k]] * q[m, k],  I[n,k] < 2^B
//
// Index k of row n occupies bits [B k, B k + B) of the row's byte string,
// least significant bit first, so the 32 indices k = 32 j .. 32 j + 31 are
// exactly the B 32-bit words j B .. j B + B - 1 of the row.
//
// Design: mma.sync m16n8k16 (fp16 x fp16 -> fp32), weight rows as the MMA's
// 16 rows, tokens as n; one warp owns 16 rows, a CTA four warps (64 rows) and
// one split of the contraction.  Within a 128-k chunk lane (gq, cl) consumes
// the 32 contiguous indices k = 32 cl .. 32 cl + 31 of its rows gq and gq + 8
// (the contraction order inside the chunk is permuted accordingly, and the
// activation fragments are staged in that order), so every index field sits
// at a compile-time bit offset of the lane's B words.  The one-time LUT
// precompute is per row and per quad lane (four replicas, entry e of row r,
// replica c at word (16 e + r) * 4 + c): the 32 lanes of a lookup hit 32
// different banks whatever the indices.
//   B = 3: a 64-entry pair table, entry p = (C[p & 7], C[p >> 3]): one lookup
//          per two weights.
//   B = 5: a 32-entry table (a pair table would need 1024 entries): two
//          lookups and a byte permute per two weights.
#include "cq_common.cuh"
#include "cq_internal.h"

#include <algorithm>

namespace cq {

constexpr int kVbWarps = 4;
constexpr int kVbChunk = 128;  // k per chunk: 8 MMA steps of 16

template <int B>
struct VbShape {
    static_assert(B == 3 || B == 5, "3- or 5-bit indices");
    static constexpr int entries = B == 3 ? 64 : 32;             // table entries per row
    static constexpr size_t table_bytes = (size_t)kVbWarps * 16 * 4 * entries * 4;
};

// 4 activation codes at k0 .. k0 + 3 of a code row -> 4 fp16 (exact).
CQ_DEV uint2 codes4_to_half(const uint8_t *row, int k0, int bits) {
    __align__(8) __half v[4];
    if (bits == 4) {
        const uint32_t w = *reinterpret_cast<const uint16_t *>(row + k0 / 2);
#pragma unroll
        for (int e = 0; e < 4; e++) v[e] = __short2half_rn((short)(((int)(w << (28 - 4 * e))) >> 28));
    } else {
        const uint32_t w = *reinterpret_cast<const uint32_t *>(row + k0);
#pragma unroll
        for (int e = 0; e < 4; e++) v[e] = __short2half_rn((short)(((int)(w << (24 - 8 * e))) >> 24));
    }
    return *reinterpret_cast<const uint2 *>(v);
}

// Bits [off, off + width) of the lane's index words (off and width are
// compile-time after unrolling).
template <int B>
CQ_DEV uint32_t field(const uint32_t (&w)[B], int off, int width) {
    const int wi = off >> 5, sh = off & 31;
    uint32_t v = w[wi] >> sh;
    if (sh + width > 32) v |= w[wi + 1] << (32 - sh);
    return v & ((1u << width) - 1u);
}

template <int B, int NT>
__global__ void __launch_bounds__(kVbWarps * 32) k_lut_vb(const LutLaunch L, const LutPlan P) {
    using Sh = VbShape<B>;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint32_t *tab = reinterpret_cast<uint32_t *>(smem_raw);                 // [warps][entries][16][4]
    uint2 *bfrag = reinterpret_cast<uint2 *>(smem_raw + Sh::table_bytes);  // [chunks][8][NT][32]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gq = lane >> 2, cl = lane & 3;
    const int K = L.K, N = L.N;
    const int rt = blockIdx.x % P.n_row_tiles, sp = blockIdx.x / P.n_row_tiles;
    const int tok0 = blockIdx.y * 8 * NT;
    const int C = P.chunks_total;
    const int ch_lo = sp * P.chunks_per_split;
    const int ch_hi = min(C, ch_lo + P.chunks_per_split);
    const int nch = ch_hi - ch_lo;
    const int64_t rowbytes = (int64_t)K * B / 8;
    const int nA = rt * 64 + warp * 16 + gq;   // rows gq and gq + 8 of the warp's tile

    griddep_launch();
    // ---- the one-time LUT precompute (weights only: overlaps the previous kernel)
    uint32_t *wtab = tab + (size_t)warp * Sh::entries * 64;
    {
        // lane: row r = lane & 15 of the warp's tile, replicas lane >> 4 and + 2
        const int r = lane & 15;
        const __half *cb =
            reinterpret_cast<const __half *>(L.cb0) + (int64_t)(rt * 64 + warp * 16 + r) * (1 << B);
        uint32_t c16[1 << B];
#pragma unroll
        for (int e = 0; e < (1 << B); e++) c16[e] = (uint32_t)__half_as_ushort(cb[e]);
#pragma unroll
        for (int e = 0; e < Sh::entries; e++) {
            const uint32_t v = B == 3 ? (c16[e & 7] | (c16[e >> 3] << 16)) : c16[e];
            wtab[(e * 16 + r) * 4 + (lane >> 4)] = v;
            wtab[(e * 16 + r) * 4 + (lane >> 4) + 2] = v;
        }
    }
    griddep_wait();  // the activation codes come from the previous kernel
    // ---- activation fragments of this split, in the permuted fragment order
    for (int it = tid; it < nch * 8 * NT * 32; it += kVbWarps * 32) {
        const int ln = it & 31, nt = (it >> 5) % NT, step = (it >> 5) / NT % 8, ch = (it >> 5) / NT / 8;
        const int tok = tok0 + 8 * nt + (ln >> 2);
        const int k0 = (ch_lo + ch) * kVbChunk + 32 * (ln & 3) + 4 * step;
        uint2 v = make_uint2(0, 0);
        if (tok < L.uniform_rows && k0 < K)
            v = codes4_to_half(L.codes + (int64_t)tok * L.ld_codes, k0, L.act_bits);
        bfrag[it] = v;
    }
    __syncthreads();

    float acc[NT][4];
#pragma unroll
    for (int t = 0; t < NT; t++)
#pragma unroll
        for (int e = 0; e < 4; e++) acc[t][e] = 0.0f;
    const uint8_t *pa = L.idx0 + (int64_t)nA * rowbytes + 4 * B * cl;
    const uint8_t *pb = pa + 8 * rowbytes;
    const uint32_t tabA = (uint32_t)__cvta_generic_to_shared(wtab) + 4u * (gq * 4 + cl);
    const uint32_t tabB = tabA + 4u * 32;  // row gq + 8
    auto load = [&](int ch, uint32_t (&a)[B], uint32_t (&b)[B]) {
        const bool live = (ch_lo + ch) * kVbChunk + 32 * cl < K;
        const int64_t off = (int64_t)(ch_lo + ch) * (16 * B);
#pragma unroll
        for (int i = 0; i < B; i++) {
            a[i] = live ? __ldg(reinterpret_cast<const unsigned int *>(pa + off) + i) : 0u;
            b[i] = live ? __ldg(reinterpret_cast<const unsigned int *>(pb + off) + i) : 0u;
        }
    };
    uint32_t wa[B], wb[B], na[B], nb[B];
    if (nch > 0) load(0, wa, wb);
    for (int ch = 0; ch < nch; ch++) {
        if (ch + 1 < nch) load(ch + 1, na, nb);
        const bool live = (ch_lo + ch) * kVbChunk + 32 * cl < K;
        const uint2 *bf = bfrag + (size_t)ch * 8 * NT * 32 + lane;
#pragma unroll
        for (int step = 0; step < 8; step++) {
            uint32_t af[4];
#pragma unroll
            for (int h = 0; h < 2; h++) {
                const int j = 2 * step + h;  // pair j: indices 2j, 2j + 1 of the lane's 32
                uint32_t va, vb;
                if (B == 3) {
                    va = lds32(tabA + field<B>(wa, 6 * j, 6) * (64u * 4u));
                    vb = lds32(tabB + field<B>(wb, 6 * j, 6) * (64u * 4u));
                } else {
                    const uint32_t a0 = lds32(tabA + field<B>(wa, 10 * j, 5) * (64u * 4u));
                    const uint32_t a1 = lds32(tabA + field<B>(wa, 10 * j + 5, 5) * (64u * 4u));
                    const uint32_t b0 = lds32(tabB + field<B>(wb, 10 * j, 5) * (64u * 4u));
                    const uint32_t b1 = lds32(tabB + field<B>(wb, 10 * j + 5, 5) * (64u * 4u));
                    va = prmt(a0, a1, 0x5410u);
                    vb = prmt(b0, b1, 0x5410u);
                }
                af[2 * h] = live ? va : 0u;
                af[2 * h + 1] = live ? vb : 0u;
            }
#pragma unroll
            for (int t = 0; t < NT; t++) {
                const uint2 bv = bf[(step * NT + t) * 32];
                mma_16816(acc[t], af, bv.x, bv.y);
            }
        }
#pragma unroll
        for (int i = 0; i < B; i++) {
            wa[i] = na[i];
            wb[i] = nb[i];
        }
    }
    // ---- split-K partial sums: out[sp][token][n]
    float *out = L.out + (int64_t)sp * L.out_split_stride;
#pragma unroll
    for (int t = 0; t < NT; t++)
#pragma unroll
        for (int e = 0; e < 2; e++) {
            const int tok = tok0 + 8 * t + 2 * cl + e;
            if (tok < L.uniform_rows) {
                out[(int64_t)tok * N + nA] = acc[t][e];
                out[(int64_t)tok * N + nA + 8] = acc[t][2 + e];
            }
        }
}

LutPlan plan_lut_vb(int M, int N, int K, int idx_bits) {
    LutPlan P{};
    P.nt = M <= 8 ? 1 : 2;
    P.warps = kVbWarps;
    P.rows_per_rt = 64;
    P.n_row_tiles = N / 64;
    P.chunks_total = (K + kVbChunk - 1) / kVbChunk;
    P.streamk = 0;
    const int tiles = (M + 8 * P.nt - 1) / (8 * P.nt);
    const size_t table = idx_bits == 3 ? VbShape<3>::table_bytes : VbShape<5>::table_bytes;
    const size_t per_chunk = (size_t)P.nt * 8 * 32 * sizeof(uint2);
    const size_t budget = 112 * 1024;  // two CTAs per SM
    const int cps_max = (int)std::max<size_t>(1, (budget - table) / per_chunk);
    const int C = P.chunks_total;
    const int64_t base = (int64_t)P.n_row_tiles * tiles;
    const int capacity = 2 * sm_count();
    int splits = base < capacity ? (int)(capacity / base) : 1;
    splits = std::max(std::min(splits, C), (C + cps_max - 1) / cps_max);
    P.chunks_per_split = (C + splits - 1) / splits;
    P.splits = (C + P.chunks_per_split - 1) / P.chunks_per_split;
    P.cps_max = P.chunks_per_split;
    P.grid = P.n_row_tiles * P.splits;
    P.uniform_rows = M;
    P.smem = table + per_chunk * P.chunks_per_split;
    P.tc = 0;
    return P;
}

template <int B, int NT>
static cudaError_t launch_vb_t(const LutLaunch &L, const LutPlan &P, int tiles, cudaStream_t st) {
    return launch_pdl(k_lut_vb<B, NT>, dim3(P.grid, tiles), dim3(kVbWarps * 32), P.smem, st, 1, L,
                      P);
}

cudaError_t launch_lut_vb(const LutLaunch &L, const LutPlan &P, int idx_bits, cudaStream_t st) {
    const int tiles = (L.uniform_rows + 8 * P.nt - 1) / (8 * P.nt);
    if (P.grid == 0 || tiles == 0) return cudaSuccess;
    const bool timed = timing_on();
    if (timed) timing_begin(st, CQ_KERNEL_LUT_VB);
    count_launch();
    cudaError_t e;
    if (idx_bits == 3)
        e = P.nt == 1 ? launch_vb_t<3, 1>(L, P, tiles, st) : launch_vb_t<3, 2>(L, P, tiles, st);
    else
        e = P.nt == 1 ? launch_vb_t<5, 1>(L, P, tiles, st) : launch_vb_t<5, 2>(L, P, tiles, st);
    if (timed) timing_end(st);
    return e;
}

}  // namespace cq
