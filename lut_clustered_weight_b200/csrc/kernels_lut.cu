// kernels_lut.cu -- LUT (codebook) GEMM for small token counts on sm_100a.
//
//   y[m, n] = s_x[m] * sum_k C[n, I[n,k]] * q[m, k]
//
// Design (CodeQuant2 Figure 4: one-time LUT precompute, then lookups):
//  * The one-time precompute turns each weight row's 16 fp16 centroids into
//    two 16-byte byte-plane tables (low bytes, high bytes) held in eight
//    registers.  A lookup of four 4-bit indices is then two byte permutes per
//    plane plus a select on index bit 3 -- about 2.75 integer instructions
//    per weight, with no shared-memory traffic.  (On B200 one HBM byte per
//    SM-cycle budget leaves ~2-3 issue slots per weight; a data-indexed
//    shared-memory lookup per weight would exceed the 32 lanes/cycle the
//    shared memory can serve, and its bank conflicts are what the CodeQuant
//    podcast transcript, "Improvements", warns about.)
//  * The looked-up fp16 weights feed mma.sync m16n8k16 (fp16 x fp16 -> fp32)
//    with the tokens as the n dimension: int codes are exact in fp16 and the
//    fp16 products are exact in fp32.  Weights are the HBM stream; every
//    packed index byte is read once with a 128-bit non-allocating load.
//  * The contraction order inside a 128-k chunk is permuted so that each lane
//    consumes 16 contiguous bytes of its rows; the activations are written
//    into shared memory in exactly that permuted fragment order.
//  * A CTA is 4 warps; a warp owns 16 weight rows (plain) or 8 gate rows plus
//    the 8 matching up rows (dual, so SwiGLU needs no data exchange).
//    Split-K partial sums go to a workspace and are reduced in a fixed order.
#include "cq_common.cuh"
#include "cq_internal.h"

namespace cq {

constexpr int kLutThreads = 128;
constexpr int kTokTile = 16;  // largest token tile (two n8 MMA tiles)
constexpr int kPrefetch = 4;  // 128-k chunks in flight per lane
constexpr size_t kLutSmemCap = 96 * 1024;

// Byte-plane tables of one codebook row: lo[j] holds the low bytes of
// C[4j..4j+3], hi[j] the high bytes.
CQ_DEV void build_tables(const __half *cb, uint32_t (&lo)[4], uint32_t (&hi)[4]) {
    const uint4 a = *reinterpret_cast<const uint4 *>(cb);
    const uint4 b = *reinterpret_cast<const uint4 *>(cb + 8);
    const uint32_t u[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int j = 0; j < 4; j++) {
        lo[j] = prmt(u[2 * j], u[2 * j + 1], 0x6420);
        hi[j] = prmt(u[2 * j], u[2 * j + 1], 0x7531);
    }
}

// Eight 4-bit indices (nibble i of w = index of element i) -> four half2:
// h[0] = (C[i0], C[i1]), h[1] = (C[i2], C[i3]), h[2] = (C[i4], C[i5]),
// h[3] = (C[i6], C[i7]).  Selector nibble bit 3 switches prmt to
// sign-replicate mode, so entries 0-7 and 8-15 are fetched from the two
// halves of each plane and merged with a per-byte mask built from bit 3.
CQ_DEV void dequant8(uint32_t w, const uint32_t (&lo)[4], const uint32_t (&hi)[4],
                     uint32_t (&h)[4]) {
    const uint32_t s0 = w, s1 = w >> 16;
    const uint32_t x0 = s0 ^ 0x8888u, x1 = s1 ^ 0x8888u;
    const uint32_t w4 = w << 4;
    const uint32_t m0 = prmt(w4, w, 0xD9C8);  // 0xFF in byte i iff nibble i >= 8
    const uint32_t m1 = prmt(w4, w, 0xFBEA);
    {
        const uint32_t l = (prmt(lo[0], lo[1], s0) & ~m0) | (prmt(lo[2], lo[3], x0) & m0);
        const uint32_t g = (prmt(hi[0], hi[1], s0) & ~m0) | (prmt(hi[2], hi[3], x0) & m0);
        h[0] = prmt(l, g, 0x5140);
        h[1] = prmt(l, g, 0x7362);
    }
    {
        const uint32_t l = (prmt(lo[0], lo[1], s1) & ~m1) | (prmt(lo[2], lo[3], x1) & m1);
        const uint32_t g = (prmt(hi[0], hi[1], s1) & ~m1) | (prmt(hi[2], hi[3], x1) & m1);
        h[2] = prmt(l, g, 0x5140);
        h[3] = prmt(l, g, 0x7362);
    }
}

CQ_DEV __half code_to_half(int v) { return __short2half_rn((short)v); }

template <int NT>
__global__ void __launch_bounds__(kLutThreads) k_lut_mma(LutLaunch L, LutPlan P) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint2 *bfrag = reinterpret_cast<uint2 *>(smem_raw);
    __shared__ int s_code_row[kTokTile];
    __shared__ float s_scale[kTokTile];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int row_tile = blockIdx.x % P.n_row_tiles;
    const int split = blockIdx.x / P.n_row_tiles;
    const int tile = blockIdx.y;

    // ---- which group / token tile
    int g, row0, nrows;
    constexpr int TT = 8 * NT;  // token rows per tile
    if (L.uniform_rows > 0) {
        const int tpg = (L.uniform_rows + TT - 1) / TT;
        g = tile / tpg;
        if (g >= L.G) return;
        row0 = g * L.uniform_rows + (tile - g * tpg) * TT;
        nrows = min(TT, (g + 1) * L.uniform_rows - row0);
    } else {
        if (tile >= L.grp_tiles[L.G]) return;
        int lo = 0, hi = L.G;  // largest g with grp_tiles[g] <= tile
        while (hi - lo > 1) {
            int mid = (lo + hi) >> 1;
            if (L.grp_tiles[mid] <= tile) lo = mid; else hi = mid;
        }
        g = lo;
        row0 = L.grp_rows[g] + (tile - L.grp_tiles[g]) * TT;
        nrows = min(TT, L.grp_rows[g + 1] - row0);
    }
    const int ch0 = split * P.chunks_per_split;
    const int ch1 = min(ch0 + P.chunks_per_split, P.chunks_total);
    const int nch = ch1 - ch0;
    if (nch <= 0 || nrows <= 0) return;
    const int K = L.K;

    if (tid < TT) {
        int cr = -1;
        if (tid < nrows) {
            const int p = row0 + tid;
            cr = L.map_mode == kMapPerm ? L.perm[p] / L.topk
               : L.map_mode == kMapModT ? p % L.T : p;
        }
        s_code_row[tid] = cr;
        s_scale[tid] = (cr >= 0 && L.direct) ? L.scales[cr] : 0.0f;
    }
    __syncthreads();

    // ---- activation fragments for chunks [ch0, ch1): 8 consecutive k per item
    const int items = NT * 8 * nch * 16;
    for (int it = tid; it < items; it += kLutThreads) {
        const int j = it / (nch * 16);
        const int rem = it - j * (nch * 16);
        const int ch = rem >> 4, o8 = rem & 15;
        const int k = (ch0 + ch) * 128 + o8 * 8;
        const int cr = s_code_row[j];
        __align__(8) __half v[8];
#pragma unroll
        for (int e = 0; e < 8; e++) v[e] = __ushort_as_half(0);
        if (cr >= 0 && k < K) {
            if (L.act_bits == 4) {
                const uint32_t w = *reinterpret_cast<const uint32_t *>(
                    L.codes + (int64_t)cr * L.ld_codes + k / 2);
#pragma unroll
                for (int e = 0; e < 8; e++) v[e] = code_to_half(((int)(w << (28 - 4 * e))) >> 28);
            } else {
                const uint2 w = *reinterpret_cast<const uint2 *>(
                    L.codes + (int64_t)cr * L.ld_codes + k);
#pragma unroll
                for (int e = 0; e < 4; e++) {
                    v[e] = code_to_half(((int)(w.x << (24 - 8 * e))) >> 24);
                    v[4 + e] = code_to_half(((int)(w.y << (24 - 8 * e))) >> 24);
                }
            }
        }
        const int c = o8 >> 2, i = 2 * (o8 & 3);
        const int ln = 4 * (j & 7) + c, nt = j >> 3;
        const uint2 *vv = reinterpret_cast<const uint2 *>(v);
        bfrag[((ch * 8 + i) * NT + nt) * 32 + ln] = vv[0];
        bfrag[((ch * 8 + i + 1) * NT + nt) * 32 + ln] = vv[1];
    }
    __syncthreads();

    // ---- this lane's two weight rows
    const int gq = lane >> 2, cl = lane & 3;
    const int64_t rowbytes = K / 2;
    const uint8_t *pA, *pB;
    const __half *cA, *cB;
    int nA, nB;
    if (L.dual) {
        nA = nB = row_tile * 32 + warp * 8 + gq;
        pA = L.idx0 + (int64_t)g * L.w_stride + (int64_t)nA * rowbytes;
        pB = L.idx1 + (int64_t)g * L.w_stride + (int64_t)nB * rowbytes;
        cA = reinterpret_cast<const __half *>(L.cb0) + (int64_t)g * L.cb_stride + nA * 16;
        cB = reinterpret_cast<const __half *>(L.cb1) + (int64_t)g * L.cb_stride + nB * 16;
    } else {
        nA = row_tile * 64 + warp * 16 + gq;
        nB = nA + 8;
        pA = L.idx0 + (int64_t)g * L.w_stride + (int64_t)nA * rowbytes;
        pB = pA + 8 * rowbytes;
        cA = reinterpret_cast<const __half *>(L.cb0) + (int64_t)g * L.cb_stride + nA * 16;
        cB = cA + 8 * 16;
    }
    uint32_t loA[4], hiA[4], loB[4], hiB[4];
    build_tables(cA, loA, hiA);
    build_tables(cB, loB, hiB);

    float acc[NT][4];
#pragma unroll
    for (int t = 0; t < NT; t++)
#pragma unroll
        for (int e = 0; e < 4; e++) acc[t][e] = 0.0f;

    // lanes whose 32-k slice lies beyond K (ragged last chunk) read nothing;
    // their activations are zero so index 0 contributes nothing
    const int tailc = (K & 127) >> 5;  // valid 32-k slices in a ragged last chunk
    auto load = [&](int ch, uint4 &a, uint4 &b) {
        const int gch = ch0 + ch;
        const bool ok = !(gch == P.chunks_total - 1 && tailc != 0 && cl >= tailc);
        if (ok) {
            a = ldg_stream(pA + (int64_t)gch * 64 + cl * 16);
            b = ldg_stream(pB + (int64_t)gch * 64 + cl * 16);
        } else {
            a = make_uint4(0, 0, 0, 0);
            b = make_uint4(0, 0, 0, 0);
        }
    };

    uint4 ra[kPrefetch], rb[kPrefetch];
#pragma unroll
    for (int p = 0; p < kPrefetch; p++)
        if (p < nch) load(p, ra[p], rb[p]);

    for (int base = 0; base < nch; base += kPrefetch) {
#pragma unroll
        for (int p = 0; p < kPrefetch; p++) {
            const int ch = base + p;
            if (ch < nch) {
                const uint32_t wa[4] = {ra[p].x, ra[p].y, ra[p].z, ra[p].w};
                const uint32_t wb[4] = {rb[p].x, rb[p].y, rb[p].z, rb[p].w};
                if (ch + kPrefetch < nch) load(ch + kPrefetch, ra[p], rb[p]);
                const uint2 *bf = bfrag + (size_t)ch * 8 * NT * 32 + lane;
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    uint32_t hA[4], hB[4];
                    dequant8(wa[j], loA, hiA, hA);
                    dequant8(wb[j], loB, hiB, hB);
#pragma unroll
                    for (int hh = 0; hh < 2; hh++) {
                        const int i = 2 * j + hh;
                        const uint32_t af[4] = {hA[2 * hh], hB[2 * hh], hA[2 * hh + 1],
                                                hB[2 * hh + 1]};
#pragma unroll
                        for (int t = 0; t < NT; t++) {
                            const uint2 bv = bf[(i * NT + t) * 32];
                            mma_16816(acc[t], af, bv.x, bv.y);
                        }
                    }
                }
            }
        }
    }

    // ---- epilogue: acc[t][0..1] row A, tokens 8t + 2cl + {0,1}; acc[t][2..3] row B
    float *out = L.out + (int64_t)split * L.out_split_stride;
#pragma unroll
    for (int t = 0; t < NT; t++) {
#pragma unroll
        for (int e = 0; e < 2; e++) {
            const int tok = 8 * t + 2 * cl + e;
            if (tok < nrows) {
                const int64_t p = row0 + tok;
                if (L.dual) {
                    *reinterpret_cast<float2 *>(out + p * L.out_row_stride + 2 * nA) =
                        make_float2(acc[t][e], acc[t][2 + e]);
                } else if (L.direct) {
                    const float s = s_scale[tok];
                    out[p * L.out_row_stride + nA] = s * acc[t][e];
                    out[p * L.out_row_stride + nB] = s * acc[t][2 + e];
                } else {
                    out[p * L.out_row_stride + nA] = acc[t][e];
                    out[p * L.out_row_stride + nB] = acc[t][2 + e];
                }
            }
        }
    }
}

int sm_count() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

LutPlan plan_lut(int N, int K, bool dual, int max_rows_per_group, int64_t est_tiles) {
    LutPlan P;
    P.nt = max_rows_per_group <= 8 ? 1 : 2;
    P.n_row_tiles = dual ? N / 32 : N / 64;
    P.chunks_total = (K + 127) / 128;
    const size_t per_chunk = (size_t)P.nt * 8 * 128 * 2;  // fp16 fragments
    const int max_cps = (int)(kLutSmemCap / per_chunk);
    // aim for ~3 resident CTAs per SM worth of independent CTAs
    const int64_t target = (int64_t)sm_count() * 3;
    const int64_t base = (int64_t)P.n_row_tiles * (est_tiles > 0 ? est_tiles : 1);
    int splits = (int)((target + base - 1) / base);
    if (splits < 1) splits = 1;
    const int min_splits = (P.chunks_total + max_cps - 1) / max_cps;
    if (splits < min_splits) splits = min_splits;
    if (splits > P.chunks_total) splits = P.chunks_total;
    P.chunks_per_split = (P.chunks_total + splits - 1) / splits;
    P.splits = (P.chunks_total + P.chunks_per_split - 1) / P.chunks_per_split;
    P.smem = per_chunk * P.chunks_per_split;
    return P;
}

cudaError_t launch_lut(const LutLaunch &L, const LutPlan &P, cudaStream_t st) {
    dim3 grid(P.n_row_tiles * P.splits, L.max_tiles);
    if (grid.y == 0 || grid.x == 0) return cudaSuccess;
    const bool timed = timing_on();
    if (timed) timing_begin(st);
    count_launch();
    if (P.nt == 1) {
        cudaFuncSetAttribute(k_lut_mma<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kLutSmemCap);
        k_lut_mma<1><<<grid, kLutThreads, P.smem, st>>>(L, P);
    } else {
        cudaFuncSetAttribute(k_lut_mma<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kLutSmemCap);
        k_lut_mma<2><<<grid, kLutThreads, P.smem, st>>>(L, P);
    }
    if (timed) timing_end(st);
    return cudaGetLastError();
}

// ---------------------------------------------------------------- split-K reduce
__global__ void k_reduce_plain(const float *__restrict__ part, int splits, int64_t M, int64_t N,
                               const float *__restrict__ s, float *__restrict__ y) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= M * N) return;
    float acc = 0.0f;
    for (int k = 0; k < splits; k++) acc += part[(int64_t)k * M * N + i];
    y[i] = s[i / N] * acc;
}

cudaError_t launch_reduce_plain(const float *part, int splits, int64_t M, int64_t N,
                                const float *s, float *y, cudaStream_t st) {
    const int64_t n = M * N;
    if (n == 0) return cudaSuccess;
    count_launch();
    k_reduce_plain<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(part, splits, M, N, s, y);
    return cudaGetLastError();
}

// ---------------------------------------------------------------- centroid sums (parity)
// S[m, n, c] = sum_{k : I[n,k] = c} q[m,k]; one thread per (m, n).
__global__ void k_centroid_sums(const uint8_t *__restrict__ q, int64_t M, int64_t K, int bits,
                                const uint8_t *__restrict__ w_idx, int64_t N, int32_t *S) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= M * N) return;
    const int64_t m = i / N, n = i % N;
    int32_t acc[16];
#pragma unroll
    for (int c = 0; c < 16; c++) acc[c] = 0;
    const uint8_t *wr = w_idx + n * (K / 2);
    for (int64_t k = 0; k < K; k++) {
        const int c = (wr[k / 2] >> (4 * (k & 1))) & 15;
        int v;
        if (bits == 4) {
            const int nib = (q[m * (K / 2) + k / 2] >> (4 * (k & 1))) & 15;
            v = nib >= 8 ? nib - 16 : nib;
        } else {
            v = (int)reinterpret_cast<const int8_t *>(q)[m * K + k];
        }
#pragma unroll
        for (int cc = 0; cc < 16; cc++) acc[cc] += (cc == c) ? v : 0;
    }
#pragma unroll
    for (int c = 0; c < 16; c++) S[i * 16 + c] = acc[c];
}

cudaError_t launch_centroid_sums(const void *q, int64_t M, int64_t K, int bits,
                                 const uint8_t *w_idx, int64_t N, int32_t *S, cudaStream_t st) {
    const int64_t n = M * N;
    if (n == 0) return cudaSuccess;
    count_launch();
    k_centroid_sums<<<(unsigned)((n + 127) / 128), 128, 0, st>>>(
        reinterpret_cast<const uint8_t *>(q), M, K, bits, w_idx, N, S);
    return cudaGetLastError();
}

}  // namespace cq
