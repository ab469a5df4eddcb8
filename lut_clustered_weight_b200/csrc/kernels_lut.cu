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
#include "lut_lookup.cuh"

#include <algorithm>

namespace cq {

constexpr int kTokTile = 16;  // largest token tile (two n8 MMA tiles)

CQ_DEV __half code_to_half(int v) { return __short2half_rn((short)v); }

CQ_DEV void cp_async16(void *smem_dst, const void *gsrc) {
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(smem_dst);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gsrc) : "memory");
}
CQ_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
CQ_DEV void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

constexpr int kStages = 6;  // per-lane cp.async ring: kStages-1 chunks in flight

// One CTA = W warps.  Shared memory: the activation fragments of the chunk
// range being processed ([cps_max][8 mma][NT][32 lanes] x 4 fp16), then the
// weight ring ([kStages][W warps][row A/B][32 lanes] x 16 bytes).  Every lane
// copies exactly the 16 bytes it will consume, so a lane only waits for its
// own copies (cp.async.wait_group) and reads are conflict-free.
template <int NT, int W>
__global__ void __launch_bounds__(W * 32, W == 8 ? 2 : 4) k_lut_mma(const LutLaunch L,
                                                                    const LutPlan P) {
    constexpr int TT = 8 * NT;  // token rows per tile
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint2 *bfrag = reinterpret_cast<uint2 *>(smem_raw);
    uint4 *ring = reinterpret_cast<uint4 *>(smem_raw + (size_t)P.cps_max * NT * 2048);
    __shared__ float s_scale[kTokTile];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gq = lane >> 2, cl = lane & 3;
    const int K = L.K;
    griddep_launch();
    // routed launches: the group tables come from the previous kernels; uniform
    // launches prefetch weights and build tables first (see below)
    if (L.uniform_rows == 0) griddep_wait();
    const int C = P.chunks_total;
    const int64_t rowbytes = K / 2;
    const int tailc = (K & 127) >> 5;  // valid 32-k slices of a ragged last chunk

    // ---- this CTA's range of units (work item * C + chunk)
    int64_t u, u_end;
    int fixed_split = 0;
    if (P.streamk) {
        u = (int64_t)blockIdx.x * P.units / P.grid;
        u_end = ((int64_t)blockIdx.x + 1) * P.units / P.grid;
    } else {
        const int rt = blockIdx.x % P.n_row_tiles;
        fixed_split = blockIdx.x / P.n_row_tiles;
        const int64_t w = (int64_t)blockIdx.y * P.n_row_tiles + rt;
        u = w * C + (int64_t)fixed_split * P.chunks_per_split;
        u_end = min(u + P.chunks_per_split, w * C + C);
    }

    float acc[NT][4];
    uint4 cbv[4];          // codebook rows A and B of a new item, loaded ahead
    bool tables_pending = false;
    int64_t cur_w = -1;
    int cur_s = 0, row0 = 0, nrows = 0, nA = 0, nB = 0;
    const uint8_t *pA = nullptr, *pB = nullptr;
    uint32_t loA[4], hiA[4], loB[4], hiB[4];

    auto flush = [&]() {
        float *out = L.out + (int64_t)cur_s * L.out_split_stride;
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
                        const float sc = s_scale[tok];
                        out[p * L.out_row_stride + nA] = sc * acc[t][e];
                        out[p * L.out_row_stride + nB] = sc * acc[t][2 + e];
                    } else {
                        out[p * L.out_row_stride + nA] = acc[t][e];
                        out[p * L.out_row_stride + nB] = acc[t][2 + e];
                    }
                }
            }
        }
    };

    uint4 *my_slots = ring + (size_t)warp * 64 + lane;  // + (slot * W * 64) + r * 32
    auto issue = [&](int gch, int slot) {
        const bool ok = !(gch == C - 1 && tailc != 0 && cl >= tailc);
        if (ok) {
            uint4 *dst = my_slots + (size_t)slot * W * 64;
            cp_async16(dst, pA + (int64_t)gch * 64 + cl * 16);
            cp_async16(dst + 32, pB + (int64_t)gch * 64 + cl * 16);
        }
    };

    while (u < u_end) {
        const int64_t w = u / C;
        const int ch_lo = (int)(u - w * C);
        const int ch_hi = (int)min((int64_t)C, ch_lo + min(u_end - u, (int64_t)P.cps_max));
        const int nch = ch_hi - ch_lo;
        const bool new_item = (w != cur_w);
        if (new_item) {
            if (cur_w >= 0) flush();
            const int64_t tile = w / P.n_row_tiles;
            const int rt = (int)(w - tile * P.n_row_tiles);
            int g;
            if (L.uniform_rows > 0) {
                const int tpg = (L.uniform_rows + TT - 1) / TT;
                g = (int)(tile / tpg);
                row0 = g * L.uniform_rows + (int)(tile - (int64_t)g * tpg) * TT;
                nrows = min(TT, (g + 1) * L.uniform_rows - row0);
            } else {
                if (tile >= L.grp_tiles[L.G]) return;  // beyond the routed tiles (fixed mode)
                g = L.tile_grp[tile];
                row0 = L.grp_rows[g] + (int)(tile - L.grp_tiles[g]) * TT;
                nrows = min(TT, L.grp_rows[g + 1] - row0);
            }
            cur_w = w;
            cur_s = P.streamk ? (int)(blockIdx.x - lut_cta_of_unit(P, w * C)) : fixed_split;
            const __half *cA, *cB;
            if (L.dual) {
                nA = nB = rt * P.rows_per_rt + warp * 8 + gq;
                pA = L.idx0 + (int64_t)g * L.w_stride + (int64_t)nA * rowbytes;
                pB = L.idx1 + (int64_t)g * L.w_stride + (int64_t)nB * rowbytes;
                cA = reinterpret_cast<const __half *>(L.cb0) + (int64_t)g * L.cb_stride + nA * 16;
                cB = reinterpret_cast<const __half *>(L.cb1) + (int64_t)g * L.cb_stride + nB * 16;
            } else {
                nA = rt * P.rows_per_rt + warp * 16 + gq;
                nB = nA + 8;
                pA = L.idx0 + (int64_t)g * L.w_stride + (int64_t)nA * rowbytes;
                pB = pA + 8 * rowbytes;
                cA = reinterpret_cast<const __half *>(L.cb0) + (int64_t)g * L.cb_stride + nA * 16;
                cB = cA + 8 * 16;
            }
            // the 64 codebook bytes go out ahead of the weight stream (behind
            // several KB of weights per lane they would wait in the DRAM queues),
            // then the stream, whose latency overlaps the set-up below
            cbv[0] = *reinterpret_cast<const uint4 *>(cA);
            cbv[1] = *reinterpret_cast<const uint4 *>(cA + 8);
            cbv[2] = *reinterpret_cast<const uint4 *>(cB);
            cbv[3] = *reinterpret_cast<const uint4 *>(cB + 8);
            tables_pending = true;  // built once the activation loads are out too
            // first stage of the weight stream now; the rest once the set-up
            // loads are out, so they do not queue behind the whole burst
            if (nch > 0) issue(ch_lo, 0);
            cp_async_commit();
#pragma unroll
            for (int t = 0; t < NT; t++)
#pragma unroll
                for (int e = 0; e < 4; e++) acc[t][e] = 0.0f;
            __syncthreads();  // previous piece is done with s_scale / bfrag
            griddep_wait();   // activations and scales come from the previous kernel
            if (tid < TT && L.direct) {
                int cr = -1;
                if (tid < nrows) {
                    const int p = row0 + tid;
                    cr = L.map_mode == kMapPerm ? L.perm[p] / L.topk
                       : L.map_mode == kMapModT ? p % L.T : p;
                }
                s_scale[tid] = cr >= 0 ? L.scales[cr] : 0.0f;
            }
        } else {
            if (nch > 0) issue(ch_lo, 0);
            cp_async_commit();
        }
        __syncthreads();  // bfrag free (the first piece of an item synchronised above)

        // ---- activation fragments for chunks [ch_lo, ch_hi).  An item is the
        // 32 consecutive k of one token that one lane consumes (lane = 4*(token
        // % 8) + k-slice); consecutive threads write consecutive lanes, and each
        // thread issues the wide loads of up to 4 items before converting.
        {
            const int items = nch * NT * 32;  // (chunk, n8 tile, lane)
            constexpr int FB = 4;
            for (int it0 = tid; it0 < items; it0 += FB * W * 32) {
                uint4 raw[FB][2];
#pragma unroll
                for (int f = 0; f < FB; f++) {
                    raw[f][0] = raw[f][1] = make_uint4(0, 0, 0, 0);
                    const int it = it0 + f * W * 32;
                    if (it < items) {
                        const int ln = it & 31, nt = (it >> 5) % NT, ch = (it >> 5) / NT;
                        const int tok = 8 * nt + (ln >> 2);
                        int cr = -1;
                        if (tok < nrows) {
                            const int p = row0 + tok;
                            cr = L.map_mode == kMapPerm ? L.perm[p] / L.topk
                               : L.map_mode == kMapModT ? p % L.T : p;
                        }
                        const int k0 = (ch_lo + ch) * 128 + 32 * (ln & 3);
                        if (cr >= 0 && k0 < K) {
                            const uint8_t *src = L.codes + (int64_t)cr * L.ld_codes;
                            if (L.act_bits == 4) {
                                raw[f][0] = *reinterpret_cast<const uint4 *>(src + k0 / 2);
                            } else {
                                raw[f][0] = *reinterpret_cast<const uint4 *>(src + k0);
                                raw[f][1] = *reinterpret_cast<const uint4 *>(src + k0 + 16);
                            }
                        }
                    }
                }
                if (tables_pending) {  // the codebook loads went out with the weights
                    build_tables(cbv[0], cbv[1], loA, hiA);
                    build_tables(cbv[2], cbv[3], loB, hiB);
                    tables_pending = false;
                }
#pragma unroll
                for (int f = 0; f < FB; f++) {
                    const int it = it0 + f * W * 32;
                    if (it < items) {
                        const int ln = it & 31, nt = (it >> 5) % NT, ch = (it >> 5) / NT;
                        const uint32_t wd[8] = {raw[f][0].x, raw[f][0].y, raw[f][0].z,
                                                raw[f][0].w, raw[f][1].x, raw[f][1].y,
                                                raw[f][1].z, raw[f][1].w};
#pragma unroll
                        for (int i = 0; i < 8; i++) {
                            // codes of k0 + 4i .. k0 + 4i + 3
                            __align__(8) __half v[4];
                            if (L.act_bits == 4) {
                                const uint32_t x = wd[i >> 1] >> (16 * (i & 1));
#pragma unroll
                                for (int e = 0; e < 4; e++)
                                    v[e] = code_to_half(((int)(x << (28 - 4 * e))) >> 28);
                            } else {
#pragma unroll
                                for (int e = 0; e < 4; e++)
                                    v[e] = code_to_half(((int)(wd[i] << (24 - 8 * e))) >> 24);
                            }
                            bfrag[((ch * 8 + i) * NT + nt) * 32 + ln] =
                                *reinterpret_cast<const uint2 *>(v);
                        }
                    }
                }
            }
        }
        if (tables_pending) {  // no activation items for this thread
            build_tables(cbv[0], cbv[1], loA, hiA);
            build_tables(cbv[2], cbv[3], loB, hiB);
            tables_pending = false;
        }
#pragma unroll
        for (int sl = 1; sl < kStages - 1; sl++) {
            if (sl < nch) issue(ch_lo + sl, sl);
            cp_async_commit();
        }
        __syncthreads();

        // ---- the chunk pipeline
        for (int ch = 0; ch < nch; ch++) {
            cp_async_wait<kStages - 2>();
            const int gch = ch_lo + ch;
            const bool ok = !(gch == C - 1 && tailc != 0 && cl >= tailc);
            const uint4 *src = my_slots + (size_t)(ch % kStages) * W * 64;
            uint4 ra = ok ? src[0] : make_uint4(0, 0, 0, 0);
            uint4 rb = ok ? src[32] : make_uint4(0, 0, 0, 0);
            if (ch + kStages - 1 < nch) issue(gch + kStages - 1, (ch + kStages - 1) % kStages);
            cp_async_commit();
            const uint32_t wa[4] = {ra.x, ra.y, ra.z, ra.w};
            const uint32_t wb[4] = {rb.x, rb.y, rb.z, rb.w};
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
        u += nch;
    }
    if (cur_w >= 0) flush();
}

int sm_count() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

LutPlan plan_lut(int N, int K, bool dual, int max_rows_per_group, int64_t est_tiles,
                 int uniform_rows, int n_groups) {
    LutPlan P{};
    P.nt = max_rows_per_group <= 8 ? 1 : 2;
    const int tt = 8 * P.nt;
    // 8 warps when the row tile divides N, else 4
    P.warps = (dual ? N % 64 == 0 : N % 128 == 0) ? 8 : 4;
    P.rows_per_rt = dual ? 8 * P.warps : 16 * P.warps;
    P.n_row_tiles = N / P.rows_per_rt;
    P.chunks_total = (K + 127) / 128;
    const int ctas_per_sm = P.warps == 8 ? 2 : 4;  // what __launch_bounds__ and smem allow
    const size_t smem_cap = (size_t)(227 * 1024) / ctas_per_sm - 1024;
    const size_t ring = (size_t)kStages * P.warps * 1024;
    const size_t per_chunk = (size_t)P.nt * 2048;
    P.cps_max = (int)std::min<size_t>(32, (smem_cap - ring) / per_chunk);
    const int capacity = sm_count() * ctas_per_sm;
    const int C = P.chunks_total;
    if (uniform_rows > 0) {
        const int64_t tiles = (int64_t)n_groups * ((uniform_rows + tt - 1) / tt);
        P.streamk = 1;
        P.uniform_rows = uniform_rows;
        P.units = tiles * P.n_row_tiles * C;
        P.grid = (int)std::min<int64_t>(capacity, P.units);
        // partial slots: the most CTAs that share one work item
        int smax = 1;
        const int64_t items = tiles * P.n_row_tiles;
        for (int64_t w = 0; w < items; w++) smax = std::max(smax, lut_item_splits(P, w));
        P.splits = smax;
        P.chunks_per_split = P.cps_max;
    } else {
        P.streamk = 0;
        const int64_t base = (int64_t)P.n_row_tiles * std::max<int64_t>(est_tiles, 1);
        int splits = base < capacity ? (int)(capacity / base) : 1;
        const int min_splits = (C + P.cps_max - 1) / P.cps_max;
        splits = std::max(std::min(splits, C), min_splits);
        P.chunks_per_split = (C + splits - 1) / splits;
        P.splits = (C + P.chunks_per_split - 1) / P.chunks_per_split;
        P.grid = P.n_row_tiles * P.splits;
        P.cps_max = P.chunks_per_split;  // the activation region holds one split
    }
    P.smem = ring + per_chunk * P.cps_max;
    return P;
}

template <int NT, int W>
static cudaError_t launch_lut_t(const LutLaunch &L, const LutPlan &P, cudaStream_t st) {
    dim3 grid(P.grid, P.streamk ? 1 : L.max_tiles);
    return launch_pdl(k_lut_mma<NT, W>, grid, dim3(W * 32), P.smem, st, 1, L, P);
}

cudaError_t launch_lut(const LutLaunch &L, const LutPlan &P, cudaStream_t st) {
    if (P.grid == 0 || (!P.streamk && L.max_tiles == 0)) return cudaSuccess;
    const bool timed = timing_on();
    if (timed) timing_begin(st, CQ_KERNEL_LUT_MMA);
    count_launch();
    if (P.nt == 1)
        P.warps == 8 ? launch_lut_t<1, 8>(L, P, st) : launch_lut_t<1, 4>(L, P, st);
    else
        P.warps == 8 ? launch_lut_t<2, 8>(L, P, st) : launch_lut_t<2, 4>(L, P, st);
    if (timed) timing_end(st);
    return cudaGetLastError();
}

// ---------------------------------------------------------------- split-K reduce
// grid: (column blocks of 256, M rows)
__global__ void __launch_bounds__(256) k_reduce_plain(const float *__restrict__ part, const LutPlan P,
                                                      int64_t M, int64_t N, const float *__restrict__ s,
                                                      float *__restrict__ y) {
    __shared__ int s_ns[8];
    griddep_wait();
    griddep_launch();
    const int64_t m = blockIdx.y;
    const int n0 = blockIdx.x * 256;
    const int rt0 = n0 / P.rows_per_rt;
    const int nrt = (min((int64_t)n0 + 255, N - 1)) / P.rows_per_rt - rt0 + 1;
    if (threadIdx.x < nrt) s_ns[threadIdx.x] = lut_splits_at(P, m, (rt0 + threadIdx.x) * P.rows_per_rt);
    __syncthreads();
    const int n = n0 + threadIdx.x;
    if (n >= N) return;
    const int64_t i = m * N + n;
    const float *pp[1] = {part + i};
    const int ns[1] = {s_ns[n / P.rows_per_rt - rt0]};
    float acc[1] = {0.0f};
    sum_slots<1, 8>(pp, ns, M * N, acc);
    y[i] = s[m] * acc[0];
}

cudaError_t launch_reduce_plain(const float *part, const LutPlan &P, int64_t M, int64_t N,
                                const float *s, float *y, cudaStream_t st) {
    const int64_t n = M * N;
    if (n == 0) return cudaSuccess;
    TimedScope ts(st, CQ_KERNEL_REDUCE);
    count_launch();
    dim3 grid((unsigned)((N + 255) / 256), (unsigned)M);
    return launch_pdl(k_reduce_plain, grid, dim3(256), 0, st, 1, part, P, M, N, s, y);
}

// ---------------------------------------------------------------- centroid sums (parity)
// S[m, n, c] = sum_{k : I[n,k] = c} q[m,k]; one thread per (m, n).
__global__ void k_centroid_sums(const uint8_t *__restrict__ q, int64_t M, int64_t K, int bits,
                                const uint8_t *__restrict__ w_idx, int64_t N, int32_t *S) {
    griddep_wait();
    griddep_launch();
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
    TimedScope ts(st, CQ_KERNEL_CENTROID_SUMS);
    count_launch();
    return launch_pdl(k_centroid_sums, dim3((unsigned)((n + 127) / 128)), dim3(128), 0, st, 1,
                      reinterpret_cast<const uint8_t *>(q), M, K, bits, w_idx, N, S);
}

}  // namespace cq
