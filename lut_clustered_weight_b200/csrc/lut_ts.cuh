// lut_ts.cuh -- LUT (codebook) GEMM for token groups of at most 32 rows on the
// sm_100a tensor cores: the decode kernel.  Included by kernels_lut_tc.cu only
// (it shares that unit's device error word and tensor-map encoder).
//
//   y[m, n] = s_x[m] * sum_k C[n, I[n,k]] * q[m, k]
//
// CodeQuant2 Figure 4: a one-time LUT precompute held in shared memory, then
// table lookups.  Here the precompute is, per weight row, the 256-entry pair
// table T[b] = (C[b & 15], C[b >> 4]) (the two fp16 centroids an index byte b
// selects).  One thread owns one weight row of a 128-row tile, so the table
// entries of the 32 rows a warp serves sit in 32 different banks (entry b of
// row t at (128 b + t) * 4): every lookup is conflict-free whatever the
// indices, with no replicated tables.  A lookup turns one index byte into the
// fp16 pair of two weights.
//
// The looked-up pairs are stored to tensor memory (row t = TMEM lane t) and
// are the A operand of tcgen05.mma kind::f16 (M = 128, K = 16); the tokens are
// N (16 or 32), their int codes as fp16 (exact) the B operand.  On B200 such
// an MMA issues every ~50-60 cycles for any N <= 64: 2048 weights, i.e. ~0.8
// of the HBM rate of 4-bit indices per SM.
//
// Roles (one CTA per SM, persistent over stream-K or fixed-split work):
//   warps 0-7   expand: warp w serves TMEM lane quarter w % 4 and half
//               w / 4 of every 256-k group (64 index bytes of its row);
//               builds the pair tables, looks up, stores A, drains the
//               accumulator (fp32 partial sums) once a segment is done
//   warp 8      lane 0 issues the MMAs; the warp owns the TMEM allocation
//   warp 9      lane 0 streams the index bytes: one 2-D TMA tile (128 rows x
//               128 B, 128-byte swizzle) per group into a 4-stage ring
//   warp 10     lane 0 loads the B tiles (fp16 codes, 64 k x NTOK rows,
//               128-byte swizzle) per group into their own ring, ahead of
//               the MMAs, which consume them later than the index bytes
// Rings: index stages (4), A slots in TMEM (3 groups, columns [0, 384)), B
// stages, accumulators (2 x NTOK columns after the A ring, so a segment's
// drain overlaps the next segment's MMAs).  Every wait is bounded.
#pragma once

namespace cq {

// Timeline hooks for tuning (global-timer stamps per role and group); compiled
// out unless the library is built with CQ_TS_TRACE.
#ifdef CQ_TS_TRACE
constexpr int kTsTraceSlots = 2048;
__device__ unsigned long long g_ts_trace[160 * kTsTraceSlots];
// slot 2047: global timer at the start of the CTA; other slots: SM clock
#define TS_TRACE(slot)                                                              \
    do {                                                                            \
        const int s_ = (slot);                                                      \
        if (s_ >= 0 && s_ < kTsTraceSlots && blockIdx.x < 160)                      \
            g_ts_trace[blockIdx.x * kTsTraceSlots + s_] = clock64();                \
    } while (0)
#define TS_TRACE_ANCHOR()                                                           \
    do {                                                                            \
        if (blockIdx.x < 160)                                                       \
            g_ts_trace[blockIdx.x * kTsTraceSlots + 2047] = globaltimer_ns();       \
    } while (0)
#else
#define TS_TRACE(slot) \
    do {               \
    } while (0)
#define TS_TRACE_ANCHOR() \
    do {                  \
    } while (0)
#endif

constexpr int kTsExpandWarps = 8;
constexpr int kTsWarpMma = 8;
constexpr int kTsWarpTma = 9;
constexpr int kTsWarpB = 10;
constexpr int kTsThreads = 32 * 11;
constexpr int kTsA = 3;                      // A slots (groups) in TMEM
constexpr int kTsI = 4;                      // index stages
constexpr uint32_t kTsIStage = kTcRows * 128;  // one group of 128 rows: 16 KB
constexpr uint32_t kTsTableBytes = 256 * kTcRows * 4;  // 128 KB

template <int NTOK>
struct TsShape {
    static_assert(NTOK == 16 || NTOK == 32, "token tiles of 16 or 32 rows");
    static constexpr int nb = NTOK == 16 ? 4 : 2;          // B stages (groups)
    static constexpr uint32_t b_chunk = NTOK * 128;        // one 64-k chunk tile
    static constexpr uint32_t b_stage = kTcG * b_chunk;    // one group
    static constexpr size_t smem = 1024 + kTsI * kTsIStage + nb * b_stage + kTsTableBytes + 512;
};

template <int NTOK>
__global__ void __launch_bounds__(kTsThreads, 1)
k_lut_ts(const __grid_constant__ CUtensorMap tmI0, const __grid_constant__ CUtensorMap tmI1,
         const __grid_constant__ CUtensorMap tmB, const LutLaunch L, const LutPlan P,
         int b_row_mod) {
    using Sh = TsShape<NTOK>;
    constexpr int NB = Sh::nb;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t *sm = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    uint8_t *istages = sm;                                   // [kTsI][128 rows][128 B]
    uint8_t *bstages = istages + kTsI * kTsIStage;           // [NB][4 chunks][NTOK][128 B]
    uint8_t *tables = bstages + NB * Sh::b_stage;            // [256 entries][128 rows] x 4 B
    uint64_t *i_full = reinterpret_cast<uint64_t *>(tables + kTsTableBytes);
    uint64_t *i_empty = i_full + kTsI;
    uint64_t *a_full = i_empty + kTsI, *a_empty = a_full + kTsA;
    uint64_t *b_full = a_empty + kTsA, *b_empty = b_full + NB;
    uint64_t *d_full = b_empty + NB, *d_empty = d_full + 2;
    uint64_t *tab_free = d_empty + 2, *tab_ready = tab_free + 4, *fin = tab_ready + 4;
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(fin + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const TcSchedule S{&L, &P};
    const bool tr0 = tid == 0;  // trace: expand warp 0
    if (tr0) {
        TS_TRACE(0);
        TS_TRACE_ANCHOR();
    }

    if (warp == kTsWarpMma) {
        tmem_alloc(s_tmem, 512);
        tmem_relinquish();
        if (lane == 0) {
            for (int s = 0; s < kTsA; s++) {
                mbar_init(&a_full[s], kTsExpandWarps);
                mbar_init(&a_empty[s], 1);
            }
            for (int s = 0; s < NB; s++) {
                mbar_init(&b_full[s], 1);
                mbar_init(&b_empty[s], 1);
            }
            for (int s = 0; s < 2; s++) {
                mbar_init(&d_full[s], 1);
                mbar_init(&d_empty[s], kTsExpandWarps);
            }
            for (int qq = 0; qq < 4; qq++) {
                mbar_init(&tab_free[qq], 2);
                mbar_init(&tab_ready[qq], 2);
            }
            mbar_init(fin, 1);
            fence_barrier_init();
        }
    }
    // routed launches: the group tables come from the previous kernels.  A
    // uniform launch reads only weights until its activations (B loads) and
    // outputs (drains), so its set-up overlaps the previous kernel.
    const bool routed = L.uniform_rows == 0;
    // index stream: the first stages go out before the CTA barrier (uniform
    // launches), the HBM latency of the weights overlaps the set-up
    TcWalk tw{};
    int tgi = 0;
    auto issue_index = [&]() {
        const int s = tgi % kTsI;
        int g, row0, nrows, rt;
        S.item(tw.w, g, row0, nrows, rt);
        mbar_arrive_expect_tx(&i_full[s], kTsIStage);
        uint8_t *dst = istages + s * kTsIStage;
        const int x = tw.c0 * (kTcChunk / 2);  // byte offset of the group in a row
        if (L.dual) {
            const int y = max(g, 0) * L.N + rt * 64;
            tma_load_2d(dst, &tmI0, x, y, &i_full[s]);
            tma_load_2d(dst + kTsIStage / 2, &tmI1, x, y, &i_full[s]);
        } else {
            tma_load_2d(dst, &tmI0, x, max(g, 0) * L.N + rt * kTcRows, &i_full[s]);
        }
        TS_TRACE(1400 + tgi);
        tgi++;
        tw.next();
    };
    if (warp == kTsWarpTma && lane == 0) {
        for (int s = 0; s < kTsI; s++) {
            mbar_init(&i_full[s], 1);
            mbar_init(&i_empty[s], kTsExpandWarps);
        }
        fence_barrier_init();
        prefetch_tmap(&tmI0);
        if (L.dual) prefetch_tmap(&tmI1);
        if (!routed) {
            tw.init(P, 0);
            while (tw.valid && tgi < kTsI) issue_index();
        }
    }
    if (warp == kTsWarpB && lane == 0) prefetch_tmap(&tmB);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    griddep_launch();
    if (routed) griddep_wait();
    const uint32_t tmem = *s_tmem;
    const uint32_t tmem_a = tmem;                      // columns [0, 384): A slots
    const uint32_t tmem_d = tmem + kTsA * 128;         // [384, 384 + 2 NTOK): accumulators
    const int n_pieces = tc_pieces(L, P);
    if (tr0) TS_TRACE(1);

    if (warp == kTsWarpTma) {
        // ====================== index stream (one thread) ======================
        if (lane == 0) {
            if (routed) tw.init(P, n_pieces);
            TS_TRACE(1399);
            while (tw.valid) {
                const int s = tgi % kTsI;
                if (tgi >= kTsI && !mbar_wait(&i_empty[s], (uint32_t)(tgi / kTsI - 1) & 1u)) break;
                issue_index();
            }
            // loads still in flight land before the CTA may leave
            for (int j = max(0, tgi - kTsI); j < tgi; j++)
                mbar_wait(&i_full[j % kTsI], (uint32_t)(j / kTsI) & 1u);
        }
    } else if (warp == kTsWarpMma) {
        // ====================== MMA issue (one thread) ======================
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_f16(kTcRows, NTOK);
            TcWalk mw;
            mw.init(P, n_pieces);
            int segs = 0;
            bool ok = true;
            for (int gi = 0; mw.valid && ok; gi++, mw.next()) {
                const int slot = gi % kTsA, bs = gi % NB;
                const bool first = mw.seg_first(), last = mw.seg_last();
                const int buf = segs & 1;
                if (first && segs >= 2)
                    ok = mbar_wait(&d_empty[buf], (uint32_t)(segs / 2 - 1) & 1u, 32);
                ok = ok && mbar_wait(&a_full[slot], (uint32_t)(gi / kTsA) & 1u, 32);
                TS_TRACE(700 + 3 * gi);
                ok = ok && mbar_wait(&b_full[bs], (uint32_t)(gi / NB) & 1u, 32);
                TS_TRACE(701 + 3 * gi);
                if (!ok) break;
                tc_fence_after();
                for (int i = 0; i < mw.gn; i++) {
                    const uint64_t bd =
                        smem_desc_sw128(smem_u32(bstages + bs * Sh::b_stage + i * Sh::b_chunk));
#pragma unroll
                    for (int kk = 0; kk < kTcChunk / 16; kk++)
                        tc_mma_ts(tmem_d + buf * NTOK, tmem_a + slot * 128 + i * 32 + kk * 8,
                                  bd + (uint64_t)(2 * kk), idesc,
                                  (first && i == 0 && kk == 0) ? 0u : 1u);
                }
                tc_commit(&b_empty[bs]);
                tc_commit(&a_empty[slot]);
                TS_TRACE(702 + 3 * gi);
                if (last) {
                    tc_commit(&d_full[buf]);
                    segs++;
                }
            }
            // every MMA is complete before tensor memory is freed
            tc_commit(fin);
            mbar_wait(fin, 0);
        }
    } else if (warp < kTsExpandWarps) {
        // ====================== expand + drain ======================
        const int q = warp & 3, h = warp >> 2;
        const int t = q * 32 + lane;                 // row of the tile = TMEM lane
        const uint32_t lane_base = ((uint32_t)(q * 32)) << 16;
        const int srow = L.dual ? ((t & 1) * 64 + (t >> 1)) : t;  // row in an index stage
        uint32_t *tab = reinterpret_cast<uint32_t *>(tables) + t;  // entry b at tab[128 b]
        const uint32_t tab_s = smem_u32(tab);
        bool ok = true, waited = routed;
        // the accumulator of a finished segment, drained once the next
        // segment's first group is out (or at the end)
        bool pend = false;
        int pend_buf = 0, pend_ph = 0, pend_row0 = 0, pend_nrows = 0, pend_col = 0, pend_slot = 0;
        auto drain = [&]() {
            if (!waited) {
                griddep_wait();  // no global write before the previous kernel is done
                waited = true;
            }
            ok = mbar_wait(&d_full[pend_buf], (uint32_t)pend_ph);
            if (!ok) return;
            tc_fence_after();
            constexpr int HC = NTOK / 2;  // token columns of this warp
            uint32_t d[HC];
            tmem_ld_cols(tmem_d + lane_base + pend_buf * NTOK + h * HC, d);
            tmem_wait_ld();
            float *out = L.out + (int64_t)pend_slot * L.out_split_stride;
#pragma unroll
            for (int c = 0; c < HC; c++) {
                const int tok = h * HC + c;
                if (tok < pend_nrows)
                    out[(int64_t)(pend_row0 + tok) * L.out_row_stride + pend_col] =
                        __uint_as_float(d[c]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&d_empty[pend_buf]);
        };
        auto codebook = [&](const TcWalk &wk, uint4 &c0, uint4 &c1) {
            if (!wk.valid) return;
            int gg, r0, nr, rtt, cc;
            const uint8_t *ip;
            const __half *cbp;
            S.item(wk.w, gg, r0, nr, rtt);
            S.row_ptrs(max(gg, 0), rtt, t, ip, cbp, cc);
            c0 = ldg_stream(cbp);
            c1 = ldg_stream(cbp + 8);
        };
        TcWalk cw;
        cw.init(P, n_pieces);
        uint4 cbn0 = make_uint4(0, 0, 0, 0), cbn1 = cbn0;  // codebook of the coming segment
        codebook(cw, cbn0, cbn1);
        int segs = 0, row0 = 0, nrows = 0, col = 0;
        for (int gi = 0; cw.valid && ok; gi++, cw.next()) {
            const int slot = gi % kTsA, is = gi % kTsI;
            if (cw.seg_first()) {
                int g, rt;
                S.item(cw.w, g, row0, nrows, rt);
                const uint8_t *ip;
                const __half *cbp;
                S.row_ptrs(max(g, 0), rt, t, ip, cbp, col);
                if (segs > 0) {
                    // both warps of the quarter are done with the previous table
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&tab_free[q]);
                    ok = mbar_wait(&tab_free[q], (uint32_t)(segs - 1) & 1u);
                    if (!ok) break;
                }
                if (tr0) TS_TRACE(650 + segs);
                const uint4 c0v = cbn0, c1v = cbn1;
                {
                    TcWalk nx = cw;  // prefetch the next segment's codebook
                    nx.c0 = nx.c_end;
                    nx.next();
                    codebook(nx, cbn0, cbn1);
                }
                // the one-time LUT precompute: this warp builds entries
                // [128 h, 128 h + 128) of its 32 rows' pair tables
                const uint32_t cu[8] = {c0v.x, c0v.y, c0v.z, c0v.w, c1v.x, c1v.y, c1v.z, c1v.w};
#pragma unroll
                for (int i = 0; i < 8; i++) {
                    const int hh = 8 * h + i;  // high nibble of the entries
                    const uint32_t wv = h ? cu[4 + (i >> 1)] : cu[i >> 1];
                    const uint32_t hv = (i & 1) ? (wv >> 16) : (wv & 0xFFFFu);
#pragma unroll
                    for (int l = 0; l < 16; l++)
                        tab[(hh * 16 + l) * kTcRows] =
                            prmt(cu[l >> 1], hv, (l & 1) ? 0x5432u : 0x5410u);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&tab_ready[q]);
                ok = mbar_wait(&tab_ready[q], (uint32_t)segs & 1u);
                if (tr0) TS_TRACE(600 + segs);
                if (!ok) break;
            }
            // this thread's 64 index bytes of the group (chunks 2h, 2h + 1)
            if (!mbar_wait(&i_full[is], (uint32_t)(gi / kTsI) & 1u)) {
                ok = false;
                break;
            }
            if (tr0) TS_TRACE(2 + 5 * gi);
            uint32_t wd[16];
            {
                const uint8_t *rp = istages + is * kTsIStage + srow * 128;
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    const int j = 4 * h + i;  // 16-byte chunk of the 128-byte row
                    const uint4 v4 = *reinterpret_cast<const uint4 *>(rp + ((j ^ (srow & 7)) << 4));
                    wd[4 * i] = v4.x;
                    wd[4 * i + 1] = v4.y;
                    wd[4 * i + 2] = v4.z;
                    wd[4 * i + 3] = v4.w;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&i_empty[is]);
            const bool mine = 2 * h < cw.gn;
            uint32_t v[64];
            if (mine) {
#pragma unroll
                for (int b = 0; b < 64; b++) {
                    const uint32_t byte = prmt(wd[b >> 2], 0u, 0x4440u | (uint32_t)(b & 3));
                    v[b] = lds32(tab_s + byte * (kTcRows * 4));
                }
            }
            if (tr0) TS_TRACE(3 + 5 * gi);
            if (gi >= kTsA) {
                ok = mbar_wait(&a_empty[slot], (uint32_t)(gi / kTsA - 1) & 1u);
                if (!ok) break;
                tc_fence_after();
            }
            if (tr0) TS_TRACE(4 + 5 * gi);
            if (mine) {
                const uint32_t ta = tmem_a + lane_base + slot * 128 + h * 64;
                tmem_st32(ta, *reinterpret_cast<const uint32_t(*)[32]>(&v[0]));
                if (2 * h + 1 < cw.gn)
                    tmem_st32(ta + 32, *reinterpret_cast<const uint32_t(*)[32]>(&v[32]));
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&a_full[slot]);
            if (tr0) TS_TRACE(5 + 5 * gi);
            if (pend) {
                drain();
                pend = false;
                if (tr0) TS_TRACE(6 + 5 * gi);
                if (!ok) break;
            }
            if (cw.seg_last()) {
                pend = true;
                pend_buf = segs & 1;
                pend_ph = (segs >> 1) & 1;
                pend_row0 = row0;
                pend_nrows = nrows;
                pend_col = col;
                pend_slot = cw.slot;
                segs++;
            }
        }
        if (pend && ok) drain();
    } else if (warp == kTsWarpB) {
        // ====================== B tiles (one thread) ======================
        if (lane == 0) {
            if (!routed) griddep_wait();  // the fp16 codes come from the previous kernel
            TcWalk w;
            w.init(P, n_pieces);
            int gi = 0, b_y = 0;
            for (; w.valid; w.next(), gi++) {
                const int s = gi % NB;
                if (gi >= NB && !mbar_wait(&b_empty[s], (uint32_t)(gi / NB - 1) & 1u)) break;
                if (w.seg_first()) {
                    int g, row0, nrows, rt;
                    S.item(w.w, g, row0, nrows, rt);
                    b_y = b_row_mod > 0 ? row0 % b_row_mod : row0;
                }
                mbar_arrive_expect_tx(&b_full[s], Sh::b_chunk * w.gn);
                for (int i = 0; i < w.gn; i++)
                    tma_load_2d(bstages + s * Sh::b_stage + i * Sh::b_chunk, &tmB,
                                (w.c0 + i) * kTcChunk, b_y, &b_full[s]);
            }
            for (int j = max(0, gi - NB); j < gi; j++)
                mbar_wait(&b_full[j % NB], (uint32_t)(j / NB) & 1u);
        }
    }
    // ---- teardown: all MMAs and tensor-memory reads are complete
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kTsWarpMma) tmem_dealloc(tmem, 512);
    if (tr0) TS_TRACE(1999);
}

}  // namespace cq
