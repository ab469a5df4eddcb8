// kernels_lut_tc.cu -- LUT (codebook) GEMM on the sm_100a tensor cores
// (tcgen05 / tensor memory).
//
//   y[m, n] = s_x[m] * sum_k C[n, I[n,k]] * q[m, k]
//
// CodeQuant2 Figure 4 describes the LUT kernel as a one-time LUT precompute
// held in shared memory followed by table lookups.  Here:
//  * Four threads per weight row: row t of a 128-row tile is lane t of tensor
//    memory (TMEM); of the sixteen "expand" warps, warps w, w + 4, w + 8 and
//    w + 12 serve TMEM lane quarter w, each taking one 64-k chunk of every
//    4-chunk (256-k) group.
//  * PAIR mode (16-token tiles): the one-time precompute is a 256-entry pair
//    table per row in shared memory -- entry b holds the two fp16 centroids
//    selected by an index byte b (low nibble = even k).  Entry b of thread t
//    sits at b * 512 + 4 t, so the 32 lanes of a warp always hit 32 different
//    banks, whatever the indices.  One byte (two weights) costs one byte
//    extract, one address multiply-add and one 4-byte shared load.
//  * PRMT mode (64- to 256-token tiles): the codebook is held as two
//    byte-plane tables in registers and looked up with byte permutes; no
//    shared memory is spent on tables, which leaves room for wide B tiles.
//  * The looked-up fp16 weights of a group are stored to TMEM (tcgen05.st,
//    32 columns per row and chunk, a 2-group ring) and used as the A operand
//    of tcgen05.mma kind::f16; the activations (int codes converted to fp16,
//    exact) are the B operand, 128-byte-swizzled shared tiles loaded by TMA.
//    The fp32 accumulator lives in TMEM and is read back with tcgen05.ld; the
//    epilogue writes fp32 partial sums, or fp16 h = silu(s g) (s u) when the
//    launch has one partial slot per output (SwiGLU fused; for 256-token
//    tiles staged in shared memory and written as whole 128-byte rows).  A
//    finished item is drained after the next item's first group; tiles of up
//    to 128 tokens keep two accumulators, so the drain overlaps MMAs.
//  * Roles: warps 0-15 expand (each thread streams its row's index bytes
//    through a private cp.async ring) and drain the accumulator; lane 0 of
//    warp 16 issues the MMAs; lane 0 of warp 17 issues the TMA loads of the
//    activation tiles.  mbarriers connect them (the A ring per slot and
//    chunk); every wait is bounded.
//  * Persistent: one CTA per SM works through (128-row tile x token tile)
//    items cut into 64-k chunks -- contiguous stream-K ranges when there are
//    few items, else whole (item, split) pieces strided over the CTAs.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "cq_common.cuh"
#include "cq_internal.h"
#include "lut_lookup.cuh"
#include "sm100.cuh"
#include "tc_walk.cuh"
#include "lut_ts.cuh"

namespace cq {

// Expand warps per TMEM lane quarter; each takes kTcG / kTcWq chunks of every
// group.  Four warps per quarter (one 64-k chunk each) keep four expand warps
// on every SM sub-partition, so one warp's index loads and tensor-memory
// stores overlap the others' lookups.
constexpr int kTcWq = 4;
constexpr int kTcCpw = kTcG / kTcWq;              // chunks per expand warp and group
constexpr int kTcPieces = 2 * kTcCpw;             // 16-byte index pieces per thread and group
constexpr int kTcExpandWarps = 4 * kTcWq;
constexpr int kTcExpand = kTcExpandWarps * 32;
constexpr int kWarpMma = kTcExpandWarps;          // TMEM allocation + MMA issue (lane 0)
constexpr int kWarpTma = kTcExpandWarps + 1;      // B tile loads (lane 0)
constexpr int kTcThreads = kTcExpand + 64;
constexpr int kTcA = 2;              // A ring depth in groups (TMEM columns [0, 256))
// B ring (shared memory, NTOK x 128 B per chunk tile): kTcB stages of kBG
// chunk tiles; a stage is freed by the commit of the MMAs that read it.
// Small token tiles take a whole group per stage (one wait and one commit
// per group instead of per chunk).
template <int NTOK> struct TcB { static constexpr int n = NTOK <= 64 ? 4 : NTOK <= 128 ? 8 : 4; };
template <int NTOK> struct TcBG { static constexpr int n = NTOK <= 64 ? kTcG : 1; };
// Independent accumulators: a chain of small MMAs into one accumulator is
// bound by the MMA latency, so tiles of few tokens spread the four K steps
// of a chunk over four accumulators (summed in the epilogue).
template <int NTOK> struct TcAcc { static constexpr int n = NTOK <= 32 ? 4 : 1; };
// Tiles of up to 128 tokens keep two accumulator buffers (2 x 128 TMEM
// columns beside the A ring): the MMAs of one work item run while the
// previous item's accumulator is drained.
template <int NTOK> struct TcDB { static constexpr bool on = NTOK <= 128; };
constexpr int kTcWStages = 4;        // index-byte ring per thread, in groups (3 in flight)
constexpr size_t kPairTableBytes = 256 * kTcRows * 4;  // 128 KB
// 256-token tiles with SwiGLU in the epilogue: h of one item is staged in
// shared memory per expand-warp group (64 tokens x 64 columns, fp16) and
// written as whole 128-byte rows
template <int NTOK> struct TcHStage { static constexpr size_t bytes = NTOK == 256 ? kTcWq * 64 * 128 : 0; };

// 18 warps: five on two of the four SM sub-partitions, whose register files
// hold 16K registers each, so at most 96 registers per thread.
template <int NTOK, bool PAIR>
__global__ void __launch_bounds__(kTcThreads, 1)
k_lut_tc(const __grid_constant__ CUtensorMap tmB, const LutLaunch L, const LutPlan P, int b_row_mod) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t pad = ((raw_addr + 1023u) & ~1023u) - raw_addr;
    uint8_t *sm = smem_raw + pad;
    constexpr uint32_t kBSlot = NTOK * 128;  // bytes of one B chunk tile
    constexpr int kTcB = TcB<NTOK>::n;
    constexpr int kBG = TcBG<NTOK>::n;
    constexpr int kAcc = TcAcc<NTOK>::n;
    uint8_t *bslots = sm;                                     // [kTcB][kBG][NTOK][128 B]
    uint8_t *tables = sm + kTcB * kBG * kBSlot;               // PAIR: [256][128 rows] x 4 B
    uint8_t *wring_raw = tables + (PAIR ? kPairTableBytes : 0);  // [stage][pieces][thr] x 16 B
    uint8_t *hstage = wring_raw + kTcWStages * kTcPieces * kTcExpand * 16;  // [kTcWq][64][128 B]
    uint64_t *bars = reinterpret_cast<uint64_t *>(hstage + TcHStage<NTOK>::bytes);
    // A ring barriers per (slot, chunk): the expand warps of one chunk and the
    // MMAs of that chunk hand a TMEM slot back and forth on their own, so the
    // warps of a lane quarter do not run in lockstep
    uint64_t *a_full = bars, *a_empty = bars + kTcA * kTcG;  // [kTcA][kTcG]
    uint64_t *b_full = bars + 2 * kTcA * kTcG, *b_empty = b_full + kTcB;
    uint64_t *d_full = b_empty + kTcB, *d_empty = d_full + 2, *fin = d_full + 4;  // d_*: [2]
    uint64_t *tab_ready = fin + 1;  // [4]: PAIR table of a lane quarter built
    uint64_t *tab_free = tab_ready + 4;  // [4]: both warps of the quarter done with it
    uint64_t *hs_bar = tab_free + 4;     // [kTcWq]: staged h of a token range (4 warps)
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(hs_bar + kTcWq);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool tr0 = tid == 0;  // trace: expand warp 0
    if (tr0) {
        TS_TRACE(0);
        TS_TRACE_ANCHOR();
    }
    constexpr bool kDB = TcDB<NTOK>::on;
    constexpr uint32_t kTmemCols = 512;  // A ring 256 + (kDB ? 2 : 1) x kAcc x NTOK (<= 256)
    static_assert(kTcA * 128 + (kDB ? 2 : 1) * kAcc * NTOK <= (int)kTmemCols, "TMEM columns");
    const TcSchedule S{&L, &P};

    if (warp == kWarpMma) {
        tmem_alloc(s_tmem, kTmemCols);
        tmem_relinquish();
        if (lane == 0) {
            for (int s = 0; s < kTcA * kTcG; s++) {
                mbar_init(&a_full[s], 4);  // the chunk's warp in each lane quarter
                mbar_init(&a_empty[s], 1);
            }
            for (int s = 0; s < kTcB; s++) {
                mbar_init(&b_full[s], 1);
                mbar_init(&b_empty[s], 1);
            }
            for (int bb = 0; bb < 2; bb++) {
                mbar_init(&d_full[bb], 1);
                mbar_init(&d_empty[bb], kTcExpandWarps);
            }
            mbar_init(fin, 1);
            for (int qq = 0; qq < 4; qq++) {
                mbar_init(&tab_ready[qq], kTcWq);
                mbar_init(&tab_free[qq], kTcWq);
            }
            for (int hh = 0; hh < kTcWq; hh++) mbar_init(&hs_bar[hh], 4);
            fence_barrier_init();
            prefetch_tmap(&tmB);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // everything below may read what the previous kernels wrote
    griddep_wait();
    griddep_launch();
    const uint32_t tmem = *s_tmem;
    const uint32_t tmem_a = tmem;                 // columns [0, 256): A ring (2 x 128)
    const uint32_t tmem_d = tmem + kTcA * 128;    // columns [256, 256 + (1|2) kAcc NTOK)
    // accumulator buffer of work item j, and the phase of its j-th use
    auto acc_buf = [&](int j) { return kDB ? (j & 1) : 0; };
    auto acc_use = [&](int j) { return kDB ? (j >> 1) : j; };

    // ---- this CTA's groups and chunks (every thread walks the same sequence)
    const int n_pieces = tc_pieces(L, P);
    int ngroups = 0, nchunks = 0;
    {
        TcWalk cnt;
        cnt.init(P, n_pieces);
        while (cnt.valid) {
            ngroups += (cnt.c_end - cnt.c_begin + kTcG - 1) / kTcG;
            nchunks += cnt.c_end - cnt.c_begin;
            cnt.c0 = cnt.c_end;
            cnt.next();
        }
    }

    if (warp == kWarpTma) {
        // ====================== B loads (one thread) ======================
        if (lane == 0 && nchunks > 0) {
            TcWalk bw;
            bw.init(P, n_pieces);
            int b_item = -1;
            int b_y = 0;
            bool ok = true;
            for (int jc = 0, gi = 0; bw.valid && ok; bw.next(), gi++) {
                if (bw.w != b_item) {
                    int g, row0, nrows, rt;
                    S.item(bw.w, g, row0, nrows, rt);
                    b_item = bw.w;
                    b_y = b_row_mod > 0 ? row0 % b_row_mod : row0;
                }
                for (int i = 0; i < bw.gn; i++, jc++) {
                    // stage js: one chunk (kBG = 1) or the whole group (kBG = kTcG)
                    const int js = kBG == 1 ? jc : gi;
                    const int s = js % kTcB;
                    if (kBG == 1 || i == 0) {
                        if (js >= kTcB &&
                            !mbar_wait(&b_empty[s], (uint32_t)(js / kTcB - 1) & 1u)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&b_full[s], kBSlot * (kBG == 1 ? 1 : bw.gn));
                    }
                    tma_load_2d(bslots + (s * kBG + (kBG == 1 ? 0 : i)) * kBSlot, &tmB,
                                (bw.c0 + i) * kTcChunk, b_y, &b_full[s]);
                }
            }
        }
    } else if (warp == kWarpMma) {
        // ====================== MMA issuer (one thread) ======================
        if (lane == 0 && nchunks > 0) {
            uint32_t idesc = idesc_f16(kTcRows, NTOK);
            TcWalk mw;
            mw.init(P, n_pieces);
            int items = 0, consumed = 0, jc = 0;
            bool ok = true;
            for (int gi = 0; mw.valid && ok; gi++, mw.next()) {
                const int gs = gi % kTcA;
                const bool first = mw.seg_first(), last = mw.seg_last();
                const int ab = acc_buf(items);
                const uint32_t dbase = tmem_d + (uint32_t)(ab * kAcc * NTOK);
                if (first) {
                    // MMA width = the item's rows rounded up to 16: the last tile
                    // of a token group costs what its rows need, not a full tile
                    int g_, r0_, nr_, rt_;
                    S.item(mw.w, g_, r0_, nr_, rt_);
                    idesc = idesc_f16(kTcRows, min(NTOK, max(16, (nr_ + 15) & ~15)));
                }
                if (first && acc_use(items) > 0)
                    ok = mbar_wait(&d_empty[ab], (uint32_t)(acc_use(items) - 1) & 1u);
                if (!ok) break;
                TS_TRACE(1100 + 2 * gi);
                // every chunk barrier of the slot completes once per group (short
                // groups included), so its phase is (gi / kTcA) & 1
                for (int i = 0; i < kTcG; i++) {
                    if (!mbar_wait(&a_full[gs * kTcG + i], (uint32_t)(gi / kTcA) & 1u)) {
                        ok = false;
                        break;
                    }
                    if (i >= mw.gn) {
                        tc_commit(&a_empty[gs * kTcG + i]);
                        continue;
                    }
                    tc_fence_after();
                    const int js = kBG == 1 ? jc : gi;
                    const int sb = js % kTcB;
                    if (kBG == 1 || i == 0) {
                        if (!mbar_wait(&b_full[sb], (uint32_t)(js / kTcB) & 1u)) {
                            ok = false;
                            break;
                        }
                        consumed++;
                    }
                    const uint64_t bd = smem_desc_sw128(
                        smem_u32(bslots + (sb * kBG + (kBG == 1 ? 0 : i)) * kBSlot));
                    const bool fresh = first && i == 0;
#pragma unroll
                    for (int kk = 0; kk < kTcChunk / 16; kk++) {
                        const uint32_t dcol = (uint32_t)((kk % kAcc) * NTOK);
                        tc_mma_ts(dbase + dcol, tmem_a + gs * 128 + i * 32 + kk * 8,
                                  bd + (uint64_t)(2 * kk), idesc,
                                  (fresh && kk < kAcc) ? 0u : 1u);
                    }
                    if (kBG == 1 || i == mw.gn - 1) tc_commit(&b_empty[sb]);
                    tc_commit(&a_empty[gs * kTcG + i]);
                    jc++;
                }
                if (!ok) break;
                TS_TRACE(1101 + 2 * gi);
                if (last) {
                    tc_commit(&d_full[ab]);
                    items++;
                }
            }
            // nothing may still be writing shared or tensor memory when the CTA
            // leaves: the B loads of chunks not consumed, and all MMAs
            const int nstages = kBG == 1 ? nchunks : ngroups;
            for (int j = consumed; j < nstages && j < consumed + kTcB; j++)
                mbar_wait(&b_full[j % kTcB], (uint32_t)(j / kTcB) & 1u);
            tc_commit(fin);
            mbar_wait(fin, 0);
        }
    } else {
        // ====================== expand warps ======================
        // warp e: TMEM lane quarter q = e % 4 (row t), part h = e / 4 of every
        // group: chunks cpw h .. cpw h + cpw - 1 (cpw = kTcCpw), i.e. 32 cpw
        // index bytes -> 32 cpw TMEM columns
        const int q = warp & 3, h = warp >> 2;
        const int t = q * 32 + lane;  // row within the tile = TMEM lane
        const uint32_t lane_base = ((uint32_t)(q * 32)) << 16;
        uint32_t *tab = reinterpret_cast<uint32_t *>(tables) + t;  // entry b at tab[b * 128]
        uint32_t lo[4] = {0, 0, 0, 0}, hi[4] = {0, 0, 0, 0};      // PRMT mode tables
        uint4 *wring = reinterpret_cast<uint4 *>(wring_raw);
        // producer: this thread's index bytes of the coming groups (3 ahead)
        TcWalk pw;
        pw.init(P, n_pieces);
        int gp = 0;
        int p_item = -1;
        const uint8_t *p_row = nullptr;
        auto issue_group = [&]() {
            if (pw.valid) {
                if (pw.w != p_item) {
                    int gg, r0, nr, rtt, cc;
                    S.item(pw.w, gg, r0, nr, rtt);
                    const __half *cbx;
                    S.row_ptrs(max(gg, 0), rtt, t, p_row, cbx, cc);
                    p_item = pw.w;
                }
                uint4 *dst = wring + (size_t)(gp % kTcWStages) * kTcPieces * kTcExpand + tid;
#pragma unroll
                for (int i = 0; i < kTcPieces; i++) {
                    // piece i: k = c0*64 + 64 cpw h + 32i .. +32 (chunk cpw h + i/2 of the group)
                    const int k0 = pw.c0 * kTcChunk + kTcChunk * kTcCpw * h + 32 * i;
                    const bool live = (kTcCpw * h + (i >> 1)) < pw.gn && k0 < L.K;
                    cp_async16_zfill(dst + i * kTcExpand, live ? p_row + k0 / 2 : p_row,
                                     live ? 16 : 0);
                }
                pw.next();
                gp++;
            }
            cp_async_commit_group();
        };
        for (int i = 0; i < kTcWStages - 1; i++) issue_group();

        int g = 0, row0 = 0, nrows = 0, rt = 0, col = 0, items = 0;
        // epilogue: this warp's slice of the NTOK token columns
        constexpr int kEpi = NTOK / kTcWq >= 16 ? NTOK / kTcWq : 16;
        constexpr int kScl = (kEpi + 31) / 32;
        const int cbeg = h * kEpi;
        float scl[kScl];  // fused SwiGLU: token scales of the slice, lane l holds c = cbeg + l + 32 i
#pragma unroll
        for (int i = 0; i < kScl; i++) scl[i] = 0.0f;
        bool ok = true;
        // this warp's chunks of A slot gs free again (the MMAs of group gi - kTcA done)
        auto wait_slot = [&](int gs, int gi) -> bool {
#pragma unroll
            for (int j = 0; j < kTcCpw; j++)
                if (!mbar_wait(&a_empty[gs * kTcG + kTcCpw * h + j], (uint32_t)(gi / kTcA - 1) & 1u))
                    return false;
            return true;
        };
        // ---- epilogue of a finished item (deferred: see the group loop)
        // kLd 16-column loads in flight per wait.  One accumulator buffer:
        // 32-column slices, all drained at once (the MMAs are idle until the
        // drain ends).  Two buffers: 16-column slices, one after each of the
        // next item's groups.  The token scale of the warp's column
        // cbeg + 32 r + l sits in lane l of pd_scl[r].
        constexpr int kLd = kDB ? 1 : (kEpi >= 32 ? 2 : 1);
        static_assert(kEpi % (16 * kLd) == 0, "drain slices");
        constexpr int kSlices = kEpi / (16 * kLd);
        int pd_left = 0;  // slices of the pending item still to drain
        uint32_t hs_phase = 0;  // completed phases of hs_bar[h]
        // the four warps of this token range meet (bounded wait)
        auto group_sync = [&]() -> bool {
            __syncwarp();
            if (lane == 0) mbar_arrive(&hs_bar[h]);
            return mbar_wait(&hs_bar[h], hs_phase++ & 1u);
        };
        int pd_item = 0, pd_row0 = 0, pd_nrows = 0, pd_col = 0, pd_slot = 0;
        float pd_scl[kScl];
#pragma unroll
        for (int i = 0; i < kScl; i++) pd_scl[i] = 0.0f;
        auto drain = [&](int n, int gi_tr) -> bool {
            const int ab = acc_buf(pd_item);
            const uint32_t dbase = tmem_d + (uint32_t)(ab * kAcc * NTOK);
            for (; n > 0 && pd_left > 0; n--) {
                const int it = kSlices - pd_left;
                if (it == 0) {
                    if (!mbar_wait(&d_full[ab], (uint32_t)acc_use(pd_item) & 1u)) return false;
                    if (tr0) TS_TRACE(6 + 6 * gi_tr);
                    tc_fence_after();
                }
                const int off = (it * 16 * kLd) & 31;  // slice start within its 32-column block
                const int c0 = cbeg + it * 16 * kLd;
                if (cbeg < NTOK && c0 < pd_nrows) {  // columns past the rows: nothing to store
                    // the kAcc accumulators summed one at a time (few live registers)
                    float acc[kLd][16];
#pragma unroll
                    for (int a = 0; a < kAcc; a++) {
                        uint32_t d[kLd][16];
#pragma unroll
                        for (int bb = 0; bb < kLd; bb++)
                            tmem_ld16(dbase + lane_base + a * NTOK + c0 + 16 * bb, d[bb]);
                        tmem_wait_ld();
                        if (tr0) TS_TRACE(1400 + 8 * (pd_item % 60) + 2 * it);
#pragma unroll
                        for (int bb = 0; bb < kLd; bb++)
#pragma unroll
                            for (int qq = 0; qq < 16; qq++)
                                acc[bb][qq] = a == 0 ? __uint_as_float(d[bb][qq])
                                                     : acc[bb][qq] + __uint_as_float(d[bb][qq]);
                    }
                    if (L.h_out) {
                        // SwiGLU.  Lanes 2j (gate) and 2j + 1 (up) hold the same output
                        // column; the even lane finishes token c and the odd lane token
                        // c + 1 after one exchange.  All values first (independent
                        // chains, no branches), then the predicated stores.
                        const int odd = lane & 1;
                        __half hv[kLd * 8];
#pragma unroll
                        for (int bb = 0; bb < kLd; bb++)
#pragma unroll
                            for (int qq = 0; qq < 16; qq += 2) {
                                const float a0 = acc[bb][qq], a1 = acc[bb][qq + 1];
                                const float recv = __shfl_xor_sync(0xffffffffu, odd ? a0 : a1, 1);
                                const float gv = odd ? recv : a0, uv = odd ? a1 : recv;
                                float sreg = pd_scl[0];
#pragma unroll
                                for (int i = 1; i < kScl; i++)
                                    if (((it * 16 * kLd + 16 * bb) >> 5) == i) sreg = pd_scl[i];
                                const float sx = __shfl_sync(0xffffffffu, sreg,
                                                             (off + 16 * bb) % 32 + qq + odd);
                                hv[bb * 8 + qq / 2] = __float2half_rn(silu_mul(gv * sx, uv * sx));
                            }
                        if (TcHStage<NTOK>::bytes > 0) {
                            // into this group's tile: token c - cbeg, column t / 2
                            __half *st = reinterpret_cast<__half *>(hstage + h * (64 * 128));
#pragma unroll
                            for (int j = 0; j < kLd * 8; j++)
                                st[(c0 - cbeg + 2 * j + odd) * 64 + (t >> 1)] = hv[j];
                        } else {
#pragma unroll
                            for (int j = 0; j < kLd * 8; j++) {
                                const int c = c0 + 2 * j + odd;
                                if (c < pd_nrows)
                                    L.h_out[(int64_t)(pd_row0 + c) * L.h_row_stride +
                                            (pd_col >> 1)] = hv[j];
                            }
                        }
                    } else {
                        float *out = L.out + (int64_t)pd_slot * L.out_split_stride;
#pragma unroll
                        for (int bb = 0; bb < kLd; bb++)
#pragma unroll
                            for (int qq = 0; qq < 16; qq++) {
                                const int c = c0 + 16 * bb + qq;
                                if (c < pd_nrows)
                                    out[(int64_t)(pd_row0 + c) * L.out_row_stride + pd_col] =
                                        acc[bb][qq];
                            }
                    }
                }
                if (tr0) TS_TRACE(1401 + 8 * (pd_item % 60) + 2 * it);
                if (TcHStage<NTOK>::bytes > 0 && L.h_out && pd_left == 1) {
                    // the four warps of this token range (one per lane quarter)
                    // have staged their columns: 64 rows of 128 B as 16-byte stores
                    if (!group_sync()) return false;
                    const int gt = q * 32 + lane;  // thread within the group
                    const uint4 *src = reinterpret_cast<const uint4 *>(hstage + h * (64 * 128));
                    const int n0 = pd_col >> 1 & ~63;  // the tile's first output column
#pragma unroll
                    for (int k = gt; k < 64 * 8; k += 128) {
                        const int r = k >> 3, part = k & 7;
                        if (cbeg + r < pd_nrows)
                            *reinterpret_cast<uint4 *>(L.h_out + (int64_t)(pd_row0 + cbeg + r) *
                                                                     L.h_row_stride +
                                                       n0 + 8 * part) = src[k];
                    }
                    if (!group_sync()) return false;  // the tile is free for the next item
                }
                if (--pd_left == 0) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&d_empty[ab]);
                    if (tr0) TS_TRACE(7 + 6 * gi_tr);
                }
            }
            return true;
        };
        TcWalk cw;
        cw.init(P, n_pieces);
        // the codebook of the coming segment is loaded one segment ahead, so a
        // new work item does not wait for its codebook's HBM round trip
        auto codebook = [&](const TcWalk &wk, uint4 &a, uint4 &b) {
            if (!wk.valid) return;
            int gg, r0, nr, rtt, cc;
            const uint8_t *ip;
            const __half *cp;
            S.item(wk.w, gg, r0, nr, rtt);
            S.row_ptrs(max(gg, 0), rtt, t, ip, cp, cc);
            a = ldg_stream(cp);
            b = ldg_stream(cp + 8);
        };
        uint4 cbn0 = make_uint4(0, 0, 0, 0), cbn1 = cbn0;
        codebook(cw, cbn0, cbn1);
        for (int gi = 0; cw.valid; gi++, cw.next()) {
            const int gs = gi % kTcA;
            if (cw.seg_first()) {
                const uint8_t *idxp;
                const __half *cbp;
                S.item(cw.w, g, row0, nrows, rt);
                S.row_ptrs(max(g, 0), rt, t, idxp, cbp, col);
                const uint4 c0v = cbn0, c1v = cbn1;
                {
                    TcWalk nx = cw;
                    nx.c0 = nx.c_end;
                    nx.next();
                    codebook(nx, cbn0, cbn1);
                }
                if (L.h_out) {  // loads in flight during the segment; used by its epilogue
#pragma unroll
                    for (int i = 0; i < kScl; i++) {
                        const int c = cbeg + lane + 32 * i;
                        scl[i] = (c < nrows && c < cbeg + kEpi) ? tc_row_scale(L, row0 + c) : 0.0f;
                    }
                }
                // the one-time LUT precompute for this row
                const uint32_t cu[8] = {c0v.x, c0v.y, c0v.z, c0v.w, c1v.x, c1v.y, c1v.z, c1v.w};
                if (PAIR) {
                    // the two warps of the quarter build half of the table each,
                    // once both have finished looking up the previous item
                    if (items > 0 && !mbar_wait(&tab_free[q], (uint32_t)(items - 1) & 1u)) {
                        ok = false;
                        break;
                    }
                    // warp h: entries whose high nibble is in [16 h / kTcWq, 16 (h + 1) / kTcWq)
                    constexpr int kHi = 16 / kTcWq;
#pragma unroll
                    for (int i = 0; i < kHi; i++) {
                        uint32_t wv = cu[i >> 1];  // centroid word of high nibble kHi h + i
#pragma unroll
                        for (int hq = 1; hq < kTcWq; hq++)
                            if (h == hq) wv = cu[(kHi * hq + i) >> 1];
                        const uint32_t hv = ((kHi * h + i) & 1) ? (wv >> 16) : (wv & 0xFFFFu);
                        const int hh = kHi * h + i;
#pragma unroll
                        for (int l = 0; l < 16; l++)
                            tab[(hh * 16 + l) * kTcRows] =
                                prmt(cu[l >> 1], hv, (l & 1) ? 0x5432u : 0x5410u);
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&tab_ready[q]);
                    ok = mbar_wait(&tab_ready[q], (uint32_t)items & 1u);
                    if (!ok) break;
                } else {
#pragma unroll
                    for (int qq = 0; qq < 4; qq++) {
                        lo[qq] = prmt(cu[2 * qq], cu[2 * qq + 1], 0x6420);
                        hi[qq] = prmt(cu[2 * qq], cu[2 * qq + 1], 0x7531);
                    }
                }
            }
            cp_async_wait_group<kTcWStages - 2>();
            if (tr0) TS_TRACE(2 + 6 * gi);
            uint32_t wd[4 * kTcPieces];
            {
                const uint4 *src = wring + (size_t)(gi % kTcWStages) * kTcPieces * kTcExpand + tid;
#pragma unroll
                for (int i = 0; i < kTcPieces; i++) {
                    const uint4 v4 = src[i * kTcExpand];
                    wd[4 * i] = v4.x;
                    wd[4 * i + 1] = v4.y;
                    wd[4 * i + 2] = v4.z;
                    wd[4 * i + 3] = v4.w;
                }
            }
            issue_group();
            if (tr0) TS_TRACE(3 + 6 * gi);
            if (kTcCpw * h < cw.gn) {
                // 64 cpw weights -> 32 cpw fp16 pairs (k = 2b, 2b + 1 in column b)
                constexpr int kB = 32 * kTcCpw;
                uint32_t v[kB];
                if (PAIR) {
                    // independent shared loads (32-bit shared addresses)
                    const uint32_t tab_s = smem_u32(tab);
#pragma unroll
                    for (int b = 0; b < kB; b++) {
                        const uint32_t byte = prmt(wd[b >> 2], 0u, 0x4440u | (uint32_t)(b & 3));
                        v[b] = lds32(tab_s + byte * (kTcRows * 4));
                    }
                } else {
#pragma unroll
                    for (int qq = 0; qq < kB / 4; qq++) {
                        uint32_t h4[4];
                        dequant8(wd[qq], lo, hi, h4);
                        v[4 * qq] = h4[0];
                        v[4 * qq + 1] = h4[1];
                        v[4 * qq + 2] = h4[2];
                        v[4 * qq + 3] = h4[3];
                    }
                }
                if (tr0) TS_TRACE(4 + 6 * gi - 0);  // looked up (slot shared with the wait below)
                if (gi >= kTcA) {
                    ok = wait_slot(gs, gi);
                    if (!ok) break;
                    tc_fence_after();
                }
                const uint32_t ta = tmem_a + lane_base + gs * 128 + h * kB;
                tmem_st32(ta, *reinterpret_cast<const uint32_t(*)[32]>(&v[0]));
                if (kTcCpw == 2 && kTcCpw * h + 1 < cw.gn)
                    tmem_st32(ta + 32, *reinterpret_cast<const uint32_t(*)[32]>(&v[kB - 32]));
                tmem_wait_st();
            } else if (gi >= kTcA) {
                // nothing to store (short group), but the slot must be free
                // before this warp reports it filled
                ok = wait_slot(gs, gi);
                if (!ok) break;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
#pragma unroll
                for (int j = 0; j < kTcCpw; j++) mbar_arrive(&a_full[gs * kTcG + kTcCpw * h + j]);
            }
            if (tr0) TS_TRACE(5 + 6 * gi);
            // the previous item's accumulator: one slice after each group with
            // two buffers (its drain overlaps this item's MMAs), all of it
            // after the first group with one buffer
            if (pd_left > 0 && !drain(kDB ? 1 : kSlices, gi)) {
                ok = false;
                break;
            }
            if (cw.seg_last()) {
                if (PAIR) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&tab_free[q]);
                }
                // a short item may still have its predecessor pending
                if (pd_left > 0 && !drain(kSlices, gi)) {
                    ok = false;
                    break;
                }
                pd_item = items;
                pd_row0 = row0;
                pd_nrows = nrows;
                pd_col = col;
                pd_slot = cw.slot;
#pragma unroll
                for (int i = 0; i < kScl; i++) pd_scl[i] = scl[i];
                pd_left = kSlices;
                items++;
            }
        }
        if (ok && pd_left > 0) ok = drain(kSlices, 0);
        cp_async_wait_group<0>();
    }
    // ---- teardown: all MMAs and TMEM reads are complete before TMEM is freed
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpMma) tmem_dealloc(tmem, kTmemCols);
    if (tr0) TS_TRACE(1999);
}

// ---------------------------------------------------------------- host side
static PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Tensor map over fp16 [rows][K] (row stride K), box [ntok rows][64 k], 128-byte swizzle.
static bool make_b_map(CUtensorMap *m, const void *base, int64_t rows, int K, int ntok) {
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    cuuint32_t box[2] = {(cuuint32_t)kTcChunk, (cuuint32_t)ntok};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int tc_ntok_for(int max_rows_per_group) {
    return max_rows_per_group <= 16 ? 16 : max_rows_per_group <= 64 ? 64
         : max_rows_per_group <= 128 ? 128 : 256;
}

LutPlan plan_lut_tc(int N, int K, bool dual, int max_rows_per_group, int64_t est_tiles,
                    int uniform_rows, int n_groups) {
    LutPlan P{};
    const int ntok = tc_ntok_for(max_rows_per_group);
    P.nt = ntok / 8;
    P.rows_per_rt = dual ? 64 : kTcRows;
    P.n_row_tiles = N / P.rows_per_rt;
    P.chunks_total = (K + kTcChunk - 1) / kTcChunk;
    P.cps_max = P.chunks_total;
    const int capacity = sm_count();  // one CTA per SM
    const int C = P.chunks_total;
    const int64_t u_tiles =
        uniform_rows > 0 ? (int64_t)n_groups * ((uniform_rows + ntok - 1) / ntok) : 0;
    if (uniform_rows > 0 && u_tiles * P.n_row_tiles < 3LL * capacity) {
        // few work items: stream-K balances them over the SMs
        const int64_t tiles = u_tiles;
        P.streamk = 1;
        P.uniform_rows = uniform_rows;
        P.units = tiles * P.n_row_tiles * C;
        P.grid = (int)std::min<int64_t>(capacity, P.units);
        int smax = 1;
        const int64_t items = tiles * P.n_row_tiles;
        for (int64_t w = 0; w < items; w++) smax = std::max(smax, lut_item_splits(P, w));
        P.splits = smax;
        P.chunks_per_split = C;
    } else {
        // many work items (or routed groups): whole items per CTA, split-K only
        // when there are fewer items than SMs
        P.streamk = 0;
        P.uniform_rows = uniform_rows;
        const int64_t base = (int64_t)P.n_row_tiles * std::max<int64_t>(est_tiles, 1);
        int splits = base < capacity ? (int)(capacity / base) : 1;
        splits = std::max(1, std::min(splits, C));
        P.chunks_per_split = (C + splits - 1) / splits;
        P.splits = (C + P.chunks_per_split - 1) / P.chunks_per_split;
        // persistent: at most one CTA per SM, striding over the pieces
        P.grid = (int)std::min<int64_t>(capacity, base * P.splits);
    }
    const bool pair = ntok <= 16;
    const int nb = ntok <= 64 ? 4 * kTcG : ntok <= 128 ? 8 : 4;  // chunk tiles in the B ring
    P.smem = 1024 + (size_t)nb * ntok * 128 + (pair ? kPairTableBytes : 0) +
             (size_t)kTcWStages * kTcPieces * kTcExpand * 16 +
             (ntok == 256 ? TcHStage<256>::bytes : 0) + 512;
    P.tc = 1;
    return P;
}

template <int NTOK, bool PAIR>
static cudaError_t launch_tc_t(const CUtensorMap &m, const LutLaunch &L, const LutPlan &P,
                               int b_row_mod, cudaStream_t st) {
    return launch_pdl(k_lut_tc<NTOK, PAIR>, dim3(P.grid), dim3(kTcThreads), P.smem, st, 1, m, L, P,
                      b_row_mod);
}

cudaError_t launch_lut_tc(const LutLaunch &L, const LutPlan &P, const void *b_f16,
                          int64_t b_rows, int b_row_mod, cudaStream_t st) {
    if (P.grid == 0 || (!P.streamk && L.max_tiles == 0)) return cudaSuccess;
    const int ntok = 8 * P.nt;
    CUtensorMap m;
    std::memset(&m, 0, sizeof(m));
    if (!make_b_map(&m, b_f16, b_rows, L.K, ntok)) return cudaErrorInvalidValue;
    const bool timed = timing_on();
    if (timed) timing_begin(st, CQ_KERNEL_LUT_TC);
    count_launch();
    cudaError_t e;
    switch (ntok) {
    case 16: e = launch_tc_t<16, true>(m, L, P, b_row_mod, st); break;
    case 64: e = launch_tc_t<64, false>(m, L, P, b_row_mod, st); break;
    case 128: e = launch_tc_t<128, false>(m, L, P, b_row_mod, st); break;
    default: e = launch_tc_t<256, false>(m, L, P, b_row_mod, st); break;
    }
    if (timed) timing_end(st);
    return e;
}

// ---------------------------------------------------------------- decode kernel (lut_ts.cuh)
// Tensor map over packed index bytes uint8 [rows][K/2] (row stride K/2), box
// [box_rows rows][128 B] (one 256-k group), 128-byte swizzle; bytes past K/2
// read as zero.
static bool make_idx_map(CUtensorMap *m, const void *base, int64_t rows, int K, int box_rows) {
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
    cuuint32_t box[2] = {128u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int ts_ntok_for(int max_rows_per_group) { return max_rows_per_group <= 16 ? 16 : 32; }

LutPlan plan_lut_ts(int N, int K, bool dual, int max_rows_per_group, int64_t est_tiles,
                    int uniform_rows, int n_groups) {
    LutPlan P{};
    const int ntok = ts_ntok_for(max_rows_per_group);
    P.nt = ntok / 8;
    P.rows_per_rt = dual ? 64 : kTcRows;
    P.n_row_tiles = N / P.rows_per_rt;
    P.chunks_total = (K + kTcChunk - 1) / kTcChunk;
    P.cps_max = P.chunks_total;
    const int capacity = sm_count();  // one CTA per SM
    const int C = P.chunks_total;
    P.uniform_rows = uniform_rows;
    if (uniform_rows > 0) {
        // stream-K: every SM gets the same number of chunks
        const int64_t tiles = (int64_t)n_groups * ((uniform_rows + ntok - 1) / ntok);
        P.streamk = 1;
        P.units = tiles * P.n_row_tiles * C;
        P.grid = (int)std::min<int64_t>(capacity, P.units);
        int smax = 1;
        const int64_t items = tiles * P.n_row_tiles;
        for (int64_t w = 0; w < items; w++) smax = std::max(smax, lut_item_splits(P, w));
        P.splits = smax;
        P.chunks_per_split = C;
    } else {
        // routed groups: whole (item, split) pieces strided over the CTAs,
        // split-K only when there are fewer items than SMs
        P.streamk = 0;
        const int64_t base = (int64_t)P.n_row_tiles * std::max<int64_t>(est_tiles, 1);
        int splits = base < capacity ? (int)(capacity / base) : 1;
        splits = std::max(1, std::min(splits, C));
        P.chunks_per_split = (C + splits - 1) / splits;
        P.splits = (C + P.chunks_per_split - 1) / P.chunks_per_split;
        P.grid = (int)std::min<int64_t>(capacity, base * P.splits);
    }
    P.smem = ntok == 16 ? TsShape<16>::smem : TsShape<32>::smem;
    P.tc = 2;
    return P;
}

template <int NTOK>
static cudaError_t launch_ts_t(const CUtensorMap &m0, const CUtensorMap &m1, const CUtensorMap &mb,
                               const LutLaunch &L, const LutPlan &P, int b_row_mod,
                               cudaStream_t st) {
    return launch_pdl(k_lut_ts<NTOK>, dim3(P.grid), dim3(kTsThreads), P.smem, st, 1, m0, m1, mb,
                      L, P, b_row_mod);
}

cudaError_t launch_lut_ts(const LutLaunch &L, const LutPlan &P, const void *b_f16,
                          int64_t b_rows, int b_row_mod, cudaStream_t st) {
    if (P.grid == 0 || (!P.streamk && L.max_tiles == 0)) return cudaSuccess;
    const int64_t rows = (int64_t)std::max(L.G, 1) * L.N;
    const int box = L.dual ? 64 : kTcRows;
    const int ntok = 8 * P.nt;
    CUtensorMap m0, m1, mb;
    std::memset(&m0, 0, sizeof(m0));
    std::memset(&m1, 0, sizeof(m1));
    std::memset(&mb, 0, sizeof(mb));
    if (!make_idx_map(&m0, L.idx0, rows, L.K, box)) return cudaErrorInvalidValue;
    if (L.dual && !make_idx_map(&m1, L.idx1, rows, L.K, box)) return cudaErrorInvalidValue;
    if (!make_b_map(&mb, b_f16, b_rows, L.K, ntok)) return cudaErrorInvalidValue;
    const bool timed = timing_on();
    if (timed) timing_begin(st, CQ_KERNEL_LUT_TS);
    count_launch();
    const CUtensorMap &m1r = L.dual ? m1 : m0;
    const cudaError_t e = ntok == 16 ? launch_ts_t<16>(m0, m1r, mb, L, P, b_row_mod, st)
                                     : launch_ts_t<32>(m0, m1r, mb, L, P, b_row_mod, st);
    if (timed) timing_end(st);
    return e;
}

// ---------------------------------------------------------------- codes -> fp16 rows
// out[p, k] = fp16(code of row map(p), position k): the B operand of the
// tensor-core kernel.  One thread per 8 codes.
__global__ void k_codes_to_f16(const uint8_t *__restrict__ codes, int64_t ld_codes, int bits,
                               int K, int64_t rows, int map_mode, const int32_t *__restrict__ perm,
                               int topk, int T, __half *__restrict__ out,
                               const float *__restrict__ scales_in, float *__restrict__ scales_out) {
    griddep_wait();
    griddep_launch();
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int per_row = K / 8;
    if (i >= rows * per_row) return;
    const int64_t p = i / per_row;
    const int k = (int)(i - p * per_row) * 8;
    const int64_t cr = map_mode == kMapPerm ? perm[p] / topk : map_mode == kMapModT ? p % T : p;
    if (scales_in && k == 0) scales_out[p] = scales_in[cr];
    const uint8_t *src = codes + cr * ld_codes;
    __align__(16) __half v[8];
    if (bits == 4) {
        const uint32_t w = *reinterpret_cast<const uint32_t *>(src + k / 2);
#pragma unroll
        for (int e = 0; e < 8; e++) v[e] = __short2half_rn((short)(((int)(w << (28 - 4 * e))) >> 28));
    } else {
        const uint2 w = *reinterpret_cast<const uint2 *>(src + k);
#pragma unroll
        for (int e = 0; e < 4; e++) {
            v[e] = __short2half_rn((short)(((int)(w.x << (24 - 8 * e))) >> 24));
            v[4 + e] = __short2half_rn((short)(((int)(w.y << (24 - 8 * e))) >> 24));
        }
    }
    *reinterpret_cast<uint4 *>(out + p * K + k) = *reinterpret_cast<const uint4 *>(v);
}

cudaError_t launch_codes_to_f16(const void *codes, int64_t ld_codes, int bits, int K,
                                int64_t rows, int map_mode, const int32_t *perm, int topk, int T,
                                void *out, cudaStream_t st, const float *scales_in,
                                float *scales_out) {
    const int64_t n = rows * (K / 8);
    if (n == 0) return cudaSuccess;
    TimedScope ts(st, CQ_KERNEL_CODES_F16);
    count_launch();
    return launch_pdl(k_codes_to_f16, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, 1,
                      reinterpret_cast<const uint8_t *>(codes), ld_codes, bits, K, rows, map_mode,
                      perm, topk, T, reinterpret_cast<__half *>(out), scales_in, scales_out);
}

LutPath lut_path() {
    static LutPath p = [] {
        const char *e = getenv("CQ_LUT_PATH");
        if (e && !strcmp(e, "mma")) return kPathMma;
        if (e && !strcmp(e, "tc")) return kPathTc;
        if (e && !strcmp(e, "ts")) return kPathTs;
        return kPathAuto;
    }();
    return p;
}

// One thread waits on an mbarrier that nothing ever arrives on: the bounded
// wait gives up after about a second, records kErrWaitTimeout and the kernel
// returns -- the error path every tensor-core kernel takes when a wait runs out.
__global__ void k_selftest_wait() {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
        mbar_wait(&bar, 0);
    }
}

cudaError_t launch_selftest_wait(cudaStream_t st) {
    count_launch();
    k_selftest_wait<<<1, 32, 0, st>>>();
    return cudaGetLastError();
}

int read_device_error() {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)) != cudaSuccess) return -1;
    if (v) {
        const int zero = 0;
        cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
    }
    return v;
}

}  // namespace cq

#ifdef CQ_TS_TRACE
// Copies the decode kernel's timeline stamps to host memory (tuning builds only).
extern "C" CQ_API int cq_ts_trace_read(void *dst, size_t bytes) {
    return cudaMemcpyFromSymbol(dst, cq::g_ts_trace, bytes) == cudaSuccess ? 0 : 1;
}
#endif
