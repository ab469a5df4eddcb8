// tc_walk.cuh -- work schedule shared by the tensor-memory LUT GEMM kernels:
// which rows, weights and k-chunks a CTA processes, in which order.
#pragma once

#include "cq_common.cuh"
#include "cq_internal.h"

namespace cq {

constexpr int kTcRows = 128;         // rows per tile (TMEM lanes)
constexpr int kTcChunk = 64;         // k per chunk: 4 MMAs of K = 16, 32 TMEM columns
constexpr int kTcG = 4;              // chunks per group (256 k)

// All work counts of a tensor-memory launch fit in 31 bits (the host plans only
// launches whose units * grid < 2^31), so the schedule uses 32-bit integer
// arithmetic: 64-bit division is a long software sequence on the GPU.
struct TcSchedule {
    const LutLaunch *L;
    const LutPlan *P;
    // work item -> (group, first row, rows, row tile)
    CQ_DEV void item(int w, int &g, int &row0, int &nrows, int &rt) const {
        const int TT = 8 * P->nt;
        const int tile = w / P->n_row_tiles;
        rt = w - tile * P->n_row_tiles;
        if (L->uniform_rows > 0) {
            const int tpg = (L->uniform_rows + TT - 1) / TT;
            g = tile / tpg;
            row0 = g * L->uniform_rows + (tile - g * tpg) * TT;
            nrows = min(TT, (g + 1) * L->uniform_rows - row0);
        } else {
            if (tile >= L->grp_tiles[L->G]) {
                g = -1;
                row0 = nrows = 0;
                return;
            }
            g = L->tile_grp[tile];
            row0 = L->grp_rows[g] + (tile - L->grp_tiles[g]) * TT;
            nrows = min(TT, L->grp_rows[g + 1] - row0);
        }
    }
    // this thread's weight row: index bytes and codebook (t = 0..127)
    CQ_DEV void row_ptrs(int g, int rt, int t, const uint8_t *&idx, const __half *&cb, int &col) const {
        const int64_t rowbytes = L->K / 2;
        if (L->dual) {
            // gate and up rows of one output column in adjacent lanes, so the
            // epilogue's stores of a warp cover 32 consecutive partial columns
            const int n = rt * 64 + (t >> 1);
            const bool up = t & 1;
            idx = (up ? L->idx1 : L->idx0) + (int64_t)g * L->w_stride + (int64_t)n * rowbytes;
            cb = reinterpret_cast<const __half *>(up ? L->cb1 : L->cb0) + (int64_t)g * L->cb_stride + n * 16;
            col = 2 * n + (up ? 1 : 0);
        } else {
            const int n = rt * kTcRows + t;
            idx = L->idx0 + (int64_t)g * L->w_stride + (int64_t)n * rowbytes;
            cb = reinterpret_cast<const __half *>(L->cb0) + (int64_t)g * L->cb_stride + n * 16;
            col = n;
        }
    }
};

// The chunks a CTA works through, as segments (work item, chunk range) cut
// into groups of at most kTcG chunks (a group never spans two segments).
// Stream-K (uniform launches): one contiguous range of units (item x chunk),
// cut at item boundaries.  Fixed split (routed launches): pieces (item,
// split) p = blockIdx.x, blockIdx.x + gridDim.x, ... below the number of
// pieces the routing produced, so the grid stays one CTA per SM whatever the
// tile count.  Every role of the CTA walks the same sequence.
struct TcWalk {
    const LutPlan *P;
    int w;            // work item of the current segment
    int c0, gn;       // first chunk (item-relative) and chunk count of the group
    int c_begin, c_end;
    int slot;         // partial-sum slot the segment writes
    int nxt, lim;
    bool valid;

    CQ_DEV void init(const LutPlan &Pl, int n_pieces) {
        P = &Pl;
        if (Pl.streamk) {
            const int U = (int)Pl.units;
            nxt = (int)blockIdx.x * U / Pl.grid;
            lim = ((int)blockIdx.x + 1) * U / Pl.grid;
        } else {
            nxt = blockIdx.x;
            lim = n_pieces;
        }
        load();
    }
    CQ_DEV void load() {
        valid = nxt < lim;
        if (!valid) return;
        const int C = P->chunks_total;
        if (P->streamk) {
            w = nxt / C;
            c_begin = nxt - w * C;
            const int e = min(lim, (w + 1) * C);
            c_end = e - w * C;
            // first CTA of the item: the one whose range holds its unit w * C
            const int first = ((w * C + 1) * P->grid - 1) / (int)P->units;
            slot = (int)blockIdx.x - first;
            nxt = e;
        } else {
            w = nxt / P->splits;
            const int sp = nxt - w * P->splits;
            c_begin = sp * P->chunks_per_split;
            c_end = min(C, c_begin + P->chunks_per_split);
            slot = sp;
            nxt += gridDim.x;
        }
        c0 = c_begin;
        gn = min(kTcG, c_end - c0);
    }
    CQ_DEV bool seg_first() const { return c0 == c_begin; }
    CQ_DEV bool seg_last() const { return c0 + gn == c_end; }
    CQ_DEV void next() {
        c0 += gn;
        if (c0 >= c_end) load();
        else gn = min(kTcG, c_end - c0);
    }
};

// Pieces of a fixed-split launch that hold rows (the routing decides how many
// token tiles there are; the host only knows an upper bound).
CQ_DEV int tc_pieces(const LutLaunch &L, const LutPlan &P) {
    if (P.streamk) return 0;
    const int TT = 8 * P.nt;
    const int tiles = L.uniform_rows > 0 ? L.G * ((L.uniform_rows + TT - 1) / TT)
                                         : min(L.grp_tiles[L.G], L.max_tiles);
    return tiles * P.n_row_tiles * P.splits;
}

// Activation scale of output row p (the row's token).
// Issued as a volatile load at segment start, so the compiler cannot sink it to
// the epilogue, where it would stall the drain of the accumulator.
CQ_DEV float tc_row_scale(const LutLaunch &L, int64_t p) {
    const float *src = L.row_scales ? L.row_scales + p
                     : L.scales + (L.map_mode == kMapModT ? p % L.T : p);
    float v;
    asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(v) : "l"(src));
    return v;
}

}  // namespace cq
