// rotate_quantize.cuh -- exact block Walsh-Hadamard rotation and per-token
// absmax quantization of one row held in shared memory (one CTA per row).
//
// The rotated values are kept in fp64.  fp16 inputs are multiples of 2^-24
// and every butterfly sum stays below 65504 * 8192 < 2^29, so all of them are
// integers below 2^53 in units of 2^-24: the fp64 butterflies are exact and
// the order of the levels does not matter.  The quantization decision
// round_half_even(qmax * v / A) is then taken exactly with int64 arithmetic.
#pragma once

#include "cq_common.cuh"
#include "cq_internal.h"

namespace cq {

// Index bits 8.. of the transform: one thread per column of R = b / 256
// elements at stride 256 (R known at compile time so the column stays in
// registers).
template <int THREADS, int R>
__device__ void fwht_columns(double *buf, int K, int log2b) {
    const int ncols = K >> (log2b - 8);
    for (int col = threadIdx.x; col < ncols; col += THREADS) {
        const int blk = col >> 8, c = col & 255;
        double *p = buf + ((size_t)blk << log2b) + c;
        double v[R];
#pragma unroll
        for (int r = 0; r < R; r++) v[r] = p[256 * r];
#pragma unroll
        for (int h = 1; h < R; h <<= 1) {
#pragma unroll
            for (int r = 0; r < R; r++) {
                if ((r & h) == 0) {
                    const double a = v[r], d = v[r + h];
                    v[r] = a + d;
                    v[r + h] = a - d;
                }
            }
        }
#pragma unroll
        for (int r = 0; r < R; r++) p[256 * r] = v[r];
    }
}

// In-place Walsh-Hadamard transform (Sylvester order) of every contiguous
// block of b = 2^log2b elements of buf[0, K).  K % 8 == 0, K % b == 0.
//   levels 0..4 (index bits 0-4): lanes of a warp, via shuffles
//   levels 5..7 (bits 5-7):       8 registers per lane (stride 32)
//   levels 8..  (bits 8..):       one thread per column, stride 256
template <int THREADS>
__device__ void block_fwht(double *buf, int K, int log2b) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int NW = THREADS / 32;
    const int lv1 = log2b < 8 ? log2b : 8;
    if (lv1 > 0) {
        for (int base = warp * 256; base < K; base += NW * 256) {
            double v[8];
#pragma unroll
            for (int j = 0; j < 8; j++) {
                int k = base + lane + 32 * j;
                v[j] = k < K ? buf[k] : 0.0;
            }
            // bits 0..4: across lanes
            for (int L = 0; L < (lv1 < 5 ? lv1 : 5); L++) {
                const int bit = 1 << L;
                const bool upper = lane & bit;
#pragma unroll
                for (int j = 0; j < 8; j++) {
                    double p = __shfl_xor_sync(0xffffffffu, v[j], bit);
                    v[j] = upper ? (p - v[j]) : (v[j] + p);
                }
            }
            // bits 5..7: inside the thread
            for (int L = 5; L < lv1; L++) {
                const int h = 1 << (L - 5);
#pragma unroll
                for (int j = 0; j < 8; j++) {
                    if ((j & h) == 0) {
                        double a = v[j], c = v[j + h];
                        v[j] = a + c;
                        v[j + h] = a - c;
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < 8; j++) {
                int k = base + lane + 32 * j;
                if (k < K) buf[k] = v[j];
            }
        }
        __syncthreads();
    }
    if (log2b > 8) {
        switch (log2b - 8) {
        case 1: fwht_columns<THREADS, 2>(buf, K, log2b); break;
        case 2: fwht_columns<THREADS, 4>(buf, K, log2b); break;
        case 3: fwht_columns<THREADS, 8>(buf, K, log2b); break;
        case 4: fwht_columns<THREADS, 16>(buf, K, log2b); break;
        default: fwht_columns<THREADS, 32>(buf, K, log2b); break;
        }
        __syncthreads();
    }
}

// max |buf[k]| over the row, returned to every thread.  red: >= 32 doubles.
template <int THREADS>
__device__ double block_absmax(const double *buf, int K, double *red) {
    double m = 0.0;
    for (int k = threadIdx.x; k < K; k += THREADS) m = fmax(m, fabs(buf[k]));
    m = warp_max_d(m);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) red[warp] = m;
    __syncthreads();
    if (warp == 0) {
        double v = lane < THREADS / 32 ? red[lane] : 0.0;
        v = warp_max_d(v);
        if (lane == 0) red[32] = v;
    }
    __syncthreads();
    double A = red[32];
    __syncthreads();  // red may be reused by the caller
    return A;
}

// round_half_even(qmax * v / A) for v, A multiples of 2^-24 (|.| < 2^29), A > 0.
CQ_DEV int quantize_exact(double v, long long Ai, int qmax) {
    const long long vi = __double2ll_rn(v * 16777216.0);  // exact integer
    const long long av = vi < 0 ? -vi : vi;
    const long long num = (long long)qmax * av;            // < 2^60
    // fp64 estimate of the quotient, then exact integer correction
    long long q0 = (long long)floor(__ddiv_rn((double)num, (double)Ai));
    long long r = num - q0 * Ai;
    if (r < 0) { q0 -= 1; r += Ai; }
    if (r >= Ai) { q0 += 1; r -= Ai; }
    if (2 * r > Ai || (2 * r == Ai && (q0 & 1))) q0 += 1;
    return (int)(vi < 0 ? -q0 : q0);
}

// s = (float)((A / sqrt(b)) / qmax), each step IEEE round-to-nearest fp64.
CQ_DEV float quant_scale(double A, int log2b, int qmax) {
    return __double2float_rn(__ddiv_rn(__ddiv_rn(A, __dsqrt_rn((double)(1 << log2b))),
                                       (double)qmax));
}

// Code of one rotated value: round_half_even(qmax * |v| / A) with the sign
// of v.  t = |v| * (qmax / A) in fp64 is within 3e-14 of the exact quotient
// (which is at most 127), so unless t lies within 1e-9 of a half-integer
// rint(t) is already the exact decision; near a half-integer the exact int64
// rational decision is taken instead.
CQ_DEV int quantize_fast(double v, double R, long long Ai, int qmax) {
    const double t = fabs(v) * R;
    const double fr = t - floor(t);
    int q;
    if (fabs(fr - 0.5) < 1e-9) {
        q = quantize_exact(fabs(v), Ai, qmax);
    } else {
        q = (int)rint(t);
    }
    return v < 0 ? -q : q;
}

// The exact decision of quantize_fast's near-tie branch, for the rare values
// whose fp64 quotient lies within 1e-9 of a tie.
CQ_DEV int quantize_tie(double v, long long Ai, int qmax) {
    const int q = quantize_exact(fabs(v), Ai, qmax);
    return v < 0 ? -q : q;
}

// Code of one rotated value, as quantize_fast, for callers that quantize many
// values in registers: t = v * R rounded to the nearest integer (ties to even)
// by adding and subtracting 1.5 * 2^52 -- the sum lies in [2^52, 2^53), where
// the fp64 spacing is 1 -- and the integer read from the low word of the sum.
// Sets *near_tie when |t - round(t)| > 0.5 - 1e-9: the caller then takes
// quantize_tie instead (|t| <= 127, so outside that window the rounding of t
// cannot change the decision).
CQ_DEV int quantize_round(double v, double R, bool &near_tie) {
    constexpr double kMagic = 6755399441055744.0;  // 1.5 * 2^52
    const double t = v * R;
    const double big = t + kMagic;
    const double r = t - (big - kMagic);
    near_tie = fabs(r) > 0.5 - 1e-9;
    return __double2loint(big);
}

// The fp16 copies of the codes of row positions (e, e + 1) of row mrow: the
// tensor-core B rows an RqF16 names (rows of K halves; small integers are
// exact in fp16).
CQ_DEV void store_code_copies(const RqF16 &f, int64_t mrow, int K, int e, int q0, int q1) {
    const __half2 h = __halves2half2(__short2half_rn((short)q0), __short2half_rn((short)q1));
    for (int d = 0; d < f.ncopy; d++) {
        const int64_t row = f.map ? (int64_t)f.map[mrow * f.ncopy + d] : mrow;
        *reinterpret_cast<__half2 *>(f.rows + row * K + e) = h;
    }
    if (f.ident) *reinterpret_cast<__half2 *>(f.ident + mrow * K + e) = h;
}
// The row's scale beside each routed copy (RqF16::row_scales).
CQ_DEV void store_copy_scales(const RqF16 &f, int64_t mrow, float sq) {
    if (!f.row_scales) return;
    for (int d = 0; d < f.ncopy; d++)
        f.row_scales[f.map ? (int64_t)f.map[mrow * f.ncopy + d] : mrow] = sq;
}
CQ_DEV bool has_copies(const RqF16 &f) { return f.ncopy > 0 || f.ident != nullptr; }

// Quantize buf[0, n) (rotated values of row positions [e0, e0 + n)) and
// store the codes: bits 4 -> packed bytes (low nibble = even position),
// bits 8 -> int8.  e0 and n are even.  A is the absmax of the whole row.
// With copies (f16 non-empty), also the fp16 copies of row mrow's codes.
template <int THREADS>
__device__ void block_quantize_range(const double *buf, int n, int e0, int bits, double A,
                                     uint8_t *qrow, const RqF16 &f16, int64_t mrow, int K) {
    const bool copies = has_copies(f16);
    const int qmax = (1 << (bits - 1)) - 1;
    const long long Ai = __double2ll_rn(A * 16777216.0);
    const double R = Ai > 0 ? __ddiv_rn((double)qmax, A) : 0.0;
    const double2 *b2 = reinterpret_cast<const double2 *>(buf);
    for (int p = threadIdx.x; p < n / 2; p += THREADS) {
        const double2 v = b2[p];
        int q0 = 0, q1 = 0;
        if (Ai > 0) {
            q0 = quantize_fast(v.x, R, Ai, qmax);
            q1 = quantize_fast(v.y, R, Ai, qmax);
        }
        if (bits == 4) {
            qrow[e0 / 2 + p] = (uint8_t)((q0 & 15) | ((q1 & 15) << 4));
        } else {
            char2 c;
            c.x = (char)q0;
            c.y = (char)q1;
            reinterpret_cast<char2 *>(qrow + e0)[p] = c;
        }
        if (copies) store_code_copies(f16, mrow, K, e0 + 2 * p, q0, q1);
    }
}

// ---------------------------------------------------------------- one warp per row
// Rotation blocks of b <= 256: the whole transform of a 256-aligned chunk is
// inside one warp (index bits 0-4 across lanes, 5-7 in registers).  buf holds
// the row (K doubles; K a multiple of b, so a ragged last chunk holds whole
// blocks); returns max |.|.
CQ_DEV double warp_fwht_absmax(double *buf, int K, int log2b) {
    const int lane = threadIdx.x & 31;
    double amax = 0.0;
    // two 256-element chunks per pass: 16 independent butterfly chains
    for (int base = 0; base < K; base += 512) {
        double v[16];
#pragma unroll
        for (int j = 0; j < 16; j++) {
            const int k = base + lane + 32 * j;
            v[j] = k < K ? buf[k] : 0.0;
        }
        for (int L = 0; L < (log2b < 5 ? log2b : 5); L++) {
            const int bit = 1 << L;
            // partner p: lower lane keeps v + p, upper lane p - v (one
            // correctly rounded fma with an exact +-1 product)
            const double sg = (lane & bit) ? -1.0 : 1.0;
#pragma unroll
            for (int j = 0; j < 16; j++) {
                const double p = __shfl_xor_sync(0xffffffffu, v[j], bit);
                v[j] = fma(sg, v[j], p);
            }
        }
        // levels 5..7 pair registers of the same lane (within each 256-chunk);
        // unrolled so that the register indices are compile-time constants
#pragma unroll
        for (int L = 5; L < 8; L++) {
            if (L < log2b) {
                const int h = 1 << (L - 5);
#pragma unroll
                for (int j = 0; j < 16; j++) {
                    if ((j & h) == 0) {
                        const double a = v[j], c = v[j + h];
                        v[j] = a + c;
                        v[j + h] = a - c;
                    }
                }
            }
        }
#pragma unroll
        for (int j = 0; j < 16; j++) {
            const int k = base + lane + 32 * j;
            if (k < K) {
                buf[k] = v[j];
                amax = fmax(amax, fabs(v[j]));
            }
        }
    }
    __syncwarp();
    return warp_max_d(amax);
}

// Quantize a rotated row held by one warp and store codes and scale (and the
// fp16 copies of row mrow's codes, when f16 names any).
CQ_DEV void warp_quantize_row(const double *buf, int K, int log2b, int bits, double A,
                              uint8_t *qrow, float *s_out, const RqF16 &f16, int64_t mrow) {
    const bool copies = has_copies(f16);
    const int lane = threadIdx.x & 31;
    const int qmax = (1 << (bits - 1)) - 1;
    const long long Ai = __double2ll_rn(A * 16777216.0);
    const double R = Ai > 0 ? __ddiv_rn((double)qmax, A) : 0.0;
    const double2 *b2 = reinterpret_cast<const double2 *>(buf);
    for (int p = lane; p < K / 2; p += 32) {
        const double2 v = b2[p];
        int q0 = 0, q1 = 0;
        if (Ai > 0) {
            q0 = quantize_fast(v.x, R, Ai, qmax);
            q1 = quantize_fast(v.y, R, Ai, qmax);
        }
        if (bits == 4) {
            qrow[p] = (uint8_t)((q0 & 15) | ((q1 & 15) << 4));
        } else {
            char2 c;
            c.x = (char)q0;
            c.y = (char)q1;
            reinterpret_cast<char2 *>(qrow)[p] = c;
        }
        if (copies) store_code_copies(f16, mrow, K, 2 * p, q0, q1);
    }
    if (lane == 0) {
        const float sq = Ai > 0 ? quant_scale(A, log2b, qmax) : 0.0f;
        *s_out = sq;
        store_copy_scales(f16, mrow, sq);
    }
}

}  // namespace cq
