// lut_lookup.cuh -- register-resident codebook lookup: the 16 fp16
// centroids of one weight row as two 16-byte byte-plane tables (low and high
// bytes), looked up four indices at a time with byte permutes.
#pragma once

#include "cq_common.cuh"

namespace cq {

// Byte-plane tables of one codebook row: lo[j] holds the low bytes of
// C[4j..4j+3], hi[j] the high bytes.
CQ_DEV void build_tables(const uint4 a, const uint4 b, uint32_t (&lo)[4], uint32_t (&hi)[4]) {
    const uint32_t u[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int j = 0; j < 4; j++) {
        lo[j] = prmt(u[2 * j], u[2 * j + 1], 0x6420);
        hi[j] = prmt(u[2 * j], u[2 * j + 1], 0x7531);
    }
}
CQ_DEV void build_tables(const __half *cb, uint32_t (&lo)[4], uint32_t (&hi)[4]) {
    build_tables(*reinterpret_cast<const uint4 *>(cb), *reinterpret_cast<const uint4 *>(cb + 8), lo,
                 hi);
}

// Eight 4-bit indices (nibble i of w = index of element i) -> four half2:
// h[0] = (C[i0], C[i1]), h[1] = (C[i2], C[i3]), h[2] = (C[i4], C[i5]),
// h[3] = (C[i6], C[i7]).  Selector nibble bit 3 switches prmt to
// sign-replicate mode, so entries 0-7 and 8-15 are fetched from the two
// halves of each plane and merged with a per-byte mask built from bit 3.
CQ_DEV void dequant8(uint32_t w, const uint32_t (&lo)[4], const uint32_t (&hi)[4],
                     uint32_t (&h)[4]) {
    // (the integer/logic pipe runs at half rate: the two right shifts and the
    // left shift are multiplies, which issue to the FMA pipe)
    const uint32_t wx = w ^ 0x88888888u;
    const uint32_t s0 = w, s1 = __umulhi(w, 0x10000u);
    const uint32_t x0 = wx, x1 = __umulhi(wx, 0x10000u);
    const uint32_t w4 = w * 16u;
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

}  // namespace cq
