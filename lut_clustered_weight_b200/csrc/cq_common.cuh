// cq_common.cuh -- shared device helpers for the sm_100a CodeQuant kernels.
#pragma once

#include <mutex>
#include <utility>
#include <vector>

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/cq.h"

#define CQ_DEV __device__ __forceinline__

namespace cq {

constexpr int kWarp = 32;

// byte permute: selects bytes of {b:a} by the nibbles of sel (bit 3 = sign mode)
CQ_DEV uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// 128-bit streaming load that skips L1 (weights are read exactly once)
CQ_DEV uint4 ldg_stream(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// 32-bit shared-memory load at a shared-window address.
CQ_DEV uint32_t lds32(uint32_t saddr) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(saddr));
    return v;
}

CQ_DEV float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

CQ_DEV double warp_max_d(double v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// mma.sync m16n8k16, fp16 x fp16 -> fp32 (accumulate in place)
CQ_DEV void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// fp32 silu(g) * u with the fast exponential and division (a few ulp in
// fp32, far below the fp16 rounding of h that follows)
CQ_DEV float silu_mul(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

// ---------------------------------------------------------------- programmatic dependent launch
// Every kernel of the library is launched with programmatic stream
// serialization: it may start while the previous kernel on the stream is
// still running.  griddep_wait() blocks until that kernel has completed and
// its writes are visible; nothing that kernel produces may be read, and no
// global memory may be written, before it.  griddep_launch() lets the next
// kernel start early (it waits for this one in turn).  Both are no-ops for a
// kernel launched without the attribute.
CQ_DEV void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
CQ_DEV void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------- split-K slot sums
CQ_DEV void vadd(float &a, float b) { a += b; }
CQ_DEV void vadd(float2 &a, float2 b) {
    a.x += b.x;
    a.y += b.y;
}
CQ_DEV void vadd(float4 &a, float4 b) {
    a.x += b.x;
    a.y += b.y;
    a.z += b.z;
    a.w += b.w;
}

// acc[f] += p[f][0] + p[f][stride] + ... (ns[f] slots, added in slot order),
// for F independent sums at once: every round issues the loads of U slots of
// all F sums before the first add, so F * U loads are in flight instead of a
// chain of dependent round trips.
template <int F, int U = 2, typename T>
CQ_DEV void sum_slots(const T *const (&p)[F], const int (&ns)[F], int64_t stride, T (&acc)[F]) {
    int nsmax = 0;
#pragma unroll
    for (int f = 0; f < F; f++) nsmax = max(nsmax, ns[f]);
    for (int s0 = 0; s0 < nsmax; s0 += U) {
        T v[F][U];
#pragma unroll
        for (int f = 0; f < F; f++)
#pragma unroll
            for (int u = 0; u < U; u++)
                v[f][u] = s0 + u < ns[f] ? p[f][(int64_t)(s0 + u) * stride] : T{};
#pragma unroll
        for (int f = 0; f < F; f++)
#pragma unroll
            for (int u = 0; u < U; u++)
                if (s0 + u < ns[f]) vadd(acc[f], v[f][u]);
    }
}

// Once per kernel and device (host): allow the largest dynamic shared memory a
// CTA may have and ask for the full shared-memory carveout.  Every kernel of
// the library then runs with the same L1 / shared-memory split, so the SMs
// never re-split it between consecutive kernels, and no launch pays a
// cudaFuncSetAttribute call.
inline void configure_kernel_once(const void *kern) {
    static std::mutex mu;
    static std::vector<std::pair<const void *, int>> done;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return;
    std::lock_guard<std::mutex> lk(mu);
    for (const auto &d : done)
        if (d.first == kern && d.second == dev) return;
    int optin = 0;
    cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    cudaFuncAttributes fa{};
    cudaFuncGetAttributes(&fa, kern);  // dynamic + static shared memory <= opt-in limit
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         optin - (int)fa.sharedSizeBytes);
    cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                         cudaSharedmemCarveoutMaxShared);
    done.emplace_back(kern, dev);
}

// Launch with programmatic stream serialization (and a cluster if cluster_x > 1).
template <typename... KArgs, typename... Args>
static inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                     cudaStream_t st, int cluster_x, Args &&...args) {
    configure_kernel_once(reinterpret_cast<const void *>(kern));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int na = 0;
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    na++;
    if (cluster_x > 1) {
        attr[na].id = cudaLaunchAttributeClusterDimension;
        attr[na].val.clusterDim.x = (unsigned)cluster_x;
        attr[na].val.clusterDim.y = 1;
        attr[na].val.clusterDim.z = 1;
        na++;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

}  // namespace cq
