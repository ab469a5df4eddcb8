// noalloc.cu -- cq_lut_gemm_noalloc: the LUT GEMM for callers that cannot
// allocate device memory.
//
// Some callers hand a kernel nothing but its inputs and outputs: plugins and
// custom-op hosts whose framework owns every byte of device memory and offers
// no allocator hook, and serving processes that forbid cudaMalloc once they
// are up, because it synchronizes the device and fragments a pre-sized pool.
// They cannot provide cq_lut_gemm's workspace.  This entry point keeps the
// split-K partial sums in a fixed array compiled into the library instead.
//
// The array is kNoAllocScratchBytes (4 MiB) of device memory.  Every GPU that
// loads the library holds it until the process exits.  All calls share it and
// it keeps whatever the last call left there; every partial sum the kernel
// reads was written by the same call, so nothing needs clearing first.  Two
// calls whose work overlaps on the GPU (different streams, or different host
// threads) race on the array: serialize them.
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "../../include/cq.h"
#include "cq_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = CQ_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices];  // device address of g_scratch, per device

// Device address of g_scratch on the current device.  In host code the name
// g_scratch is only a host-side stand-in; the address must come from
// cudaGetSymbolAddress, once per device, with that device current.
cudaError_t scratch_on_current_device(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" CQ_API cq_status cq_lut_gemm_noalloc(const void *q, const float *s_x, int64_t M,
                                                int64_t K, int32_t act_bits,
                                                const uint8_t *w_idx, const void *codebook,
                                                int64_t N, float *y, cq_stream_t stream) {
    using namespace cq;
    if (M < 0 || K <= 0 || N <= 0) return CQ_ERR_INVALID_ARGUMENT;
    if (act_bits != 4 && act_bits != 8) return CQ_ERR_INVALID_ARGUMENT;
    if (K % 2) return CQ_ERR_INVALID_ARGUMENT;
    if (!w_idx || !codebook || !y || (M > 0 && (!q || !s_x))) return CQ_ERR_INVALID_ARGUMENT;
    if (!aligned16(q) || !aligned16(s_x) || !aligned16(w_idx) || !aligned16(codebook) ||
        !aligned16(y))
        return CQ_ERR_INVALID_ARGUMENT;
    if (K % 32 || N % 64 || K > (int64_t(1) << 30) || N > (int64_t(1) << 30) ||
        M > (int64_t(1) << 30))
        return CQ_ERR_UNSUPPORTED;
    if (M == 0) return CQ_OK;

    // exactly the plan and kernels of cq_lut_gemm, with the scratch in the array
    const LutGemmPlan g = plan_gemm(M, N, K);
    if (g.ws > kNoAllocScratchBytes) return CQ_ERR_UNSUPPORTED;  // beyond the fixed scratch

    void *p = nullptr;
    if (scratch_on_current_device(&p) != cudaSuccess) return CQ_ERR_CUDA;
    const cudaError_t e = run_lut_gemm(g, q, s_x, M, K, act_bits, w_idx, codebook, N, y, p,
                                       reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? CQ_OK : CQ_ERR_CUDA;
}
