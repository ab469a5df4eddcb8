// timing.cu -- measurement aids: a count of kernel launches and optional
// CUDA-event bracketing of every LUT GEMM launch.  They never change what is
// computed; when timing is off the only cost is one atomic increment per launch.
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "../../include/cq.h"
#include "cq_internal.h"

namespace cq {

static std::atomic<long long> g_launches{0};
static std::atomic<int> g_timing{0};
static std::mutex g_mu;
struct EventPair {
    cudaEvent_t a, b;
    int kind;
};
static std::vector<EventPair> g_pending, g_free;

void count_launch(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

bool timing_on() { return g_timing.load(std::memory_order_relaxed) != 0; }
bool timing_on_all() { return g_timing.load(std::memory_order_relaxed) == 2; }

// Record the opening event of a timed launch (closed by timing_end).
void timing_begin(cudaStream_t st, int kind) {
    std::lock_guard<std::mutex> lk(g_mu);
    EventPair p;
    if (!g_free.empty()) {
        p = g_free.back();
        g_free.pop_back();
    } else {
        if (cudaEventCreate(&p.a) != cudaSuccess) return;
        if (cudaEventCreate(&p.b) != cudaSuccess) {
            cudaEventDestroy(p.a);
            return;
        }
    }
    p.kind = kind;
    cudaEventRecord(p.a, st);
    g_pending.push_back(p);
}

void timing_end(cudaStream_t st) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_pending.empty()) cudaEventRecord(g_pending.back().b, st);
}

}  // namespace cq

extern "C" {

CQ_API int64_t cq_launch_count(void) { return cq::g_launches.load(); }

CQ_API int32_t cq_device_error(void) { return cq::read_device_error(); }

CQ_API cq_status cq_selftest_wait_timeout(cq_stream_t stream) {
    return cq::launch_selftest_wait(reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
               ? CQ_OK
               : CQ_ERR_CUDA;
}

CQ_API cq_status cq_timing_enable(int32_t on) {
    cq::g_timing.store(on == 2 ? 2 : on ? 1 : 0);
    return CQ_OK;
}

CQ_API cq_status cq_timing_read_launches(int32_t *kinds, float *ms, int64_t cap, int64_t *n) {
    if (!n || cap < 0 || (cap > 0 && (!kinds || !ms))) return CQ_ERR_INVALID_ARGUMENT;
    std::lock_guard<std::mutex> lk(cq::g_mu);
    int64_t i = 0;
    cq_status st = CQ_OK;
    for (auto &p : cq::g_pending) {
        float t = 0.0f;
        if (cudaEventSynchronize(p.b) != cudaSuccess ||
            cudaEventElapsedTime(&t, p.a, p.b) != cudaSuccess) {
            st = CQ_ERR_CUDA;
            t = -1.0f;
        }
        if (i < cap) {
            kinds[i] = p.kind;
            ms[i] = t;
        }
        i++;
        cq::g_free.push_back(p);
    }
    cq::g_pending.clear();
    *n = i;
    return st;
}

CQ_API cq_status cq_timing_read(int64_t *launches, double *total_ms) {
    if (!launches || !total_ms) return CQ_ERR_INVALID_ARGUMENT;
    std::lock_guard<std::mutex> lk(cq::g_mu);
    double tot = 0.0;
    int64_t n = 0;
    cq_status st = CQ_OK;
    for (auto &p : cq::g_pending) {
        float ms = 0.0f;
        if (cudaEventSynchronize(p.b) != cudaSuccess ||
            cudaEventElapsedTime(&ms, p.a, p.b) != cudaSuccess) {
            st = CQ_ERR_CUDA;
        } else {
            tot += ms;
            n++;
        }
        cq::g_free.push_back(p);
    }
    cq::g_pending.clear();
    *launches = n;
    *total_ms = tot;
    return st;
}

}  // extern "C"
