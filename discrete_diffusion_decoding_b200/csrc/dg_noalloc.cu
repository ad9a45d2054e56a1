// Allocation-free entry point: the fused logits / softmax / entropy / argmax /
// self-conditioning pass and its split-vocabulary combine, with every scratch
// buffer taken from a fixed array that the library itself owns in device
// memory instead of a caller-provided workspace.
//
// Who needs it: callers that cannot allocate device memory at the point of
// the call - code that runs inside a framework whose allocator is off limits to
// plugins, a process whose memory budget is fixed up front, or a host thread
// that must not touch the allocator on a latency-critical path.  They pass only
// their inputs and outputs.
//
// Cost of the convenience: every GPU that loads the library holds
// kNoAllocScratchBytes for the fused pass until the process exits, and all calls
// on one device share it (calls whose GPU work overlaps would race).
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/dg.h"
#include "dg_common.cuh"
#include "dg_fused.h"
#include "dg_host.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;   // 64 MiB, stated in include/dg.h

}  // namespace

// The library-owned scratch.  In host code this name is only a stand-in for the
// symbol: its device address comes from cudaGetSymbolAddress, per device.
static __device__ __align__(256) uint8_t g_dg_noalloc_scratch[kNoAllocScratchBytes];

namespace {

struct DeviceScratch {
    void* ptr = nullptr;
    bool resolved = false;
};
DeviceScratch g_device_scratch[64];
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device (resolved once per device).
dg_status scratch_on_current_device(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DG_ECUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    DeviceScratch& e = g_device_scratch[dev];
    if (!e.resolved) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_dg_noalloc_scratch) != cudaSuccess || ptr == nullptr) return DG_ECUDA;
        e.ptr = ptr;
        e.resolved = true;
    }
    *out = e.ptr;
    return DG_OK;
}

// Zero the canvas stop flags (every canvas takes part), the error word and the
// fused kernel's group counters left over from the previous call.
__global__ void dg_noalloc_clear_kernel(int32_t* stop, int C, int32_t* err, uint32_t* counters, int n_words) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < C || i < n_words || i < 4; i += gridDim.x * blockDim.x) {
        if (i < C) stop[i] = 0;
        if (i < 4) err[i] = 0;
        if (i < n_words) counters[i] = 0u;
    }
}

}  // namespace

extern "C" dg_status dg_denoise_stats_noalloc(const dg_params* p, int step, const void* h_dev, const void* W_dev,
                                              const void* E_dev, float* entropy_dev, int32_t* argmax_dev,
                                              float* lse_dev, float* selfcond_dev, void* stream) {
    using namespace dg;
    host::set_last_launches(0);
    if (!p || step < 1 || step > p->max_steps) return DG_EINVAL;
    if (p->logits_format != 0) return DG_EUNSUPPORTED;      // bf16 logits only
    if (!h_dev || !W_dev || !E_dev || !entropy_dev || !argmax_dev) return DG_EINVAL;
    const uintptr_t mis = reinterpret_cast<uintptr_t>(h_dev) | reinterpret_cast<uintptr_t>(W_dev) |
                          reinterpret_cast<uintptr_t>(E_dev) | reinterpret_cast<uintptr_t>(selfcond_dev);
    if (mis & 15u) return DG_EINVAL;
    Plan pl;
    const dg_status planned = host::plan_current_device(p, &pl);   // also validates the shape
    if (planned != DG_OK) return planned;
    const Layout L = make_layout(pl);
    if (L.total > kNoAllocScratchBytes) return DG_ENOMEM;    // beyond the fixed scratch

    void* ws = nullptr;
    const dg_status got = scratch_on_current_device(&ws);
    if (got != DG_OK) return got;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* base = static_cast<uint8_t*>(ws);
    dg_noalloc_clear_kernel<<<4, 256, 0, s>>>(reinterpret_cast<int32_t*>(base + L.stop), pl.C,
                                              reinterpret_cast<int32_t*>(base + L.err),
                                              reinterpret_cast<uint32_t*>(base + L.counters), pl.n_groups * 128);
    if (cudaGetLastError() != cudaSuccess) return DG_ECUDA;

    // statistics only: no seeds, no sampler state, and the argmax mode (no sample is drawn)
    dg_params q = *p;
    q.accept_mode = 0;
    q.accept_rule = 0;
    host::PassIO io{};
    io.h = h_dev;
    io.W = W_dev;
    io.E = E_dev;
    io.entropy = entropy_dev;
    io.argmax = argmax_dev;
    io.lse = lse_dev;
    io.selfcond = selfcond_dev;
    io.vocab_offset = 0;
    io.vocab_rows = pl.V;
    const dg_status r = host::launch_fused_and_combine(&q, pl, L, ws, step, io, s);
    if (r != DG_OK) return r;
    host::set_last_launches(3);
    return DG_OK;
}
