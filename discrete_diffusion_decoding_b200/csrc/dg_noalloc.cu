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

#include <cstring>
#include <mutex>

#include "../../include/dg.h"
#include "dg_common.cuh"
#include "dg_fused.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;   // 64 MiB, stated in include/dg.h
constexpr int kNoAllocSmem = dg::kFusedSmemBytes;

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

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encoder() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 3-D view {64 columns, rows, cols/64 column blocks} of a row-major bf16 matrix:
// one box of {64, box_rows, box_blocks} fills box_blocks consecutive 128-byte
// swizzle atoms (the layout the UMMA descriptors use: K-major for h and W,
// MN-major for P^T and E).
bool encode_blocks_3d(EncodeTiledFn enc, CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                      uint32_t box_rows, uint32_t box_blocks) {
    if (!enc || cols % 64 != 0) return false;
    cuuint64_t dims[3] = {64, rows, cols / 64};
    cuuint64_t strides[2] = {cols * 2, 128};
    cuuint32_t box[3] = {64, box_rows, box_blocks};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <class T>
T* at(void* base, size_t off) {
    return reinterpret_cast<T*>(static_cast<uint8_t*>(base) + off);
}

}  // namespace

extern "C" dg_status dg_denoise_stats_noalloc(const dg_params* p, int step, const void* h_dev, const void* W_dev,
                                              const void* E_dev, float* entropy_dev, int32_t* argmax_dev,
                                              float* lse_dev, float* selfcond_dev, void* stream) {
    using namespace dg;
    if (!p || step < 1 || step > p->max_steps) return DG_EINVAL;
    if (!h_dev || !W_dev || !E_dev || !entropy_dev || !argmax_dev) return DG_EINVAL;
    const uintptr_t mis = reinterpret_cast<uintptr_t>(h_dev) | reinterpret_cast<uintptr_t>(W_dev) |
                          reinterpret_cast<uintptr_t>(E_dev) | reinterpret_cast<uintptr_t>(selfcond_dev);
    if (mis & 15u) return DG_EINVAL;
    int G = 0, n_groups = 0, slice = 0;
    const dg_status planned = dg_plan(p, &G, &n_groups, &slice);   // also validates the shape
    if (planned != DG_OK) return planned;

    Plan pl{};
    pl.C = p->n_canvas;
    pl.N = p->n_canvas * kCanvas;
    pl.V = p->vocab;
    pl.d = p->hidden;
    pl.group = G;
    pl.slice = slice;
    pl.n_groups = n_groups;
    pl.steps_per_tile = (p->vocab + G * kBV - 1) / (G * kBV);
    pl.max_seg = 1;
    for (int n_ct = 1; n_ct <= pl.C; ++n_ct) {
        const int pg = pieces_per_group(n_ct, pl.n_groups);
        if (pg > pl.max_seg) pl.max_seg = pg;
    }
    pl.n_slots = pl.n_groups * pl.max_seg;
    const Layout L = make_layout(pl);
    if (L.total > kNoAllocScratchBytes) return DG_ENOMEM;    // beyond the fixed scratch

    void* ws = nullptr;
    const dg_status got = scratch_on_current_device(&ws);
    if (got != DG_OK) return got;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    int32_t* stop = at<int32_t>(ws, L.stop);
    uint32_t* counters = at<uint32_t>(ws, L.counters);
    dg_noalloc_clear_kernel<<<4, 256, 0, s>>>(stop, pl.C, at<int32_t>(ws, L.err), counters, pl.n_groups * 128);
    if (cudaGetLastError() != cudaSuccess) return DG_ECUDA;

    const float T = dg_temperature(p, step);
    FusedArgs fa;
    std::memset(&fa, 0, sizeof(fa));
    const uint64_t prow_total = static_cast<uint64_t>(pl.n_groups) * 2 * pl.group * kCanvas;
    if (!encode_blocks_3d(encoder(), &fa.map_h, h_dev, pl.N, pl.d, kTileM, kKChunk / 64) ||
        !encode_blocks_3d(encoder(), &fa.map_w, W_dev, pl.V, pl.d, kBV / 2, kKChunk / 64) ||
        !encode_blocks_3d(encoder(), &fa.map_e, E_dev, pl.V, pl.d, kVChunk, pl.slice / 128) ||
        !encode_blocks_3d(encoder(), &fa.map_p, at<void>(ws, L.pbuf), prow_total, kCanvas, kVChunk, 2))
        return DG_ECUDA;
    fa.stop = stop;
    fa.counters = counters;
    fa.rowmax = at<float>(ws, L.rowmax);
    fa.pbuf = at<__nv_bfloat16>(ws, L.pbuf);
    fa.stats = at<float4>(ws, L.stats);
    fa.stat_idx = at<int32_t>(ws, L.stat_idx);
    fa.opart = at<float>(ws, L.opart);
    fa.err = at<int>(ws, L.err);
    fa.C = pl.C;
    fa.V = pl.V;
    fa.d = pl.d;
    fa.G = pl.group;
    fa.keep_w_stages = E_dev == W_dev ? (pl.d / kKChunk) * kKeepWTenths / 10 : 0;
    fa.slice = pl.slice;
    fa.n_groups = pl.n_groups;
    fa.steps_per_tile = pl.steps_per_tile;
    fa.max_seg = pl.max_seg;
    fa.scale_log2 = static_cast<float>(1.4426950408889634 / static_cast<double>(T));

    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(2 * pl.n_groups * pl.group);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kNoAllocSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, dg_fused_kernel, fa) != cudaSuccess) return DG_ECUDA;

    CombineArgs ca;
    ca.stop = stop;
    ca.counters = counters;
    ca.stats = fa.stats;
    ca.stat_idx = fa.stat_idx;
    ca.skey = nullptr;          // statistics only: no acceptance, so no sample
    ca.sidx = nullptr;
    ca.accept_mode = 0;
    ca.accept_rule = 0;
    ca.kept = nullptr;
    ca.opart = fa.opart;
    ca.entropy = entropy_dev;
    ca.argmax = argmax_dev;
    ca.lse = lse_dev;
    ca.selfcond = selfcond_dev;
    ca.C = pl.C;
    ca.d = pl.d;
    ca.G = pl.group;
    ca.n_groups = pl.n_groups;
    ca.steps_per_tile = pl.steps_per_tile;
    ca.max_seg = pl.max_seg;
    ca.seeds = nullptr;
    ca.tokens = nullptr;     // no sampler state in this entry point
    ca.accept = nullptr;
    ca.bound = 0.f;
    ca.step = step;
    ca.V = pl.V;
    dg_combine_kernel<<<combine_grid(pl.N, pl.d), 256, 0, s>>>(ca);
    if (cudaGetLastError() != cudaSuccess) return DG_ECUDA;
    return DG_OK;
}
