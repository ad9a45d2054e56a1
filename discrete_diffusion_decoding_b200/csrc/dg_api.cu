// C ABI of the denoise-sampling stage: argument checks, planning, workspace
// layout, TMA descriptor encoding and the launch sequence of one step.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/dg.h"
#include "dg_common.cuh"
#include "dg_fused.h"

using namespace dg;

namespace {

constexpr int kFusedSmem = kFusedSmemBytes;
thread_local int g_last_launches = 0;

// Event pairs recorded around fused-kernel launches while profiling is enabled.
struct ProfileState {
    bool on = false;
    int max_records = 0;
    std::vector<cudaEvent_t> start, stop;
    int used = 0;
};
thread_local ProfileState g_prof;

void profile_release() {
    for (auto e : g_prof.start) cudaEventDestroy(e);
    for (auto e : g_prof.stop) cudaEventDestroy(e);
    g_prof.start.clear();
    g_prof.stop.clear();
    g_prof.used = 0;
    g_prof.on = false;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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

int device_sm_count() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    return sms;
}

bool fused_attr_set() {
    static std::once_flag once;
    static cudaError_t err = cudaSuccess;
    std::call_once(once, [] {
        err = cudaFuncSetAttribute(dg_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kFusedSmem);
        if (err == cudaSuccess)
            err = cudaFuncSetAttribute(dg_fused_sample_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kFusedSmem);
    });
    return err == cudaSuccess;
}

// How many CTA pairs of the fused kernel can be resident at once on the current
// device (a pair is a cluster of two CTAs, one CTA per SM).
int resident_pairs() {
    static int cache[64];
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
    std::lock_guard<std::mutex> lock(mu);
    if (cache[dev] > 0) return cache[dev];
    if (!fused_attr_set()) return -1;
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(2 * 64);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kFusedSmem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, dg_fused_kernel, &cfg) != cudaSuccess || n <= 0) return -1;
    cache[dev] = n;
    return n;
}

bool params_ok(const dg_params* p) {
    if (!p) return false;
    if (p->n_canvas < 1 || p->n_canvas > kMaxCanvas) return false;
    if (p->canvas_len != kCanvas) return false;
    if (p->vocab < kBV || p->vocab % kBV != 0) return false;
    if (p->hidden < 64 || p->hidden % 64 != 0) return false;
    if (p->max_steps < 1) return false;
    if (!(p->t_start > 0.f) || !(p->t_end > 0.f)) return false;
    if (p->stability < 0) return false;
    if (p->accept_mode != 0 && p->accept_mode != 1) return false;
    if (p->accept_rule != 0 && p->accept_rule != 1) return false;
    return true;
}

// Returns DG_OK and fills `pl`, or the reason the shape is not handled.
// `pairs` is the number of CTA pairs resident at once.
dg_status make_plan(const dg_params* p, int pairs, Plan* pl) {
    if (!params_ok(p)) return DG_EINVAL;
    int slice = 0;
    if (p->group > 0) {
        if (p->hidden % p->group != 0) return DG_EUNSUPPORTED;
        slice = p->hidden / p->group;
        if (slice % 128 != 0 || slice > kMaxSlice) return DG_EUNSUPPORTED;
    } else {
        for (int s = kMaxSlice; s >= 128; s -= 128)
            if (p->hidden % s == 0) {
                slice = s;
                break;
            }
        if (slice == 0) return DG_EUNSUPPORTED;
    }
    const int G = p->hidden / slice;
    if (pairs < G) return DG_EUNSUPPORTED;
    Plan q{};
    q.C = p->n_canvas;
    q.N = p->n_canvas * kCanvas;
    q.V = p->vocab;
    q.d = p->hidden;
    q.group = G;
    q.slice = slice;
    q.n_groups = pairs / G;
    q.steps_per_tile = (p->vocab + G * kBV - 1) / (G * kBV);
    // partial slots per group: the most pieces any active-canvas count can give a group
    q.max_seg = 1;
    for (int n_ct = 1; n_ct <= q.C; ++n_ct) {
        const int pg = pieces_per_group(n_ct, q.n_groups);
        if (pg > q.max_seg) q.max_seg = pg;
    }
    q.n_slots = q.n_groups * q.max_seg;
    *pl = q;
    return DG_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

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
T* at(void* ws, size_t off) {
    return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

}  // namespace

extern "C" {

void dg_params_default(dg_params* p, int n_canvas, int vocab, int hidden) {
    if (!p) return;
    std::memset(p, 0, sizeof(*p));
    p->n_canvas = n_canvas;
    p->canvas_len = kCanvas;
    p->vocab = vocab;
    p->hidden = hidden;
    p->max_steps = 48;
    p->t_start = 0.8f;
    p->t_end = 0.4f;
    p->eb_bound = 0.1f;
    p->stop_thresh = 0.005f;
    p->stability = 2;
    p->tied = 1;
    p->group = 0;
    p->accept_mode = 0;
    p->accept_rule = 0;
}

float dg_temperature(const dg_params* p, int step) {
    if (!p) return NAN;
    double t = p->t_start;
    if (p->max_steps > 1)
        t = static_cast<double>(p->t_start) +
            (static_cast<double>(p->t_end) - static_cast<double>(p->t_start)) * (step - 1) / (p->max_steps - 1);
    return static_cast<float>(t);
}

const char* dg_status_string(dg_status s) {
    switch (s) {
        case DG_OK: return "ok";
        case DG_EINVAL: return "invalid argument";
        case DG_ECUDA: return "CUDA error";
        case DG_EUNSUPPORTED: return "unsupported shape";
        case DG_ETIMEOUT: return "in-kernel wait timed out";
        case DG_ENOMEM: return "workspace too small";
    }
    return "unknown status";
}

int dg_last_launch_count(void) { return g_last_launches; }

dg_status dg_plan(const dg_params* p, int* group, int* n_groups, int* slice_cols) {
    const int pairs = resident_pairs();
    if (pairs <= 0) return DG_ECUDA;
    Plan pl;
    dg_status st = make_plan(p, pairs, &pl);
    if (st != DG_OK) return st;
    if (group) *group = pl.group;
    if (n_groups) *n_groups = pl.n_groups;
    if (slice_cols) *slice_cols = pl.slice;
    return DG_OK;
}

size_t dg_workspace_size(const dg_params* p) {
    const int pairs = resident_pairs();
    if (pairs <= 0) return 0;
    Plan pl;
    if (make_plan(p, pairs, &pl) != DG_OK) return 0;
    return make_layout(pl).total;
}

dg_status dg_canvas_init(const dg_params* p, const uint64_t* seeds_dev, int32_t* tokens_dev, void* workspace_dev,
                         size_t workspace_bytes, void* stream) {
    g_last_launches = 0;
    const int pairs = resident_pairs();
    if (pairs <= 0) return DG_ECUDA;
    Plan pl;
    dg_status st = make_plan(p, pairs, &pl);
    if (st != DG_OK) return st;
    if (!seeds_dev || !tokens_dev || !workspace_dev) return DG_EINVAL;
    const Layout L = make_layout(pl);
    if (workspace_bytes < L.total) return DG_ENOMEM;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int threads = 256;
    const int blocks = (pl.N + threads - 1) / threads;
    dg_init_kernel<<<blocks, threads, 0, s>>>(seeds_dev, tokens_dev, at<int32_t>(workspace_dev, L.prev_argmax),
                                              at<int32_t>(workspace_dev, L.stable), at<int32_t>(workspace_dev, L.stop),
                                              at<int32_t>(workspace_dev, L.err), at<uint32_t>(workspace_dev, L.counters),
                                              pl.n_groups * 128, pl.C, pl.V);
    if (cudaGetLastError() != cudaSuccess) return DG_ECUDA;
    g_last_launches = 1;
    return DG_OK;
}

dg_status dg_denoise_step(const dg_params* p, int step, const void* h_dev, const void* W_dev, const void* E_dev,
                          const uint64_t* seeds_dev, int32_t* tokens_dev, float* entropy_dev, int32_t* argmax_dev,
                          uint8_t* accept_dev, float* lse_dev, float* selfcond_dev, void* workspace_dev,
                          size_t workspace_bytes, void* stream) {
    g_last_launches = 0;
    const int pairs = resident_pairs();
    if (pairs <= 0) return DG_ECUDA;
    Plan pl;
    dg_status st = make_plan(p, pairs, &pl);
    if (st != DG_OK) return st;
    if (step < 1 || step > p->max_steps) return DG_EINVAL;
    if (!h_dev || !W_dev || !E_dev || !seeds_dev || !tokens_dev || !entropy_dev || !argmax_dev || !accept_dev ||
        !workspace_dev)
        return DG_EINVAL;
    if (!aligned16(h_dev) || !aligned16(W_dev) || !aligned16(E_dev) || (selfcond_dev && !aligned16(selfcond_dev)))
        return DG_EINVAL;
    const Layout L = make_layout(pl);
    if (workspace_bytes < L.total) return DG_ENOMEM;
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    if (!fused_attr_set()) return DG_ECUDA;

    const float T = dg_temperature(p, step);
    FusedArgs fa;
    std::memset(&fa, 0, sizeof(fa));
    const uint64_t prow_total = static_cast<uint64_t>(pl.n_groups) * 2 * pl.group * kCanvas;
    if (!encode_blocks_3d(encode_fn(), &fa.map_h, h_dev, pl.N, pl.d, kTileM, kKChunk / 64) ||
        !encode_blocks_3d(encode_fn(), &fa.map_w, W_dev, pl.V, pl.d, kBV / 2, kKChunk / 64) ||
        !encode_blocks_3d(encode_fn(), &fa.map_e, E_dev, pl.V, pl.d, kVChunk, pl.slice / 128) ||
        !encode_blocks_3d(encode_fn(), &fa.map_p, at<void>(workspace_dev, L.pbuf), prow_total, kCanvas, kVChunk, 2))
        return DG_ECUDA;
    int32_t* stop = at<int32_t>(workspace_dev, L.stop);
    fa.stop = stop;
    fa.counters = at<uint32_t>(workspace_dev, L.counters);
    fa.rowmax = at<float>(workspace_dev, L.rowmax);
    fa.pbuf = at<__nv_bfloat16>(workspace_dev, L.pbuf);
    fa.stats = at<float4>(workspace_dev, L.stats);
    fa.stat_idx = at<int32_t>(workspace_dev, L.stat_idx);
    fa.opart = at<float>(workspace_dev, L.opart);
    fa.err = at<int>(workspace_dev, L.err);
    fa.seeds = seeds_dev;
    fa.skey = at<float>(workspace_dev, L.skey);
    fa.sidx = at<int32_t>(workspace_dev, L.sidx);
    fa.step = step;
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
    cfg.dynamicSmemBytes = kFusedSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;   // CTA pairs
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const bool prof = g_prof.on && g_prof.used < g_prof.max_records;
    if (prof && cudaEventRecord(g_prof.start[g_prof.used], s) != cudaSuccess) return DG_ECUDA;
    if (cudaLaunchKernelEx(&cfg, p->accept_mode == 1 ? dg_fused_sample_kernel : dg_fused_kernel, fa) != cudaSuccess)
        return DG_ECUDA;
    if (prof) {
        if (cudaEventRecord(g_prof.stop[g_prof.used], s) != cudaSuccess) return DG_ECUDA;
        ++g_prof.used;
    }

    CombineArgs ca;
    ca.stop = stop;
    ca.counters = fa.counters;
    ca.stats = fa.stats;
    ca.stat_idx = fa.stat_idx;
    ca.skey = fa.skey;
    ca.sidx = fa.sidx;
    ca.accept_mode = p->accept_mode;
    ca.accept_rule = p->accept_rule;
    ca.kept = at<int32_t>(workspace_dev, L.kept);
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
    ca.seeds = seeds_dev;
    ca.tokens = tokens_dev;
    ca.accept = accept_dev;
    ca.bound = p->eb_bound;
    ca.step = step;
    ca.V = pl.V;
    dg_combine_kernel<<<combine_grid(pl.N, pl.d), 256, 0, s>>>(ca);
    if (cudaGetLastError() != cudaSuccess) return DG_ECUDA;

    GroupAcceptArgs ga{p->accept_rule, p->eb_bound, ca.kept, seeds_dev, tokens_dev, accept_dev, pl.V};
    dg_stop_kernel<<<pl.C, kCanvas, 0, s>>>(entropy_dev, argmax_dev, at<int32_t>(workspace_dev, L.prev_argmax),
                                            at<int32_t>(workspace_dev, L.stable), stop, p->stop_thresh, p->stability,
                                            step, ga);
    if (cudaGetLastError() != cudaSuccess) return DG_ECUDA;
    g_last_launches = 3;
    return DG_OK;
}

dg_status dg_profile_enable(int max_records) {
    if (max_records < 1) return DG_EINVAL;
    profile_release();
    g_prof.start.resize(max_records);
    g_prof.stop.resize(max_records);
    for (int i = 0; i < max_records; ++i) {
        if (cudaEventCreate(&g_prof.start[i]) != cudaSuccess || cudaEventCreate(&g_prof.stop[i]) != cudaSuccess) {
            g_prof.start.resize(i);
            g_prof.stop.resize(i);
            profile_release();
            return DG_ECUDA;
        }
    }
    g_prof.max_records = max_records;
    g_prof.used = 0;
    g_prof.on = true;
    return DG_OK;
}

dg_status dg_profile_collect(int* n_records, float* mean_ms, float* total_ms) {
    float total = 0.f;
    const int n = g_prof.used;
    for (int i = 0; i < n; ++i) {
        if (cudaEventSynchronize(g_prof.stop[i]) != cudaSuccess) {
            profile_release();
            return DG_ECUDA;
        }
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, g_prof.start[i], g_prof.stop[i]) != cudaSuccess) {
            profile_release();
            return DG_ECUDA;
        }
        total += ms;
    }
    if (n_records) *n_records = n;
    if (mean_ms) *mean_ms = n ? total / n : 0.f;
    if (total_ms) *total_ms = total;
    profile_release();
    return DG_OK;
}

dg_status dg_stop_check(const dg_params* p, void* workspace_dev, size_t workspace_bytes, int32_t* stop_flags_host,
                        int32_t* stable_host, int* n_stopped_host, void* stream) {
    const int pairs = resident_pairs();
    if (pairs <= 0) return DG_ECUDA;
    Plan pl;
    dg_status st = make_plan(p, pairs, &pl);
    if (st != DG_OK) return st;
    if (!workspace_dev) return DG_EINVAL;
    const Layout L = make_layout(pl);
    if (workspace_bytes < L.total) return DG_ENOMEM;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t err_word = 0;
    if (cudaMemcpyAsync(&err_word, at<int32_t>(workspace_dev, L.err), sizeof(int32_t), cudaMemcpyDeviceToHost, s) !=
        cudaSuccess)
        return DG_ECUDA;
    int32_t flags_local[kMaxCanvas];
    int32_t* flags = stop_flags_host ? stop_flags_host : flags_local;
    if (cudaMemcpyAsync(flags, at<int32_t>(workspace_dev, L.stop), sizeof(int32_t) * pl.C, cudaMemcpyDeviceToHost,
                        s) != cudaSuccess)
        return DG_ECUDA;
    if (stable_host && cudaMemcpyAsync(stable_host, at<int32_t>(workspace_dev, L.stable), sizeof(int32_t) * pl.C,
                                       cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return DG_ECUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return DG_ECUDA;
    if (n_stopped_host) {
        int n = 0;
        for (int c = 0; c < pl.C; ++c) n += flags[c] != 0;
        *n_stopped_host = n;
    }
    if (err_word != 0) return DG_ETIMEOUT;
    return DG_OK;
}

dg_status dg_debug_set_error(const dg_params* p, void* workspace_dev, size_t workspace_bytes, int32_t code,
                             void* stream) {
    const int pairs = resident_pairs();
    if (pairs <= 0) return DG_ECUDA;
    Plan pl;
    dg_status st = make_plan(p, pairs, &pl);
    if (st != DG_OK) return st;
    if (!workspace_dev) return DG_EINVAL;
    const Layout L = make_layout(pl);
    if (workspace_bytes < L.total) return DG_ENOMEM;
    // pageable source: the copy is complete when cudaMemcpyAsync returns, so `code` may live on the stack
    if (cudaMemcpyAsync(at<int32_t>(workspace_dev, L.err), &code, sizeof(int32_t), cudaMemcpyHostToDevice,
                        static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return DG_ECUDA;
    return DG_OK;
}

dg_status dg_stub_hidden(const dg_params* p, int step, float gain, float noise, const uint64_t* seeds_dev,
                         const void* E_dev, const int32_t* tokens_dev, void* h_dev, void* workspace_dev,
                         size_t workspace_bytes, void* stream) {
    g_last_launches = 0;
    const int pairs = resident_pairs();
    if (pairs <= 0) return DG_ECUDA;
    Plan pl;
    dg_status st = make_plan(p, pairs, &pl);
    if (st != DG_OK) return st;
    if (step < 1 || step > p->max_steps) return DG_EINVAL;
    if (!seeds_dev || !E_dev || !tokens_dev || !h_dev || !workspace_dev) return DG_EINVAL;
    if ((reinterpret_cast<uintptr_t>(E_dev) & 7u) || (reinterpret_cast<uintptr_t>(h_dev) & 7u)) return DG_EINVAL;
    const Layout L = make_layout(pl);
    if (workspace_bytes < L.total) return DG_ENOMEM;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const float a_s = static_cast<float>(static_cast<double>(step) / p->max_steps);
    const long long total = static_cast<long long>(pl.N) * (pl.d / 4);
    long long blocks = (total + 255) / 256;
    const long long cap = static_cast<long long>(device_sm_count()) * 16;
    if (cap > 0 && blocks > cap) blocks = cap;
    dg_stub_kernel<<<static_cast<int>(blocks), 256, 0, s>>>(
        seeds_dev, static_cast<const __nv_bfloat16*>(E_dev), tokens_dev, at<int32_t>(workspace_dev, L.stop),
        static_cast<__nv_bfloat16*>(h_dev), a_s, gain, noise, step, pl.d, pl.V, pl.N);
    if (cudaGetLastError() != cudaSuccess) return DG_ECUDA;
    g_last_launches = 1;
    return DG_OK;
}

}  // extern "C"
