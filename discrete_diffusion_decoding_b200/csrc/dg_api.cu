// C ABI of the denoise-sampling stage: argument checks, planning, workspace
// layout, TMA descriptor encoding and the launch sequence of one step.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include "../../include/dg.h"
#include "dg_common.cuh"
#include "dg_fused.h"
#include "dg_host.h"
#include "dg_sm100.cuh"

using namespace dg;

namespace dg {
namespace host {

namespace {

constexpr int kFusedSmem = kFusedSmemBytes;
constexpr int kMaxDevices = 64;
thread_local int g_last_launches = 0;
thread_local unsigned long long g_counter_wait_ns = DG_WAIT_LIMIT_NS;

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

// Per-device set-up state: the shared-memory attribute of the fused kernels and
// the number of CTA pairs resident at once (both belong to one device).
std::mutex g_dev_mu;
bool g_attr_done[kMaxDevices];
int g_pairs[kMaxDevices];

bool current_device(int* dev) {
    return cudaGetDevice(dev) == cudaSuccess && *dev >= 0 && *dev < kMaxDevices;
}

// Caller holds g_dev_mu; `dev` is the current device.
bool attr_set_locked(int dev) {
    if (g_attr_done[dev]) return true;
    for (auto k : {dg_fused_kernel, dg_fused_sample_kernel, dg_fused_fp8_kernel, dg_fused_fp8_sample_kernel})
        if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kFusedSmem) != cudaSuccess)
            return false;
    g_attr_done[dev] = true;
    return true;
}

bool params_ok(const dg_params* p) {
    if (!p) return false;
    if (p->n_canvas < 1 || p->n_canvas > kMaxCanvas) return false;
    if (p->canvas_len != kCanvas) return false;
    if (p->vocab < kBV || p->vocab % kBV != 0) return false;
    if (p->hidden < 128 || p->hidden % 128 != 0) return false;
    if (p->max_steps < 1) return false;
    if (!(p->t_start > 0.f) || !(p->t_end > 0.f)) return false;
    if (p->stability < 0) return false;
    if (p->accept_mode != 0 && p->accept_mode != 1) return false;
    if (p->accept_rule != 0 && p->accept_rule != 1) return false;
    if (p->logits_format != 0 && p->logits_format != 1) return false;
    if (p->head_layout != 0 && p->head_layout != 1) return false;
    return true;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <class T>
T* at(void* ws, size_t off) {
    return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

}  // namespace

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

bool encode_blocks_3d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
                      uint32_t box_blocks) {
    EncodeTiledFn enc = encode_fn();
    if (!enc || cols % 64 != 0) return false;
    cuuint64_t dims[3] = {64, rows, cols / 64};
    cuuint64_t strides[2] = {cols * 2, 128};
    cuuint32_t box[3] = {64, box_rows, box_blocks};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A bf16 [rows, cols] head in the tile-major layout (tiled_index): {64 columns, 128 rows,
// (rows/128) (cols/64) atoms}, atoms 16 KB apart, so a box of {64, 128, box_blocks} at atom z
// is box_blocks consecutive atoms of one row tile - one contiguous block of memory.
bool encode_tiled_3d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_blocks) {
    EncodeTiledFn enc = encode_fn();
    if (!enc || cols % 64 != 0 || rows % 128 != 0) return false;
    cuuint64_t dims[3] = {64, 128, (rows / 128) * (cols / 64)};
    cuuint64_t strides[2] = {128, 128 * 128};
    cuuint32_t box[3] = {64, 128, box_blocks};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The same view of a row-major matrix of 8-bit codes: {128 columns, rows, cols/128 blocks},
// so a box of {128, box_rows, box_blocks} fills box_blocks 128-byte swizzle atoms.
bool encode_bytes_3d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
                     uint32_t box_blocks) {
    EncodeTiledFn enc = encode_fn();
    if (!enc || cols % 128 != 0) return false;
    cuuint64_t dims[3] = {128, rows, cols / 128};
    cuuint64_t strides[2] = {cols, 128};
    cuuint32_t box[3] = {128, box_rows, box_blocks};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int device_sm_count() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    return sms;
}

bool fused_attr_set() {
    int dev = 0;
    if (!current_device(&dev)) return false;
    std::lock_guard<std::mutex> lock(g_dev_mu);
    return attr_set_locked(dev);
}

int resident_pairs() {
    int dev = 0;
    if (!current_device(&dev)) return -1;
    std::lock_guard<std::mutex> lock(g_dev_mu);
    if (g_pairs[dev] > 0) return g_pairs[dev];
    if (!attr_set_locked(dev)) return -1;
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
    g_pairs[dev] = n;
    return n;
}

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
    if (p->logits_format == 1 && p->hidden % 256 != 0) return DG_EUNSUPPORTED;   // 256 E4M3 values per stage
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
    q.fp8 = p->logits_format == 1;
    q.tiled = p->head_layout == 1;
    if (q.fp8 && q.tiled) return DG_EUNSUPPORTED;
    *pl = q;
    return DG_OK;
}

dg_status plan_current_device(const dg_params* p, Plan* pl) {
    const int pairs = resident_pairs();
    if (pairs <= 0) return DG_ECUDA;
    return make_plan(p, pairs, pl);
}

void set_last_launches(int n) { g_last_launches = n; }

PartialLayout partial_layout(int N, int d) {
    PartialLayout P{};
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t a = o;
        o = align_up(o + bytes, 256);
        return a;
    };
    P.stats = take(sizeof(float4) * static_cast<size_t>(N));
    P.idx = take(sizeof(int32_t) * static_cast<size_t>(N));
    P.skey = take(sizeof(float) * static_cast<size_t>(N));
    P.sidx = take(sizeof(int32_t) * static_cast<size_t>(N));
    P.o = take(sizeof(float) * static_cast<size_t>(N) * d);
    P.total = o;
    return P;
}

// Launch a kernel that consumes only what the kernel before it on the stream wrote, with
// programmatic stream serialization: it is set up while its predecessor runs and waits
// (griddepcontrol.wait at its top) for the predecessor to complete, hiding the launch gap.
template <class... KArgs, class... Args>
cudaError_t launch_after(void (*kern)(KArgs...), dim3 grid, dim3 block, cudaStream_t s, Args&&... args) {
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

dg_status launch_fused_and_combine(const dg_params* p, const Plan& pl, const Layout& L, void* ws, int step,
                                   const PassIO& io, cudaStream_t s) {
    if (!fused_attr_set()) return DG_ECUDA;
    const float T = dg_temperature(p, step);
    FusedArgs fa;
    std::memset(&fa, 0, sizeof(fa));
    const uint64_t prow_total = static_cast<uint64_t>(pl.n_groups) * 2 * pl.group * kCanvas;
    if (pl.fp8) {
        // the step's hidden states to E4M3 codes with a power-of-two scale per position
        dg_quant_rows_kernel<<<pl.N, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(io.h), pl.d,
                                                  at<uint8_t>(ws, L.hq), at<int32_t>(ws, L.hexp));
        if (cudaGetLastError() != cudaSuccess) return DG_ECUDA;
    }
    const bool maps_ok =
        pl.fp8 ? encode_bytes_3d(&fa.map_h, at<void>(ws, L.hq), pl.N, pl.d, kTileM, 2) &&
                     encode_bytes_3d(&fa.map_w, io.W, io.vocab_rows, pl.d, kBV / 2, 2)
        : pl.tiled ? encode_blocks_3d(&fa.map_h, io.h, pl.N, pl.d, kTileM, kKChunk / 64) &&
                         encode_tiled_3d(&fa.map_w, io.W, io.vocab_rows, pl.d, kKChunk / 64) &&
                         encode_tiled_3d(&fa.map_e, io.E, io.vocab_rows, pl.d, pl.slice / 128)
                   : encode_blocks_3d(&fa.map_h, io.h, pl.N, pl.d, kTileM, kKChunk / 64) &&
                         encode_blocks_3d(&fa.map_w, io.W, io.vocab_rows, pl.d, kBV / 2, kKChunk / 64) &&
                         encode_blocks_3d(&fa.map_e, io.E, io.vocab_rows, pl.d, kVChunk, pl.slice / 128);
    if (!maps_ok || (pl.fp8 && !encode_blocks_3d(&fa.map_e, io.E, io.vocab_rows, pl.d, kVChunk, pl.slice / 128)) ||
        !encode_blocks_3d(&fa.map_p, at<void>(ws, L.pbuf), prow_total, kCanvas, kVChunk, 2))
        return DG_ECUDA;
    int32_t* stop = at<int32_t>(ws, L.stop);
    fa.stop = stop;
    fa.counters = at<uint32_t>(ws, L.counters);
    fa.rowmax = at<float>(ws, L.rowmax);
    fa.pbuf = at<__nv_bfloat16>(ws, L.pbuf);
    fa.stats = at<float4>(ws, L.stats);
    fa.stat_idx = at<int32_t>(ws, L.stat_idx);
    fa.opart = at<float>(ws, L.opart);
    fa.err = at<int>(ws, L.err);
    fa.clk = at<unsigned long long>(ws, L.clk);
    fa.seeds = io.seeds;
    fa.skey = at<float>(ws, L.skey);
    fa.sidx = at<int32_t>(ws, L.sidx);
    fa.step = step;
    fa.C = pl.C;
    fa.V = io.vocab_rows;
    fa.vocab_offset = io.vocab_offset;
    fa.d = pl.d;
    fa.G = pl.group;
    fa.tiled = pl.tiled;
    fa.keep_w_stages = (io.E == io.W && !pl.fp8) ? (pl.d / kKChunk) * kKeepWTenths / 10 : 0;
    if (pl.fp8) {
        fa.row_exp = at<int32_t>(ws, L.hexp);
        fa.w_exp = p->w_scale_exp;
    }
    fa.slice = pl.slice;
    fa.n_groups = pl.n_groups;
    fa.steps_per_tile = (io.vocab_rows + pl.group * kBV - 1) / (pl.group * kBV);
    fa.max_seg = pl.max_seg;
    fa.scale_log2 = static_cast<float>(1.4426950408889634 / static_cast<double>(T));
    fa.counter_wait_ns = g_counter_wait_ns;

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
    void (*kern)(const FusedArgs) = p->accept_mode == 1 ? (pl.fp8 ? dg_fused_fp8_sample_kernel : dg_fused_sample_kernel)
                                                        : (pl.fp8 ? dg_fused_fp8_kernel : dg_fused_kernel);
    if (cudaLaunchKernelEx(&cfg, kern, fa) != cudaSuccess) return DG_ECUDA;
    if (prof) {
        if (cudaEventRecord(g_prof.stop[g_prof.used], s) != cudaSuccess) return DG_ECUDA;
        ++g_prof.used;
    }

    CombineArgs ca;
    std::memset(&ca, 0, sizeof(ca));
    ca.stop = stop;
    ca.err = fa.err;
    ca.counters = fa.counters;
    ca.stats = fa.stats;
    ca.stat_idx = fa.stat_idx;
    ca.skey = fa.skey;
    ca.sidx = fa.sidx;
    ca.accept_mode = p->accept_mode;
    ca.accept_rule = p->accept_rule;
    ca.kept = at<int32_t>(ws, L.kept);
    ca.opart = fa.opart;
    ca.entropy = io.entropy;
    ca.argmax = io.argmax;
    ca.lse = io.lse;
    ca.selfcond = io.selfcond;
    if (io.partial) {
        const PartialLayout P = partial_layout(pl.N, pl.d);
        uint8_t* base = static_cast<uint8_t*>(io.partial);
        ca.part_stats = reinterpret_cast<float4*>(base + P.stats);
        ca.part_idx = reinterpret_cast<int32_t*>(base + P.idx);
        ca.part_skey = reinterpret_cast<float*>(base + P.skey);
        ca.part_sidx = reinterpret_cast<int32_t*>(base + P.sidx);
        ca.part_o = reinterpret_cast<float*>(base + P.o);
    }
    ca.C = pl.C;
    ca.d = pl.d;
    ca.G = pl.group;
    ca.n_groups = pl.n_groups;
    ca.steps_per_tile = fa.steps_per_tile;
    ca.max_seg = pl.max_seg;
    ca.seeds = io.seeds;
    ca.tokens = io.tokens;
    ca.accept = io.accept;
    ca.bound = p->eb_bound;
    ca.step = step;
    ca.V = pl.V;
    if (launch_after(dg_combine_kernel, combine_grid(pl.N, pl.d), dim3(256), s, ca) != cudaSuccess) return DG_ECUDA;
    return DG_OK;
}

}  // namespace host
}  // namespace dg

using namespace dg::host;

namespace {

dg_status launch_stop(const dg_params* p, const Plan& pl, const Layout& L, void* ws, int step,
                      const uint64_t* seeds_dev, int32_t* tokens_dev, const float* entropy_dev,
                      const int32_t* argmax_dev, uint8_t* accept_dev, cudaStream_t s) {
    GroupAcceptArgs ga{p->accept_rule, p->eb_bound, at<int32_t>(ws, L.kept), seeds_dev, tokens_dev, accept_dev,
                       pl.V};
    const cudaError_t e = launch_after(dg_stop_kernel, dim3(pl.C), dim3(kCanvas), s, entropy_dev, argmax_dev,
                                       at<int32_t>(ws, L.prev_argmax), at<int32_t>(ws, L.stable),
                                       at<int32_t>(ws, L.stop), p->stop_thresh, p->stability, step, ga);
    return e == cudaSuccess ? DG_OK : DG_ECUDA;
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
    Plan pl;
    const dg_status st = plan_current_device(p, &pl);
    if (st != DG_OK) return st;
    if (group) *group = pl.group;
    if (n_groups) *n_groups = pl.n_groups;
    if (slice_cols) *slice_cols = pl.slice;
    return DG_OK;
}

size_t dg_workspace_size(const dg_params* p) {
    Plan pl;
    if (plan_current_device(p, &pl) != DG_OK) return 0;
    return make_layout(pl).total;
}

dg_status dg_canvas_init(const dg_params* p, const uint64_t* seeds_dev, int32_t* tokens_dev, void* workspace_dev,
                         size_t workspace_bytes, void* stream) {
    g_last_launches = 0;
    Plan pl;
    const dg_status st = plan_current_device(p, &pl);
    if (st != DG_OK) return st;
    if (!seeds_dev || !tokens_dev || !workspace_dev) return DG_EINVAL;
    const Layout L = make_layout(pl);
    if (workspace_bytes < L.total) return DG_ENOMEM;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int threads = 256;
    const int blocks = (pl.N + threads - 1) / threads;
    dg_init_kernel<<<blocks, threads, 0, s>>>(seeds_dev, tokens_dev, at<int32_t>(workspace_dev, L.prev_argmax),
                                              at<int32_t>(workspace_dev, L.stable), at<int32_t>(workspace_dev, L.stop),
                                              at<int32_t>(workspace_dev, L.err),
                                              at<unsigned long long>(workspace_dev, L.clk),
                                              at<uint32_t>(workspace_dev, L.counters),
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
    Plan pl;
    const dg_status st = plan_current_device(p, &pl);
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

    PassIO io{};
    io.h = h_dev;
    io.W = W_dev;
    io.E = E_dev;
    io.seeds = seeds_dev;
    io.tokens = tokens_dev;
    io.entropy = entropy_dev;
    io.argmax = argmax_dev;
    io.accept = accept_dev;
    io.lse = lse_dev;
    io.selfcond = selfcond_dev;
    io.vocab_offset = 0;
    io.vocab_rows = pl.V;
    dg_status r = launch_fused_and_combine(p, pl, L, workspace_dev, step, io, s);
    if (r != DG_OK) return r;
    r = launch_stop(p, pl, L, workspace_dev, step, seeds_dev, tokens_dev, entropy_dev, argmax_dev, accept_dev, s);
    if (r != DG_OK) return r;
    g_last_launches = pl.fp8 ? 4 : 3;
    return DG_OK;
}

size_t dg_partial_bytes(const dg_params* p) {
    if (!p || p->n_canvas < 1 || p->n_canvas > kMaxCanvas || p->canvas_len != kCanvas || p->hidden < 128 ||
        p->hidden % 128 != 0)
        return 0;
    return partial_layout(p->n_canvas * kCanvas, p->hidden).total;
}

dg_status dg_denoise_partial(const dg_params* p, int step, int v_begin, int v_count, const void* h_dev,
                             const void* W_shard_dev, const void* E_shard_dev, const uint64_t* seeds_dev,
                             void* partial_dev, void* workspace_dev, size_t workspace_bytes, void* stream) {
    g_last_launches = 0;
    Plan pl;
    dg_status st = plan_current_device(p, &pl);
    if (st != DG_OK) return st;
    if (step < 1 || step > p->max_steps) return DG_EINVAL;
    if (v_begin < 0 || v_count < kBV || v_begin % kBV != 0 || v_count % kBV != 0 ||
        static_cast<long long>(v_begin) + v_count > p->vocab)
        return DG_EINVAL;
    if (!h_dev || !W_shard_dev || !E_shard_dev || !seeds_dev || !partial_dev || !workspace_dev) return DG_EINVAL;
    if (!aligned16(h_dev) || !aligned16(W_shard_dev) || !aligned16(E_shard_dev) || !aligned16(partial_dev))
        return DG_EINVAL;
    const Layout L = make_layout(pl);
    if (workspace_bytes < L.total) return DG_ENOMEM;
    PassIO io{};
    io.h = h_dev;
    io.W = W_shard_dev;
    io.E = E_shard_dev;
    io.seeds = seeds_dev;
    io.partial = partial_dev;
    io.vocab_offset = v_begin;
    io.vocab_rows = v_count;
    st = launch_fused_and_combine(p, pl, L, workspace_dev, step, io, static_cast<cudaStream_t>(stream));
    if (st != DG_OK) return st;
    g_last_launches = 2;
    return DG_OK;
}

dg_status dg_denoise_merge(const dg_params* p, int step, int n_parts, const void* partials_dev,
                           const uint64_t* seeds_dev, int32_t* tokens_dev, float* entropy_dev, int32_t* argmax_dev,
                           uint8_t* accept_dev, float* lse_dev, float* selfcond_dev, void* workspace_dev,
                           size_t workspace_bytes, void* stream) {
    g_last_launches = 0;
    Plan pl;
    dg_status st = plan_current_device(p, &pl);
    if (st != DG_OK) return st;
    if (step < 1 || step > p->max_steps) return DG_EINVAL;
    if (n_parts < 1 || n_parts > kMaxParts) return DG_EINVAL;
    if (!partials_dev || !seeds_dev || !tokens_dev || !entropy_dev || !argmax_dev || !accept_dev || !workspace_dev)
        return DG_EINVAL;
    if (!aligned16(partials_dev) || (selfcond_dev && !aligned16(selfcond_dev))) return DG_EINVAL;
    const Layout L = make_layout(pl);
    if (workspace_bytes < L.total) return DG_ENOMEM;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const PartialLayout P = partial_layout(pl.N, pl.d);
    MergeArgs ma;
    std::memset(&ma, 0, sizeof(ma));
    ma.partials = static_cast<const uint8_t*>(partials_dev);
    ma.part_bytes = P.total;
    ma.off_stats = P.stats;
    ma.off_idx = P.idx;
    ma.off_skey = P.skey;
    ma.off_sidx = P.sidx;
    ma.off_o = P.o;
    ma.n_parts = n_parts;
    ma.stop = at<int32_t>(workspace_dev, L.stop);
    ma.accept_mode = p->accept_mode;
    ma.accept_rule = p->accept_rule;
    ma.kept = at<int32_t>(workspace_dev, L.kept);
    ma.entropy = entropy_dev;
    ma.argmax = argmax_dev;
    ma.lse = lse_dev;
    ma.selfcond = selfcond_dev;
    ma.seeds = seeds_dev;
    ma.tokens = tokens_dev;
    ma.accept = accept_dev;
    ma.bound = p->eb_bound;
    ma.step = step;
    ma.V = pl.V;
    ma.N = pl.N;
    ma.d = pl.d;
    dg_merge_kernel<<<combine_grid(pl.N, pl.d), 256, 0, s>>>(ma);
    if (cudaGetLastError() != cudaSuccess) return DG_ECUDA;
    st = launch_stop(p, pl, L, workspace_dev, step, seeds_dev, tokens_dev, entropy_dev, argmax_dev, accept_dev, s);
    if (st != DG_OK) return st;
    g_last_launches = 2;
    return DG_OK;
}

dg_status dg_quantize_e4m3(const void* src_dev, long long rows, int cols, int per_row, uint8_t* codes_dev,
                           int32_t* exps_dev, void* stream) {
    g_last_launches = 0;
    if (!src_dev || !codes_dev || !exps_dev || rows < 1 || cols < 2 || cols % 2 != 0) return DG_EINVAL;
    if ((reinterpret_cast<uintptr_t>(src_dev) | reinterpret_cast<uintptr_t>(codes_dev) |
         reinterpret_cast<uintptr_t>(exps_dev)) & 3u)
        return DG_EINVAL;
    if (per_row && rows > 0x7fffffffLL) return DG_EINVAL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const __nv_bfloat16* src = static_cast<const __nv_bfloat16*>(src_dev);
    if (per_row) {
        dg_quant_rows_kernel<<<static_cast<unsigned>(rows), 256, 0, s>>>(src, cols, codes_dev, exps_dev);
        if (cudaGetLastError() != cudaSuccess) return DG_ECUDA;
        g_last_launches = 1;
        return DG_OK;
    }
    const long long n_pairs = rows * static_cast<long long>(cols) / 2;
    long long blocks = (n_pairs + 255) / 256;
    const long long cap = static_cast<long long>(device_sm_count()) * 8;
    if (cap > 0 && blocks > cap) blocks = cap;
    if (cudaMemsetAsync(exps_dev, 0, sizeof(int32_t), s) != cudaSuccess) return DG_ECUDA;
    dg_amax_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(src, n_pairs, reinterpret_cast<uint32_t*>(exps_dev));
    dg_amax_to_exp_kernel<<<1, 32, 0, s>>>(exps_dev);
    dg_quant_tensor_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(src, n_pairs, codes_dev, exps_dev);
    if (cudaGetLastError() != cudaSuccess) return DG_ECUDA;
    g_last_launches = 3;
    return DG_OK;
}

dg_status dg_tile_head(const void* src_dev, void* dst_dev, long long rows, int cols, int to_rows, void* stream) {
    g_last_launches = 0;
    if (!src_dev || !dst_dev || rows < 128 || rows % 128 != 0 || cols < 64 || cols % 64 != 0) return DG_EINVAL;
    if (to_rows != 0 && to_rows != 1) return DG_EINVAL;
    if (!aligned16(src_dev) || !aligned16(dst_dev)) return DG_EINVAL;
    const uintptr_t bytes = static_cast<uintptr_t>(rows) * static_cast<uintptr_t>(cols) * 2;
    const uintptr_t a = reinterpret_cast<uintptr_t>(src_dev), b = reinterpret_cast<uintptr_t>(dst_dev);
    if (a < b + bytes && b < a + bytes) return DG_EINVAL;
    const long long work = rows * (cols / 8);
    long long blocks = (work + 255) / 256;
    const long long cap = static_cast<long long>(device_sm_count()) * 16;
    if (cap > 0 && blocks > cap) blocks = cap;
    dg_tile_head_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const __nv_bfloat16*>(src_dev), static_cast<__nv_bfloat16*>(dst_dev), rows, cols, to_rows);
    if (cudaGetLastError() != cudaSuccess) return DG_ECUDA;
    g_last_launches = 1;
    return DG_OK;
}

dg_status dg_debug_set_counter_wait_limit(unsigned long long ns) {
    g_counter_wait_ns = ns == 0 ? DG_WAIT_LIMIT_NS : ns;
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
    Plan pl;
    const dg_status st = plan_current_device(p, &pl);
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

dg_status dg_last_sm_clock(const dg_params* p, const void* workspace_dev, size_t workspace_bytes, float* mhz_host,
                           void* stream) {
    if (!workspace_dev || !mhz_host) return DG_EINVAL;
    Plan pl;
    const dg_status st = plan_current_device(p, &pl);
    if (st != DG_OK) return st;
    const Layout L = make_layout(pl);
    if (workspace_bytes < L.total) return DG_ENOMEM;
    unsigned long long v[4] = {0, 0, 0, 0};
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(v, static_cast<const uint8_t*>(workspace_dev) + L.clk, sizeof(v), cudaMemcpyDeviceToHost, s) !=
            cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return DG_ECUDA;
    *mhz_host = (v[3] > v[1] && v[2] > v[0])
                    ? static_cast<float>(static_cast<double>(v[2] - v[0]) / static_cast<double>(v[3] - v[1]) * 1e3)
                    : 0.f;
    return DG_OK;
}

dg_status dg_debug_set_error(const dg_params* p, void* workspace_dev, size_t workspace_bytes, int32_t code,
                             void* stream) {
    Plan pl;
    const dg_status st = plan_current_device(p, &pl);
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
    Plan pl;
    const dg_status st = plan_current_device(p, &pl);
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
        static_cast<__nv_bfloat16*>(h_dev), a_s, gain, noise, step, pl.d, pl.V, pl.N, pl.tiled);
    if (cudaGetLastError() != cudaSuccess) return DG_ECUDA;
    g_last_launches = 1;
    return DG_OK;
}

}  // extern "C"
