// Host-side helpers shared by the entry points (dg_api.cu, dg_noalloc.cu): the
// tensor-map encoder, the per-device set-up of the fused kernels, the plan of the
// fused kernel's grid and the launch of the fused pass with its combine.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "../../include/dg.h"
#include "dg_common.cuh"
#include "dg_fused.h"

namespace dg {
namespace host {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled from the driver (resolved once per process), or null.
EncodeTiledFn encode_fn();

// 3-D view {64 columns, rows, cols/64 column blocks} of a row-major bf16 matrix:
// one box of {64, box_rows, box_blocks} fills box_blocks consecutive 128-byte
// swizzle atoms (the layout the UMMA descriptors use: K-major for h and W,
// MN-major for P^T and E).
bool encode_blocks_3d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
                      uint32_t box_blocks);

// CTA pairs of the fused kernel resident at once on the current device (-1 on a
// CUDA error).  The first call on each device also raises the fused kernels'
// dynamic shared-memory limit there (the attribute belongs to the device).
int resident_pairs();

// Makes sure the fused kernels' shared-memory attribute is set on the current device.
bool fused_attr_set();

int device_sm_count();

// DG_OK and the plan of params p for `pairs` resident pairs, or why p is not handled.
dg_status make_plan(const dg_params* p, int pairs, Plan* pl);

// Resolve the plan of p on the current device (resident_pairs + make_plan).
dg_status plan_current_device(const dg_params* p, Plan* pl);

// Records how many kernels the calling entry point launched (dg_last_launch_count).
void set_last_launches(int n);

// Where the fused pass and its combine read and write one step's data.
struct PassIO {
    const void* h;
    const void* W;
    const void* E;
    const uint64_t* seeds;   // may be null when accept_mode is 0
    int32_t* tokens;         // null: no accept / re-noise (statistics only)
    float* entropy;
    int32_t* argmax;
    uint8_t* accept;
    float* lse;
    float* selfcond;
    void* partial;           // non-null: write this shard's merged statistics + O here instead of finishing
    int vocab_offset;        // vocabulary index of the first row of W / E (0 unless a shard)
    int vocab_rows;          // rows of W / E streamed (the shard's size, or the whole vocabulary)
};

// Launch the fused pass and the split-vocabulary combine of one step on `stream`
// (2 launches).  `ws` holds the layout L of plan pl.
dg_status launch_fused_and_combine(const dg_params* p, const Plan& pl, const Layout& L, void* ws, int step,
                                   const PassIO& io, cudaStream_t stream);

// Byte layout of one shard's partial (dg_partial_bytes): per position a float4
// {m, l, u, best}, an int32 index, a float sampled key and an int32 sampled index,
// then the unnormalised self-conditioning numerator [N, d] fp32.
struct PartialLayout {
    size_t stats, idx, skey, sidx, o, total;
};
PartialLayout partial_layout(int N, int d);

}  // namespace host
}  // namespace dg
