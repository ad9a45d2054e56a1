// Kernel argument blocks and kernel declarations shared by the launch code.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

namespace dg {

struct FusedArgs {
    // every operand as a 3-D view {64 columns, rows, column blocks of 64} of a
    // row-major bf16 matrix, so that one box fills several 128-byte swizzle atoms
    CUtensorMap map_h;   // h [N, d], box {64, 128 rows, 2}: a 128 x 128 K-major tile
    CUtensorMap map_w;   // W [V, d], box {64, 128 rows, 2} (half of a 256-row tile per CTA)
    CUtensorMap map_e;   // E [V, d], box {64, 128 vocab rows, slice/128}: MN-major B operand
    CUtensorMap map_p;   // P^T scratch [n_groups*2*G*256 vocab rows, 256 canvas rows],
                         // box {64, 128 vocab rows, 2}: MN-major A operand
    const int32_t* stop;
    uint32_t* counters;
    float* rowmax;
    __nv_bfloat16* pbuf;
    float4* stats;
    int32_t* stat_idx;
    float* opart;
    int* err;
    unsigned long long* clk;   // CTA 0 writes SM cycles and global ns at the start and end of its MMA loop
    // sampled acceptance (dg_fused_sample_kernel only): per-canvas Philox seeds, the
    // step, and the best Gumbel-max key / index of every (piece, pair, position)
    const uint64_t* seeds;
    float* skey;
    int32_t* sidx;
    int step;
    int C, V, d, G, slice, n_groups, steps_per_tile, max_seg;
    int vocab_offset;    // vocabulary index of row 0 of W / E (a shard of the vocabulary; 0 otherwise):
                         // added to the argmax and sample indices and to the sampled mode's chunk counter
    int tiled;           // W and E in the tile-major head layout (dg_tile_head): atoms of 128 rows x 64
                         // columns, [row tile][column atom], so every 3-D box is one contiguous block
    int keep_w_stages;   // E aliases W: the first keep_w_stages hidden-column stages of every W
                         // tile keep normal L2 priority, so the self-conditioning pass finds them
                         // there (0 when E is a separate matrix)
    float scale_log2;    // log2(e) / T
    // E4M3 logits (dg_fused_fp8_*): map_h / map_w view the 8-bit codes; row_exp [N] holds the hidden
    // states' per-position exponents, w_exp the head's, so z = 2^(row_exp + w_exp) S / T
    const int32_t* row_exp;
    int w_exp;
    unsigned long long counter_wait_ns;   // limit of the waits on other CTAs' counters (the drains keep theirs)
};

struct CombineArgs {
    const int32_t* stop;
    const int* err;          // the fused kernel's error word: when set, every output is poisoned (NaN, -1)
    uint32_t* counters;
    const float4* stats;
    const int32_t* stat_idx;
    const float* skey;       // sampled acceptance: Gumbel-max keys / indices (accept_mode 1)
    const int32_t* sidx;
    int accept_mode;         // 0: keep the argmax, 1: keep the Gumbel-max sample
    int accept_rule;         // 0: accept per position here; 1: only store the kept token (group rule)
    int32_t* kept;           // [N] the kept token of every position (accept_rule 1)
    const float* opart;
    float* entropy;
    int32_t* argmax;
    float* lse;
    float* selfcond;
    // entropy-bounded accept / re-noise of each position (skipped when tokens is null)
    const uint64_t* seeds;
    int32_t* tokens;
    uint8_t* accept;
    float bound;
    int step, V;
    int C, d, G, n_groups, steps_per_tile, max_seg;
    // shard mode (part_stats non-null): write the merged statistics of this vocabulary shard and
    // its unnormalised self-conditioning numerator instead of finishing (no accept / re-noise)
    float4* part_stats;      // [N] {m, l, u, best}: m absolute (log2 units), l and u relative to m
    int32_t* part_idx;       // [N] argmax of the shard (vocabulary index)
    float* part_skey;        // [N] best sampled key (accept_mode 1)
    int32_t* part_sidx;      // [N] its vocabulary index
    float* part_o;           // [N, d] sum_v 2^(y_v - m) E_v
};

// Merge of the partials of n_parts vocabulary shards (dg_denoise_merge), laid out
// back to back, part_bytes apart, each as dg_host.h's PartialLayout.
struct MergeArgs {
    const uint8_t* partials;
    size_t part_bytes, off_stats, off_idx, off_skey, off_sidx, off_o;
    int n_parts;
    const int32_t* stop;
    int accept_mode, accept_rule;
    int32_t* kept;
    float* entropy;
    int32_t* argmax;
    float* lse;
    float* selfcond;
    const uint64_t* seeds;
    int32_t* tokens;
    uint8_t* accept;
    float bound;
    int step, V, N, d;
};

// Combine grid: one CTA per (position, block of kCombineCols self-conditioning columns).
constexpr int kCombineCols = 1024;
inline dim3 combine_grid(int N, int d) { return dim3(N, (d + kCombineCols - 1) / kCombineCols); }

__global__ void dg_fused_kernel(const __grid_constant__ FusedArgs a);          // argmax acceptance
__global__ void dg_fused_sample_kernel(const __grid_constant__ FusedArgs a);   // + Gumbel-max sample
__global__ void dg_fused_fp8_kernel(const __grid_constant__ FusedArgs a);      // E4M3 logits operands
__global__ void dg_fused_fp8_sample_kernel(const __grid_constant__ FusedArgs a);
// E4M3 quantisation (dg_fp8.cu)
__global__ void dg_quant_rows_kernel(const __nv_bfloat16* src, int cols, uint8_t* codes, int32_t* exps);
__global__ void dg_amax_kernel(const __nv_bfloat16* src, long long n_pairs, uint32_t* amax_bits);
__global__ void dg_amax_to_exp_kernel(int32_t* exps);
__global__ void dg_quant_tensor_kernel(const __nv_bfloat16* src, long long n_pairs, uint8_t* codes,
                                       const int32_t* exps);
__global__ void dg_combine_kernel(const CombineArgs a);
__global__ void dg_merge_kernel(const MergeArgs a);

// small kernels (dg_small.cu)
__global__ void dg_init_kernel(const uint64_t* seeds, int32_t* tokens, int32_t* prev_argmax, int32_t* stable,
                               int32_t* stop, int32_t* err, unsigned long long* clk, uint32_t* counters,
                               int n_counter_words, int C, int V);
// Group entropy-bounded accept, applied by dg_stop_kernel before the stop reduction
// when `rule` is 1 (nothing happens with rule 0 or a null tokens pointer).
struct GroupAcceptArgs {
    int rule;
    float bound;
    const int32_t* kept;
    const uint64_t* seeds;
    int32_t* tokens;
    uint8_t* accept;
    int V;
};

__global__ void dg_stop_kernel(const float* entropy, const int32_t* argmax, int32_t* prev_argmax, int32_t* stable,
                               int32_t* stop, float stop_thresh, int stability, int step, GroupAcceptArgs ga);
__global__ void dg_stub_kernel(const uint64_t* seeds, const __nv_bfloat16* E, const int32_t* tokens,
                               const int32_t* stop, __nv_bfloat16* h, float a_s, float gain, float noise, int step,
                               int d, int V, int N, int tiled);
// Row-major [V, d] bf16 head -> tile-major (or back when to_rows is 1).
__global__ void dg_tile_head_kernel(const __nv_bfloat16* src, __nv_bfloat16* dst, long long V, int d, int to_rows);

}  // namespace dg
