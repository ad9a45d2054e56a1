// The element-wise and per-canvas kernels around the fused pass: canvas
// initialisation, the two-fold stop reduction and the benchmark-only denoiser
// stub (the entropy-bounded accept / re-noise runs inside dg_combine_kernel).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "dg_common.cuh"
#include "dg_fused.h"

namespace dg {

// Uniform-state noise for a fresh canvas (deep dive, reverse diffusion step 1;
// juhoplayground, entropy bounded sampler: start from uniform random tokens),
// plus a reset of the per-canvas state.
__global__ void dg_init_kernel(const uint64_t* seeds, int32_t* tokens, int32_t* prev_argmax, int32_t* stable,
                               int32_t* stop, int32_t* err, unsigned long long* clk, uint32_t* counters,
                               int n_counter_words, int C, int V) {
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    const int N = C * kCanvas;
    if (n < N) {
        const int c = n / kCanvas, i = n % kCanvas;
        tokens[n] = philox_token(seeds[c], static_cast<uint32_t>(i), 0u, static_cast<uint32_t>(c), kTagInit,
                                 static_cast<uint32_t>(V));
        prev_argmax[n] = -1;
    }
    if (n < C) {
        stable[n] = 0;
        stop[n] = 0;
    }
    if (n < 4) {
        err[n] = 0;
        clk[n] = 0ull;
    }
    for (int w = n; w < n_counter_words; w += gridDim.x * blockDim.x) counters[w] = 0u;
}

// Group entropy-bounded accept of one canvas (juhoplayground overview, entropy
// bounded sampler: token groups are accepted by entropy; deep dive bound 0.1):
// the positions ordered by (max(H, 0), position) - a bitonic sort of 64-bit keys
// (entropy bits, position), monotone because the entropy is non-negative - and the
// longest prefix whose cumulative entropy is <= bound keeps its token; the other
// positions take the uniform re-noise draw (Philox tag 1, this step).  The
// cumulative sum runs in sorted order in one thread.
__device__ void group_accept(const float* entropy, const GroupAcceptArgs& ga, int c, int step) {
    __shared__ unsigned long long key[kCanvas];
    __shared__ int n_acc;
    const int tid = threadIdx.x;
    // a NaN entropy (a position poisoned by a failed pass) sorts last and is never accepted
    const float hv = entropy[c * kCanvas + tid];
    const float h = hv != hv ? INFINITY : fmaxf(hv, 0.f);
    key[tid] = (static_cast<unsigned long long>(__float_as_uint(h)) << 32) | static_cast<unsigned>(tid);
    __syncthreads();
    for (int k = 2; k <= kCanvas; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            const int p = tid ^ j;
            if (p > tid) {
                const unsigned long long x = key[tid], y = key[p];
                const bool up = (tid & k) == 0;
                if ((x > y) == up) {
                    key[tid] = y;
                    key[p] = x;
                }
            }
            __syncthreads();
        }
    }
    if (tid == 0) {
        float S = 0.f;
        int k = 0;
        for (; k < kCanvas; ++k) {
            S += __uint_as_float(static_cast<uint32_t>(key[k] >> 32));
            if (!(S <= ga.bound)) break;
        }
        n_acc = k;
    }
    __syncthreads();
    const int i = static_cast<int>(key[tid] & 0xffffffffu);      // the position of sorted rank tid
    const int n = c * kCanvas + i;
    const bool acc = tid < n_acc;
    ga.tokens[n] = acc ? ga.kept[n]
                       : philox_token(ga.seeds[c], static_cast<uint32_t>(i), static_cast<uint32_t>(step),
                                      static_cast<uint32_t>(c), kTagRenoise, static_cast<uint32_t>(ga.V));
    ga.accept[n] = acc ? 1 : 0;
}

// Two-fold adaptive stop (deep dive, "Two-Fold Adaptive Stopping"): one CTA of
// 256 threads per canvas; the mean entropy is a fixed-order tree sum; the
// stable counter grows while the argmax vector repeats (0 at step 1) and resets
// on any change; stop = mean H < threshold AND stable >= stability.  With the
// group rule the canvas's accept / re-noise runs first (group_accept).
__global__ void __launch_bounds__(256) dg_stop_kernel(const float* entropy, const int32_t* argmax,
                                                      int32_t* prev_argmax, int32_t* stable, int32_t* stop,
                                                      float stop_thresh, int stability, int step, GroupAcceptArgs ga) {
    // launched after the kernel that wrote this step's entropy and argmax: wait for it
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int c = blockIdx.x;
    if (stop[c]) return;
    if (ga.rule == 1 && ga.tokens != nullptr) group_accept(entropy, ga, c, step);
    const int tid = threadIdx.x;
    const int n = c * kCanvas + tid;
    float h = entropy[n];
    const int am = argmax[n];
    const int changed = am != prev_argmax[n];
    prev_argmax[n] = am;
#pragma unroll
    for (int off = 16; off; off >>= 1) h += __shfl_xor_sync(0xffffffffu, h, off);
    const int any_changed = __syncthreads_or(changed);
    __shared__ float part[8];
    if ((tid & 31) == 0) part[tid >> 5] = h;
    __syncthreads();
    if (tid == 0) {
        float sum = 0.f;
        for (int w = 0; w < 8; ++w) sum += part[w];
        const float mean = sum * (1.0f / kCanvas);
        const int st = (step > 1 && !any_changed) ? stable[c] + 1 : 0;
        stable[c] = st;
        stop[c] = (mean < stop_thresh && st >= stability) ? 1 : 0;
    }
}

// Benchmark-only stand-in for the denoiser (not on the pages):
// h = gain (a E[tgt] + (1-a) E[x]) + noise n, n ~ N(0,1) by Box-Muller on the four
// words of Philox counter (i*d/4 + j, s, c, 3): (w0, w1) give elements 4j, 4j+1 and
// (w2, w3) give 4j+2, 4j+3 with u1 = (w+1) 2^-32 and u2 = w' 2^-32.
__global__ void dg_stub_kernel(const uint64_t* seeds, const __nv_bfloat16* E, const int32_t* tokens,
                               const int32_t* stop, __nv_bfloat16* h, float a_s, float gain, float noise, int step,
                               int d, int V, int N, int tiled) {
    const int q = d / 4;
    const long long total = static_cast<long long>(N) * q;
    for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < total;
         e += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int n = static_cast<int>(e / q), j = static_cast<int>(e % q);
        const int c = n / kCanvas, i = n % kCanvas;
        if (stop[c]) continue;
        const uint64_t seed = seeds[c];
        const int tgt = philox_token(seed, static_cast<uint32_t>(i), 0u, static_cast<uint32_t>(c), kTagStubTarget,
                                     static_cast<uint32_t>(V));
        const int x = tokens[n];
        uint32_t w[4] = {static_cast<uint32_t>(i * q + j), static_cast<uint32_t>(step), static_cast<uint32_t>(c),
                         kTagStubNoise};
        philox4x32_10(w, static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32));
        const float k32 = 2.3283064365386963e-10f;   // 2^-32
        float nz[4];
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            const float u1 = fmaf(static_cast<float>(w[2 * p]), k32, k32);
            const float rad = sqrtf(-2.0f * logf(u1));
            float sn, cs;
            sincospif(static_cast<float>(w[2 * p + 1]) * (2.0f * k32), &sn, &cs);
            nz[2 * p] = rad * cs;
            nz[2 * p + 1] = rad * sn;
        }
        // four consecutive columns of a row: contiguous in either head layout
        const size_t ot = tiled ? tiled_index(tgt, 4 * j, d) : static_cast<size_t>(tgt) * d + 4 * j;
        const size_t ox = tiled ? tiled_index(x, 4 * j, d) : static_cast<size_t>(x) * d + 4 * j;
        const uint2 et = *reinterpret_cast<const uint2*>(E + ot);
        const uint2 ex = *reinterpret_cast<const uint2*>(E + ox);
        const __nv_bfloat162* bt = reinterpret_cast<const __nv_bfloat162*>(&et);
        const __nv_bfloat162* bx = reinterpret_cast<const __nv_bfloat162*>(&ex);
        float vt[4] = {__low2float(bt[0]), __high2float(bt[0]), __low2float(bt[1]), __high2float(bt[1])};
        float vx[4] = {__low2float(bx[0]), __high2float(bx[0]), __low2float(bx[1]), __high2float(bx[1])};
        float out[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) out[m] = fmaf(noise, nz[m], gain * fmaf(a_s, vt[m], (1.0f - a_s) * vx[m]));
        __nv_bfloat162 o0 = __floats2bfloat162_rn(out[0], out[1]);
        __nv_bfloat162 o1 = __floats2bfloat162_rn(out[2], out[3]);
        uint2 pk;
        pk.x = *reinterpret_cast<uint32_t*>(&o0);
        pk.y = *reinterpret_cast<uint32_t*>(&o1);
        *reinterpret_cast<uint2*>(h + static_cast<size_t>(n) * d + 4 * j) = pk;
    }
}

// Row-major <-> tile-major head (tiled_index): one thread per 8 consecutive columns of a row
// (16 bytes, inside one 64-column atom in both layouts).
__global__ void dg_tile_head_kernel(const __nv_bfloat16* src, __nv_bfloat16* dst, long long V, int d, int to_rows) {
    const int per_row = d / 8;
    const long long total = V * per_row;
    for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < total;
         e += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long v = e / per_row;
        const int c = static_cast<int>(e % per_row) * 8;
        const size_t rm = static_cast<size_t>(v) * d + c;
        const size_t tl = tiled_index(v, c, d);
        const uint4 x = *reinterpret_cast<const uint4*>(src + (to_rows ? tl : rm));
        *reinterpret_cast<uint4*>(dst + (to_rows ? rm : tl)) = x;
    }
}

}  // namespace dg
