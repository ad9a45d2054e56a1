// E4M3 quantisation for the low-precision logits option: power-of-two scales chosen from
// the exact maximum magnitude (per row, or one for a whole tensor), then every value
// scaled exactly and rounded to the nearest E4M3 value, ties to the even mantissa.
//
// E4M3: sign bit, 4 exponent bits with bias 7, 3 mantissa bits, subnormals down to 2^-9,
// largest finite value 448, no infinities.  The pages cite quantised deployments of the
// model (axbrief.com brief, deployment on a 24 GB GPU: GGUF sizes) but define none for
// this stage; this is the reading the library takes.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "dg_common.cuh"
#include "dg_fused.h"

namespace dg {

namespace {

constexpr float kE4M3Max = 448.0f;

// The smallest integer e with amax 2^-e <= 448 (0 for a zero or non-finite maximum).  The
// comparisons use exact power-of-two scalings (ldexpf of a value in the normal range).
__device__ int pow2_exponent(float amax) {
    if (!(amax > 0.f) || !isfinite(amax)) return 0;
    int e = 0;
    frexpf(amax / kE4M3Max, &e);
    while (ldexpf(amax, -e) > kE4M3Max) ++e;
    while (ldexpf(amax, -(e - 1)) <= kE4M3Max) --e;
    return e;
}

// Two values to two E4M3 codes (round to nearest even, finite saturation); lo at the lower
// byte address.
__device__ __forceinline__ uint16_t to_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ float block_max(float v, float* sh) {
#pragma unroll
    for (int off = 16; off; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) sh[w] = v;
    __syncthreads();
    if (w == 0) {
        v = lane < static_cast<int>(blockDim.x >> 5) ? sh[lane] : 0.f;
#pragma unroll
        for (int off = 16; off; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
        if (lane == 0) sh[0] = v;
    }
    __syncthreads();
    return sh[0];
}

}  // namespace

// One CTA per row: the row's scale exponent and codes.  cols is even.
__global__ void __launch_bounds__(256) dg_quant_rows_kernel(const __nv_bfloat16* src, int cols, uint8_t* codes,
                                                            int32_t* exps) {
    __shared__ float sh[32];
    __shared__ int sh_e;
    const long long row = blockIdx.x;
    const __nv_bfloat162* s2 = reinterpret_cast<const __nv_bfloat162*>(src + row * cols);
    uint16_t* c2 = reinterpret_cast<uint16_t*>(codes + row * cols);
    const int half = cols / 2;
    float amax = 0.f;
    for (int j = threadIdx.x; j < half; j += blockDim.x) {
        const float2 v = __bfloat1622float2(s2[j]);
        amax = fmaxf(amax, fmaxf(fabsf(v.x), fabsf(v.y)));
    }
    amax = block_max(amax, sh);
    if (threadIdx.x == 0) {
        sh_e = pow2_exponent(amax);
        exps[row] = sh_e;
    }
    __syncthreads();
    const int e = sh_e;
    for (int j = threadIdx.x; j < half; j += blockDim.x) {
        const float2 v = __bfloat1622float2(s2[j]);
        c2[j] = to_e4m3x2(ldexpf(v.x, -e), ldexpf(v.y, -e));
    }
}

// Largest magnitude of a tensor: block maxima folded into *amax_bits with an integer
// atomicMax (non-negative floats order as their bit patterns); *amax_bits starts at 0.
__global__ void __launch_bounds__(256) dg_amax_kernel(const __nv_bfloat16* src, long long n_pairs,
                                                      uint32_t* amax_bits) {
    __shared__ float sh[32];
    const __nv_bfloat162* s2 = reinterpret_cast<const __nv_bfloat162*>(src);
    float amax = 0.f;
    for (long long j = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; j < n_pairs;
         j += static_cast<long long>(gridDim.x) * blockDim.x) {
        const float2 v = __bfloat1622float2(s2[j]);
        amax = fmaxf(amax, fmaxf(fabsf(v.x), fabsf(v.y)));
    }
    amax = block_max(amax, sh);
    if (threadIdx.x == 0) atomicMax(amax_bits, __float_as_uint(amax));
}

// The tensor's exponent from its maximum (exps[0] holds the maximum's bits on entry).
__global__ void dg_amax_to_exp_kernel(int32_t* exps) {
    if (threadIdx.x == 0 && blockIdx.x == 0) exps[0] = pow2_exponent(__uint_as_float(static_cast<uint32_t>(exps[0])));
}

__global__ void __launch_bounds__(256) dg_quant_tensor_kernel(const __nv_bfloat16* src, long long n_pairs,
                                                              uint8_t* codes, const int32_t* exps) {
    const int e = exps[0];
    const __nv_bfloat162* s2 = reinterpret_cast<const __nv_bfloat162*>(src);
    uint16_t* c2 = reinterpret_cast<uint16_t*>(codes);
    for (long long j = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; j < n_pairs;
         j += static_cast<long long>(gridDim.x) * blockDim.x) {
        const float2 v = __bfloat1622float2(s2[j]);
        c2[j] = to_e4m3x2(ldexpf(v.x, -e), ldexpf(v.y, -e));
    }
}

}  // namespace dg
