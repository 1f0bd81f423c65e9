// fp4_quant.cuh -- FP4 microscaling quantizers and dequantizers
// ("post-training-quantization-gptq-awq-and-rotation" (arganzheng.life)
// sections 九.1 and 九.2: E2M1 elements {0, 0.5, 1, 1.5, 2, 3, 4, 6} x sign;
// MXFP4 = one E8M0 power-of-two scale per 32 elements (the OCP standard);
// NVFP4 = one E4M3 scale per 16 elements and one fp32 scale per tensor).
//
//   MXFP4: e = clamp(floor(log2(amax_b)) - 2, -127, 127), scale byte e + 127,
//          q = e2m1(v * 2^-e) (saturating at 6); an all-zero block gets
//          scale byte 0 and codes +0.
//   NVFP4: s_t = A / 2688 (A = max |W|, 2688 = 6 * 448; 1 if A = 0),
//          c_b = e4m3_satfinite(fp32(amax_b / 6) / s_t), S_b = e4m3(c_b) * s_t,
//          q = e2m1(v / S_b), codes 0 where S_b = 0.
// E2M1 rounding is to nearest with ties to the even magnitude index and
// keeps the sign (-0 is code 8).  Codes are packed two per byte, the even
// element in the low nibble, as the INT4 weights.
#pragma once

#include <cuda_fp8.h>

#include "q4_device.cuh"
#include "q4_quant.cuh"

namespace q4dev {

// Nearest E2M1 code of a finite fp32 value: the magnitude index counts the
// rounding thresholds passed (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5, each a
// midpoint of two neighbours; at a midpoint the neighbour with mantissa bit 0
// wins, hence > at the odd-to-even steps and >= at the even-to-odd ones).
// Every magnitude at or above 5 (incl. >= 6) ends at index 7 = 6.0.
__device__ __forceinline__ uint32_t e2m1_code(float t) {
    const float a = fabsf(t);
    const uint32_t m = (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) + (a > 2.5f) +
                       (a >= 3.5f) + (a > 5.0f);
    return m | (signbit(t) ? 8u : 0u);
}

__device__ __forceinline__ float e2m1_value(uint32_t c) {
    // magnitude index m: 0, 0.5, 1, 1.5, 2, 3, 4, 6 = (m < 2 ? m / 2 : 2^(m/2 - 1) (1 + (m & 1) / 2))
    const uint32_t m = c & 7u;
    const float mag = m < 2u ? 0.5f * static_cast<float>(m)
                             : __int_as_float(static_cast<int>((126u + (m >> 1)) << 23)) *
                                   (1.0f + 0.5f * static_cast<float>(m & 1u));
    return (c & 8u) ? -mag : mag;
}

// E4M3 value of a code (1 sign, 4 exponent bits with bias 7, 3 mantissa
// bits; the NaN code 0x7F is never produced here).
__device__ __forceinline__ float e4m3_value(uint32_t c) {
    const uint32_t e = (c >> 3) & 0xFu, m = c & 7u;
    const float mag = e == 0u ? static_cast<float>(m) * 0.001953125f  // m * 2^-9
                              : static_cast<float>(8u | m) *
                                    __int_as_float(static_cast<int>((e + 117u) << 23));  // 2^(e-10)
    return (c & 0x80u) ? -mag : mag;
}

// floor(log2(a)) of a positive finite fp32 value.
__device__ __forceinline__ int floor_log2(float a) {
    const uint32_t b = __float_as_uint(a);
    const int E = static_cast<int>((b >> 23) & 0xFFu);
    if (E > 0) return E - 127;
    return (31 - __clz(static_cast<int>(b & 0x7FFFFFu))) - 149;
}

// One thread per 8 consecutive elements (16-byte load, 4-byte packed store);
// a 32-element block is 4 adjacent lanes.
template <bool BF16IN>
__global__ void __launch_bounds__(256)
    mxfp4_quantize_kernel(const void* __restrict__ W, int64_t nchunks,
                          uint32_t* __restrict__ packed, uint8_t* __restrict__ scales) {
    const int lane = threadIdx.x & 31;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i - lane < nchunks;
         i += stride) {
        const bool active = i < nchunks;
        float v[8];
        if (active) {
            load8_f32<BF16IN>(W, i * 8, v);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = 0.f;
        }
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) a = fmaxf(a, fabsf(v[e]));
        a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 1));
        a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 2));
        int ex = -127;
        if (a > 0.f) ex = min(max(floor_log2(a) - 2, -127), 127);
        // 2^-ex, with -ex in [-125, 127] (a < 2^128 keeps ex <= 125): a normal float
        const float inv = __int_as_float((127 - ex) << 23);
        uint32_t p = 0;
        if (a > 0.f) {
#pragma unroll
            for (int e = 0; e < 8; ++e) p |= e2m1_code(__fmul_rn(v[e], inv)) << (4 * e);
        }
        if (active) {
            packed[i] = p;
            if ((lane & 3) == 0) scales[(i * 8) / 32] = static_cast<uint8_t>(ex + 127);
        }
    }
}

// max |W| over the tensor into *amax_bits (the fp32 bit pattern, zeroed by
// the caller; non-negative floats order as unsigned integers).
template <bool BF16IN>
__global__ void __launch_bounds__(256)
    tensor_amax_kernel(const void* __restrict__ W, int64_t nchunks, unsigned* __restrict__ amax_bits) {
    float a = 0.f;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nchunks;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        float v[8];
        load8_f32<BF16IN>(W, i * 8, v);
#pragma unroll
        for (int e = 0; e < 8; ++e) a = fmaxf(a, fabsf(v[e]));
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, off));
    __shared__ float red[8];
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
    __syncthreads();
    if (threadIdx.x == 0) {
        float m = red[0];
        for (int w = 1; w < 8; ++w) m = fmaxf(m, red[w]);
        atomicMax(amax_bits, __float_as_uint(m));
    }
}

__device__ __forceinline__ float nvfp4_tensor_scale(unsigned amax_bits) {
    const float A = __uint_as_float(amax_bits);
    return A > 0.f ? __fdiv_rn(A, 2688.0f) : 1.0f;
}

// One thread per 8 elements; a 16-element block is 2 adjacent lanes.
template <bool BF16IN>
__global__ void __launch_bounds__(256)
    nvfp4_quantize_kernel(const void* __restrict__ W, int64_t nchunks,
                          const unsigned* __restrict__ amax_bits, uint32_t* __restrict__ packed,
                          uint8_t* __restrict__ scales) {
    const int lane = threadIdx.x & 31;
    const float st = nvfp4_tensor_scale(*amax_bits);
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i - lane < nchunks;
         i += stride) {
        const bool active = i < nchunks;
        float v[8];
        if (active) {
            load8_f32<BF16IN>(W, i * 8, v);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = 0.f;
        }
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) a = fmaxf(a, fabsf(v[e]));
        a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 1));
        const float sb = __fdiv_rn(__fdiv_rn(a, 6.0f), st);
        const uint32_t cb = static_cast<uint32_t>(__nv_cvt_float_to_fp8(sb, __NV_SATFINITE, __NV_E4M3));
        const float S = __fmul_rn(e4m3_value(cb), st);
        uint32_t p = 0;
        if (S > 0.f) {
#pragma unroll
            for (int e = 0; e < 8; ++e) p |= e2m1_code(__fdiv_rn(v[e], S)) << (4 * e);
        }
        if (active) {
            packed[i] = p;
            if ((lane & 1) == 0) scales[(i * 8) / 16] = static_cast<uint8_t>(cb);
        }
    }
}

// Writes the tensor scale s_t over the amax bits once the quantizer is done.
__global__ void nvfp4_finalize_kernel(unsigned* amax_bits) {
    if (threadIdx.x == 0 && blockIdx.x == 0)
        *reinterpret_cast<float*>(amax_bits) = nvfp4_tensor_scale(*amax_bits);
}

// Dequantization: one packed 32-bit word (8 codes) per thread step.
// MXFP4: e2m1(q) * 2^(s - 127) (exact in fp32); NVFP4: e2m1(q) * (e4m3(c) * s_t).
template <typename OutT, bool NV>
__global__ void __launch_bounds__(256)
    fp4_dequant_kernel(const uint32_t* __restrict__ packed, const uint8_t* __restrict__ scales,
                       const float* __restrict__ tensor_scale, int64_t nwords,
                       OutT* __restrict__ W_hat) {
    const float st = NV ? *tensor_scale : 1.f;
    for (int64_t i = blockIdx.x * 256LL + threadIdx.x; i < nwords; i += gridDim.x * 256LL) {
        const uint32_t p = __ldg(packed + i);
        const uint32_t sc = __ldg(scales + (NV ? (i * 8) / 16 : (i * 8) / 32));
        float S;
        if constexpr (NV) {
            S = __fmul_rn(e4m3_value(sc), st);
        } else {
            S = sc == 0u ? __int_as_float(0x00400000) : __int_as_float(static_cast<int>(sc << 23));
        }
        float o[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] = __fmul_rn(e2m1_value((p >> (4 * e)) & 0xFu), S);
        store8(W_hat + i * 8, o);
    }
}

}  // namespace q4dev
