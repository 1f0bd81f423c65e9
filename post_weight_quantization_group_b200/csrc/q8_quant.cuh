// q8_quant.cuh -- INT8 quantizers: per-output-channel INT8 weights and the
// INT8 KV cache, with their dequantizations.
//
// Weights ("量化：PTQ、GPTQ、AWQ 与 SmoothQuant" (charles2530.github.io)
// section 13, per_channel_int8_quant), one scale per row of W [out, in]:
//   s = max(max_k |w|, 1e-6) / 127,   q = clamp(rne(w / s), -127, 127)
// in fp32 with the results of IEEE divisions (int8_code); s is stored as fp32
// and w_hat = q * s.
//
// KV cache ("压缩算法" (cs-knowledge-wiki) section 7.4.1.1,
// quantize_kv_cache_int8 along the last axis), one scale per row of head_dim
// values of a [batch, heads, seq, head_dim] cache:
//   s = cache_type(max |x| / 127),   q = clamp(rne(x / s), -128, 127)
// with the stored (rounded) scale used for the codes and a zero stored scale
// giving codes 0; the dequantization is cache_type(q * s), one rounding of
// an exact fp32 product.
#pragma once

#include "q4_device.cuh"
#include "q4_quant.cuh"

namespace q4dev {

// ---------------------------------------------------------- INT8 weights

// INT8 code of one value, clamp(rne(fl(v / s)), qmin, 127), through t = v * r
// (r = 1/s correctly rounded, from quot_recip): |t - fl(v/s)| <= |t| (3u + u^2)
// (u = 2^-24), below 3.2e-5 while |t| < 178, and t - rint(t) is exact; so when
// |t - rint(t)| < 0.5 - 3.2e-5 both round to the same integer, and from
// |t| >= 178 on both clamp alike.  Otherwise (near a tie, or a NaN) the exact
// quotient is rounded as the definition states (NaN -> qmin).
__device__ __forceinline__ int int8_code(float v, float s, float r, int qmin) {
    const float t = __fmul_rn(v, r);
    const int q = __float2int_rn(t);
    if (fabsf(__fsub_rn(t, __int2float_rn(q))) < 0.4999679f) return min(max(q, qmin), 127);
    float u = rintf(__fdiv_rn(v, s));
    u = fminf(fmaxf(u, static_cast<float>(qmin)), 127.f);
    return static_cast<int>(u);
}

// Eight codes as two little-endian words (element 0 in byte 0).
__device__ __forceinline__ uint2 pack8_bytes(const int (&q)[8]) {
    uint32_t w[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint32_t lo = __byte_perm(q[4 * h], q[4 * h + 1], 0x0040);
        const uint32_t hi = __byte_perm(q[4 * h + 2], q[4 * h + 3], 0x0040);
        w[h] = __byte_perm(lo, hi, 0x5410);
    }
    return make_uint2(w[0], w[1]);
}

// One CTA per row (grid-stride over rows): the row's amax by a block
// reduction, then the codes; the second read of the row comes from L2.
template <bool BF16IN>
__global__ void __launch_bounds__(256)
    q8_quantize_rows_kernel(const void* __restrict__ W, int64_t out, int64_t in,
                            int8_t* __restrict__ q, float* __restrict__ scales) {
    __shared__ float red[8];
    __shared__ float s_row;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    for (int64_t r = blockIdx.x; r < out; r += gridDim.x) {
        float a = 0.f;
        for (int64_t k = static_cast<int64_t>(threadIdx.x) * 8; k < in; k += 256 * 8) {
            float v[8];
            load8_f32<BF16IN>(W, r * in + k, v);
#pragma unroll
            for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(v[i]));
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, off));
        if (lane == 0) red[warp] = a;
        __syncthreads();
        if (threadIdx.x == 0) {
            float m = red[0];
            for (int w = 1; w < 8; ++w) m = fmaxf(m, red[w]);
            const float s = __fdiv_rn(fmaxf(m, 1e-6f), 127.0f);
            s_row = s;
            scales[r] = s;
        }
        __syncthreads();
        const float s = s_row;
        const float rs = quot_recip(s);
        for (int64_t k = static_cast<int64_t>(threadIdx.x) * 8; k < in; k += 256 * 8) {
            float v[8];
            load8_f32<BF16IN>(W, r * in + k, v);
            int c[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) c[i] = int8_code(v[i], s, rs, -127);
            *reinterpret_cast<uint2*>(q + r * in + k) = pack8_bytes(c);
        }
        __syncthreads();  // red / s_row are reused by the next row
    }
}

template <typename OutT>
__device__ __forceinline__ OutT from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __half from_f32<__half>(float v) { return __float2half_rn(v); }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

// w_hat[r, k] = q[r, k] * s[r]: eight codes per thread step (in % 16 == 0, so
// an 8-code vector never crosses a row).
template <typename OutT>
__global__ void __launch_bounds__(256)
    q8_dequant_kernel(const int8_t* __restrict__ q, const float* __restrict__ scales,
                      int64_t nvec, int64_t in, OutT* __restrict__ W_hat) {
    for (int64_t i = blockIdx.x * 256LL + threadIdx.x; i < nvec; i += gridDim.x * 256LL) {
        const int64_t e0 = i * 8;
        const float s = __ldg(scales + e0 / in);
        const uint2 raw = __ldg(reinterpret_cast<const uint2*>(q + e0));
        const uint32_t w[2] = {raw.x, raw.y};
        OutT o[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int code = static_cast<int8_t>((w[j >> 2] >> (8 * (j & 3))) & 0xFFu);
            o[j] = from_f32<OutT>(static_cast<float>(code) * s);
        }
        if constexpr (sizeof(OutT) == 4) {
            float4* dst = reinterpret_cast<float4*>(W_hat + e0);
            dst[0] = make_float4(o[0], o[1], o[2], o[3]);
            dst[1] = make_float4(o[4], o[5], o[6], o[7]);
        } else {
            *reinterpret_cast<uint4*>(W_hat + e0) = *reinterpret_cast<const uint4*>(o);
        }
    }
}

// ---------------------------------------------------------- INT8 KV cache

template <bool BF16>
__device__ __forceinline__ uint16_t cache_bits(float v) {
    if constexpr (BF16) {
        const __nv_bfloat16 h = __float2bfloat16_rn(v);
        return *reinterpret_cast<const uint16_t*>(&h);
    } else {
        const __half h = __float2half_rn(v);
        return *reinterpret_cast<const uint16_t*>(&h);
    }
}
template <bool BF16>
__device__ __forceinline__ float cache_value(uint16_t b) {
    if constexpr (BF16) {
        return __uint_as_float(static_cast<uint32_t>(b) << 16);
    } else {
        return __half2float(__ushort_as_half(b));
    }
}


// A team of TS lanes (a power of two dividing 32) per row of d values; a lane
// holds the 8-value vectors sub and sub + TS of the row (d <= 16 * TS).  The
// warp's loop bound is uniform so that every lane takes part in the
// shuffles; lanes past the last row only skip their loads and stores.
template <bool BF16, int TS>
__global__ void __launch_bounds__(256)
    kv_quantize_int8_kernel(const uint16_t* __restrict__ kv, int64_t rows, int d,
                            int8_t* __restrict__ codes, uint16_t* __restrict__ scales) {
    constexpr int RPW = 32 / TS;  // rows per warp step
    const int lane = threadIdx.x & 31;
    const int sub = lane % TS;
    const int V = d / 8;
    const int64_t warp_g = (blockIdx.x * 256LL + threadIdx.x) >> 5;
    const int64_t nwarps = (gridDim.x * 256LL) >> 5;
    for (int64_t base = warp_g * RPW; base < rows; base += nwarps * RPW) {
        const int64_t r = base + lane / TS;
        const bool live = r < rows;
        float v[2][8];
        float a = 0.f;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int vec = sub + h * TS;
            if (live && vec < V) {
                load8_f32<BF16>(kv, r * d + vec * 8, v[h]);
#pragma unroll
                for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(v[h][i]));
            }
        }
#pragma unroll
        for (int off = TS / 2; off >= 1; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, off));
        const uint16_t sbits = cache_bits<BF16>(__fdiv_rn(a, 127.0f));
        const float s = cache_value<BF16>(sbits);
        const float rs = quot_recip(s);
        if (live && sub == 0) scales[r] = sbits;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int vec = sub + h * TS;
            if (!(live && vec < V)) continue;
            uint2 packed = make_uint2(0u, 0u);
            if (s != 0.f) {
                int q[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) q[i] = int8_code(v[h][i], s, rs, -128);
                packed = pack8_bytes(q);
            }
            *reinterpret_cast<uint2*>(codes + r * d + vec * 8) = packed;
        }
    }
}

// out = cache_type(q * s), eight values per thread step (d % 8 == 0).
template <bool BF16>
__global__ void __launch_bounds__(256)
    kv_dequant_int8_kernel(const int8_t* __restrict__ codes, const uint16_t* __restrict__ scales,
                           int64_t nvec, int d, uint16_t* __restrict__ out) {
    for (int64_t i = blockIdx.x * 256LL + threadIdx.x; i < nvec; i += gridDim.x * 256LL) {
        const int64_t e0 = i * 8;
        const float s = cache_value<BF16>(__ldg(scales + e0 / d));
        const uint2 raw = __ldg(reinterpret_cast<const uint2*>(codes + e0));
        const uint32_t w[2] = {raw.x, raw.y};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c0 = static_cast<int8_t>((w[j >> 1] >> (16 * (j & 1))) & 0xFFu);
            const int c1 = static_cast<int8_t>((w[j >> 1] >> (16 * (j & 1) + 8)) & 0xFFu);
            o[j] = static_cast<uint32_t>(cache_bits<BF16>(static_cast<float>(c0) * s)) |
                   (static_cast<uint32_t>(cache_bits<BF16>(static_cast<float>(c1) * s)) << 16);
        }
        *reinterpret_cast<uint4*>(out + e0) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

}  // namespace q4dev
