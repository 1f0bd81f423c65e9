// q4_quant.cuh -- group-wise INT4 quantize + pack, and dequantization.
//
// Quantizer ("LLM 后训练量化深度实战" (ybb.press) section 二, quantize_per_group;
// arganzheng.life post-training-quantization-gptq-awq-and-rotation section
// 二.2): per group of g consecutive elements along `in`,
//   symmetric   s = fp16(amax / 7),            q = clamp(rne(w / s), -8, 7)
//   asymmetric  s = fp16((max - min) / 15),   z = clamp(rne(-min / s), 0, 15),
//               q = clamp(rne(w / s) + z, 0, 15)
// with IEEE fp32 divisions (no reciprocal multiply), round-half-to-even, and
// the stored fp16 scale used for the codes; a zero stored scale gives codes
// 0.  Two codes per byte, the even element in the low nibble ("压缩算法"
// (cs-knowledge-wiki) section 7.4.1.2, pack_int4).
//
// The matrix is a sequence of out*in/g groups of g contiguous elements
// (g divides in).  The fast kernel gives each thread 8 consecutive elements
// (one 16-byte load, one 4-byte packed store): a group is g/8 adjacent lanes
// and its statistics are a warp-shuffle reduction.  Other even group sizes
// take a warp per group.
#pragma once

#include "q4_device.cuh"

namespace q4dev {

template <bool BF16IN>
__device__ __forceinline__ void load8_f32(const void* base, int64_t elem, float (&v)[8]) {
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(
        reinterpret_cast<const uint16_t*>(base) + elem));
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if constexpr (BF16IN) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        } else {
            __half2 h = *reinterpret_cast<const __half2*>(&w[i]);
            float2 f = __half22float2(h);
            v[2 * i] = f.x;
            v[2 * i + 1] = f.y;
        }
    }
}

// Column index perm[c] clamped into [0, in); a bad entry is recorded.
__device__ __forceinline__ int64_t perm_col(const int32_t* perm, int64_t c, int64_t in,
                                            unsigned* status) {
    int64_t k = perm[c];
    if (k < 0 || k >= in) {
        atomicOr(status, kStatusBadIndex);
        k = k < 0 ? 0 : in - 1;
    }
    return k;
}

// Eight consecutive columns c0 .. c0+7 of row r taken through perm
// (act order): element e is W[r, perm[c0 + e]].
template <bool BF16IN>
__device__ __forceinline__ void load8_perm_f32(const void* base, int64_t r, int64_t c0, int64_t in,
                                               const int32_t* perm, unsigned* status,
                                               float (&v)[8]) {
    const uint16_t* w16 = reinterpret_cast<const uint16_t*>(base) + r * in;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const uint16_t b = __ldg(w16 + perm_col(perm, c0 + e, in, status));
        if constexpr (BF16IN) {
            v[e] = __uint_as_float(static_cast<uint32_t>(b) << 16);
        } else {
            v[e] = __half2float(__ushort_as_half(b));
        }
    }
}

// clamp(rne(w / s) + z, qmin, qmax) with the result of the definition's fp32
// operations: IEEE division (through rne_quot, r = quot_recip(s)), round half
// to even, add z, clamp (NaN -> qmin).
__device__ __forceinline__ int quant_one(float w, float s, float r, float z, float qmin,
                                         float qmax) {
    float t = rne_quot(w, s, r);
    t = __fadd_rn(t, z);
    t = fminf(fmaxf(t, qmin), qmax);
    return static_cast<int>(t);
}

// Fast path: group size G in {8, 16, 32, 64, 128, 256}.  n16 = number of
// 8-element chunks = out*in/8.
// With perm (act order, may be null) the columns are read through it: the
// quantized matrix is W[:, perm] (in = row length, for the gather).
template <int G, bool SYM, bool BF16IN>
__global__ void __launch_bounds__(256) quantize_pack_kernel(const void* __restrict__ W,
                                                            int64_t nchunks,
                                                            uint32_t* __restrict__ qweight,
                                                            __half* __restrict__ scales,
                                                            __half* __restrict__ zeros,
                                                            const int32_t* __restrict__ perm,
                                                            int64_t in, unsigned* status) {
    constexpr int LANES = G / 8;  // lanes per group
    static_assert(LANES >= 1 && LANES <= 32 && (32 % LANES) == 0, "group must tile a warp");
    const int lane = threadIdx.x & 31;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
         i - lane < nchunks; i += stride) {
        const bool active = i < nchunks;
        float v[8];
        if (active) {
            if (perm != nullptr)
                load8_perm_f32<BF16IN>(W, (i * 8) / in, (i * 8) % in, in, perm, status, v);
            else
                load8_f32<BF16IN>(W, i * 8, v);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = 0.f;
        }
        uint32_t packed = 0;
        float s32, sf, zf = 0.f;
        if constexpr (SYM) {
            float a = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) a = fmaxf(a, fabsf(v[e]));
#pragma unroll
            for (int off = LANES / 2; off >= 1; off >>= 1)
                a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, off));
            s32 = __fdiv_rn(a, 7.0f);
            sf = __half2float(__float2half_rn(s32));
            if (sf != 0.f) {
                const float rf = quot_recip(sf);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int q = quant_one(v[e], sf, rf, 0.f, -8.f, 7.f);
                    packed |= (static_cast<uint32_t>(q) & 0xFu) << (4 * e);
                }
            }
        } else {
            float mn = v[0], mx = v[0];
#pragma unroll
            for (int e = 1; e < 8; ++e) {
                mn = fminf(mn, v[e]);
                mx = fmaxf(mx, v[e]);
            }
#pragma unroll
            for (int off = LANES / 2; off >= 1; off >>= 1) {
                mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, off));
                mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
            }
            s32 = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
            sf = __half2float(__float2half_rn(s32));
            if (sf != 0.f) {
                const float rf = quot_recip(sf);
                zf = static_cast<float>(quant_one(-mn, sf, rf, 0.f, 0.f, 15.f));
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int q = quant_one(v[e], sf, rf, zf, 0.f, 15.f);
                    packed |= (static_cast<uint32_t>(q) & 0xFu) << (4 * e);
                }
            }
        }
        if (active) {
            qweight[i] = packed;
            if ((lane % LANES) == 0) {
                const int64_t grp = (i * 8) / G;
                scales[grp] = __float2half_rn(s32);
                if constexpr (!SYM) zeros[grp] = __float2half_rn(zf);
            }
        }
    }
}

// Symmetric quantization with a per-group range (clipping) search
// (arganzheng.life post-training-quantization-gptq-awq-and-rotation section
// 三.2, 裁剪与舍入的权衡: scan ranges alpha from 0.8 to 1.0 of max|w| and keep
// the one with the smallest error).  Candidates alpha_j = amax (K - j) / K,
// K = 5 (n - 1), j = 0 .. n-1; s_j = fp16(amax (K - j) / (7 K)) (the product
// is exact in fp32, the division IEEE); codes clamp(rne(w / s_j), -7, 7), the
// section's symmetric grid; error sum (w - s_j q)^2 in fp64, reduced over the
// group's lanes by butterfly shuffles (every lane holds the same sum and takes
// the same decision); j replaces the best only if its error is below
// E_best (1 - 1e-12), so ties keep the wider range.  j = 0 is RTN exactly.
template <int G, bool BF16IN>
__global__ void __launch_bounds__(256) quantize_pack_clip_kernel(const void* __restrict__ W,
                                                                 int64_t nchunks, int n,
                                                                 uint32_t* __restrict__ qweight,
                                                                 __half* __restrict__ scales) {
    constexpr int LANES = G / 8;
    static_assert(LANES >= 1 && LANES <= 32 && (32 % LANES) == 0, "group must tile a warp");
    const int lane = threadIdx.x & 31;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int K = 5 * (n - 1);
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
         i - lane < nchunks; i += stride) {
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
#pragma unroll
        for (int off = LANES / 2; off >= 1; off >>= 1)
            a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, off));
        uint32_t best_packed = 0;
        __half best_s = __float2half_rn(0.f);
        double best_e = 0.0;
        for (int j = 0; j < n; ++j) {
            const float num = (n == 1) ? a : __fmul_rn(a, static_cast<float>(K - j));
            const float den = (n == 1) ? 7.0f : static_cast<float>(7 * K);
            const __half s16 = __float2half_rn(__fdiv_rn(num, den));
            const float sf = __half2float(s16);
            uint32_t packed = 0;
            double e = 0.0;
            const float rf = quot_recip(sf);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int q = (sf == 0.f) ? 0 : quant_one(v[k], sf, rf, 0.f, -7.f, 7.f);
                packed |= (static_cast<uint32_t>(q) & 0xFu) << (4 * k);
                const double d = static_cast<double>(v[k]) - static_cast<double>(sf) * q;
                e += d * d;
            }
#pragma unroll
            for (int off = LANES / 2; off >= 1; off >>= 1) e += __shfl_xor_sync(0xFFFFFFFFu, e, off);
            if (j == 0 || (sf != 0.f && e < best_e * (1.0 - 1e-12))) {
                best_e = e;
                best_packed = packed;
                best_s = s16;
            }
        }
        if (active) {
            qweight[i] = best_packed;
            if ((lane % LANES) == 0) scales[(i * 8) / G] = best_s;
        }
    }
}

// Generic path: any even group size; one warp per group, element pairs
// strided over the lanes.
template <bool SYM, bool BF16IN>
__global__ void __launch_bounds__(256) quantize_pack_generic_kernel(
    const void* __restrict__ W, int64_t ngroups, int g, uint8_t* __restrict__ qweight,
    __half* __restrict__ scales, __half* __restrict__ zeros, const int32_t* __restrict__ perm,
    int64_t in, unsigned* status) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const uint16_t* w16 = reinterpret_cast<const uint16_t*>(W);
    auto ld = [&](int64_t e) -> float {
        // element e of the (column-permuted, with perm) matrix
        const uint16_t b = perm != nullptr ? w16[(e / in) * in + perm_col(perm, e % in, in, status)]
                                           : w16[e];
        if constexpr (BF16IN) {
            return __uint_as_float(static_cast<uint32_t>(b) << 16);
        } else {
            return __half2float(__ushort_as_half(b));
        }
    };
    for (int64_t grp = warp; grp < ngroups; grp += nwarps) {
        const int64_t base = grp * g;
        float a = 0.f, mn = INFINITY, mx = -INFINITY;
        for (int k = lane; k < g; k += 32) {
            const float v = ld(base + k);
            a = fmaxf(a, fabsf(v));
            mn = fminf(mn, v);
            mx = fmaxf(mx, v);
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) {
            a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, off));
            mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, off));
            mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
        }
        float s32, zf = 0.f;
        if constexpr (SYM) {
            s32 = __fdiv_rn(a, 7.0f);
        } else {
            s32 = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
        }
        const float sf = __half2float(__float2half_rn(s32));
        const float rf = quot_recip(sf);
        if (!SYM && sf != 0.f) zf = static_cast<float>(quant_one(-mn, sf, rf, 0.f, 0.f, 15.f));
        for (int p = lane; p < g / 2; p += 32) {
            int q0 = 0, q1 = 0;
            if (sf != 0.f) {
                if constexpr (SYM) {
                    q0 = quant_one(ld(base + 2 * p), sf, rf, 0.f, -8.f, 7.f);
                    q1 = quant_one(ld(base + 2 * p + 1), sf, rf, 0.f, -8.f, 7.f);
                } else {
                    q0 = quant_one(ld(base + 2 * p), sf, rf, zf, 0.f, 15.f);
                    q1 = quant_one(ld(base + 2 * p + 1), sf, rf, zf, 0.f, 15.f);
                }
            }
            qweight[base / 2 + p] =
                static_cast<uint8_t>((q0 & 0xF) | ((q1 & 0xF) << 4));
        }
        if (lane == 0) {
            scales[grp] = __float2half_rn(s32);
            if constexpr (!SYM) zeros[grp] = __float2half_rn(zf);
        }
    }
}

// Dequantization w_hat = s * (q - z): each thread expands one packed 32-bit
// word (8 codes) into 8 outputs.  s * (q - z) is exact in fp32; 16-bit
// outputs are its round-to-nearest-even conversion.
template <typename OutT>
__device__ __forceinline__ void store8(OutT* dst, const float (&v)[8]);

template <>
__device__ __forceinline__ void store8<float>(float* dst, const float (&v)[8]) {
    reinterpret_cast<float4*>(dst)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(dst)[1] = make_float4(v[4], v[5], v[6], v[7]);
}

template <>
__device__ __forceinline__ void store8<__half>(__half* dst, const float (&v)[8]) {
    uint4 o;
    __half2 h0 = __floats2half2_rn(v[0], v[1]), h1 = __floats2half2_rn(v[2], v[3]);
    __half2 h2 = __floats2half2_rn(v[4], v[5]), h3 = __floats2half2_rn(v[6], v[7]);
    o.x = *reinterpret_cast<uint32_t*>(&h0);
    o.y = *reinterpret_cast<uint32_t*>(&h1);
    o.z = *reinterpret_cast<uint32_t*>(&h2);
    o.w = *reinterpret_cast<uint32_t*>(&h3);
    *reinterpret_cast<uint4*>(dst) = o;
}

template <>
__device__ __forceinline__ void store8<__nv_bfloat16>(__nv_bfloat16* dst, const float (&v)[8]) {
    uint4 o;
    __nv_bfloat162 h0 = __floats2bfloat162_rn(v[0], v[1]);
    __nv_bfloat162 h1 = __floats2bfloat162_rn(v[2], v[3]);
    __nv_bfloat162 h2 = __floats2bfloat162_rn(v[4], v[5]);
    __nv_bfloat162 h3 = __floats2bfloat162_rn(v[6], v[7]);
    o.x = *reinterpret_cast<uint32_t*>(&h0);
    o.y = *reinterpret_cast<uint32_t*>(&h1);
    o.z = *reinterpret_cast<uint32_t*>(&h2);
    o.w = *reinterpret_cast<uint32_t*>(&h3);
    *reinterpret_cast<uint4*>(dst) = o;
}

template <typename OutT, bool SYM>
__global__ void __launch_bounds__(256) dequant_kernel(const uint32_t* __restrict__ qweight,
                                                      const __half* __restrict__ scales,
                                                      const __half* __restrict__ zeros,
                                                      int64_t nwords, int64_t in, int g,
                                                      OutT* __restrict__ W_hat) {
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int64_t G = in / g;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nwords;
         i += stride) {
        const uint32_t w = __ldg(qweight + i);
        const int64_t e0 = i * 8;  // flat element index; 8 | in so one row
        const int64_t r = e0 / in;
        const int64_t k0 = e0 - r * in;
        float v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int64_t gi = r * G + (k0 + e) / g;
            const float s = __half2float(scales[gi]);
            int n = static_cast<int>((w >> (4 * e)) & 0xFu);
            float q;
            if constexpr (SYM) {
                q = static_cast<float>(n >= 8 ? n - 16 : n);
            } else {
                q = static_cast<float>(n) - __half2float(zeros[gi]);
            }
            v[e] = __fmul_rn(s, q);
        }
        store8<OutT>(W_hat + e0, v);
    }
}

// Activations gathered into the act order: x_perm[b, j] = x[b, perm[j]]
// (arganzheng.life section 九.2: the g_idx reorder is a gather); one thread
// per 8 outputs (16-byte store).
__global__ void __launch_bounds__(256) permute_columns_kernel(const uint16_t* __restrict__ x,
                                                              int64_t rows, int64_t in,
                                                              const int32_t* __restrict__ perm,
                                                              uint16_t* __restrict__ xo,
                                                              unsigned* status) {
    // launched as a programmatic dependent: the next kernel (the product) may
    // start and prefetch its weights at once; x is read only after the
    // preceding kernel has completed
    grid_launch_dependents();
    grid_dependency_wait();
    const int64_t n8 = rows * in / 8;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
         i += stride) {
        const int64_t r = (i * 8) / in, c0 = (i * 8) % in;
        uint16_t o[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] = __ldg(x + r * in + perm_col(perm, c0 + e, in, status));
        uint4 v;
        v.x = o[0] | (static_cast<uint32_t>(o[1]) << 16);
        v.y = o[2] | (static_cast<uint32_t>(o[3]) << 16);
        v.z = o[4] | (static_cast<uint32_t>(o[5]) << 16);
        v.w = o[6] | (static_cast<uint32_t>(o[7]) << 16);
        *reinterpret_cast<uint4*>(xo + i * 8) = v;
    }
}

}  // namespace q4dev
