// q4_gemv.cuh -- helpers shared by the streaming product kernels: chunk
// constants, the MMA row mapping, the 16-bit magic-number bases of the code
// unpacking and the output store.
#pragma once

#include "q4_device.cuh"

namespace q4dev {

// MMA row group (lane / 4) -> row inside a 16-row tile; the 3-bit reversal
// makes the lanes of one shared-memory phase hit different 16-byte columns of
// the 128-byte-swizzled tiles.
__host__ __device__ constexpr int rho(int g) {
    return ((g & 1) << 2) | (g & 2) | ((g >> 2) & 1);
}

// Chunk = 256 codes of a row = 128 bytes.
constexpr int kChunkCodes = 256;
constexpr int kChunkBytes = 128;

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

template <bool BF16>
struct Magic {
    // 16-bit float with exponent such that the low 4 mantissa bits hold a nibble
    // as an integer: bf16 0x4300 = 128.0, fp16 0x6400 = 1024.0.
    static constexpr uint32_t base2 = BF16 ? 0x43004300u : 0x64006400u;
    static constexpr float base = BF16 ? 128.0f : 1024.0f;
};

// Output store of one value.
__device__ __forceinline__ void store_y(void* y, int ydt, int64_t idx, float v) {
    if (ydt == 2) {
        reinterpret_cast<float*>(y)[idx] = v;
    } else if (ydt == 1) {
        reinterpret_cast<__nv_bfloat16*>(y)[idx] = __float2bfloat16_rn(v);
    } else {
        reinterpret_cast<__half*>(y)[idx] = __float2half_rn(v);
    }
}

}  // namespace q4dev
