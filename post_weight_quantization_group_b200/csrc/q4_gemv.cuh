// q4_gemv.cuh -- helpers shared by the streaming product kernels (chunk
// constants, the MMA row mapping, the 16-bit magic-number bases of the code
// unpacking, the output store, the thread-block-cluster reduction) and the
// unquantised bf16 reference product.
//
// The bf16 reference (ybb.press "LLM 后训练量化深度实战" section 一,
// roofline_bound; arganzheng.life post-training-quantization-gptq-awq-and-
// rotation section 二.4, the BF16 vs W4A16 batch table) is y = x W^T with fp32
// accumulation: a producer warp streams [RT rows x 64 columns] bf16 tiles
// with TMA (128-byte swizzle) into a ring of shared-memory stages; consumer
// warps multiply them with the activations on m16n8k16 tensor-core MMAs
// (n = 8 batch columns, B of them live); the K dimension is split over the
// CTAs of a thread-block cluster, whose partial tiles are reduced through
// distributed shared memory in rank order -- deterministic, and no global
// scratch memory.
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

// Cluster split-K reduction of the [RT x BP] fp32 partial tiles left in each
// CTA's shared memory (red), rows divided among the ranks; rank order fixed.
__device__ __forceinline__ void cluster_reduce_store(const float* red, int rt, int bp, int b,
                                                     int64_t row0, int64_t out, void* y,
                                                     int ydt) {
    const uint32_t S = gridDim.x;
    const uint32_t q = cluster_ctarank();
    const int per = (rt + S - 1) / S;
    const int r_beg = q * per;
    const int r_end = min(rt, r_beg + per);
    const uint32_t red_addr = smem_u32(red);
    for (int idx = threadIdx.x; idx < (r_end - r_beg) * b; idx += blockDim.x) {
        const int r = r_beg + idx / b;
        const int col = idx % b;
        const int64_t grow = row0 + r;
        const uint32_t a = red_addr + static_cast<uint32_t>((r * bp + col) * 4);
        float acc = 0.f;
        for (uint32_t p = 0; p < S; ++p) acc += ld_shared_cluster_f32(mapa_shared(a, p));
        if (grow < out) store_y(y, ydt, static_cast<int64_t>(col) * out + grow, acc);
    }
}

// -------------------------------------------------------------- bf16 GEMV
// y = x W^T for bf16 W [out, in] and B <= 8, fp32 accumulation on the tensor
// cores.  Chunk = 64 columns = 128 bytes per row; thread t reads 16 bytes
// (8 consecutive columns) per row per 32-column slot, matching the natural
// (k, k+1), (k+2, k+3) pairs of the activation fragments.
struct DenseGeom {
    size_t off_x, off_bar, total, xpitch;
};
constexpr int kDenseChunkCols = 64;

__host__ __device__ inline DenseGeom dense_geom(int rt, int stages, int cps, int b) {
    DenseGeom g{};
    size_t off = static_cast<size_t>(stages) * rt * kChunkBytes;
    g.off_x = off;
    g.xpitch = static_cast<size_t>(cps) * kDenseChunkCols * 2 + 64;  // 64 mod 128: conflict-free
    off += g.xpitch * b;
    off = (off + 15) & ~static_cast<size_t>(15);
    g.off_bar = off;
    off += static_cast<size_t>(2 * stages) * 8;
    g.total = off + 1024;
    return g;
}

template <int MT, int CW, int STAGES>
__global__ void __launch_bounds__((CW + 1) * 32)
    bf16_gemv_kernel(const __grid_constant__ CUtensorMap tmap_w, const uint16_t* __restrict__ x,
                     int B, int64_t out, int64_t in, int cps, int nchunks, void* __restrict__ y,
                     unsigned* __restrict__ status) {
    constexpr int RT = CW * MT * 16;
    constexpr int BP = 8;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const DenseGeom geo = dense_geom(RT, STAGES, cps, B);
    uint8_t* xs = smem + geo.off_x;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + geo.off_bar);
    uint64_t* empty = full + STAGES;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int split = blockIdx.x;
    const int64_t row0 = static_cast<int64_t>(blockIdx.y) * RT;
    const int c_begin = split * cps;
    const int nch = max(0, min(nchunks, c_begin + cps) - c_begin);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], CW);
        }
        fence_mbarrier_init_cluster();
    }
    __syncthreads();

    float acc[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[mt][e] = 0.f;

    if (warp == CW) {
        if (lane == 0) {
            prefetch_tmap(&tmap_w);
            bool ok = true;
            for (int c = 0; c < nch && ok; ++c) {
                const int s = c % STAGES;
                const uint32_t it = c / STAGES;
                if (c >= STAGES)
                    ok = mbar_wait_bounded(&empty[s], (it - 1) & 1, status, kWaitLimitNs);
                if (!ok) break;
                mbar_arrive_expect_tx(&full[s], RT * kChunkBytes);
                tma_load_2d(smem + static_cast<size_t>(s) * RT * kChunkBytes, &tmap_w,
                            (c_begin + c) * kDenseChunkCols, static_cast<int32_t>(row0), &full[s]);
            }
            for (int s = 0; s < STAGES && s < nch; ++s) {
                const int last = s + ((nch - 1 - s) / STAGES) * STAGES;
                mbar_wait_bounded(&full[s], (last / STAGES) & 1, status, kWaitLimitNs);
            }
        }
        __syncwarp();
    } else {
        const int ctid = threadIdx.x;
        const int64_t kbase = static_cast<int64_t>(c_begin) * kDenseChunkCols;
        const int nblk = nch * (kDenseChunkCols / 8);
        for (int idx = ctid; idx < B * nblk; idx += CW * 32) {
            const int p = idx % nblk;
            const int n = idx / nblk;
            const int64_t k = kbase + p * 8;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (k < in) v = __ldg(reinterpret_cast<const uint4*>(x + static_cast<int64_t>(n) * in + k));
            *reinterpret_cast<uint4*>(xs + n * geo.xpitch + p * 16) = v;
        }
        named_bar_sync(1, CW * 32);

        const int gid = lane >> 2;
        const int t = lane & 3;
        const int rrow = rho(gid);
        for (int c = 0; c < nch; ++c) {
            const int s = c % STAGES;
            if (!mbar_wait_bounded(&full[s], (c / STAGES) & 1, status, kWaitLimitNs)) break;
            const uint8_t* stage = smem + static_cast<size_t>(s) * RT * kChunkBytes;
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                uint4 xv = make_uint4(0, 0, 0, 0);
                if (gid < B)
                    xv = *reinterpret_cast<const uint4*>(xs + gid * geo.xpitch +
                                                         (c * kDenseChunkCols + 32 * m + 8 * t) * 2);
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    const int R0 = (warp * MT + mt) * 16 + rrow;
                    const int piece = 4 * m + t;
                    const int sw = (piece ^ (R0 & 7)) << 4;
                    const uint4 a = *reinterpret_cast<const uint4*>(stage + R0 * kChunkBytes + sw);
                    const uint4 b = *reinterpret_cast<const uint4*>(stage + (R0 + 8) * kChunkBytes + sw);
                    const uint32_t A0[4] = {a.x, b.x, a.y, b.y};
                    const uint32_t A1[4] = {a.z, b.z, a.w, b.w};
                    mma_16816<true>(acc[mt], A0, xv.x, xv.y);
                    mma_16816<true>(acc[mt], A1, xv.z, xv.w);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
    }

    const int S = gridDim.x;
    if (S == 1) {
        if (warp < CW) {
            const int gid = lane >> 2, t = lane & 3;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const int64_t r0 = row0 + (warp * MT + mt) * 16 + rho(gid);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int col = 2 * t + (e & 1);
                    const int64_t row = r0 + ((e >> 1) ? 8 : 0);
                    if (col < B && row < out) store_y(y, 1, static_cast<int64_t>(col) * out + row, acc[mt][e]);
                }
            }
        }
        return;
    }
    float* red = reinterpret_cast<float*>(smem);
    __syncthreads();
    if (warp < CW) {
        const int gid = lane >> 2, t = lane & 3;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            const int r0 = (warp * MT + mt) * 16 + rho(gid);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int col = 2 * t + (e & 1);
                const int row = r0 + ((e >> 1) ? 8 : 0);
                red[row * BP + col] = acc[mt][e];
            }
        }
    }
    cluster_sync_all();
    cluster_reduce_store(red, RT, BP, B, row0, out, y, 1);
    cluster_sync_all();
}

}  // namespace q4dev
