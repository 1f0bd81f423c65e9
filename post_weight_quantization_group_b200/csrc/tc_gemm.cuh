// tc_gemm.cuh -- streaming products on the tcgen05 tensor cores of sm_100a
// whose operands go from HBM to the tensor core without conversion: the
// W4A4 product of two FP4 microscaling operands (block-scaled MMA) and the
// unquantised bf16 reference product.
//
// W4A4 ("post-training-quantization-gptq-awq-and-rotation" (arganzheng.life),
// sections 九.1 and 九.2): the weights and the activations both hold E2M1
// codes with one scale per small block along K -- an E8M0 power of two per
// 32 elements (MXFP4) or an E4M3 value per 16 elements under one fp32 scale
// per tensor (NVFP4).  The product is
//
//   y[b, r] = g * sum_k e2m1(W[r, k]) S_W[r, k / VS] * e2m1(X[b, k]) S_X[b, k / VS]
//
// with g = s_tW s_tX (NVFP4) or 1 (MXFP4).  Blackwell's block-scaled MMA
// applies S_W and S_X inside the tensor core, so the codes go from HBM to the
// tensor core untouched: no unpacking and no per-group rescale on the CUDA
// cores (the INT4 kernels spend most of their issue slots there).
//
// bf16 reference ("LLM 后训练量化深度实战" (ybb.press) section 一,
// roofline_bound; arganzheng.life section 二.4, the BF16 vs W4A16 batch
// table): y = x W^T with fp32 accumulation, the same pipeline with bf16
// tiles (kind::f16 MMAs, K = 16 per MMA, 128 values of K per stage) and no
// scale factors.
//
// Work decomposition: the persistent stream-K split of the INT4 kernels
// (q4_gemv_sk.cuh): T = row_tiles x chunks iterations, a row tile is 128 rows
// (the MMA's M and the 128 lanes of tensor memory), a chunk is 512 codes of K;
// CTA p owns iterations [T p / P, T (p+1) / P); a tile split between CTAs is
// finished by the CTA that arrives last on its counter, adding the fp32
// partials in CTA order (deterministic).
//
// One CTA per SM, ten warps:
//  * warp 0, producer: TMA loads per chunk of the weight codes [128 x 256 B]
//    and the activation codes [NT x 256 B] (each as two 128-byte-swizzled
//    K-major boxes; activation rows >= B read as zero), and of both operands'
//    scale bytes [rows x 512/VS] (row-major, as the quantizers write them);
//  * warps 2-5, scale writers (FP4 only; one per tensor-memory lane quarter): the MMA
//    reads the scale of row m, K-block j from tensor-memory lane m mod 32
//    (in every lane quarter), column m / 32, byte j -- the 32-lane x 128-bit
//    pattern replicated four times.  Each warp reads rows lane + 32 i
//    (i = 0..3) from shared memory and writes that pattern into its own lane
//    quarter with tcgen05.st, for the weights and for the activations;
//  * warp 1, MMA issuer (one thread): eight
//    D[128 x NT] (+)= A[128 x 64] * B[NT x 64]^T block-scaled MMAs per chunk
//    into one of two fp32 accumulators in tensor memory (one per output tile
//    segment, so the epilogue of a segment overlaps the next one's MMAs);
//  * warps 6-9, epilogue: read the finished accumulator back (tcgen05.ld),
//    multiply by g and store y, or store the partial and run the fix-up.
//
// Tensor-memory columns: accumulators [0, 2 NT); scale factors of stage s at
// 2 NT + 2 SFC s (weights) and + SFC (activations), SFC = 32 (NVFP4: four
// columns per MMA) or 16 (MXFP4: four columns per pair of MMAs, the second
// of a pair reading bytes 2-3 through scale-factor id 2).
#pragma once

#include "q4_device.cuh"
#include "q4_gemv.cuh"
#include "q4_gemv_sk.cuh"
#include "q4_tcgen05.cuh"

namespace q4dev {

constexpr int kF4RT = 128;              // rows per tile: MMA M, tensor-memory lanes
constexpr int kF4ChunkCodes = 512;      // K per pipeline stage
constexpr int kF4ChunkBytes = 256;      // code bytes per row per stage (two 128-byte atoms)
constexpr int kF4Box = 128;             // bytes per row of one swizzled TMA box
constexpr int kF4KSteps = 8;            // MMAs (K = 64) per chunk
constexpr int kF4MaxStages = 4;
constexpr int kF4Threads = 320;
constexpr uint32_t kF4TmemCols = 512;

// Operand kinds of the streaming tcgen05 product.
constexpr int kKindMXFP4 = 0;
constexpr int kKindNVFP4 = 1;
constexpr int kKindBF16 = 2;

template <int KIND>
struct TcKind {
    static constexpr bool fp4 = KIND != kKindBF16;
    static constexpr bool NV = KIND == kKindNVFP4;
    static constexpr int VS = NV ? 16 : 32;                       // elements per scale (FP4)
    static constexpr int chunk_elems = fp4 ? kF4ChunkCodes : 128;  // K per stage (256 B per row)
    static constexpr int box_step = fp4 ? kF4Box : 64;  // TMA coordinate of one 128-byte box
    static constexpr int sf_bytes = fp4 ? kF4ChunkCodes / VS : 0;  // scale bytes per row per stage
    // tensor-memory columns of one operand's scales per stage: one column
    // per 32-bit word of a row's scale bytes and per row quarter
    static constexpr int sf_cols = sf_bytes;
    static constexpr uint32_t scale_format = NV ? 0u : 1u;  // E4M3 / E8M0
};

template <bool NV>
using F4Fmt = TcKind<NV ? kKindNVFP4 : kKindMXFP4>;

struct F4Geom {
    size_t off_x, off_sw, off_sx, stage_bytes, off_bar, total;
};

// Per stage: weight codes 2 x [128 x 128 B] | activation codes 2 x [nt x 128 B]
// | weight scales [128 x sfb] | activation scales [nt x sfb].
__host__ __device__ inline F4Geom f4_geom(int nt, int sfb, int stages) {
    F4Geom g{};
    g.off_x = static_cast<size_t>(kF4RT) * kF4ChunkBytes;
    g.off_sw = g.off_x + static_cast<size_t>(nt) * kF4ChunkBytes;
    g.off_sx = g.off_sw + static_cast<size_t>(kF4RT) * sfb;
    g.stage_bytes = align_up(g.off_sx + static_cast<size_t>(nt) * sfb, 1024);
    g.off_bar = g.stage_bytes * stages;
    // full, sf_ready, empty per stage; acc_full, acc_empty per accumulator;
    // drain; the fix-up's bulk copies; tensor-memory base and the
    // last-arriver flag
    g.total = g.off_bar + static_cast<size_t>(3 * kF4MaxStages + 4 + 2) * 8 + 16 + 1024;
    return g;
}

// Block-scaled instruction descriptor: A and B E2M1 (format 1 of the FP4
// kinds), both K-major, D fp32, M = 128, N = NT, K = 64, scale format per
// kind; the scale-factor ids (bits 29-30 for A, 4-5 for B) are or-ed in per
// MMA.
template <bool NV, int N>
__host__ __device__ constexpr uint32_t umma_idesc_f4() {
    return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
           (F4Fmt<NV>::scale_format << 23) | (static_cast<uint32_t>(kF4RT >> 4) << 24);
}

// D[tmem] (+)= (A * S_A)[smem] * ((B * S_B)[smem])^T for one K = 64 step;
// the scale factors are read from tensor memory at sfa / sfb (their top two
// bits the byte offset inside a column).  Issued by one thread.
template <bool NV>
__device__ __forceinline__ void umma_f4(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                        uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                        uint32_t accumulate) {
    if constexpr (NV) {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], "
            "[%6], p;\n\t}" ::"r"(tmem_d),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
            : "memory");
    } else {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "setp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], "
            "[%6], p;\n\t}" ::"r"(tmem_d),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
            : "memory");
    }
}

// Bulk copy of `bytes` (a multiple of 16, both addresses 16-byte aligned)
// from global to this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_load_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                              uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            dst),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Orders this thread's earlier generic-proxy memory accesses before its
// later async-proxy ones (bulk copies).
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async;" ::: "memory");
}

// 16 or 32 consecutive columns of this thread's lane from registers.
template <int N>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const uint32_t (&v)[N]) {
    static_assert(N == 16 || N == 32, "tcgen05.st width");
    if constexpr (N == 16) {
        asm volatile(
            "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
            "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
            "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
            "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
            "r"(v[15])
            : "memory");
    } else {
        asm volatile(
            "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
            "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
            "%28, %29, %30, %31, %32};" ::"r"(taddr),
            "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
            "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
            "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
            "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
            "r"(v[29]), "r"(v[30]), "r"(v[31])
            : "memory");
    }
}

// 16 or 32 consecutive columns of this thread's lane into registers.
template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&v)[N]) {
    static_assert(N == 16 || N == 32, "tcgen05.ld width");
    if constexpr (N == 16) {
        tmem_ld16(taddr, v);
    } else {
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
            "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
            "%28, %29, %30, %31}, [%32];"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
              "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
              "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]),
              "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
              "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]),
              "=r"(v[31])
            : "r"(taddr)
            : "memory");
    }
}

// Scale bytes of rows lane + 32 i (i = 0..3, rows < nrows; others zero) of a
// row-major [rows x SFB] shared-memory tile, arranged as the MMA reads them:
// column 4 w + i holds 32-bit word w of row lane + 32 i.
template <int SFB>
__device__ __forceinline__ void gather_scales(uint32_t tile, int lane, int nrows,
                                              uint32_t (&v)[SFB]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int row = lane + 32 * i;
        const bool on = row < nrows;
#pragma unroll
        for (int h = 0; h < SFB / 16; ++h) {
            const uint4 t = on ? lds128(tile + static_cast<uint32_t>(row * SFB + 16 * h))
                               : make_uint4(0u, 0u, 0u, 0u);
            v[(4 * h + 0) * 4 + i] = t.x;
            v[(4 * h + 1) * 4 + i] = t.y;
            v[(4 * h + 2) * 4 + i] = t.z;
            v[(4 * h + 3) * 4 + i] = t.w;
        }
    }
}

// CLUSTER: the grid is row_tiles x cluster_s CTAs in clusters of cluster_s,
// CTA p holding K part p % cluster_s of row tile p / cluster_s (one partial
// segment each); the cluster adds its partials through distributed shared
// memory instead of the workspace protocol.
template <int KIND, int NT, bool CLUSTER>
__device__ __forceinline__ void tc_gemm_body(const CUtensorMap& tmap_w, const CUtensorMap& tmap_sw,
                                             const CUtensorMap& tmap_x, const CUtensorMap& tmap_sx,
                                             const float* __restrict__ w_ts,
                                             const float* __restrict__ x_ts, int stages, int B,
                                             int64_t out, int nchunks, int64_t T,
                                             void* __restrict__ y, int ydt,
                                             float* __restrict__ ws_part,
                                             unsigned* __restrict__ ws_count,
                                             unsigned* __restrict__ status, int cluster_s) {
    using K = TcKind<KIND>;
    constexpr bool NV = K::NV;
    constexpr int SFB = K::sf_bytes;
    constexpr int SFC = K::sf_cols;
    constexpr int BOX = K::box_step;
    constexpr uint32_t kSf0 = 2 * NT;   // first scale-factor column
    constexpr uint32_t kIdesc =
        K::fp4 ? umma_idesc_f4<NV, NT>() : umma_idesc_f16<true, kF4RT, NT>();
    constexpr int PW = NT < 32 ? NT : 32;  // accumulator columns per tcgen05.ld
    constexpr int PF = 16;                 // columns per step of the fix-up
    static_assert(NT % 16 == 0 && NT >= 16 && NT <= 128, "activation tile width");
    static_assert(2 * NT + kF4MaxStages * 2 * SFC <= static_cast<int>(kF4TmemCols),
                  "tensor memory");

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const F4Geom geo = f4_geom(NT, SFB, stages);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + geo.off_bar);
    uint64_t* sf_ready = full + kF4MaxStages;
    uint64_t* empty = sf_ready + kF4MaxStages;
    uint64_t* acc_full = empty + kF4MaxStages;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* drain = acc_empty + 2;
    uint64_t* fixbar = drain + 1;
    uint32_t* tbase_s = reinterpret_cast<uint32_t*>(fixbar + 1);
    unsigned* last_flag = tbase_s + 1;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t P = gridDim.x;
    const int64_t p = blockIdx.x;
    const int64_t it_beg = (T * p) / P;
    const int64_t it_end = (T * (p + 1)) / P;
    const int nit = static_cast<int>(it_end - it_beg);
    const int tile0 = static_cast<int>(it_beg / nchunks);
    const int chunk0 = static_cast<int>(it_beg - static_cast<int64_t>(tile0) * nchunks);

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&sf_ready[s], 4);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], 4);
        }
        mbar_init(drain, 1);
        mbar_init(fixbar, 1);
        fence_mbarrier_init_cluster();
    }
    if (warp == 1) tmem_alloc(tbase_s, kF4TmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tbase_s;
    grid_launch_dependents();

    if (warp == 0) {
        // ------------------------------------------------------ producer
        if (lane == 0 && nit > 0) {
            prefetch_tmap(&tmap_w);
            prefetch_tmap(&tmap_x);
            if constexpr (K::fp4) {
                prefetch_tmap(&tmap_sw);
                prefetch_tmap(&tmap_sx);
            }
            const uint32_t tx = (kF4RT + NT) * (kF4ChunkBytes + SFB);
            auto load_w = [&](uint8_t* st, int chunk, int tile, uint64_t* bar) {
                tma_load_2d(st, &tmap_w, chunk * 2 * BOX, tile * kF4RT, bar);
                tma_load_2d(st + kF4RT * kF4Box, &tmap_w, chunk * 2 * BOX + BOX, tile * kF4RT, bar);
                if constexpr (K::fp4)
                    tma_load_2d(st + geo.off_sw, &tmap_sw, chunk * SFB, tile * kF4RT, bar);
            };
            const int pre = nit < stages ? nit : stages;
            {
                int tile = tile0, chunk = chunk0;
                for (int c = 0; c < pre; ++c) {
                    mbar_arrive_expect_tx(&full[c], tx);
                    load_w(smem + geo.stage_bytes * c, chunk, tile, &full[c]);
                    if (++chunk == nchunks) {
                        chunk = 0;
                        ++tile;
                    }
                }
            }
            grid_dependency_wait();  // the activations may come from the previous kernel
            bool ok = true;
            int tile = tile0, chunk = chunk0, s = 0;
            uint32_t ph = 0;
            for (int c = 0; c < nit; ++c) {
                if (c >= stages) ok = mbar_wait_bounded(&empty[s], ph ^ 1u, status, kWaitLimitNs);
                if (!ok) break;
                uint8_t* st = smem + geo.stage_bytes * s;
                if (c >= pre) {
                    mbar_arrive_expect_tx(&full[s], tx);
                    load_w(st, chunk, tile, &full[s]);
                }
                tma_load_2d(st + geo.off_x, &tmap_x, chunk * 2 * BOX, 0, &full[s]);
                tma_load_2d(st + geo.off_x + NT * kF4Box, &tmap_x, chunk * 2 * BOX + BOX, 0,
                            &full[s]);
                if constexpr (K::fp4) tma_load_2d(st + geo.off_sx, &tmap_sx, chunk * SFB, 0, &full[s]);
                if (++chunk == nchunks) {
                    chunk = 0;
                    ++tile;
                }
                if (++s == stages) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            // no load may still be landing when the CTA exits
            for (int s2 = 0; s2 < stages && s2 < nit; ++s2) {
                const int last = s2 + ((nit - 1 - s2) / stages) * stages;
                mbar_wait_bounded(&full[s2], (last / stages) & 1, status, kWaitLimitNs);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------- MMA issuer
        if (lane == 0 && nit > 0) {
            const uint32_t sb = smem_u32(smem);
            bool ok = true;
            int s = 0, chunk = chunk0, seg = 0;
            uint32_t ph = 0;
            bool seg_first = true;  // the next chunk starts a segment
            for (int c = 0; c < nit; ++c) {
                const int a = seg & 1;
                if (seg_first && seg >= 2)
                    ok = mbar_wait_bounded(&acc_empty[a], static_cast<uint32_t>((seg >> 1) - 1) & 1u,
                                           status, kWaitLimitNs);
                if (ok) ok = mbar_wait_bounded(&full[s], ph, status, kWaitLimitNs);
                if (K::fp4 && ok) ok = mbar_wait_bounded(&sf_ready[s], ph, status, kWaitLimitNs);
                if (!ok) break;
                tc_fence_after();
                const uint32_t st = sb + static_cast<uint32_t>(geo.stage_bytes) * s;
                const uint32_t sfa = tbase + kSf0 + static_cast<uint32_t>(2 * SFC * s);
                const uint32_t sfb = sfa + SFC;
#pragma unroll
                for (int kk = 0; kk < kF4KSteps; ++kk) {
                    const uint32_t koff = static_cast<uint32_t>((kk & 3) * 32);  // K slice in the atom
                    const uint64_t ad = umma_desc_sw128_kmajor(
                        st + static_cast<uint32_t>((kk >> 2) * kF4RT * kF4Box) + koff);
                    const uint64_t bd = umma_desc_sw128_kmajor(
                        st + static_cast<uint32_t>(geo.off_x + (kk >> 2) * NT * kF4Box) + koff);
                    const uint32_t acc = (seg_first && kk == 0) ? 0u : 1u;
                    if constexpr (K::fp4) {
                        const uint32_t col = NV ? 4u * kk : 4u * (kk >> 1);
                        const uint32_t sid = NV ? 0u : 2u * (kk & 1);
                        umma_f4<NV>(tbase + static_cast<uint32_t>(a * NT), ad, bd,
                                    kIdesc | (sid << 29) | (sid << 4), (sfa + col) | (sid << 30),
                                    (sfb + col) | (sid << 30), acc);
                    } else {
                        umma_f16_ss(tbase + static_cast<uint32_t>(a * NT), ad, bd, kIdesc, acc);
                    }
                }
                umma_commit(&empty[s]);  // the stage's codes and scales are no longer read
                const bool seg_end = chunk == nchunks - 1 || c == nit - 1;
                if (seg_end) {
                    umma_commit(&acc_full[a]);
                    ++seg;
                }
                seg_first = seg_end;
                if (++chunk == nchunks) chunk = 0;
                if (++s == stages) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            // every MMA has completed before tensor memory is released
            umma_commit(drain);
            mbar_wait_bounded(drain, 0, status, kWaitLimitNs);
        }
    } else if (warp < 6) {
        // ------------------------------------------------ scale writers
        if constexpr (K::fp4) {
        const uint32_t tl = tbase + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
        const uint32_t sb = smem_u32(smem);
        bool ok = true;
        int s = 0;
        uint32_t ph = 0;
        for (int c = 0; c < nit; ++c) {
            if (ok) ok = mbar_wait_bounded(&full[s], ph, status, kWaitLimitNs);
            ok = __all_sync(0xffffffffu, ok);
            if (ok) {
                tc_fence_after();
                const uint32_t st = sb + static_cast<uint32_t>(geo.stage_bytes) * s;
                const uint32_t col = kSf0 + static_cast<uint32_t>(2 * SFC * s);
                uint32_t v[SFC];
                gather_scales<SFB>(st + static_cast<uint32_t>(geo.off_sw), lane, kF4RT, v);
                tmem_st_cols<SFC>(tl + col, v);
                gather_scales<SFB>(st + static_cast<uint32_t>(geo.off_sx), lane, NT, v);
                tmem_st_cols<SFC>(tl + col + SFC, v);
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sf_ready[s]);
            if (++s == stages) {
                s = 0;
                ph ^= 1u;
            }
        }
        }
    } else {
        // ------------------------------------------------------- epilogue
        const int q = warp & 3;
        const int r = 32 * q + lane;  // row of the tile held in this thread's lane
        const uint32_t tl = tbase + (static_cast<uint32_t>(32 * q) << 16);
        // the drained pipeline's shared memory holds the partials of the final
        // fix-up: up to fix_cap contributors of NT x 128 fp32 each
        const uint32_t fix_smem = smem_u32(smem);
        const int fix_cap = static_cast<int>((geo.stage_bytes * stages) /
                                             (static_cast<size_t>(kF4RT) * NT * 4));
        grid_dependency_wait();  // x_ts may come from the previous kernel; y is written below
        const float g = NV ? __ldg(w_ts) * __ldg(x_ts) : 1.0f;
        bool ok = true;
        int tile = tile0, chunk = chunk0, seg = 0, c = 0;
        while (c < nit) {
            const int len = (nchunks - chunk) < (nit - c) ? (nchunks - chunk) : (nit - c);
            const bool whole = chunk == 0 && len == nchunks;
            const bool first = c == 0;
            const bool final_seg = c + len == nit;
            const int a = seg & 1;
            if (ok)
                ok = mbar_wait_bounded(&acc_full[a], static_cast<uint32_t>(seg >> 1) & 1u, status,
                                       kWaitLimitNs);
            ok = __all_sync(0xffffffffu, ok);
            tc_fence_after();
            if constexpr (CLUSTER) {
                // The CTA's one (partial) segment: its accumulator goes to the
                // drained pipeline's shared memory, [NT columns x 128 rows]
                // fp32, for the cluster's reduction after the role branches.
                if (ok) {
#pragma unroll 1
                    for (int c0 = 0; c0 < NT; c0 += PW) {
                        uint32_t v[PW];
                        tmem_ld_cols<PW>(tl + static_cast<uint32_t>(a * NT + c0), v);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < PW; ++e)
                            sts32(fix_smem + static_cast<uint32_t>(((c0 + e) * kF4RT + r) * 4), v[e]);
                    }
                }
                c += len;
                chunk = 0;
                ++tile;
                ++seg;
                continue;
            }
            const int64_t row = static_cast<int64_t>(tile) * kF4RT + r;
            const int slot = static_cast<int>(2 * p + (first ? 0 : 1));
            float* part = ws_part + static_cast<size_t>(slot) * kF4RT * NT;
            const int64_t t64 = tile;
            const int64_t q_lo = sk_owner(t64 * nchunks, T, P);
            const int64_t q_hi = sk_owner(t64 * nchunks + nchunks - 1, T, P);
            const int nothers = static_cast<int>(q_hi - q_lo);
            // at the end of the range every stage has been consumed: the
            // other partials are bulk-copied into shared memory at once
            const bool bulk = final_seg && nothers <= fix_cap;
            // A final partial segment whose tile counter already holds every
            // other contributor is certainly the last one: it keeps its
            // partial in tensor memory instead of storing it.
            bool early = false;
            if (!whole && bulk) {
                named_bar_sync(1, 128);
                if (threadIdx.x == 192) {
                    const bool e = ld_acquire_gpu(ws_count + tile) == static_cast<unsigned>(nothers);
                    if (e) ws_count[tile] = 0u;  // no other contributor touches it again
                    *last_flag = e ? 2u : 0u;
                }
                named_bar_sync(1, 128);
                early = *last_flag == 2u;
            }
            if (ok && !(early && !whole)) {
#pragma unroll 1
                for (int c0 = 0; c0 < NT; c0 += PW) {
                    uint32_t v[PW];
                    tmem_ld_cols<PW>(tl + static_cast<uint32_t>(a * NT + c0), v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < PW; ++e) {
                        const int n = c0 + e;
                        if (n >= B) continue;
                        if (whole) {
                            if (row < out)
                                store_y(y, ydt, static_cast<int64_t>(n) * out + row,
                                        g * __uint_as_float(v[e]));
                        } else {
                            __stcg(part + n * kF4RT + r, __uint_as_float(v[e]));
                        }
                    }
                }
            }
            // the final partial accumulator stays in tensor memory for the fix-up
            // (no later segment reuses its buffer)
            const bool keep = final_seg && !whole;
            if (!keep) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[a]);
            }
            if (!whole) {
                named_bar_sync(1, 128);
                if (threadIdx.x == 192) {
                    bool last = early;
                    if (!early) {
                        const unsigned prev = atom_add_acq_rel_gpu(ws_count + tile, 1u);
                        last = prev == static_cast<unsigned>(nothers);
                        if (last) ws_count[tile] = 0u;  // zero again for the next call
                    }
                    *last_flag = last ? 1u : 0u;
                    if (last && bulk) {
                        fence_proxy_async();  // the partials were written through the generic proxy
                        mbar_arrive_expect_tx(fixbar,
                                              static_cast<uint32_t>(nothers * NT * kF4RT * 4));
                        int j = 0;
                        for (int64_t qq = q_lo; qq <= q_hi; ++qq) {
                            if (qq == p) continue;
                            const bool fs = (T * qq) / P >= t64 * nchunks;
                            const float* src = ws_part + static_cast<size_t>(2 * qq + (fs ? 0 : 1)) *
                                                             kF4RT * NT;
                            for (int pi = 0; pi < NT / PF; ++pi)
                                bulk_load_g2s(fix_smem + static_cast<uint32_t>(
                                                             (pi * nothers + j) * PF * kF4RT * 4),
                                              src + pi * PF * kF4RT, PF * kF4RT * 4, fixbar);
                            ++j;
                        }
                    }
                }
                named_bar_sync(1, 128);
                if (*last_flag) {
                    if (bulk) {
                        bool okf = ok && mbar_wait_bounded(fixbar, 0, status, kWaitLimitNs);
                        okf = __all_sync(0xffffffffu, okf);
                        // contributors in CTA order, this CTA's own part from tensor memory
#pragma unroll 1
                        for (int pi = 0; pi < NT / PF; ++pi) {
                            const int c0 = pi * PF;
                            uint32_t v[PF];
                            if (okf) {
                                tmem_ld_cols<PF>(tl + static_cast<uint32_t>(a * NT + c0), v);
                                tmem_wait_ld();
                            }
                            if (okf && c0 < B && row < out) {
                                float acc[PF];
#pragma unroll
                                for (int e = 0; e < PF; ++e) acc[e] = 0.f;
                                int j = 0;
                                for (int64_t qq = q_lo; qq <= q_hi; ++qq) {
                                    if (qq == p) {
#pragma unroll
                                        for (int e = 0; e < PF; ++e) acc[e] += __uint_as_float(v[e]);
                                    } else {
                                        const uint32_t blk =
                                            fix_smem +
                                            static_cast<uint32_t>(((pi * nothers + j) * PF * kF4RT + r) * 4);
#pragma unroll
                                        for (int e = 0; e < PF; ++e)
                                            acc[e] += __uint_as_float(lds32(blk + e * kF4RT * 4));
                                        ++j;
                                    }
                                }
#pragma unroll
                                for (int e = 0; e < PF; ++e)
                                    if (c0 + e < B)
                                        store_y(y, ydt, static_cast<int64_t>(c0 + e) * out + row,
                                                g * acc[e]);
                            }
                        }
                    } else if (row < out) {
                        // a fix-up while the pipeline still runs: from global
                        // memory, PF independent loads per contributor
#pragma unroll 1
                        for (int c0 = 0; c0 < NT; c0 += PF) {
                            if (c0 < B) {
                                float acc[PF];
#pragma unroll
                                for (int e = 0; e < PF; ++e) acc[e] = 0.f;
                                for (int64_t qq = q_lo; qq <= q_hi; ++qq) {
                                    const bool fs = (T * qq) / P >= t64 * nchunks;
                                    const int qs = static_cast<int>(2 * qq + (fs ? 0 : 1));
                                    const float* pq =
                                        ws_part + static_cast<size_t>(qs) * kF4RT * NT + r;
#pragma unroll
                                    for (int e = 0; e < PF; ++e)
                                        if (c0 + e < B) acc[e] += __ldcg(pq + (c0 + e) * kF4RT);
                                }
#pragma unroll
                                for (int e = 0; e < PF; ++e)
                                    if (c0 + e < B)
                                        store_y(y, ydt, static_cast<int64_t>(c0 + e) * out + row,
                                                g * acc[e]);
                            }
                        }
                    }
                }
                named_bar_sync(1, 128);
            }
            c += len;
            chunk = 0;
            ++tile;
            ++seg;
        }
    }

    tc_fence_before();
    __syncthreads();
    if constexpr (CLUSTER) {
        // Every thread of every CTA of the cluster passes both barriers: all
        // roles have joined at the __syncthreads above.
        cluster_sync_all();  // every rank's partial is in its shared memory
        if (warp >= 6) {
            // rank rk writes y for columns [NT rk / S, NT (rk+1) / S) of the
            // tile, adding the S partials in rank order
            const int S = cluster_s;
            const int rk = static_cast<int>(cluster_ctarank());
            const int r = 32 * (warp & 3) + lane;
            const int64_t row = static_cast<int64_t>(tile0) * kF4RT + r;
            const float g = NV ? __ldg(w_ts) * __ldg(x_ts) : 1.0f;
            const uint32_t base = smem_u32(smem);
            const int n_end = min(NT * (rk + 1) / S, B);
            constexpr int U = 8;
            for (int n0 = NT * rk / S; n0 < n_end; n0 += U) {
                float acc[U];
#pragma unroll
                for (int u = 0; u < U; ++u) acc[u] = 0.f;
                for (int k = 0; k < S; ++k) {
                    float v[U];
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const int n = min(n0 + u, NT - 1);
                        v[u] = ld_shared_cluster_f32(mapa_shared(
                            base + static_cast<uint32_t>((n * kF4RT + r) * 4), static_cast<uint32_t>(k)));
                    }
#pragma unroll
                    for (int u = 0; u < U; ++u) acc[u] += v[u];
                }
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if (n0 + u < n_end && row < out)
                        store_y(y, ydt, static_cast<int64_t>(n0 + u) * out + row, g * acc[u]);
            }
        }
        __syncwarp();
        cluster_sync_all();  // no rank leaves while another still reads it
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, kF4TmemCols);
    }
}

// W4A4 product of two FP4 operands (NVFP4 or MXFP4).
template <bool NV, int NT, bool CLUSTER>
__global__ void __launch_bounds__(kF4Threads, 1)
    fp4_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_w,
                       const __grid_constant__ CUtensorMap tmap_sw,
                       const __grid_constant__ CUtensorMap tmap_x,
                       const __grid_constant__ CUtensorMap tmap_sx,
                       const float* __restrict__ w_ts, const float* __restrict__ x_ts, int stages,
                       int B, int64_t out, int nchunks, int64_t T, void* __restrict__ y, int ydt,
                       float* __restrict__ ws_part, unsigned* __restrict__ ws_count,
                       unsigned* __restrict__ status, int cluster_s) {
    tc_gemm_body<NV ? kKindNVFP4 : kKindMXFP4, NT, CLUSTER>(tmap_w, tmap_sw, tmap_x, tmap_sx, w_ts,
                                                            x_ts, stages, B, out, nchunks, T, y,
                                                            ydt, ws_part, ws_count, status,
                                                            cluster_s);
}

// The bf16 reference product y = x W^T (bf16 W and x, fp32 accumulation).
template <int NT, bool CLUSTER>
__global__ void __launch_bounds__(kF4Threads, 1)
    bf16_gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_w,
                        const __grid_constant__ CUtensorMap tmap_x, int stages, int B, int64_t out,
                        int nchunks, int64_t T, void* __restrict__ y, int ydt,
                        float* __restrict__ ws_part, unsigned* __restrict__ ws_count,
                        unsigned* __restrict__ status, int cluster_s) {
    tc_gemm_body<kKindBF16, NT, CLUSTER>(tmap_w, tmap_w, tmap_x, tmap_x, nullptr, nullptr, stages,
                                         B, out, nchunks, T, y, ydt, ws_part, ws_count, status,
                                         cluster_s);
}

}  // namespace q4dev
