// q4_skinny_tc.cuh -- W4A16 product on the tcgen05 tensor cores for batches
// of 9 to 128 rows (the skinny-GEMM regime).
//
//   y[b, r] = sum_j s[r, j] * sum_{k in group j} (q[r, k] - z[r, j]) * x[b, k]
//
// Work decomposition: the same persistent stream-K split as the small-batch
// kernel (q4_gemv_sk.cuh): T = row_tiles x chunks iterations, a row tile is
// 128 rows (the MMA's M and the 128 lanes of tensor memory), a chunk 256
// codes of K; CTA p owns iterations [T p / P, T (p+1) / P), partial tiles are
// finished by the CTA that arrives last on the tile's counter, adding the
// partials in CTA order.
//
// Data flow of one chunk (a pipeline stage):
//  * producer warp: TMA loads of the weight tile [128 rows x 128 B] (128-byte
//    swizzle), of the activations [NT rows x 256] as four 128-byte-swizzled
//    K-major atoms (rows >= B are filled with zeros by the TMA unit), and of
//    the scale (and zero-point) window;
//  * 4 (NT <= 32) or 16 converter warps, one weight row per thread and
//    lane, in shares of four warps (one per tensor-memory lane quarter): each
//    group's codes are unpacked to exact 16-bit integers q (or q - z) and
//    stored into a tensor-memory A buffer, the 16-byte chunks of a row divided
//    among the shares (arganzheng.life post-training-quantization-gptq-awq-
//    and-rotation, section 二.3: the int4 weights are dequantized on chip,
//    never in HBM);
//  * MMA warp, one thread: per group, GS/16 tcgen05.mma steps
//    D[128 x NT] (+)= A[128 x 16] * X[NT x 16]^T into a fresh fp32
//    accumulator in tensor memory, then a commit;
//  * the converter warps read each finished group accumulator back, each
//    share its own columns, and add it times the group's fp32 scale into
//    registers (section 二.2: per-group scales are applied inside the K
//    accumulation, one partial per group).  The rescale of a group runs one
//    or two groups after its unpack, so the MMAs overlap the next unpacks.
//
// Unpacking keeps K in natural order: for the byte holding codes k and k+1,
// one PRMT places it and the same byte of the word shifted right by 4 at the
// two halves of a register, one LOP3 masks the two low nibbles into the
// mantissas of 128.0 (bf16) / 1024.0 (fp16) and flips the sign bit of
// two's-complement codes, and one packed subtraction of 136 / 1032 (or
// 128 + z / 1024 + z) leaves the exact integers: a k, k+1 pair is exactly the
// 32-bit column layout of a 16-bit A operand, and the activations need no
// reordering.
#pragma once

#include "q4_device.cuh"
#include "q4_gemv.cuh"
#include "q4_gemv_sk.cuh"
#include "q4_tcgen05.cuh"

namespace q4dev {

constexpr int kTcRT = 128;        // rows per tile: MMA M, tensor-memory lanes
constexpr int kTcMaxStages = 4;
constexpr int kTcMaxBuf = 4;      // group buffers in tensor memory

template <int NT>
struct TcCfg {
    // CTAs per SM: tensor memory (512 columns per SM) is split between them
    static constexpr int ctas_per_sm = NT <= 32 ? 2 : 1;
    static constexpr uint32_t tmem_cols = NT <= 32 ? 256u : 512u;
    // converter warps: H shares of 4 warps (one per tensor-memory lane
    // quarter); share h unpacks the 16-byte chunks c with c % H == h and
    // rescales accumulator columns [h NT / H, (h + 1) NT / H).  Narrow tiles
    // are bound by the MMA rate (one M = 128, K = 16 step takes as long at
    // N = 16 as at N = 128), wide ones by the rescale work.
    static constexpr int conv_warps = NT <= 32 ? 4 : 16;
    static constexpr int threads = (2 + conv_warps) * 32;
};

struct TcGeom {
    size_t off_x, off_sc, off_zc, stage_bytes, off_bar, total;
};

// Per stage: weights [128 x 128 B] | activations 4 x [nt x 128 B] |
// scale window [128 x 8] fp16 | zero-point window [128 x 8] fp16 (asymmetric).
__host__ __device__ inline TcGeom tc_geom(int nt, int stages, bool sym) {
    TcGeom g{};
    g.off_x = static_cast<size_t>(kTcRT) * kChunkBytes;
    g.off_sc = g.off_x + static_cast<size_t>(4) * nt * 128;
    g.off_zc = g.off_sc + static_cast<size_t>(kTcRT) * 16;
    const size_t end = g.off_zc + (sym ? 0 : static_cast<size_t>(kTcRT) * 16);
    g.stage_bytes = align_up(end, 1024);
    g.off_bar = g.stage_bytes * stages;
    // full, empty per stage; a_full, mma_done, acc_free per buffer; drain;
    // tensor-memory base and the last-arriver flag
    g.total = g.off_bar + static_cast<size_t>(2 * kTcMaxStages + 3 * kTcMaxBuf + 1) * 8 + 16 + 1024;
    return g;
}

// Selector of PRMT placing byte j of a at byte 0 and byte j of b at byte 2.
template <int J>
struct PairSel {
    static constexpr uint32_t v = J | (J << 4) | ((4 + J) << 8) | ((4 + J) << 12);
};

// Eight codes of one 32-bit word -> four (k, k+1) pairs of exact 16-bit values.
template <bool BF16>
__device__ __forceinline__ void unpack_word_pairs(uint32_t w, uint32_t magic, uint32_t c2,
                                                  uint32_t* o) {
    const uint32_t u = shr_fma<4>(w);
    o[0] = sub2<BF16>(lop3_and_xor(prmt(w, u, PairSel<0>::v), 0x000F000Fu, magic), c2);
    o[1] = sub2<BF16>(lop3_and_xor(prmt(w, u, PairSel<1>::v), 0x000F000Fu, magic), c2);
    o[2] = sub2<BF16>(lop3_and_xor(prmt(w, u, PairSel<2>::v), 0x000F000Fu, magic), c2);
    o[3] = sub2<BF16>(lop3_and_xor(prmt(w, u, PairSel<3>::v), 0x000F000Fu, magic), c2);
}

template <bool BF16, int GS, int NT>
__global__ void __launch_bounds__(TcCfg<NT>::threads, TcCfg<NT>::ctas_per_sm)
    q4_skinny_tc_kernel(const __grid_constant__ CUtensorMap tmap_w,
                        const __grid_constant__ CUtensorMap tmap_x,
                        const __grid_constant__ CUtensorMap tmap_s,
                        const __grid_constant__ CUtensorMap tmap_z, int meta_tma,
                        const uint16_t* __restrict__ scales, const uint16_t* __restrict__ zeros,
                        int sym, int stages, int B, int64_t out, int64_t in, int nchunks, int64_t T,
                        void* __restrict__ y, int ydt, float* __restrict__ ws_part,
                        unsigned* __restrict__ ws_count, unsigned* __restrict__ status) {
    constexpr int GPC = kChunkCodes / GS;      // groups per chunk
    constexpr int KSG = GS / 16;               // MMA K steps per group
    constexpr int ACOLS = GS / 2;              // tensor-memory columns of one group's A
    constexpr uint32_t TCOLS = TcCfg<NT>::tmem_cols;
    constexpr int NBF = static_cast<int>(TCOLS) / (ACOLS + NT);
    constexpr int NB = NBF < kTcMaxBuf ? NBF : kTcMaxBuf;
    static_assert(NB >= 2, "tensor memory too small for two group buffers");
    constexpr uint32_t kIdesc = umma_idesc_f16<BF16, kTcRT, NT>();
    constexpr uint32_t kDcol0 = NB * ACOLS;    // first accumulator column
    constexpr int CONV = TcCfg<NT>::conv_warps;
    constexpr int H = CONV / 4;
    constexpr int NH = NT / H;                 // accumulator columns per converter warp
    constexpr int LAG = NB >= 3 ? 2 : 1;       // groups between a group's unpack and its rescale
    static_assert(NH % 8 == 0, "columns per converter warp");

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const TcGeom geo = tc_geom(NT, stages, sym != 0);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + geo.off_bar);
    uint64_t* empty = full + kTcMaxStages;
    uint64_t* a_full = empty + kTcMaxStages;
    uint64_t* mma_done = a_full + kTcMaxBuf;
    uint64_t* acc_free = mma_done + kTcMaxBuf;
    uint64_t* drain = acc_free + kTcMaxBuf;
    uint32_t* tbase_s = reinterpret_cast<uint32_t*>(drain + 1);
    unsigned* last_flag = tbase_s + 1;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t P = gridDim.x;
    const int64_t p = blockIdx.x;
    const int64_t it_beg = (T * p) / P;
    const int64_t it_end = (T * (p + 1)) / P;
    const int nit = static_cast<int>(it_end - it_beg);
    const int64_t G = in / GS;
    const int tile0 = static_cast<int>(it_beg / nchunks);
    const int chunk0 = static_cast<int>(it_beg - static_cast<int64_t>(tile0) * nchunks);

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], CONV + 1);  // converter warps + the MMA commit
        }
        for (int b = 0; b < NB; ++b) {
            mbar_init(&a_full[b], CONV);
            mbar_init(&mma_done[b], 1);
            mbar_init(&acc_free[b], CONV);
        }
        mbar_init(drain, 1);
        fence_mbarrier_init_cluster();
    }
    if (warp == 1) tmem_alloc(tbase_s, TCOLS);
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
            const uint32_t tx = kTcRT * kChunkBytes + 4 * NT * 128 +
                                (meta_tma ? kTcRT * 16 * (sym ? 1 : 2) : 0);
            const int pre = nit < stages ? nit : stages;
            {
                int tile = tile0, chunk = chunk0;
                for (int c = 0; c < pre; ++c) {
                    uint8_t* st = smem + geo.stage_bytes * c;
                    mbar_arrive_expect_tx(&full[c], tx);
                    tma_load_2d(st, &tmap_w, chunk * kChunkBytes, tile * kTcRT, &full[c]);
                    if (meta_tma) {
                        const int win = (chunk * GPC) & ~7;
                        tma_load_2d(st + geo.off_sc, &tmap_s, win, tile * kTcRT, &full[c]);
                        if (!sym) tma_load_2d(st + geo.off_zc, &tmap_z, win, tile * kTcRT, &full[c]);
                    }
                    if (++chunk == nchunks) {
                        chunk = 0;
                        ++tile;
                    }
                }
            }
            grid_dependency_wait();
            bool ok = true;
            int tile = tile0, chunk = chunk0, s = 0;
            uint32_t ph = 0;
            for (int c = 0; c < nit; ++c) {
                if (c >= stages) ok = mbar_wait_bounded(&empty[s], ph ^ 1u, status, kWaitLimitNs);
                if (!ok) break;
                uint8_t* st = smem + geo.stage_bytes * s;
                if (c >= pre) {
                    mbar_arrive_expect_tx(&full[s], tx);
                    tma_load_2d(st, &tmap_w, chunk * kChunkBytes, tile * kTcRT, &full[s]);
                    if (meta_tma) {
                        const int win = (chunk * GPC) & ~7;
                        tma_load_2d(st + geo.off_sc, &tmap_s, win, tile * kTcRT, &full[s]);
                        if (!sym) tma_load_2d(st + geo.off_zc, &tmap_z, win, tile * kTcRT, &full[s]);
                    }
                }
#pragma unroll
                for (int a = 0; a < 4; ++a)
                    tma_load_2d(st + geo.off_x + a * NT * 128, &tmap_x, chunk * kChunkCodes + a * 64,
                                0, &full[s]);
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
            const uint32_t xs0 = smem_u32(smem) + static_cast<uint32_t>(geo.off_x);
            const uint32_t sbytes = static_cast<uint32_t>(geo.stage_bytes);
            bool ok = true;
            int s = 0, i = 0;
            uint32_t ph = 0;
            for (int c = 0; c < nit && ok; ++c) {
                ok = mbar_wait_bounded(&full[s], ph, status, kWaitLimitNs);
                if (!ok) break;
                const uint32_t xb = xs0 + sbytes * static_cast<uint32_t>(s);
#pragma unroll
                for (int gq = 0; gq < GPC; ++gq, ++i) {
                    const int b = i % NB;
                    const uint32_t u = static_cast<uint32_t>(i / NB);
                    ok = mbar_wait_bounded(&a_full[b], u & 1u, status, kWaitLimitNs);
                    if (ok && i >= NB)
                        ok = mbar_wait_bounded(&acc_free[b], (u - 1u) & 1u, status, kWaitLimitNs);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < KSG; ++kk) {
                        const int ks = gq * KSG + kk;  // K step inside the chunk
                        const uint64_t bd = umma_desc_sw128_kmajor(
                            xb + static_cast<uint32_t>((ks >> 2) * NT * 128 + (ks & 3) * 32));
                        umma_f16_ts(tbase + kDcol0 + b * NT, tbase + b * ACOLS + kk * 8, bd, kIdesc,
                                    kk > 0 ? 1u : 0u);
                    }
                    umma_commit(&mma_done[b]);
                }
                if (!ok) break;
                umma_commit(&empty[s]);  // the stage's activations are no longer read
                if (++s == stages) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            // every MMA has completed before tensor memory is released
            umma_commit(drain);
            mbar_wait_bounded(drain, 0, status, kWaitLimitNs);
        }
    } else {
        // ------------------------------------------------------ converters
        const int q = warp & 3;          // tensor-memory lane quarter (warp % 4)
        const int h = (warp - 2) >> 2;   // this warp's share of the work
        const int r = 32 * q + lane;     // weight row of this thread
        const uint32_t tl = tbase + (static_cast<uint32_t>(32 * q) << 16);
        const uint32_t magic = Magic<BF16>::base2 ^ (sym ? 0x00080008u : 0u);
        const uint32_t csym = static_cast<uint32_t>(small_int_bits<BF16>(Magic<BF16>::base + 8.0f)) *
                              0x00010001u;
        grid_dependency_wait();  // y and the workspace are written below

        float yacc[NH];
#pragma unroll
        for (int e = 0; e < NH; ++e) yacc[e] = 0.f;

        const uint32_t sbase = smem_u32(smem);
        const uint32_t sbytes = static_cast<uint32_t>(geo.stage_bytes);
        bool ok = true;
        int cur_tile = tile0, cur_chunk = chunk0, s = 0, i = 0;
        uint32_t ph = 0;
        int seg_start = 0;

        // A group waiting for its rescale: its scale and, if it ends a
        // segment, the segment's tile and kind.
        struct Pend {
            float scale;
            bool end, whole, first;
            int tile;
        };
        Pend p0{0.f, false, false, false, 0}, p1{0.f, false, false, false, 0};

        // Rescale of group j (accumulator buffer j % NB): this warp's NH
        // columns times the group's scale into yacc; then, if the group ends
        // a segment, the segment's epilogue.
        auto rescale = [&](int j, const Pend& pd) {
            const int b = j % NB;
            if (ok) ok = mbar_wait_bounded(&mma_done[b], static_cast<uint32_t>(j / NB) & 1u, status,
                                           kWaitLimitNs);
            tc_fence_after();
            if (ok) {
                uint32_t v[NH];
#pragma unroll
                for (int c0 = 0; c0 < NH; c0 += 8)
                    tmem_ld8(tl + kDcol0 + b * NT + h * NH + c0,
                             *reinterpret_cast<uint32_t(*)[8]>(&v[c0]));
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < NH; ++e) yacc[e] = fmaf(pd.scale, __uint_as_float(v[e]), yacc[e]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_free[b]);
            if (!pd.end) return;
            const int64_t row = static_cast<int64_t>(pd.tile) * kTcRT + r;
            if (pd.whole) {
                if (row < out) {
#pragma unroll
                    for (int e = 0; e < NH; ++e) {
                        const int n = h * NH + e;
                        if (n < B) store_y(y, ydt, static_cast<int64_t>(n) * out + row, yacc[e]);
                    }
                }
            } else {
                const int slot = static_cast<int>(2 * p + (pd.first ? 0 : 1));
                float* part = ws_part + static_cast<size_t>(slot) * kTcRT * NT;
#pragma unroll
                for (int e = 0; e < NH; ++e) {
                    const int n = h * NH + e;
                    if (n < B) __stcg(part + n * kTcRT + r, yacc[e]);
                }
                const int64_t t64 = pd.tile;
                const int64_t q_lo = sk_owner(t64 * nchunks, T, P);
                const int64_t q_hi = sk_owner(t64 * nchunks + nchunks - 1, T, P);
                named_bar_sync(1, CONV * 32);
                if (threadIdx.x == 64) {
                    const unsigned prev = atom_add_acq_rel_gpu(ws_count + pd.tile, 1u);
                    const bool last = prev == static_cast<unsigned>(q_hi - q_lo);
                    *last_flag = last ? 1u : 0u;
                    if (last) ws_count[pd.tile] = 0u;  // zero again for the next call
                }
                named_bar_sync(1, CONV * 32);
                if (*last_flag) {
                    // contributors in CTA order
#pragma unroll
                    for (int e = 0; e < NH; ++e) yacc[e] = 0.f;
                    for (int64_t qq = q_lo; qq <= q_hi; ++qq) {
                        const bool fs = (T * qq) / P >= t64 * nchunks;
                        const int qs = static_cast<int>(2 * qq + (fs ? 0 : 1));
                        const float* pq = ws_part + static_cast<size_t>(qs) * kTcRT * NT;
#pragma unroll
                        for (int e = 0; e < NH; ++e) {
                            const int n = h * NH + e;
                            if (n < B) yacc[e] += __ldcg(pq + n * kTcRT + r);
                        }
                    }
                    if (row < out) {
#pragma unroll
                        for (int e = 0; e < NH; ++e) {
                            const int n = h * NH + e;
                            if (n < B) store_y(y, ydt, static_cast<int64_t>(n) * out + row, yacc[e]);
                        }
                    }
                }
                named_bar_sync(1, CONV * 32);
            }
#pragma unroll
            for (int e = 0; e < NH; ++e) yacc[e] = 0.f;
        };

        for (int c = 0; c < nit; ++c) {
            if (ok) ok = mbar_wait_bounded(&full[s], ph, status, kWaitLimitNs);
            const uint32_t sa = sbase + sbytes * static_cast<uint32_t>(s);
            const int win = (cur_chunk * GPC) & ~7;
            const int64_t row = static_cast<int64_t>(cur_tile) * kTcRT + r;
#pragma unroll
            for (int gq = 0; gq < GPC; ++gq, ++i) {
                const int b = i % NB;
                const int64_t g = static_cast<int64_t>(cur_chunk) * GPC + gq;
                float sc = 0.f;
                if (ok) {
                    uint32_t c2 = csym;
                    if (meta_tma) {
                        const uint32_t so = static_cast<uint32_t>(geo.off_sc) + r * 16 +
                                            static_cast<uint32_t>(g - win) * 2;
                        sc = __half2float(__ushort_as_half(lds16(sa + so)));
                        if (!sym) {
                            const float z = __half2float(__ushort_as_half(
                                lds16(sa + so + static_cast<uint32_t>(geo.off_zc - geo.off_sc))));
                            c2 = static_cast<uint32_t>(small_int_bits<BF16>(Magic<BF16>::base + z)) *
                                 0x00010001u;
                        }
                    } else {
                        const bool okg = row < out && g < G;
                        sc = okg ? __half2float(__ushort_as_half(__ldg(scales + row * G + g))) : 0.f;
                        if (!sym) {
                            const float z = okg ? __half2float(__ushort_as_half(__ldg(zeros + row * G + g))) : 0.f;
                            c2 = static_cast<uint32_t>(small_int_bits<BF16>(Magic<BF16>::base + z)) *
                                 0x00010001u;
                        }
                    }
#pragma unroll
                    for (int t = 0; t < GS / 32; ++t) {
                        const int c16 = gq * (GS / 32) + t;
                        if (c16 % H != h) continue;
                        const uint4 w = lds128(sa + r * kChunkBytes + ((c16 ^ (r & 7)) << 4));
                        uint32_t v0[8], v1[8];
                        unpack_word_pairs<BF16>(w.x, magic, c2, v0);
                        unpack_word_pairs<BF16>(w.y, magic, c2, v0 + 4);
                        unpack_word_pairs<BF16>(w.z, magic, c2, v1);
                        unpack_word_pairs<BF16>(w.w, magic, c2, v1 + 4);
                        tmem_st8(tl + b * ACOLS + (2 * t) * 8, v0);
                        tmem_st8(tl + b * ACOLS + (2 * t + 1) * 8, v1);
                    }
                    tmem_wait_st();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&a_full[b]);
                    if (gq == GPC - 1) mbar_arrive(&empty[s]);  // weights and scales consumed
                }
                // this group ends a segment at the tile's last group or the range's last
                const bool seg_end = gq == GPC - 1 && (cur_chunk == nchunks - 1 || c == nit - 1);
                const Pend cur{sc, seg_end,
                               seg_end && (c - seg_start) == cur_chunk && cur_chunk == nchunks - 1,
                               seg_start == 0, cur_tile};
                if (seg_end) seg_start = c + 1;
                if constexpr (LAG == 2) {
                    if (i >= 2) rescale(i - 2, p0);
                    p0 = p1;
                    p1 = cur;
                } else {
                    if (i >= 1) rescale(i - 1, p0);
                    p0 = cur;
                }
            }
            if (++cur_chunk == nchunks) {
                cur_chunk = 0;
                ++cur_tile;
            }
            if (++s == stages) {
                s = 0;
                ph ^= 1u;
            }
        }
        if constexpr (LAG == 2) {
            if (i >= 2) rescale(i - 2, p0);
            if (i >= 1) rescale(i - 1, p1);
        } else {
            if (i >= 1) rescale(i - 1, p0);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tbase, TCOLS);
    }
}

}  // namespace q4dev
