// q4_gemv_sk.cuh -- persistent stream-K W4A16 decode product for B <= 8.
//
//   y[b, r] = sum_j s[r, j] * sum_{k in group j} (q[r, k] - z[r, j]) * x[b, k]
//
// Work decomposition.  The product is T = row_tiles x chunks iterations (a
// row tile is RT = 16 * CW rows, a chunk 256 codes of K).  A persistent grid
// of P CTAs (two per SM) gives CTA p the contiguous range
// [T p / P, T (p+1) / P) in tile-major order, so every CTA streams the same
// number of bytes whatever the shape.  A range covers whole row tiles and at
// most two partial ones.  A partial tile's fp32 partial goes to a workspace
// slot; the CTA that arrives last on the tile's counter adds all partials of
// the tile in CTA order -- the result does not depend on timing -- writes y
// and resets the counter, so the counters are zero again for the next call.
// No CTA ever waits for another.
//
// The host picks P per shape; the same split then yields two special plans.
//  * Cluster fix-up (template flag CLUSTER): P = row_tiles x S, launched in
//    clusters of S <= 8.  CTA p holds K part p % S of row tile p / S, so the
//    S CTAs of a tile are one cluster.  Each keeps its partial tile in shared
//    memory, and after a cluster barrier rank r adds rows
//    [RT r / S, RT (r+1) / S) of the S partials in rank order through
//    distributed shared memory.  No workspace, counter or atomic.  Every
//    thread of every CTA passes both cluster barriers.
//  * Whole-tile grid: P = row_tiles, every range one whole tile, y stored
//    directly (the stream-K instance; its fix-up path is never reached).
//
// Launch overlap: the kernel lets the next kernel of the stream launch as
// soon as it has started (programmatic dependent launch), and itself issues
// the loads of its first stages of weights and scales -- which no preceding
// kernel of this library writes -- before waiting for the preceding kernel;
// activations, outputs and the workspace are touched only after that wait.
//
// Warp roles inside a CTA:
//  * CW consumer warps, one 16-row MMA tile each;
//  * a producer warp: one thread issues, per iteration, TMA loads of the
//    weight tile [RT rows x 128 B] (128-byte swizzle), the activation chunk
//    [B rows x 256 values] and the aligned window of 8 groups of scales
//    (and zero points) [RT rows x 8] that holds the chunk's groups, into a
//    ring of `stages` shared-memory stages;
//  * one helper warp (two for B >= 4, taking alternate chunks): per stage it
//    rewrites the activation chunk in MMA fragment order and sums it per
//    group, shared memory to shared memory, so the consumer threads do
//    nothing but unpack, multiply and rescale.
//    (Scale rows that are not 16-byte aligned cannot be copied by TMA; the
//    helper then loads the chunk's scales itself.)
//
// Arithmetic (arganzheng.life post-training-quantization-gptq-awq-and-rotation,
// section 二.3: codes unpacked on chip and multiplied on 16-bit tensor cores;
// section 二.2: per-group scales applied inside the K accumulation): one LOP3
// turns a code pair into the bf16 (fp16) values 128 + q' (1024 + q'), q' =
// q + 8 for two's-complement symmetric codes and q' = q for asymmetric ones;
// m16n8k16 MMAs multiply them exactly with the activations and accumulate one
// group in fp32; the offset is removed per group as
//   sum (c + q') x - c * sum x,   c = 136 | 128 + z (bf16), 1032 | 1024 + z (fp16),
// and the group partial is multiplied by its fp32 scale.  The accumulator
// restarts every group, so the cancellation costs 6 (bf16) to 9 (fp16) of
// fp32's 24 bits of one group's partial.  Codes meet activations out of
// natural order inside a group: each thread takes 8 consecutive codes per
// 32-bit word and pairs nibbles (0,4), (1,5), (2,6), (3,7), and the helper
// stores the activations in the matching order.
#pragma once

#include "q4_device.cuh"
#include "q4_gemv.cuh"

namespace q4dev {

constexpr int kSkMaxStages = 4;

// Up to kSkMaxGroup products that share their activations (one call covers,
// e.g., the q, k and v projections of a layer): their row tiles are
// concatenated into one stream-K iteration space, product i owning the global
// row tiles [tile_beg[i], tile_beg[i + 1]).
constexpr int kSkMaxGroup = 4;
struct SkGroup {
    CUtensorMap w[kSkMaxGroup], s[kSkMaxGroup], z[kSkMaxGroup];
    const uint16_t* scales[kSkMaxGroup];
    const uint16_t* zeros[kSkMaxGroup];
    void* y[kSkMaxGroup];
    int64_t out[kSkMaxGroup];
    int64_t tile_beg[kSkMaxGroup + 1];
    int n;
};

// Product that owns global row tile `tile`.
__device__ __forceinline__ int sk_product(const SkGroup& g, int64_t tile) {
    int i = 0;
#pragma unroll
    for (int k = 1; k < kSkMaxGroup; ++k) i += (k < g.n && tile >= g.tile_beg[k]) ? 1 : 0;
    return i;
}

struct SkGeom {
    size_t w_bytes, off_m, m_bytes;              // weight tiles, per-stage slots
    size_t off_x, off_xp, off_sx, off_sc, off_zc;  // inside a per-stage slot
    size_t off_bar, off_red, total;
};

// All stages' weight tiles [rt x 128 B] first (each 1024-byte aligned for
// the 128-byte swizzle), then per stage: activations [b x 512 B] as loaded,
// rewritten in place by the helper into MMA fragment order [8 slots x 8
// batch x 4 threads x 16 B] | group sums [8 groups x 8 batch] fp32 | scale
// window [rt x 8] fp16 | zero-point window [rt x 8] fp16 (asymmetric only).
__host__ __device__ inline SkGeom sk_geom(int rt, int stages, int b, bool sym, bool cluster) {
    SkGeom g{};
    (void)b;  // the activation area is 8 x 512 B for every b <= 8
    g.w_bytes = static_cast<size_t>(rt) * kChunkBytes;
    g.off_m = g.w_bytes * stages;
    g.off_x = 0;
    g.off_xp = 0;
    g.off_sx = 8 * 8 * 64;
    g.off_sc = g.off_sx + 8 * 8 * 4;
    g.off_zc = g.off_sc + static_cast<size_t>(rt) * 16;
    g.m_bytes = align_up(g.off_zc + (sym ? 0 : static_cast<size_t>(rt) * 16), 128);
    g.off_bar = align_up(g.off_m + g.m_bytes * stages, 8);
    // with the cluster fix-up: the partial tile the cluster reduces through
    // distributed shared memory
    g.off_red = align_up(g.off_bar + static_cast<size_t>(3 * kSkMaxStages) * 8 + 64, 16);
    g.total = g.off_red + (cluster ? static_cast<size_t>(rt) * 8 * 4 : 0) + 1024;
    return g;
}

// The two cluster barriers of the reduction, for warps with no part in it.
__device__ __forceinline__ void cluster_idle(int n) {
    for (int i = 0; i < n; ++i) cluster_sync_all();
}

// CTA that owns iteration i of T split over P CTAs: it_beg(q) = T q / P.
__device__ __forceinline__ int64_t sk_owner(int64_t i, int64_t T, int64_t P) {
    return ((i + 1) * P - 1) / T;
}

__device__ __forceinline__ uint32_t pair_lo(uint32_t a, uint32_t b) { return prmt(a, b, 0x5410); }
__device__ __forceinline__ uint32_t pair_hi(uint32_t a, uint32_t b) { return prmt(a, b, 0x7632); }

__device__ __forceinline__ unsigned atom_add_acq_rel_gpu(unsigned* p, unsigned v) {
    unsigned old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;"
                 : "=r"(old)
                 : "l"(p), "r"(v)
                 : "memory");
    return old;
}

// NH helper warps per CTA: the helper's per-chunk work grows with B, so
// larger batches split the chunks between two helpers (chunk c to helper
// c % 2).  NH is a template parameter so that each variant gets the register
// budget of its own block size.
template <bool BF16, int GS, bool SYM, int CW, int NH, bool CLUSTER>
__global__ void __launch_bounds__((CW + 1 + NH) * 32, 2)
    q4_gemv_sk_kernel(const __grid_constant__ SkGroup grp,
                      const __grid_constant__ CUtensorMap tmap_x, int meta_tma, int stages, int B,
                      int64_t in, int nchunks, int64_t T, int ydt, float* __restrict__ ws_part,
                      unsigned* __restrict__ ws_count, unsigned* __restrict__ status,
                      int cluster_s) {
    constexpr int RT = CW * 16;
    constexpr int GPC = kChunkCodes / GS;  // groups per chunk
    constexpr int WPG = GS / 32;           // 32-bit words per thread per row per group
    constexpr uint32_t kMagic = Magic<BF16>::base2 ^ (SYM ? 0x00080008u : 0u);

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const SkGeom geo = sk_geom(RT, stages, B, SYM, CLUSTER);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + geo.off_bar);
    uint64_t* sxful = full + kSkMaxStages;
    uint64_t* empty = sxful + kSkMaxStages;
    unsigned* last_flag = reinterpret_cast<unsigned*>(empty + kSkMaxStages);

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
            mbar_init(&sxful[s], 1);
            mbar_init(&empty[s], CW);
        }
        fence_mbarrier_init_cluster();
    }
    // fragment-order rows n >= B are never read: consumer threads of batch
    // columns n >= B skip their activation loads
    __syncthreads();
    grid_launch_dependents();

    if (warp == CW) {
        // ------------------------------------------------------ producer
        if (lane == 0 && nit > 0) {
            for (int i = 0; i < grp.n; ++i) prefetch_tmap(&grp.w[i]);
            prefetch_tmap(&tmap_x);
            const uint32_t tx = RT * kChunkBytes + B * 512 +
                                (meta_tma ? RT * 16 * (SYM ? 1 : 2) : 0);
            // weights and scales of the first stages before the dependency wait
            const int pre = nit < stages ? nit : stages;
            {
                int tile = tile0, chunk = chunk0;
                for (int c = 0; c < pre; ++c) {
                    uint8_t* ms = smem + geo.off_m + geo.m_bytes * c;
                    mbar_arrive_expect_tx(&full[c], tx);
                    const int pi = sk_product(grp, tile);
                    const int lt = static_cast<int>(tile - grp.tile_beg[pi]);
                    tma_load_2d(smem + geo.w_bytes * c, &grp.w[pi], chunk * kChunkBytes, lt * RT, &full[c]);
                    if (meta_tma) {
                        const int win = (chunk * GPC) & ~7;
                        tma_load_2d(ms + geo.off_sc, &grp.s[pi], win, lt * RT, &full[c]);
                        if constexpr (!SYM) tma_load_2d(ms + geo.off_zc, &grp.z[pi], win, lt * RT, &full[c]);
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
            for (int c = 0; c < nit && ok; ++c) {
                if (c >= stages) ok = mbar_wait_bounded(&empty[s], ph ^ 1u, status, kWaitLimitNs);
                if (!ok) break;
                uint8_t* ms = smem + geo.off_m + geo.m_bytes * s;
                if (c >= pre) {
                    mbar_arrive_expect_tx(&full[s], tx);
                    const int pi = sk_product(grp, tile);
                    const int lt = static_cast<int>(tile - grp.tile_beg[pi]);
                    tma_load_2d(smem + geo.w_bytes * s, &grp.w[pi], chunk * kChunkBytes, lt * RT, &full[s]);
                    if (meta_tma) {
                        const int win = (chunk * GPC) & ~7;
                        tma_load_2d(ms + geo.off_sc, &grp.s[pi], win, lt * RT, &full[s]);
                        if constexpr (!SYM) tma_load_2d(ms + geo.off_zc, &grp.z[pi], win, lt * RT, &full[s]);
                    }
                }
                tma_load_2d(ms + geo.off_x, &tmap_x, chunk * kChunkCodes, 0, &full[s]);
                if (++chunk == nchunks) {
                    chunk = 0;
                    ++tile;
                }
                if (++s == stages) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            for (int s2 = 0; s2 < stages && s2 < nit; ++s2) {
                const int last = s2 + ((nit - 1 - s2) / stages) * stages;
                mbar_wait_bounded(&full[s2], (last / stages) & 1, status, kWaitLimitNs);
            }
        }
        __syncwarp();
        if constexpr (CLUSTER) cluster_idle(2);
        return;
    }

    if (warp >= CW + 1) {
        // -------------------------------------------------------- helpers
        // helper hw of nh (launched warps beyond the producer) takes the
        // chunks c with c % nh == hw
        // Lane l owns the 8-value block l of each activation row of a chunk
        // (256 = 32 x 8): it stores the block pair-permuted at the fragment
        // slot of the consumer thread that multiplies those codes, and adds
        // its values; GS/8 consecutive lanes form a group, reduced by
        // shuffles in a fixed order.
        const int hgq = lane / (GS / 8);
        const int rem = lane % (GS / 8);
        const int ht = rem / WPG;
        const int hi = rem % WPG;
        // A helper must own fixed ring slots: waiting for phase k of a slot
        // before phase k-1 is known complete would read the parity of phase
        // k-1 as done.  So nh divides the ring depth; otherwise one helper.
        const int hw = warp - (CW + 1);
        const int nh = stages % NH == 0 ? NH : 1;
        if (hw >= nh) {
            if constexpr (CLUSTER) cluster_idle(2);
            return;
        }
        grid_dependency_wait();
        int tile = tile0, chunk = chunk0, s = 0;
        uint32_t ph = 0;
        const uint32_t sbase = smem_u32(smem) + static_cast<uint32_t>(geo.off_m);
        const uint32_t sbytes = static_cast<uint32_t>(geo.m_bytes);
        const uint32_t oX = static_cast<uint32_t>(geo.off_x), oXP = static_cast<uint32_t>(geo.off_xp);
        const uint32_t oSX = static_cast<uint32_t>(geo.off_sx);
        const uint32_t xp_lane = oXP + static_cast<uint32_t>((((hgq * WPG + hi) * 8) * 4 + ht) * 16);
        for (int c = 0; c < nit; ++c) {
            if (c % nh != hw) {  // another helper's chunk
                if (++chunk == nchunks) {
                    chunk = 0;
                    ++tile;
                }
                if (++s == stages) {
                    s = 0;
                    ph ^= 1u;
                }
                continue;
            }
            if (!mbar_wait_bounded(&full[s], ph, status, kWaitLimitNs)) break;
            uint8_t* st = smem + geo.off_m + geo.m_bytes * s;
            const uint32_t sa = sbase + sbytes * static_cast<uint32_t>(s);
            // the fragment order overwrites the activations in place: every
            // lane reads its blocks of all rows before any lane writes
            uint4 qv[8];
#pragma unroll
            for (int n = 0; n < 8; ++n)
                if (n < B) qv[n] = lds128(sa + oX + n * 512 + lane * 16);
            __syncwarp();
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                if (n >= B) break;
                const uint4 q = qv[n];
                uint4 o;
                o.x = pair_lo(q.x, q.z);  // (x0, x4)
                o.y = pair_hi(q.x, q.z);  // (x1, x5)
                o.z = pair_lo(q.y, q.w);  // (x2, x6)
                o.w = pair_hi(q.y, q.w);  // (x3, x7)
                sts128(sa + xp_lane + n * 64, o);
                const uint32_t wv[4] = {q.x, q.y, q.z, q.w};
                float v = 0.f;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    if constexpr (BF16) {
                        v += __uint_as_float(wv[e] << 16);
                        v += __uint_as_float(wv[e] & 0xFFFF0000u);
                    } else {
                        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&wv[e]));
                        v += f.x;
                        v += f.y;
                    }
                }
#pragma unroll
                for (int off = GS / 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
                if (rem == 0) sts32(sa + oSX + (hgq * 8 + n) * 4, __float_as_uint(v));
            }
            // sums of the absent batch rows are zero
            for (int idx = lane; idx < GPC * 8; idx += 32) {
                if ((idx & 7) >= B) sts32(sa + oSX + idx * 4, 0u);
            }
            if (!meta_tma) {
                // scales (and zero points) at their places in the window
                uint16_t* scs = reinterpret_cast<uint16_t*>(st + geo.off_sc);
                uint16_t* zcs = reinterpret_cast<uint16_t*>(st + geo.off_zc);
                const int64_t g0 = static_cast<int64_t>(chunk) * GPC;
                const int wofs = (chunk * GPC) & 7;
                const int pi = sk_product(grp, tile);
                const int64_t out_p = grp.out[pi];
                const uint16_t* scales = grp.scales[pi];
                const uint16_t* zeros = grp.zeros[pi];
                const int64_t row_p = (static_cast<int64_t>(tile) - grp.tile_beg[pi]) * RT;
                for (int idx = lane; idx < RT * GPC; idx += 32) {
                    const int r = idx / GPC;
                    const int gq = idx % GPC;
                    const int64_t row = row_p + r;
                    const bool okg = row < out_p && g0 + gq < G;
                    scs[r * 8 + wofs + gq] = okg ? __ldg(scales + row * G + g0 + gq) : 0;
                    if constexpr (!SYM) zcs[r * 8 + wofs + gq] = okg ? __ldg(zeros + row * G + g0 + gq) : 0;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sxful[s]);
            if (++chunk == nchunks) {
                chunk = 0;
                ++tile;
            }
            if (++s == stages) {
                s = 0;
                ph ^= 1u;
            }
        }
        __syncwarp();
        if constexpr (CLUSTER) cluster_idle(2);
        return;
    }

    // ---------------------------------------------------------- consumers
    const int gid = lane >> 2;
    const int t = lane & 3;
    const int R0 = warp * 16 + rho(gid);  // rows R0 and R0 + 8 of the tile
    // byte offset (swizzled) of this thread's words of group gq inside a row
    int swo[GPC];
#pragma unroll
    for (int gq = 0; gq < GPC; ++gq) {
        const int byte = gq * (GS / 2) + t * (GS / 8);
        swo[gq] = (((byte >> 4) ^ (R0 & 7)) << 4) | (byte & 15);
    }
    // batch columns n >= B are zero: their threads skip the activation loads
    const bool x_live = gid < B;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    int seg_start = 0;  // first iteration (relative) of the current segment
    int cur_tile = tile0, cur_chunk = chunk0, s = 0;
    uint32_t ph = 0;
    grid_dependency_wait();  // y and the workspace are written below

    // 32-bit shared addresses of this thread's loads inside a stage
    const uint32_t wbase = smem_u32(smem);
    const uint32_t wbytes = static_cast<uint32_t>(geo.w_bytes);
    const uint32_t sbase = wbase + static_cast<uint32_t>(geo.off_m);
    const uint32_t sbytes = static_cast<uint32_t>(geo.m_bytes);
    const uint32_t a_xp = static_cast<uint32_t>(geo.off_xp) + (gid * 4 + t) * 16;
    const uint32_t a_sx = static_cast<uint32_t>(geo.off_sx) + 2 * t * 4;
    const uint32_t a_sc0 = static_cast<uint32_t>(geo.off_sc) + R0 * 16;
    const uint32_t a_zc0 = static_cast<uint32_t>(geo.off_zc) + R0 * 16;
    uint32_t a_w[GPC];
#pragma unroll
    for (int gq = 0; gq < GPC; ++gq) a_w[gq] = R0 * kChunkBytes + swo[gq];

    bool ok = true;
    for (int c = 0; c < nit; ++c) {
        // One wait per stage: the helper arrives on sxful only after it has
        // observed the TMA loads of the stage complete (full), so by the
        // release/acquire chain the weights and scales are visible here too;
        // each mbarrier wait costs ~100 cycles even when the phase is done.
        if (ok) ok = mbar_wait_bounded(&sxful[s], ph, status, kWaitLimitNs);
        if (ok) {
            const uint32_t sa = sbase + sbytes * static_cast<uint32_t>(s);
            const uint32_t wofs2 = ((cur_chunk * GPC) & 7) * 2;  // byte offset in the window
#pragma unroll
            for (int gq = 0; gq < GPC; ++gq) {
                uint32_t xf[WPG][4];
#pragma unroll
                for (int i = 0; i < WPG; ++i) {
                    const uint4 v = lds128_if(sa + a_xp + (gq * WPG + i) * 8 * 64, x_live);
                    xf[i][0] = v.x;
                    xf[i][1] = v.y;
                    xf[i][2] = v.z;
                    xf[i][3] = v.w;
                }
                uint32_t w0[WPG], w1[WPG];
                const uint32_t p0 = wbase + wbytes * static_cast<uint32_t>(s) + a_w[gq];
                const uint32_t p1 = p0 + 8 * kChunkBytes;
                if constexpr (WPG == 4) {
                    const uint4 a = lds128(p0);
                    const uint4 b = lds128(p1);
                    w0[0] = a.x; w0[1] = a.y; w0[2] = a.z; w0[3] = a.w;
                    w1[0] = b.x; w1[1] = b.y; w1[2] = b.z; w1[3] = b.w;
                } else if constexpr (WPG == 2) {
                    const uint2 a = lds64(p0);
                    const uint2 b = lds64(p1);
                    w0[0] = a.x; w0[1] = a.y;
                    w1[0] = b.x; w1[1] = b.y;
                } else {
                    w0[0] = lds32(p0);
                    w1[0] = lds32(p1);
                }
                float pa[4] = {0.f, 0.f, 0.f, 0.f};
                float pb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int i = 0; i < WPG; ++i) {
                    const uint32_t a = w0[i], b = w1[i];
                    const uint32_t A0[4] = {lop3_and_xor(a, 0x000F000Fu, kMagic),
                                            lop3_and_xor(b, 0x000F000Fu, kMagic),
                                            lop3_and_xor((a >> 4), 0x000F000Fu, kMagic),
                                            lop3_and_xor((b >> 4), 0x000F000Fu, kMagic)};
                    const uint32_t A1[4] = {lop3_and_xor((a >> 8), 0x000F000Fu, kMagic),
                                            lop3_and_xor((b >> 8), 0x000F000Fu, kMagic),
                                            lop3_and_xor((a >> 12), 0x000F000Fu, kMagic),
                                            lop3_and_xor((b >> 12), 0x000F000Fu, kMagic)};
                    mma_16816<BF16>(pa, A0, xf[i][0], xf[i][1]);
                    mma_16816<BF16>(pb, A1, xf[i][2], xf[i][3]);
                }
                const uint2 sxw = lds64(sa + a_sx + gq * 32);
                const float2 sxv = make_float2(__uint_as_float(sxw.x), __uint_as_float(sxw.y));
                const float s0 = __half2float(__ushort_as_half(lds16(sa + a_sc0 + wofs2 + gq * 2)));
                const float s1 = __half2float(__ushort_as_half(lds16(sa + a_sc0 + 128 + wofs2 + gq * 2)));
                float c0, c1;
                if constexpr (SYM) {
                    c0 = c1 = Magic<BF16>::base + 8.0f;
                } else {
                    c0 = Magic<BF16>::base + __half2float(__ushort_as_half(lds16(sa + a_zc0 + wofs2 + gq * 2)));
                    c1 = Magic<BF16>::base + __half2float(__ushort_as_half(lds16(sa + a_zc0 + 128 + wofs2 + gq * 2)));
                }
                acc[0] = fmaf(s0, fmaf(-c0, sxv.x, pa[0] + pb[0]), acc[0]);
                acc[1] = fmaf(s0, fmaf(-c0, sxv.y, pa[1] + pb[1]), acc[1]);
                acc[2] = fmaf(s1, fmaf(-c1, sxv.x, pa[2] + pb[2]), acc[2]);
                acc[3] = fmaf(s1, fmaf(-c1, sxv.y, pa[3] + pb[3]), acc[3]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);

        // ---------------------------------------------- segment epilogue
        if (cur_chunk == nchunks - 1 || c == nit - 1) {
            const int64_t tile = cur_tile;
            const int pi = sk_product(grp, tile);
            const int64_t out = grp.out[pi];
            void* const y = grp.y[pi];
            const int64_t row0 = (tile - grp.tile_beg[pi]) * RT;
            const bool whole = (c - seg_start) == cur_chunk && cur_chunk == nchunks - 1;
            if (whole) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int col = 2 * t + (e & 1);
                    const int64_t row = row0 + R0 + ((e >> 1) ? 8 : 0);
                    if (col < B && row < out) store_y(y, ydt, static_cast<int64_t>(col) * out + row, acc[e]);
                }
            } else if constexpr (CLUSTER) {
                // the CTA's one segment: its partial tile stays in shared
                // memory for the cluster's reduction after the loop
                float* red = reinterpret_cast<float*>(smem + geo.off_red);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int col = 2 * t + (e & 1);
                    const int row = R0 + ((e >> 1) ? 8 : 0);
                    red[row * 8 + col] = acc[e];
                }
            } else {
                // partial tile: slot 2p (the range's first segment) or 2p + 1
                const int slot = static_cast<int>(2 * p + (seg_start == 0 ? 0 : 1));
                float* part = ws_part + static_cast<size_t>(slot) * RT * 8;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int col = 2 * t + (e & 1);
                    const int row = R0 + ((e >> 1) ? 8 : 0);
                    __stcg(part + row * 8 + col, acc[e]);
                }
                const int64_t q_lo = sk_owner(tile * nchunks, T, P);
                const int64_t q_hi = sk_owner(tile * nchunks + nchunks - 1, T, P);
                // one release-acquire atomic per CTA, after the barrier that
                // orders every consumer's partial stores before it
                named_bar_sync(1, CW * 32);
                if (threadIdx.x == 0) {
                    const unsigned prev = atom_add_acq_rel_gpu(ws_count + tile, 1u);
                    const bool last = prev == static_cast<unsigned>(q_hi - q_lo);
                    *last_flag = last ? 1u : 0u;
                    if (last) ws_count[tile] = 0u;  // zero again for the next call
                }
                named_bar_sync(1, CW * 32);
                if (*last_flag) {
                    float sum[4] = {0.f, 0.f, 0.f, 0.f};
                    // contributors in CTA order; 8 loads issued before their adds
                    for (int64_t q0 = q_lo; q0 <= q_hi; q0 += 8) {
                        float v[8][4];
#pragma unroll
                        for (int u = 0; u < 8; ++u) {
                            const int64_t q = q0 + u;
                            const bool live = q <= q_hi;
                            const bool first_seg = (T * q) / P >= tile * nchunks;
                            const int qs = static_cast<int>(2 * q + (first_seg ? 0 : 1));
                            const float* pq = ws_part + static_cast<size_t>(live ? qs : 0) * RT * 8;
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int col = 2 * t + (e & 1);
                                const int row = R0 + ((e >> 1) ? 8 : 0);
                                v[u][e] = live ? __ldcg(pq + row * 8 + col) : 0.f;
                            }
                        }
#pragma unroll
                        for (int u = 0; u < 8; ++u)
#pragma unroll
                            for (int e = 0; e < 4; ++e) sum[e] += v[u][e];
                    }
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int col = 2 * t + (e & 1);
                        const int64_t row = row0 + R0 + ((e >> 1) ? 8 : 0);
                        if (col < B && row < out) store_y(y, ydt, static_cast<int64_t>(col) * out + row, sum[e]);
                    }
                }
                named_bar_sync(1, CW * 32);
            }
            acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
            seg_start = c + 1;
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
    if constexpr (CLUSTER) {
        // The S CTAs of a cluster share one row tile (rank r holds K range r
        // of S): rank r adds rows [RT r / S, RT (r+1) / S) of the S partial
        // tiles in rank order through distributed shared memory and writes y.
        __syncwarp();
        cluster_sync_all();  // every rank's partial tile is in its shared memory
        const int S = cluster_s;
        const int r = static_cast<int>(cluster_ctarank());
        const int pi = sk_product(grp, tile0);
        const int64_t out = grp.out[pi];
        void* const y = grp.y[pi];
        const int64_t row0 = (static_cast<int64_t>(tile0) - grp.tile_beg[pi]) * RT;
        const uint32_t red = smem_u32(smem + geo.off_red);
        const int v_end = (RT * (r + 1) / S) * 8;
        for (int v = (RT * r / S) * 8 + static_cast<int>(threadIdx.x); v < v_end; v += CW * 32) {
            const int row = v >> 3, col = v & 7;
            // all S remote loads in flight at once, then the sum in rank order
            float part[8];
#pragma unroll
            for (int q = 0; q < 8; ++q)
                part[q] = q < S ? ld_shared_cluster_f32(mapa_shared(red + static_cast<uint32_t>(v) * 4,
                                                                    static_cast<uint32_t>(q)))
                                : 0.f;
            float sum = 0.f;
#pragma unroll
            for (int q = 0; q < 8; ++q)
                if (q < S) sum += part[q];
            if (col < B && row0 + row < out)
                store_y(y, ydt, static_cast<int64_t>(col) * out + row0 + row, sum);
        }
        __syncwarp();
        cluster_sync_all();  // no rank leaves while another still reads it
    }
}

}  // namespace q4dev
