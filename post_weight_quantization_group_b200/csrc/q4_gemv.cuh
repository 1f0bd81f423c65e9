// q4_gemv.cuh -- fused W4A16 decode product for small batches (B <= 8) and
// the bf16 reference product, both as HBM-streaming kernels.
//
//   y[b, r] = sum_j s[r, j] * sum_{k in group j} (q[r, k] - z[r, j]) * x[b, k]
//
// Dataflow (arganzheng.life post-training-quantization-gptq-awq-and-rotation,
// section 二.3: INT4 + scale/zero read from HBM, dequantised on chip, 16-bit
// tensor-core multiply-add; section 二.2: a per-group scale has to be applied
// inside the K accumulation):
//
//  * one producer warp streams [RT rows x 128 B] tiles of the packed weights
//    into a ring of shared-memory stages with TMA (128-byte swizzle), paced by
//    full / empty mbarriers;
//  * consumer warps turn each 32-bit word (8 codes) into exact 16-bit
//    integers with one LOP3 per code pair: code | 0x4300 is the bf16 value
//    128 + code (0x6400: fp16 1024 + code; symmetric codes are XORed with 8
//    in the same LOP3 to make them 0..15).  These raw values are the A
//    operand of m16n8k16 tensor-core MMAs whose B operand is the activation
//    batch (n = 8 columns, B of them live).  The products are exact and the
//    MMA accumulates one group in fp32; the constant offset is removed per
//    group as  sum (c + q') x = c * sum x + sum q' x,  with c = 136 (bf16,
//    symmetric), 128 + z (bf16, asymmetric) or 1024 + 8 / 1024 + z (fp16) and
//    sum x of the group precomputed once per CTA.  The accumulator restarts
//    every group, so the cancellation costs about 6 (bf16) to 9 (fp16) of
//    fp32's 24 bits on one group's partial; the partial is then multiplied
//    by the group's fp32 scale and added to the running fp32 accumulator;
//  * the K dimension is split over the CTAs of a thread-block cluster; each
//    CTA leaves its [RT x B] fp32 partial in shared memory and the cluster
//    reduces them through distributed shared memory, in rank order, so the
//    result is deterministic and no global scratch memory is used.
//
// Codes may be paired with activations in any order inside a group (the sum
// is the same); each thread takes 8 consecutive codes per 32-bit word and the
// activations are stored in shared memory in the matching order, (x0,x4),
// (x1,x5), (x2,x6), (x3,x7) per 8-element block.
#pragma once

#include "q4_device.cuh"

namespace q4dev {

// MMA row group (lane / 4) -> row inside a 16-row tile; the 3-bit reversal
// makes the lanes of one shared-memory phase hit different 16-byte columns of
// the 128-byte-swizzled tiles.
__host__ __device__ constexpr int rho(int g) {
    return ((g & 1) << 2) | (g & 2) | ((g >> 2) & 1);
}

struct GemvGeom {
    int rt;           // rows per CTA
    int stages;       // weight ring depth
    int cps;          // chunks per split
    int b;            // batch
    int gpc;          // groups per chunk
    int glp;          // groups per CTA, padded to a multiple of 8 (16 bytes of fp16)
    bool sym;
    // byte offsets in dynamic shared memory
    size_t off_x, off_s, off_z, off_sx, off_bar, total;
};

// Chunk = 256 codes of a row = 128 bytes.
constexpr int kChunkCodes = 256;
constexpr int kChunkBytes = 128;

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

__host__ __device__ inline GemvGeom gemv_geom(int rt, int stages, int cps, int b, int gs,
                                              bool sym) {
    GemvGeom g{};
    g.rt = rt;
    g.stages = stages;
    g.cps = cps;
    g.b = b;
    g.gpc = kChunkCodes / gs;
    g.glp = static_cast<int>(align_up(static_cast<size_t>(cps) * g.gpc, 8));
    g.sym = sym;
    size_t off = static_cast<size_t>(stages) * rt * kChunkBytes;  // stages, 1024-aligned
    g.off_x = off;
    off += static_cast<size_t>(b) * cps * 512;                     // permuted x
    off = align_up(off, 1024);
    g.off_s = off;                                                 // scales [rt][glp] fp16
    off = align_up(off + static_cast<size_t>(rt) * g.glp * 2, 1024);
    g.off_z = off;                                                 // zeros  [rt][glp] fp16
    if (!sym) off = align_up(off + static_cast<size_t>(rt) * g.glp * 2, 1024);
    g.off_sx = off;                                                // group sums of x [glp][8] fp32
    off += static_cast<size_t>(g.glp) * 8 * 4;
    g.off_bar = off;
    off += static_cast<size_t>(2 * stages + 1) * 8;
    g.total = off + 1024;  // slack to align the base to 1024 bytes
    return g;
}

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

// ---------------------------------------------------------------- INT4 GEMV
// Template parameters:
//   BF16  activations / MMA operands are bf16 (else fp16)
//   GS    group size (32, 64, 128)
//   SYM   symmetric codes (two's complement, z = 0)
//   MT    16-row m-tiles per consumer warp
//   CW    consumer warps; rows per CTA RT = CW * MT * 16
//   STAGES weight ring depth
// grid = (S splits of K, ceil(out / RT)); cluster = (S, 1, 1) when S > 1.
template <bool BF16, int GS, bool SYM, int MT, int CW, int STAGES>
__global__ void __launch_bounds__((CW + 1) * 32)
    q4_gemv_kernel(const __grid_constant__ CUtensorMap tmap_w,
                   const __grid_constant__ CUtensorMap tmap_s,
                   const __grid_constant__ CUtensorMap tmap_z, int meta_tma,
                   const __half* __restrict__ scales, const __half* __restrict__ zeros,
                   const uint16_t* __restrict__ x, int B, int64_t out, int64_t in, int cps,
                   int nchunks, void* __restrict__ y, int ydt, unsigned* __restrict__ status) {
    constexpr int RT = CW * MT * 16;
    constexpr int GPC = kChunkCodes / GS;  // groups per chunk
    constexpr int WPG = GS / 32;           // 32-bit words per thread per row per group
    constexpr int BP = 8;                  // padded batch (one n8 tile)
    constexpr uint32_t kMagic = Magic<BF16>::base2 ^ (SYM ? 0x00080008u : 0u);

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const GemvGeom geo = gemv_geom(RT, STAGES, cps, B, GS, SYM);
    uint8_t* xs = smem + geo.off_x;
    uint16_t* ss16 = reinterpret_cast<uint16_t*>(smem + geo.off_s);
    uint16_t* zs16 = reinterpret_cast<uint16_t*>(smem + geo.off_z);
    float* sxs = reinterpret_cast<float*>(smem + geo.off_sx);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + geo.off_bar);
    uint64_t* empty = full + STAGES;
    uint64_t* meta = empty + STAGES;  // scales / zeros tile landed
    const int GLP = geo.glp;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int split = blockIdx.x;
    const int64_t row0 = static_cast<int64_t>(blockIdx.y) * RT;
    const int c_begin = split * cps;
    const int nch = max(0, min(nchunks, c_begin + cps) - c_begin);
    const int64_t G = in / GS;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], CW);
        }
        mbar_init(meta, 1);
        fence_mbarrier_init_cluster();
    }
    __syncthreads();

    float acc[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[mt][e] = 0.f;

    if (warp == CW) {
        // ------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&tmap_w);
            if (meta_tma && nch > 0) {
                // the CTA's [RT x GLP] scale (and zero) tiles, group index c_begin*GPC
                mbar_arrive_expect_tx(meta, RT * GLP * 2 * (SYM ? 1 : 2));
                tma_load_2d(ss16, &tmap_s, c_begin * GPC, static_cast<int32_t>(row0), meta);
                if constexpr (!SYM)
                    tma_load_2d(zs16, &tmap_z, c_begin * GPC, static_cast<int32_t>(row0), meta);
            }
            bool ok = true;
            for (int c = 0; c < nch && ok; ++c) {
                const int s = c % STAGES;
                const uint32_t it = c / STAGES;
                if (c >= STAGES)
                    ok = mbar_wait_bounded(&empty[s], (it - 1) & 1, status, kWaitLimitNs);
                if (!ok) break;
                mbar_arrive_expect_tx(&full[s], RT * kChunkBytes);
                tma_load_2d(smem + static_cast<size_t>(s) * RT * kChunkBytes, &tmap_w,
                            (c_begin + c) * kChunkBytes, static_cast<int32_t>(row0), &full[s]);
            }
            if (meta_tma && nch > 0) mbar_wait_bounded(meta, 0, status, kWaitLimitNs);
            // drain: the last phase of every stage that was filled must have
            // landed before shared memory is reused or released
            for (int s = 0; s < STAGES && s < nch; ++s) {
                const int last = s + ((nch - 1 - s) / STAGES) * STAGES;
                mbar_wait_bounded(&full[s], (last / STAGES) & 1, status, kWaitLimitNs);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------ consumers
        const int ctid = threadIdx.x;  // 0 .. CW*32-1
        // permuted activations: block p of chunk c for batch n goes to word
        // slot w = G*WPG + i of thread t, where p = G*(GS/8) + t*WPG + i.
        // All loads of a batch are issued before any store.
        const int kbase = c_begin * kChunkCodes;
        const int nitems = B * nch * 32;
        constexpr int XU = 4;
        for (int base = ctid; base < nitems; base += XU * CW * 32) {
            uint4 v[XU];
#pragma unroll
            for (int u = 0; u < XU; ++u) {
                const int idx = base + u * CW * 32;
                v[u] = make_uint4(0, 0, 0, 0);
                if (idx < nitems) {
                    const int p = idx & 31;
                    const int c = (idx >> 5) % nch;
                    const int n = (idx >> 5) / nch;
                    const int64_t k = static_cast<int64_t>(kbase) + c * kChunkCodes + p * 8;
                    if (k < in)
                        v[u] = __ldg(reinterpret_cast<const uint4*>(x + static_cast<int64_t>(n) * in + k));
                }
            }
#pragma unroll
            for (int u = 0; u < XU; ++u) {
                const int idx = base + u * CW * 32;
                if (idx < nitems) {
                    const int p = idx & 31;
                    const int c = (idx >> 5) % nch;
                    const int n = (idx >> 5) / nch;
                    uint4 o;
                    o.x = prmt(v[u].x, v[u].z, 0x5410);  // (x0, x4)
                    o.y = prmt(v[u].x, v[u].z, 0x7632);  // (x1, x5)
                    o.z = prmt(v[u].y, v[u].w, 0x5410);  // (x2, x6)
                    o.w = prmt(v[u].y, v[u].w, 0x7632);  // (x3, x7)
                    const int gq = p / (GS / 8);
                    const int rem = p % (GS / 8);
                    const int t = rem / WPG;
                    const int i = rem % WPG;
                    const int w = gq * WPG + i;
                    *reinterpret_cast<uint4*>(xs + ((static_cast<size_t>(c) * 8 + w) * B + n) * 64 + 16 * t) = o;
                }
            }
        }
        if (!meta_tma) {
            // scales / zeros whose rows are not 16-byte aligned: plain loads into
            // the same [RT][GLP] layout the tensor-map copy produces
            const int GL = nch * GPC;
            const int64_t gbase = static_cast<int64_t>(c_begin) * GPC;
            for (int idx = ctid; idx < RT * GLP; idx += CW * 32) {
                const int gl = idx % GLP;
                const int r = idx / GLP;
                const int64_t grow = row0 + r;
                const int64_t gg = gbase + gl;
                uint16_t sv = 0, zv = 0;
                if (gl < GL && grow < out && gg < G) {
                    sv = __half_as_ushort(scales[grow * G + gg]);
                    if constexpr (!SYM) zv = __half_as_ushort(zeros[grow * G + gg]);
                }
                ss16[idx] = sv;
                if constexpr (!SYM) zs16[idx] = zv;
            }
        }
        named_bar_sync(1, CW * 32);
        // per (group, batch) sums of the activations, in a fixed order
        {
            const int GL = nch * GPC;
            for (int idx = ctid; idx < GLP * 8; idx += CW * 32) {
                const int gl = idx >> 3;
                const int n = idx & 7;
                float sum = 0.f;
                if (n < B && gl < GL) {
                    const int c = gl / GPC;
                    const int gq = gl % GPC;
#pragma unroll
                    for (int i = 0; i < WPG; ++i) {
#pragma unroll
                        for (int t = 0; t < 4; ++t) {
                            const uint4 v = *reinterpret_cast<const uint4*>(
                                xs + ((static_cast<size_t>(c) * 8 + gq * WPG + i) * B + n) * 64 + 16 * t);
                            const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                float lo, hi;
                                if constexpr (BF16) {
                                    lo = __uint_as_float(wv[e] << 16);
                                    hi = __uint_as_float(wv[e] & 0xFFFF0000u);
                                } else {
                                    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&wv[e]));
                                    lo = f.x;
                                    hi = f.y;
                                }
                                sum += lo;
                                sum += hi;
                            }
                        }
                    }
                }
                sxs[idx] = sum;
            }
        }
        named_bar_sync(1, CW * 32);
        if (meta_tma && nch > 0) mbar_wait_bounded(meta, 0, status, kWaitLimitNs);

        const int gid = lane >> 2;
        const int t = lane & 3;
        const int rrow = rho(gid);
        bool ok = true;
        for (int c = 0; c < nch; ++c) {
            const int s = c % STAGES;
            if (!mbar_wait_bounded(&full[s], (c / STAGES) & 1, status, kWaitLimitNs)) {
                ok = false;
                break;
            }
            const uint8_t* stage = smem + static_cast<size_t>(s) * RT * kChunkBytes;
#pragma unroll
            for (int gq = 0; gq < GPC; ++gq) {
                // activation fragments of this group's word slots
                uint32_t xf[WPG][4];
#pragma unroll
                for (int i = 0; i < WPG; ++i) {
                    if (gid < B) {
                        const uint4 v = *reinterpret_cast<const uint4*>(
                            xs + ((static_cast<size_t>(c) * 8 + gq * WPG + i) * B + gid) * 64 + 16 * t);
                        xf[i][0] = v.x;
                        xf[i][1] = v.y;
                        xf[i][2] = v.z;
                        xf[i][3] = v.w;
                    } else {
                        xf[i][0] = xf[i][1] = xf[i][2] = xf[i][3] = 0u;
                    }
                }
                // group sums for this lane's accumulator columns n = 2t, 2t+1
                const float2 sx = *reinterpret_cast<const float2*>(sxs + (c * GPC + gq) * 8 + 2 * t);
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    const int mtile = warp * MT + mt;
                    const int R0 = mtile * 16 + rrow;  // rows R0 and R0 + 8, same swizzle phase
                    // packed words of rows R0, R0+8 for this group
                    const int byte = gq * (GS / 2) + t * (GS / 8);
                    const int piece = byte >> 4;
                    const int within = byte & 15;
                    const int sw = ((piece ^ (R0 & 7)) << 4) | within;
                    uint32_t w0[WPG], w1[WPG];
                    const uint8_t* p0 = stage + R0 * kChunkBytes + sw;
                    const uint8_t* p1 = p0 + 8 * kChunkBytes;
                    if constexpr (WPG == 4) {
                        const uint4 a = *reinterpret_cast<const uint4*>(p0);
                        const uint4 b = *reinterpret_cast<const uint4*>(p1);
                        w0[0] = a.x; w0[1] = a.y; w0[2] = a.z; w0[3] = a.w;
                        w1[0] = b.x; w1[1] = b.y; w1[2] = b.z; w1[3] = b.w;
                    } else if constexpr (WPG == 2) {
                        const uint2 a = *reinterpret_cast<const uint2*>(p0);
                        const uint2 b = *reinterpret_cast<const uint2*>(p1);
                        w0[0] = a.x; w0[1] = a.y;
                        w1[0] = b.x; w1[1] = b.y;
                    } else {
                        w0[0] = *reinterpret_cast<const uint32_t*>(p0);
                        w1[0] = *reinterpret_cast<const uint32_t*>(p1);
                    }
                    const int gl = c * GPC + gq;
                    const float2 sc = make_float2(
                        __half2float(__ushort_as_half(ss16[R0 * GLP + gl])),
                        __half2float(__ushort_as_half(ss16[(R0 + 8) * GLP + gl])));
                    // offset of the raw values: base + 8 (symmetric) or base + z
                    float cst0, cst1;
                    if constexpr (SYM) {
                        cst0 = cst1 = Magic<BF16>::base + 8.0f;
                    } else {
                        cst0 = Magic<BF16>::base + __half2float(__ushort_as_half(zs16[R0 * GLP + gl]));
                        cst1 = Magic<BF16>::base + __half2float(__ushort_as_half(zs16[(R0 + 8) * GLP + gl]));
                    }
                    // two independent MMA accumulation chains per group
                    float pa[4] = {0.f, 0.f, 0.f, 0.f};
                    float pb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int i = 0; i < WPG; ++i) {
                        const uint32_t a = w0[i], b = w1[i];
                        // nibbles (0,4), (1,5), (2,6), (3,7) of each word
                        const uint32_t A0[4] = {lop3_and_xor(a, 0x000F000Fu, kMagic),
                                                lop3_and_xor(b, 0x000F000Fu, kMagic),
                                                lop3_and_xor(a >> 4, 0x000F000Fu, kMagic),
                                                lop3_and_xor(b >> 4, 0x000F000Fu, kMagic)};
                        const uint32_t A1[4] = {lop3_and_xor(a >> 8, 0x000F000Fu, kMagic),
                                                lop3_and_xor(b >> 8, 0x000F000Fu, kMagic),
                                                lop3_and_xor(a >> 12, 0x000F000Fu, kMagic),
                                                lop3_and_xor(b >> 12, 0x000F000Fu, kMagic)};
                        mma_16816<BF16>(pa, A0, xf[i][0], xf[i][1]);
                        mma_16816<BF16>(pb, A1, xf[i][2], xf[i][3]);
                    }
                    // sum (c + q') x  ->  sum q' x  (q' = q - z), then scale
                    acc[mt][0] = fmaf(sc.x, fmaf(-cst0, sx.x, pa[0] + pb[0]), acc[mt][0]);
                    acc[mt][1] = fmaf(sc.x, fmaf(-cst0, sx.y, pa[1] + pb[1]), acc[mt][1]);
                    acc[mt][2] = fmaf(sc.y, fmaf(-cst1, sx.x, pa[2] + pb[2]), acc[mt][2]);
                    acc[mt][3] = fmaf(sc.y, fmaf(-cst1, sx.y, pa[3] + pb[3]), acc[mt][3]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
        (void)ok;
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
                    if (col < B && row < out) store_y(y, ydt, static_cast<int64_t>(col) * out + row, acc[mt][e]);
                }
            }
        }
        return;
    }
    // split-K across the cluster: partial tiles through distributed smem
    float* red = reinterpret_cast<float*>(smem);  // reuses the (drained) stage ring
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
    cluster_reduce_store(red, RT, BP, B, row0, out, y, ydt);
    cluster_sync_all();
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
