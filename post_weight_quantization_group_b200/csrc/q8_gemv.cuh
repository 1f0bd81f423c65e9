// q8_gemv.cuh -- persistent stream-K W8A16 decode product for B <= 8 with
// per-output-channel INT8 weights ("量化：PTQ、GPTQ、AWQ 与 SmoothQuant"
// (charles2530.github.io) section 13, per_channel_int8_quant: one scale per
// row, w_hat = q * s):
//
//   y[b, r] = s[r] * sum_k q[r, k] * x[b, k]
//
// Work decomposition, launch overlap and the deterministic stream-K fix-up
// follow the W4A16 kernel of q4_gemv_sk.cuh: T = row_tiles x chunks
// iterations, a row tile RT = 16 * CW rows and a chunk 128 codes of K (128
// bytes of every row, the same bytes per iteration as the 4-bit kernel); CTA
// p of P takes the contiguous range [T p / P, T (p+1) / P); a partial tile's
// fp32 partial goes to a workspace slot and the CTA that arrives last on the
// tile's counter adds the partials in CTA order, writes y and re-zeroes the
// counter.  The weight loads of the first stages are issued before the wait
// for the preceding kernel (griddepcontrol); activations, scales, outputs and
// the workspace only after it.
//
// Warp roles: CW consumer warps, one 16-row MMA tile each, and a producer
// warp whose elected thread issues per chunk the TMA loads of the weight tile
// [RT rows x 128 B] and of the activations [B rows x 128 values] as two
// boxes of 64 values, all with the 128-byte swizzle, into a ring of `stages`
// shared-memory stages.  There is no helper warp: the activations are read
// in their natural order, and the swizzle makes those reads conflict-free.
//
// Arithmetic.  Consumer thread (gid, t) owns rows R0 and R0 + 8 of its warp's
// tile and, of every row, the 16-byte units t and t + 4 of the chunk (codes
// 16t .. 16t+15 and 64+16t .. 64+16t+15).  Each 4-code word feeds one
// m16n8k16 MMA: codes (c0, c1) at logical k (2t, 2t+1) and (c2, c3) at
// (2t+8, 2t+9), against the activations of the same four K positions, which
// are two consecutive 32-bit words of the thread's activation unit.  A code
// byte b (two's complement q) becomes an exact 16-bit float:
//   bf16: a PRMT puts b under the exponent byte 0x43; then
//         (0x43 | b & 0x7F) - (0x43 | b & 0x80) = (128 + low7) - (128 or 256)
//         = low7 - 128 * bit7 = q;
//   fp16: a PRMT puts b under 0x64, XOR 0x80 gives 1024 + (q + 128), and
//         subtracting 1152 gives q.
// Both subtractions are exact.  The MMAs accumulate in fp32 over a segment's
// whole K range (two chains, one per 64-code half of the chunk) and the row
// scale multiplies the sum once, in the epilogue.
#pragma once

#include "q4_device.cuh"
#include "q4_gemv.cuh"
#include "q4_gemv_sk.cuh"

namespace q4dev {

constexpr int kQ8ChunkCodes = 128;  // codes (= bytes) of a weight row per chunk
constexpr int kQ8MaxStages = 6;
constexpr int kQ8XBoxBytes = 1024;  // one activation box: up to 8 rows x 128 B

struct Q8Geom {
    size_t w_bytes, stage_bytes, off_bar, total;
};

// Stage s: weight tile [rt x 128 B] | activation box 0 | activation box 1,
// every part 1024-byte aligned (rt a multiple of 8); then the barriers.
__host__ __device__ inline Q8Geom q8_geom(int rt, int stages) {
    Q8Geom g{};
    g.w_bytes = static_cast<size_t>(rt) * kChunkBytes;
    g.stage_bytes = g.w_bytes + 2 * kQ8XBoxBytes;
    g.off_bar = g.stage_bytes * stages;
    g.total = g.off_bar + static_cast<size_t>(2 * kQ8MaxStages) * 8 + 64 + 1024;
    return g;
}

// Two codes of a word (bytes selected by `sel`: 0x4140 for bytes 0, 1 and
// 0x4342 for bytes 2, 3) as a pair of exact 16-bit floats.
template <bool BF16>
__device__ __forceinline__ uint32_t q8_pair(uint32_t w, uint32_t sel) {
    if constexpr (BF16) {
        const uint32_t p = prmt(w, 0x43u, sel);  // 0x43 b' 0x43 b
        return sub2<true>(p & 0xFF7FFF7Fu, p & 0xFF80FF80u);
    } else {
        const uint32_t p = prmt(w, 0x64u, sel) ^ 0x00800080u;
        return sub2<false>(p, 0x64806480u);
    }
}

// Four MMAs of one 16-byte unit per row: wa, wb the units of rows R0 and
// R0 + 8, xa, xb the activation units of its codes 0-7 and 8-15.
template <bool BF16>
__device__ __forceinline__ void q8_unit_mma(float (&acc)[4], const uint4& wa, const uint4& wb,
                                            const uint4& xa, const uint4& xb) {
    const uint32_t A[4] = {wa.x, wa.y, wa.z, wa.w};
    const uint32_t Bw[4] = {wb.x, wb.y, wb.z, wb.w};
    const uint32_t X[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t a[4] = {q8_pair<BF16>(A[i], 0x4140u), q8_pair<BF16>(Bw[i], 0x4140u),
                               q8_pair<BF16>(A[i], 0x4342u), q8_pair<BF16>(Bw[i], 0x4342u)};
        mma_16816<BF16>(acc, a, X[2 * i], X[2 * i + 1]);
    }
}

template <bool BF16, int CW>
__global__ void __launch_bounds__((CW + 1) * 32, 2)
    q8_gemv_sk_kernel(const __grid_constant__ CUtensorMap tmap_w,
                      const __grid_constant__ CUtensorMap tmap_x,
                      const float* __restrict__ scales, int stages, int B, int64_t out,
                      int64_t in, int nchunks, int64_t T, void* __restrict__ y, int ydt,
                      float* __restrict__ ws_part, unsigned* __restrict__ ws_count,
                      unsigned* __restrict__ status) {
    constexpr int RT = CW * 16;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const Q8Geom geo = q8_geom(RT, stages);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + geo.off_bar);
    uint64_t* empty = full + kQ8MaxStages;
    unsigned* last_flag = reinterpret_cast<unsigned*>(empty + kQ8MaxStages);

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
            mbar_init(&empty[s], CW);
        }
        fence_mbarrier_init_cluster();
    }
    __syncthreads();
    grid_launch_dependents();

    if (warp == CW) {
        // ------------------------------------------------------ producer
        if (lane == 0 && nit > 0) {
            prefetch_tmap(&tmap_w);
            prefetch_tmap(&tmap_x);
            // the second activation box of a chunk exists only where the
            // chunk reaches past 64 codes; a box wholly beyond `in` is not loaded
            auto tx_of = [&](int chunk) -> uint32_t {
                const bool hi = static_cast<int64_t>(chunk) * kQ8ChunkCodes + 64 < in;
                return static_cast<uint32_t>(RT * kChunkBytes + (hi ? 2 : 1) * B * 128);
            };
            const int pre = nit < stages ? nit : stages;
            {
                int tile = tile0, chunk = chunk0;
                for (int c = 0; c < pre; ++c) {
                    mbar_arrive_expect_tx(&full[c], tx_of(chunk));
                    tma_load_2d(smem + geo.stage_bytes * c, &tmap_w, chunk * kChunkBytes, tile * RT,
                                &full[c]);
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
                uint8_t* st = smem + geo.stage_bytes * s;
                if (c >= pre) {
                    mbar_arrive_expect_tx(&full[s], tx_of(chunk));
                    tma_load_2d(st, &tmap_w, chunk * kChunkBytes, tile * RT, &full[s]);
                }
                tma_load_2d(st + geo.w_bytes, &tmap_x, chunk * kQ8ChunkCodes, 0, &full[s]);
                if (static_cast<int64_t>(chunk) * kQ8ChunkCodes + 64 < in)
                    tma_load_2d(st + geo.w_bytes + kQ8XBoxBytes, &tmap_x, chunk * kQ8ChunkCodes + 64,
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
            // the CTA exits only after its last loads have landed
            for (int s2 = 0; s2 < stages && s2 < nit; ++s2) {
                const int last = s2 + ((nit - 1 - s2) / stages) * stages;
                mbar_wait_bounded(&full[s2], (last / stages) & 1, status, kWaitLimitNs);
            }
        }
        __syncwarp();
        return;
    }

    // ---------------------------------------------------------- consumers
    const int gid = lane >> 2;
    const int t = lane & 3;
    const int R0 = warp * 16 + rho(gid);  // rows R0 and R0 + 8 of the tile (same swizzle phase)
    const int sw = R0 & 7;
    const uint32_t a_w0 = static_cast<uint32_t>(R0 * kChunkBytes + ((t ^ sw) << 4));
    const uint32_t a_w1 = static_cast<uint32_t>(R0 * kChunkBytes + (((t + 4) ^ sw) << 4));
    // activation row gid, units 2t and 2t + 1 of a 64-value box
    const uint32_t a_x0 = static_cast<uint32_t>(gid * 128 + (((2 * t) ^ (gid & 7)) << 4));
    const uint32_t a_x1 = static_cast<uint32_t>(gid * 128 + (((2 * t + 1) ^ (gid & 7)) << 4));
    // batch columns n >= B are zero: their threads skip the activation loads
    const bool x_live = gid < B;
    float acc0[4] = {0.f, 0.f, 0.f, 0.f};
    float acc1[4] = {0.f, 0.f, 0.f, 0.f};
    int seg_start = 0;
    int cur_tile = tile0, cur_chunk = chunk0, s = 0;
    uint32_t ph = 0;
    grid_dependency_wait();  // y, the scales and the workspace are read or written below

    const uint32_t sbase = smem_u32(smem);
    const uint32_t sbytes = static_cast<uint32_t>(geo.stage_bytes);
    const uint32_t wbytes = static_cast<uint32_t>(geo.w_bytes);

    bool ok = true;
    for (int c = 0; c < nit; ++c) {
        if (ok) ok = mbar_wait_bounded(&full[s], ph, status, kWaitLimitNs);
        if (ok) {
            const uint32_t st = sbase + sbytes * static_cast<uint32_t>(s);
            const uint32_t xs = st + wbytes;
            const uint4 wa0 = lds128(st + a_w0);
            const uint4 wb0 = lds128(st + a_w0 + 8 * kChunkBytes);
            const uint4 xa0 = lds128_if(xs + a_x0, x_live);
            const uint4 xb0 = lds128_if(xs + a_x1, x_live);
            q8_unit_mma<BF16>(acc0, wa0, wb0, xa0, xb0);
            if (static_cast<int64_t>(cur_chunk) * kQ8ChunkCodes + 64 < in) {
                const uint4 wa1 = lds128(st + a_w1);
                const uint4 wb1 = lds128(st + a_w1 + 8 * kChunkBytes);
                const uint4 xa1 = lds128_if(xs + kQ8XBoxBytes + a_x0, x_live);
                const uint4 xb1 = lds128_if(xs + kQ8XBoxBytes + a_x1, x_live);
                q8_unit_mma<BF16>(acc1, wa1, wb1, xa1, xb1);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);

        // ---------------------------------------------- segment epilogue
        if (cur_chunk == nchunks - 1 || c == nit - 1) {
            float acc[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[e] = acc0[e] + acc1[e];
            const int64_t tile = cur_tile;
            const int64_t row0 = tile * RT;
            const int64_t ra = row0 + R0;
            const int64_t rb = ra + 8;
            const float sa = ra < out ? __ldg(scales + ra) : 0.f;
            const float sb = rb < out ? __ldg(scales + rb) : 0.f;
            const bool whole = (c - seg_start) == cur_chunk && cur_chunk == nchunks - 1;
            if (whole) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int col = 2 * t + (e & 1);
                    const int64_t row = (e >> 1) ? rb : ra;
                    if (col < B && row < out)
                        store_y(y, ydt, static_cast<int64_t>(col) * out + row, acc[e] * ((e >> 1) ? sb : sa));
                }
            } else {
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
                named_bar_sync(1, CW * 32);
                if (threadIdx.x == 0) {
                    const unsigned prev = atom_add_acq_rel_gpu(ws_count + tile, 1u);
                    const bool last = prev == static_cast<unsigned>(q_hi - q_lo);
                    *last_flag = last ? 1u : 0u;
                    if (last) ws_count[tile] = 0u;
                }
                named_bar_sync(1, CW * 32);
                if (*last_flag) {
                    float sum[4] = {0.f, 0.f, 0.f, 0.f};
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
                        const int64_t row = (e >> 1) ? rb : ra;
                        if (col < B && row < out)
                            store_y(y, ydt, static_cast<int64_t>(col) * out + row,
                                    sum[e] * ((e >> 1) ? sb : sa));
                    }
                }
                named_bar_sync(1, CW * 32);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) acc0[e] = acc1[e] = 0.f;
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
}

}  // namespace q4dev
