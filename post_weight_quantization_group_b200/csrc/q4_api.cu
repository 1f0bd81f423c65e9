// q4_api.cu -- the C ABI of include/q4.h: argument validation, launch
// planning, TMA descriptor encoding and kernel launches.  All kernels live in
// this translation unit (q4_quant.cuh, q4_gemv.cuh, q4_gemv_sk.cuh,
// q4_skinny_tc.cuh, q4_skinny_f16.cuh, q8_gemv.cuh, q8_quant.cuh, fp4_quant.cuh, tc_gemm.cuh).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include "q4.h"
#include "q4_device.cuh"
#include "q4_gemv.cuh"
#include "q4_gemv_sk.cuh"
#include "q4_quant.cuh"
#include "q4_skinny_tc.cuh"
#include "q4_skinny_f16.cuh"
#include "q8_gemv.cuh"
#include "q8_quant.cuh"
#include "fp4_quant.cuh"
#include "tc_gemm.cuh"

namespace {

using namespace q4dev;

// Device-side error word (see q4dev::kStatusTimeout); read and cleared by
// q4_sync_status.
__device__ unsigned g_q4_status;

// --------------------------------------------------------------- helpers
constexpr int kMaxDevices = 64;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int current_device() {
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess) return -1;
    return d;
}

int sm_count(int dev) {
    static std::atomic<int> cache[kMaxDevices];
    if (dev < 0 || dev >= kMaxDevices) return 148;
    int v = cache[dev].load(std::memory_order_relaxed);
    if (v > 0) return v;
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        n = 148;
    cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

int max_smem_optin(int dev) {
    static std::atomic<int> cache[kMaxDevices];
    if (dev < 0 || dev >= kMaxDevices) return 227 * 1024;
    int v = cache[dev].load(std::memory_order_relaxed);
    if (v > 0) return v;
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
        n <= 0)
        n = 227 * 1024;
    cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda
// link dependency).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2-D row-major tensor [rows, cols] of `elem` bytes, box [box_rows, box_cols],
// out-of-bounds elements read as zero.
bool make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int elem,
                  uint64_t rows, uint64_t cols, uint32_t box_rows, uint32_t box_cols,
                  CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * static_cast<uint64_t>(elem)};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

q4_status launch_status(cudaError_t e) {
    if (e == cudaSuccess) e = cudaGetLastError();
    return e == cudaSuccess ? Q4_OK : Q4_ERR_CUDA;
}

// Per-(kernel, device) one-time attribute setup.
template <typename K>
bool set_kernel_attrs(K kernel, int smem_bytes, bool nonportable_cluster) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         smem_bytes);
    if (e != cudaSuccess) return false;
    if (nonportable_cluster) {
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return false;
    }
    return true;
}

// Launch with an optional cluster shape and, for kernels written for it,
// programmatic stream serialization (the kernel may start before the previous
// kernel of the stream has finished; it waits with griddepcontrol.wait).
template <typename... KArgs, typename... Args>
q4_status launch_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                    int cluster_x, bool pdl, cudaStream_t stream, Args&&... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    int n = 0;
    if (cluster_x > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = cluster_x;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    if (pdl) {
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    cfg.attrs = n ? attr : nullptr;
    cfg.numAttrs = n;
    return launch_status(cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...));
}

bool valid_dtype(int d) { return d == Q4_F16 || d == Q4_BF16 || d == Q4_F32; }

q4_status validate_weight(const q4_weight* w) {
    if (!w) return Q4_ERR_INVALID_ARG;
    if (w->bits != 4) return Q4_ERR_UNSUPPORTED;
    if (w->out < 0 || w->in <= 0 || w->group_size <= 0) return Q4_ERR_SHAPE;
    if ((w->group_size & 1) || (w->in % w->group_size) != 0) return Q4_ERR_SHAPE;
    if (w->symmetric != 0 && w->symmetric != 1) return Q4_ERR_INVALID_ARG;
    if (w->out > 0 && (!w->qweight || !w->scales)) return Q4_ERR_INVALID_ARG;
    if (w->out > 0 && !w->symmetric && !w->zeros) return Q4_ERR_INVALID_ARG;
    if (w->symmetric && w->zeros) return Q4_ERR_INVALID_ARG;
    if (!aligned(w->scales, 2) || (w->zeros && !aligned(w->zeros, 2))) return Q4_ERR_ALIGNMENT;
    return Q4_OK;
}

// A wait that can never be satisfied, bounded by limit_ns.
__global__ void selftest_wait_kernel(uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbarrier_init_cluster();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait_bounded(&bar, 0, &g_q4_status, limit_ns);
}

// --------------------------------------------------------- quantize_pack
template <bool SYM, bool BF16IN>
q4_status run_quantize(const void* W, int64_t out, int64_t in, int g, uint8_t* qweight,
                       __half* scales, __half* zeros, cudaStream_t st,
                       const int32_t* perm = nullptr) {
    unsigned* status = nullptr;
    if (perm != nullptr &&
        cudaGetSymbolAddress(reinterpret_cast<void**>(&status), g_q4_status) != cudaSuccess)
        return Q4_ERR_CUDA;
    const int dev = current_device();
    const int sms = sm_count(dev);
    const int64_t ngroups = out * (in / g);
    if (ngroups == 0) return Q4_OK;
    const bool fast = (g == 8 || g == 16 || g == 32 || g == 64 || g == 128 || g == 256) &&
                      aligned(qweight, 4);
    if (fast) {
        const int64_t nchunks = out * in / 8;
        const int64_t want = (nchunks + 255) / 256;
        const int blocks = static_cast<int>(want < 8LL * sms ? want : 8LL * sms);
        uint32_t* qw = reinterpret_cast<uint32_t*>(qweight);
        switch (g) {
#define Q4_QCASE(GV)                                                                              \
    case GV:                                                                                      \
        quantize_pack_kernel<GV, SYM, BF16IN><<<blocks, 256, 0, st>>>(W, nchunks, qw, scales, zeros, \
                                                                     perm, in, status);           \
        break;
            Q4_QCASE(8) Q4_QCASE(16) Q4_QCASE(32) Q4_QCASE(64) Q4_QCASE(128) Q4_QCASE(256)
#undef Q4_QCASE
        }
        return launch_status(cudaSuccess);
    }
    const int64_t want = (ngroups * 32 + 255) / 256;
    const int blocks = static_cast<int>(want < 8LL * sms ? want : 8LL * sms);
    quantize_pack_generic_kernel<SYM, BF16IN><<<blocks, 256, 0, st>>>(W, ngroups, g, qweight,
                                                                      scales, zeros, perm, in,
                                                                      status);
    return launch_status(cudaSuccess);
}

template <bool BF16IN>
q4_status run_quantize_clip(const void* W, int64_t out, int64_t in, int g, int n,
                            uint8_t* qweight, __half* scales, cudaStream_t st) {
    const int sms = sm_count(current_device());
    const int64_t nchunks = out * in / 8;
    const int64_t want = (nchunks + 255) / 256;
    const int blocks = static_cast<int>(want < 8LL * sms ? want : 8LL * sms);
    uint32_t* qw = reinterpret_cast<uint32_t*>(qweight);
    switch (g) {
#define Q4_CCASE(GV)                                                                         \
    case GV:                                                                                 \
        quantize_pack_clip_kernel<GV, BF16IN><<<blocks, 256, 0, st>>>(W, nchunks, n, qw, scales); \
        break;
        Q4_CCASE(8) Q4_CCASE(16) Q4_CCASE(32) Q4_CCASE(64) Q4_CCASE(128) Q4_CCASE(256)
#undef Q4_CCASE
        default: return Q4_ERR_UNSUPPORTED;
    }
    return launch_status(cudaSuccess);
}

// ------------------------------------------------------------------ GEMV
// Tile shape of the small-batch kernels (compile-time tunables).
// Small-batch stream-K kernel: CW consumer warps (16 rows each), 2 CTAs/SM.
#ifndef Q4_SK_CW
#define Q4_SK_CW 8
#endif
constexpr int kSkCW = Q4_SK_CW;
static_assert(Q4_GROUP_MAX == kSkMaxGroup, "group size of the ABI and the kernel");
constexpr int kSkRT = kSkCW * 16;
constexpr int kSkCtasPerSm = 2;
constexpr int kSkMinIters = 2;

// Workspace layout, the same for every shape, batch and kernel so that one
// buffer can serve any sequence of calls: [one counter per row tile, at most
// 65535 tiles: kWsCounterBytes] [partial slots of the launch's grid].
// Counters are reset by every call that uses them; partial slots never
// overlap counters.
constexpr size_t kWsCounterBytes = static_cast<size_t>(65536) * 4;

struct SkPlan {
    int64_t row_tiles, T, P;
    int nchunks;
    size_t ws_part_bytes, ws_bytes;
};

// Stream-K plan over row tiles of `rt` rows and chunks of `chunk_codes`
// codes of K: at least `min_iters` iterations per CTA (tiny problems use
// fewer SMs rather than paying a fixup for every chunk), at most `pmax` CTAs;
// each CTA has two partial slots of rt x `cols` fp32.
SkPlan stream_k_plan(int64_t out, int64_t in, int rt, int64_t pmax, int min_iters, int cols,
                     int chunk_codes = kChunkCodes) {
    SkPlan p{};
    p.nchunks = static_cast<int>((in + chunk_codes - 1) / chunk_codes);
    p.row_tiles = (out + rt - 1) / rt;
    p.T = p.row_tiles * p.nchunks;
    p.P = std::min<int64_t>(std::max<int64_t>(1, p.T / min_iters), pmax);
    p.ws_part_bytes = static_cast<size_t>(2 * pmax) * rt * cols * 4;
    p.ws_bytes = kWsCounterBytes + p.ws_part_bytes;
    return p;
}

SkPlan sk_plan(int64_t out, int64_t in, int sms) {
    return stream_k_plan(out, in, kSkRT, static_cast<int64_t>(kSkCtasPerSm) * sms, kSkMinIters, 8);
}

// Cluster fix-up of the B <= 8 kernel.  With P = row_tiles x S the stream-K
// split gives CTA p the K part p % S of row tile p / S, so the S CTAs of a
// tile are one aligned cluster: they add their partial tiles through
// distributed shared memory instead of the workspace, counter and
// last-arriver pass.  Taken with the largest S <= 8 whose clusters the
// device holds all at once, unless its CTAs run more than kSkClusterSlack
// chunks beyond the longest stream-K range; otherwise stream-K.  (Measured:
// a slack of 2 takes the 70B k_proj, 8 tiles x 32 chunks, from 8.8 to 5.6 us
// and the 70B q/k/v group from 18.6 to 17.6 us; 3 would also move the 70B
// down_proj, 28 chunks against 25, which is slower.)
#ifndef Q4_SK_CLUSTER_SLACK
#define Q4_SK_CLUSTER_SLACK 2
#endif
constexpr int kSkClusterSlack = Q4_SK_CLUSTER_SLACK;

// Whole-tile grid of the B <= 8 kernel: when the row tiles alone nearly fill
// the grid (and no cluster plan is taken), one CTA per row tile has no
// partial tile and no fix-up at all.  Stream-K's shorter ranges pay two
// partial-tile epilogues per CTA (partial stores, counter atomic, the last
// arriver's reads), measured at about four chunks' worth of time per CTA; so
// the whole-tile grid is taken when it costs at most kSkWholeTileSlack chunks
// over the longest stream-K range (8B gate/up, 224 tiles x 16 chunks: 18.5
// against 20.2 us; 70B gate, 224 x 32 chunks, 7 more: 35.7 against 33.0).
constexpr int kSkWholeTileSlack = 3;

// Clusters of `s` CTAs of `kernel` resident at once on the current device
// (cached per kernel, cluster size and shared-memory size; 0 if the query
// fails, which leaves the caller on stream-K).
template <typename K>
int max_active_clusters(K kernel, int s, dim3 block, size_t smem) {
    struct Entry {
        const void* k;
        int dev, s;
        size_t smem;
        int n;
    };
    static std::mutex mu;
    static std::vector<Entry> cache;
    const int dev = current_device();
    const void* key = reinterpret_cast<const void*>(kernel);
    std::lock_guard<std::mutex> lock(mu);
    for (const Entry& e : cache)
        if (e.k == key && e.dev == dev && e.s == s && e.smem == smem) return e.n;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(s));
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = s;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) {
        (void)cudaGetLastError();
        n = 0;
    }
    cache.push_back({key, dev, s, smem, n});
    return n;
}

// Skinny-GEMM (tcgen05) kernel: activation tile width NT per batch size.
constexpr int kTcMinIters = 4;
int tc_nt(int64_t B) { return B <= 16 ? 16 : B <= 32 ? 32 : B <= 64 ? 64 : 128; }
int tc_ctas_per_sm(int nt) { return nt <= 32 ? 2 : 1; }

SkPlan tc_plan(int64_t out, int64_t in, int64_t B, int sms) {
    const int nt = tc_nt(B);
    SkPlan p = stream_k_plan(out, in, kTcRT, static_cast<int64_t>(tc_ctas_per_sm(nt)) * sms,
                             kTcMinIters, nt);
    // NT = 128 runs the scaled-fp16 kernel, whose bf16 activations are first
    // converted to fp16 into the workspace, after the partial slots
    if (nt == 128) p.ws_bytes += align_up(static_cast<size_t>(B) * in * 2, 256);
    return p;
}

SkPlan product_plan(int64_t out, int64_t in, int64_t B, int sms) {
    return B <= 8 ? sk_plan(out, in, sms) : tc_plan(out, in, B, sms);
}

// One launch over n products that share x (same in, group size, symmetry):
// their row tiles are concatenated into one stream-K iteration space.
template <bool BF16, int GS, bool SYM>
q4_status run_gemv(const q4_weight* const* wv, int n, const void* x, int64_t B, void* const* ys,
                   int ydt, void* ws, size_t ws_bytes, cudaStream_t st) {
    const int dev = current_device();
    SkGroup grp;
    std::memset(&grp, 0, sizeof(grp));
    grp.n = n;
    int64_t tiles = 0;
    for (int i = 0; i < n; ++i) {
        grp.tile_beg[i] = tiles;
        tiles += (wv[i]->out + kSkRT - 1) / kSkRT;
    }
    grp.tile_beg[n] = tiles;
    if (tiles > 65536) return Q4_ERR_SHAPE;  // one workspace counter per row tile
    const int64_t in = wv[0]->in;
    const SkPlan p = sk_plan(tiles * kSkRT, in, sm_count(dev));
    if (!ws || ws_bytes < p.ws_bytes) return Q4_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return Q4_ERR_ALIGNMENT;
    // Deepest ring that still lets two CTAs share an SM.  From B = 4 on, two
    // helper warps split the activation work; they need an even ring (each
    // owns fixed slots), so the ring is cut to an even depth.
    const int per_sm = 228 * 1024;
    int stages = kSkMaxStages;
    SkGeom geo = sk_geom(kSkRT, stages, static_cast<int>(B), SYM, false);
    while (stages > 2 && kSkCtasPerSm * (geo.total + 1024) > static_cast<size_t>(per_sm)) {
        --stages;
        geo = sk_geom(kSkRT, stages, static_cast<int>(B), SYM, false);
    }
    const bool two_helpers = B >= 4;
    if (two_helpers && (stages & 1)) geo = sk_geom(kSkRT, --stages, static_cast<int>(B), SYM, false);
    // TMA destinations: weight tiles 1024-byte aligned (128-byte swizzle),
    // the activation chunk and the scale / zero-point windows 128-byte aligned
    if (geo.w_bytes % 1024 || geo.off_m % 1024 || geo.m_bytes % 128 || geo.off_x % 128 ||
        geo.off_sc % 128 || geo.off_zc % 128)
        return Q4_ERR_CUDA;
    const int helpers = two_helpers ? 2 : 1;
    const dim3 block((kSkCW + 1 + helpers) * 32);
    auto kernel = two_helpers ? q4_gemv_sk_kernel<BF16, GS, SYM, kSkCW, 2, false>
                              : q4_gemv_sk_kernel<BF16, GS, SYM, kSkCW, 1, false>;
    // the cluster fix-up, when its clusters fit (see kSkClusterSlack), else
    // the whole-tile grid when it fits (see kSkWholeTileSlack), else stream-K
    const int64_t pmax = static_cast<int64_t>(kSkCtasPerSm) * sm_count(dev);
    const int64_t sk_iters = (p.T + p.P - 1) / p.P;
    int cluster_s = 1;
    {
        const SkGeom gcl = sk_geom(kSkRT, stages, static_cast<int>(B), SYM, true);
        auto kcl = two_helpers ? q4_gemv_sk_kernel<BF16, GS, SYM, kSkCW, 2, true>
                               : q4_gemv_sk_kernel<BF16, GS, SYM, kSkCW, 1, true>;
        const bool fits = kSkCtasPerSm * (gcl.total + 1024) <= static_cast<size_t>(per_sm);
        for (int S = 8; fits && S >= 2 && cluster_s == 1; --S) {
            if (S > p.nchunks || p.row_tiles * S > pmax) continue;
            if ((p.nchunks + S - 1) / S > sk_iters + kSkClusterSlack) break;
            if (!set_kernel_attrs(kcl, static_cast<int>(gcl.total), false)) return Q4_ERR_CUDA;
            if (max_active_clusters(kcl, S, block, gcl.total) >= p.row_tiles) {
                cluster_s = S;
                kernel = kcl;
                geo = gcl;
            }
        }
    }
    int64_t grid = p.P;
    if (cluster_s > 1)
        grid = p.row_tiles * cluster_s;
    else if (p.row_tiles <= pmax && p.nchunks <= sk_iters + kSkWholeTileSlack)
        grid = p.row_tiles;  // T p / P = p nchunks: CTA p owns row tile p whole
    const int64_t G = in / GS;
    // scale / zero windows by TMA when every product's rows are 16-byte aligned
    bool meta_tma = (G % 8) == 0;
    for (int i = 0; i < n; ++i)
        meta_tma = meta_tma && aligned(wv[i]->scales, 16) && (SYM || aligned(wv[i]->zeros, 16));
    for (int i = 0; i < n; ++i) {
        const q4_weight* w = wv[i];
        grp.scales[i] = reinterpret_cast<const uint16_t*>(w->scales);
        grp.zeros[i] = reinterpret_cast<const uint16_t*>(w->zeros);
        grp.y[i] = ys[i];
        grp.out[i] = w->out;
        if (!make_tmap_2d(&grp.w[i], w->qweight, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1,
                          static_cast<uint64_t>(w->out), static_cast<uint64_t>(in / 2), kSkRT,
                          kChunkBytes))
            return Q4_ERR_CUDA;
        if (meta_tma) {
            if (!make_tmap_2d(&grp.s[i], w->scales, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                              static_cast<uint64_t>(w->out), static_cast<uint64_t>(G), kSkRT, 8,
                              CU_TENSOR_MAP_SWIZZLE_NONE))
                return Q4_ERR_CUDA;
            if (!SYM && !make_tmap_2d(&grp.z[i], w->zeros, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                                      static_cast<uint64_t>(w->out), static_cast<uint64_t>(G),
                                      kSkRT, 8, CU_TENSOR_MAP_SWIZZLE_NONE))
                return Q4_ERR_CUDA;
        }
    }
    CUtensorMap tmap_x;
    if (!make_tmap_2d(&tmap_x, x,
                      BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                      static_cast<uint64_t>(B), static_cast<uint64_t>(in),
                      static_cast<uint32_t>(B), kChunkCodes, CU_TENSOR_MAP_SWIZZLE_NONE))
        return Q4_ERR_CUDA;
    if (!set_kernel_attrs(kernel, static_cast<int>(geo.total), false)) return Q4_ERR_CUDA;
    unsigned* status = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&status), g_q4_status) != cudaSuccess)
        return Q4_ERR_CUDA;
    unsigned* ws_count = reinterpret_cast<unsigned*>(ws);
    float* ws_part = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) + kWsCounterBytes);
    return launch_ex(kernel, dim3(static_cast<unsigned>(grid)), block, geo.total, cluster_s, true,
                     st, grp, tmap_x, meta_tma ? 1 : 0, stages, static_cast<int>(B), in,
                     p.nchunks, p.T, ydt, ws_part, ws_count, status, cluster_s);
}

template <bool BF16>
q4_status dispatch_gemv(const q4_weight* const* wv, int n, const void* x, int64_t B,
                        void* const* ys, int ydt, void* ws, size_t wsb, cudaStream_t st) {
    const bool sym = wv[0]->symmetric != 0;
    switch (wv[0]->group_size) {
        case 32: return sym ? run_gemv<BF16, 32, true>(wv, n, x, B, ys, ydt, ws, wsb, st)
                            : run_gemv<BF16, 32, false>(wv, n, x, B, ys, ydt, ws, wsb, st);
        case 64: return sym ? run_gemv<BF16, 64, true>(wv, n, x, B, ys, ydt, ws, wsb, st)
                            : run_gemv<BF16, 64, false>(wv, n, x, B, ys, ydt, ws, wsb, st);
        case 128: return sym ? run_gemv<BF16, 128, true>(wv, n, x, B, ys, ydt, ws, wsb, st)
                             : run_gemv<BF16, 128, false>(wv, n, x, B, ys, ydt, ws, wsb, st);
        default: return Q4_ERR_UNSUPPORTED;
    }
}

template <bool BF16>
q4_status dispatch_gemv(const q4_weight* w, const void* x, int64_t B, void* y, int ydt, void* ws,
                        size_t wsb, cudaStream_t st) {
    const q4_weight* wv[1] = {w};
    void* ys[1] = {y};
    return dispatch_gemv<BF16>(wv, 1, x, B, ys, ydt, ws, wsb, st);
}

// ------------------------------------------- W8A16 (per-channel INT8)
constexpr int kQ8CW = 8;
constexpr int kQ8RT = kQ8CW * 16;

SkPlan q8_plan(int64_t out, int64_t in, int sms) {
    return stream_k_plan(out, in, kQ8RT, static_cast<int64_t>(kSkCtasPerSm) * sms, kSkMinIters, 8,
                         kQ8ChunkCodes);
}

template <bool BF16>
q4_status run_q8_gemv(const int8_t* qweight, const float* scales, int64_t out, int64_t in,
                      const void* x, int64_t B, void* y, int ydt, void* ws, size_t ws_bytes,
                      cudaStream_t st) {
    const int dev = current_device();
    const SkPlan p = q8_plan(out, in, sm_count(dev));
    if (!ws || ws_bytes < p.ws_bytes) return Q4_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return Q4_ERR_ALIGNMENT;
    // deepest ring that still lets two CTAs share an SM
    const size_t per_sm = 228 * 1024;
    int stages = kQ8MaxStages;
    Q8Geom geo = q8_geom(kQ8RT, stages);
    while (stages > 2 && kSkCtasPerSm * (geo.total + 1024) > per_sm) geo = q8_geom(kQ8RT, --stages);
    CUtensorMap tmap_w, tmap_x;
    if (!make_tmap_2d(&tmap_w, qweight, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1,
                      static_cast<uint64_t>(out), static_cast<uint64_t>(in), kQ8RT, kChunkBytes))
        return Q4_ERR_CUDA;
    if (!make_tmap_2d(&tmap_x, x,
                      BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                      static_cast<uint64_t>(B), static_cast<uint64_t>(in),
                      static_cast<uint32_t>(B), 64))
        return Q4_ERR_CUDA;
    auto kernel = q8_gemv_sk_kernel<BF16, kQ8CW>;
    if (!set_kernel_attrs(kernel, static_cast<int>(geo.total), false)) return Q4_ERR_CUDA;
    unsigned* status = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&status), g_q4_status) != cudaSuccess)
        return Q4_ERR_CUDA;
    unsigned* ws_count = reinterpret_cast<unsigned*>(ws);
    float* ws_part = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) + kWsCounterBytes);
    return launch_ex(kernel, dim3(static_cast<unsigned>(p.P)), dim3((kQ8CW + 1) * 32), geo.total,
                     1, true, st, tmap_w, tmap_x, scales, stages, static_cast<int>(B), out, in,
                     p.nchunks, p.T, y, ydt, ws_part, ws_count, status);
}

template <bool BF16, int GS, int NT>
q4_status run_skinny(const q4_weight* w, const void* x, int64_t B, void* y, int ydt, void* ws,
                     size_t ws_bytes, cudaStream_t st) {
    const int dev = current_device();
    const SkPlan p = tc_plan(w->out, w->in, B, sm_count(dev));
    if (!ws || ws_bytes < p.ws_bytes) return Q4_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return Q4_ERR_ALIGNMENT;
    const bool sym = w->symmetric != 0;
    constexpr int cps = TcCfg<NT>::ctas_per_sm;
    const size_t per_sm = 228 * 1024;
    const size_t smax = static_cast<size_t>(max_smem_optin(dev));
    // deepest ring with `cps` CTAs per SM
    int stages = kTcMaxStages;
    TcGeom geo = tc_geom(NT, stages, sym);
    while (stages > 2 && (cps * (geo.total + 1024) > per_sm || geo.total > smax)) {
        --stages;
        geo = tc_geom(NT, stages, sym);
    }
    if (cps * (geo.total + 1024) > per_sm || geo.total > smax) return Q4_ERR_UNSUPPORTED;
    const int64_t G = w->in / GS;
    const bool meta_tma = (G % 8) == 0 && aligned(w->scales, 16) && (sym || aligned(w->zeros, 16));
    CUtensorMap tmap_w, tmap_x, tmap_s, tmap_z;
    std::memset(&tmap_s, 0, sizeof(tmap_s));
    std::memset(&tmap_z, 0, sizeof(tmap_z));
    if (!make_tmap_2d(&tmap_w, w->qweight, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1,
                      static_cast<uint64_t>(w->out), static_cast<uint64_t>(w->in / 2), kTcRT,
                      kChunkBytes))
        return Q4_ERR_CUDA;
    // activations: NT-row boxes of 64 values, rows >= B read as zeros
    if (!make_tmap_2d(&tmap_x, x,
                      BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                      static_cast<uint64_t>(B), static_cast<uint64_t>(w->in), NT, 64,
                      CU_TENSOR_MAP_SWIZZLE_128B))
        return Q4_ERR_CUDA;
    if (meta_tma) {
        if (!make_tmap_2d(&tmap_s, w->scales, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                          static_cast<uint64_t>(w->out), static_cast<uint64_t>(G), kTcRT, 8,
                          CU_TENSOR_MAP_SWIZZLE_NONE))
            return Q4_ERR_CUDA;
        if (!sym && !make_tmap_2d(&tmap_z, w->zeros, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                                  static_cast<uint64_t>(w->out), static_cast<uint64_t>(G), kTcRT,
                                  8, CU_TENSOR_MAP_SWIZZLE_NONE))
            return Q4_ERR_CUDA;
    }
    auto kernel = q4_skinny_tc_kernel<BF16, GS, NT>;
    if (!set_kernel_attrs(kernel, static_cast<int>(geo.total), false)) return Q4_ERR_CUDA;
    unsigned* status = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&status), g_q4_status) != cudaSuccess)
        return Q4_ERR_CUDA;
    unsigned* ws_count = reinterpret_cast<unsigned*>(ws);
    float* ws_part = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) + kWsCounterBytes);
    return launch_ex(kernel, dim3(static_cast<unsigned>(p.P)), dim3(TcCfg<NT>::threads), geo.total,
                     1, true,
                     st, tmap_w, tmap_x, tmap_s, tmap_z, meta_tma ? 1 : 0,
                     reinterpret_cast<const uint16_t*>(w->scales),
                     reinterpret_cast<const uint16_t*>(w->zeros), sym ? 1 : 0, stages,
                     static_cast<int>(B), w->out, w->in, p.nchunks, p.T, y, ydt, ws_part, ws_count,
                     status);
}

// The scaled-fp16 tcgen05 kernel (q4_skinny_f16.cuh) for NT = 128; bf16
// activations are converted to fp16 first, into the workspace.
template <bool BF16, int GS, int NT>
q4_status run_skinny_f16(const q4_weight* w, const void* x, int64_t B, void* y, int ydt, void* ws,
                         size_t ws_bytes, cudaStream_t st) {
    const int dev = current_device();
    const SkPlan p = tc_plan(w->out, w->in, B, sm_count(dev));
    if (!ws || ws_bytes < p.ws_bytes) return Q4_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return Q4_ERR_ALIGNMENT;
    const bool sym = w->symmetric != 0;
    constexpr int cps = F16Cfg<NT>::ctas_per_sm;
    const size_t per_sm = 228 * 1024;
    const size_t smax = static_cast<size_t>(max_smem_optin(dev));
    int stages = kTcMaxStages;
    TcGeom geo = tc_geom(NT, stages, sym);
    while (stages > 2 && (cps * (geo.total + 1024) > per_sm || geo.total > smax)) {
        --stages;
        geo = tc_geom(NT, stages, sym);
    }
    if (cps * (geo.total + 1024) > per_sm || geo.total > smax) return Q4_ERR_UNSUPPORTED;
    const int64_t G = w->in / GS;
    const bool meta_tma = (G % 8) == 0 && aligned(w->scales, 16) && (sym || aligned(w->zeros, 16));
    CUtensorMap tmap_w, tmap_x, tmap_s, tmap_z;
    std::memset(&tmap_s, 0, sizeof(tmap_s));
    std::memset(&tmap_z, 0, sizeof(tmap_z));
    if (!make_tmap_2d(&tmap_w, w->qweight, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1,
                      static_cast<uint64_t>(w->out), static_cast<uint64_t>(w->in / 2), kTcRT,
                      kChunkBytes))
        return Q4_ERR_CUDA;
    unsigned* status = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&status), g_q4_status) != cudaSuccess)
        return Q4_ERR_CUDA;
    const void* xf = x;
    if (BF16) {
        void* xw = reinterpret_cast<uint8_t*>(ws) + kWsCounterBytes + p.ws_part_bytes;
        const int64_t n8 = B * w->in / 8;
        const int blocks = static_cast<int>(std::min<int64_t>((n8 + 255) / 256, 4LL * sm_count(dev)));
        const q4_status s0 = launch_ex(x_to_f16_kernel, dim3(static_cast<unsigned>(blocks)),
                                       dim3(256), 0, 1, true, st,
                                       reinterpret_cast<const uint4*>(x), n8,
                                       reinterpret_cast<uint4*>(xw), status);
        if (s0 != Q4_OK) return s0;
        xf = xw;
    }
    if (!make_tmap_2d(&tmap_x, xf, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, static_cast<uint64_t>(B),
                      static_cast<uint64_t>(w->in), NT, 64, CU_TENSOR_MAP_SWIZZLE_128B))
        return Q4_ERR_CUDA;
    if (meta_tma) {
        if (!make_tmap_2d(&tmap_s, w->scales, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                          static_cast<uint64_t>(w->out), static_cast<uint64_t>(G), kTcRT, 8,
                          CU_TENSOR_MAP_SWIZZLE_NONE))
            return Q4_ERR_CUDA;
        if (!sym && !make_tmap_2d(&tmap_z, w->zeros, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                                  static_cast<uint64_t>(w->out), static_cast<uint64_t>(G), kTcRT,
                                  8, CU_TENSOR_MAP_SWIZZLE_NONE))
            return Q4_ERR_CUDA;
    }
    auto kernel = q4_skinny_f16_kernel<GS, NT>;
    if (!set_kernel_attrs(kernel, static_cast<int>(geo.total), false)) return Q4_ERR_CUDA;
    unsigned* ws_count = reinterpret_cast<unsigned*>(ws);
    float* ws_part = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) + kWsCounterBytes);
    return launch_ex(kernel, dim3(static_cast<unsigned>(p.P)), dim3(F16Cfg<NT>::threads),
                     geo.total, 1, true, st, tmap_w, tmap_x, tmap_s, tmap_z, meta_tma ? 1 : 0,
                     reinterpret_cast<const uint16_t*>(w->scales),
                     reinterpret_cast<const uint16_t*>(w->zeros), sym ? 1 : 0, stages,
                     static_cast<int>(B), w->out, w->in, p.nchunks, p.T, y, ydt, ws_part, ws_count,
                     status);
}

template <bool BF16, int NT>
q4_status dispatch_skinny_nt(const q4_weight* w, const void* x, int64_t B, void* y, int ydt,
                             void* ws, size_t wsb, cudaStream_t st) {
    // B > 64: the scales go into the fp16 A operand and one accumulator
    // covers a segment (the exact kernel's per-group rescale of 128 columns
    // bounds it there); B <= 64: exact codes, per-group rescale
    if constexpr (NT == 128) {
        switch (w->group_size) {
            case 32: return run_skinny_f16<BF16, 32, NT>(w, x, B, y, ydt, ws, wsb, st);
            case 64: return run_skinny_f16<BF16, 64, NT>(w, x, B, y, ydt, ws, wsb, st);
            case 128: return run_skinny_f16<BF16, 128, NT>(w, x, B, y, ydt, ws, wsb, st);
            default: return Q4_ERR_UNSUPPORTED;
        }
    } else {
        switch (w->group_size) {
            case 32: return run_skinny<BF16, 32, NT>(w, x, B, y, ydt, ws, wsb, st);
            case 64: return run_skinny<BF16, 64, NT>(w, x, B, y, ydt, ws, wsb, st);
            case 128: return run_skinny<BF16, 128, NT>(w, x, B, y, ydt, ws, wsb, st);
            default: return Q4_ERR_UNSUPPORTED;
        }
    }
}

template <bool BF16>
q4_status dispatch_skinny(const q4_weight* w, const void* x, int64_t B, void* y, int ydt, void* ws,
                          size_t wsb, cudaStream_t st) {
    switch (tc_nt(B)) {
        case 16: return dispatch_skinny_nt<BF16, 16>(w, x, B, y, ydt, ws, wsb, st);
        case 32: return dispatch_skinny_nt<BF16, 32>(w, x, B, y, ydt, ws, wsb, st);
        case 64: return dispatch_skinny_nt<BF16, 64>(w, x, B, y, ydt, ws, wsb, st);
        default: return dispatch_skinny_nt<BF16, 128>(w, x, B, y, ydt, ws, wsb, st);
    }
}

q4_status validate_product(const q4_weight* w, const void* x, q4_dtype x_dtype, int64_t B,
                           void* y, q4_dtype y_dtype, int64_t bmax) {
    q4_status s = validate_weight(w);
    if (s != Q4_OK) return s;
    if (!valid_dtype(x_dtype) || !valid_dtype(y_dtype)) return Q4_ERR_INVALID_ARG;
    if (x_dtype == Q4_F32) return Q4_ERR_UNSUPPORTED;
    if (y_dtype != x_dtype && y_dtype != Q4_F32) return Q4_ERR_UNSUPPORTED;
    if (B < 1 || B > bmax) return Q4_ERR_SHAPE;
    if (w->group_size != 32 && w->group_size != 64 && w->group_size != 128)
        return Q4_ERR_UNSUPPORTED;
    if ((w->in % 32) != 0) return Q4_ERR_SHAPE;
    if (w->in > (int64_t(1) << 30) || w->out > int64_t(65535) * 128) return Q4_ERR_SHAPE;
    if (w->out == 0) return Q4_OK;  // nothing to read or write
    if (!x || !y) return Q4_ERR_INVALID_ARG;
    if (!aligned(w->qweight, 16) || !aligned(x, 16) || !aligned(y, 16)) return Q4_ERR_ALIGNMENT;
    return Q4_OK;
}

// ------------------------------------------- static scratch (no allocation)
constexpr size_t kNoAllocScratchBytes = Q4_NOALLOC_SCRATCH_BYTES;

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices];      // scratch address per device, once set up
bool g_noalloc_reclear[kMaxDevices];   // zero-fill again before the next call

}  // namespace

// Stream-K scratch of q4_gemv_noalloc: partial sums and per-row-tile
// counters, the same layout as a q4_gemv workspace.  Zero at module load and
// zero-filled again at setup; the counters must start at zero.
static __device__ __align__(256) unsigned char g_q4_noalloc_scratch[kNoAllocScratchBytes];

namespace {

// Scratch address on the current device `dev`.  The symbol's address is
// looked up on every call (with `dev` current): when it differs from the
// cached one -- the first call on the device, or a context that was torn down
// and created again, whose module load zeroed a fresh array -- the scratch
// is treated as new: zero-filled on `st`, and `st` waited for.
q4_status noalloc_scratch(int dev, cudaStream_t st, void** out) {
    if (dev < 0 || dev >= kMaxDevices) return Q4_ERR_UNSUPPORTED;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_q4_noalloc_scratch) != cudaSuccess || p == nullptr)
        return Q4_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_ptr[dev] != p) {
        if (cudaMemsetAsync(p, 0, kNoAllocScratchBytes, st) != cudaSuccess) return Q4_ERR_CUDA;
        if (cudaStreamSynchronize(st) != cudaSuccess) return Q4_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
        g_noalloc_reclear[dev] = false;
    } else if (g_noalloc_reclear[dev]) {
        if (cudaMemsetAsync(p, 0, kNoAllocScratchBytes, st) != cudaSuccess) return Q4_ERR_CUDA;
        g_noalloc_reclear[dev] = false;
    }
    *out = p;
    return Q4_OK;
}

// A bounded wait ran out: counters in the static scratch may be left set.
void noalloc_mark_reclear() {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    for (int d = 0; d < kMaxDevices; ++d) g_noalloc_reclear[d] = g_noalloc_ptr[d] != nullptr;
}

}  // namespace

// ======================================================================= ABI
// FP4 helpers of the ABI below
namespace {
q4_status fp4_check_quant(const void* W, q4_dtype w_dtype, int64_t out, int64_t in, int block,
                          const uint8_t* packed, const uint8_t* scales) {
    if (w_dtype != Q4_F16 && w_dtype != Q4_BF16) {
        return valid_dtype(w_dtype) ? Q4_ERR_UNSUPPORTED : Q4_ERR_INVALID_ARG;
    }
    if (out < 0 || in <= 0 || (in % block) != 0) return Q4_ERR_SHAPE;
    if (out == 0) return Q4_OK;
    if (!W || !packed || !scales) return Q4_ERR_INVALID_ARG;
    if (!aligned(W, 16) || !aligned(packed, 4)) return Q4_ERR_ALIGNMENT;
    return Q4_OK;
}

int fp4_blocks(int64_t nchunks, int sms) {
    const int64_t want = (nchunks + 255) / 256;
    return static_cast<int>(want < 8LL * sms ? want : 8LL * sms);
}

template <bool NV>
q4_status fp4_dequant(const uint8_t* packed, const uint8_t* scales, const float* tensor_scale,
                      int64_t out, int64_t in, void* W_hat, q4_dtype out_dtype, cudaStream_t st) {
    const int64_t nwords = out * in / 8;
    const int blocks = fp4_blocks(nwords, sm_count(current_device()));
    const uint32_t* pw = reinterpret_cast<const uint32_t*>(packed);
    if (out_dtype == Q4_F32)
        fp4_dequant_kernel<float, NV><<<blocks, 256, 0, st>>>(pw, scales, tensor_scale, nwords,
                                                              reinterpret_cast<float*>(W_hat));
    else if (out_dtype == Q4_F16)
        fp4_dequant_kernel<__half, NV><<<blocks, 256, 0, st>>>(pw, scales, tensor_scale, nwords,
                                                               reinterpret_cast<__half*>(W_hat));
    else
        fp4_dequant_kernel<__nv_bfloat16, NV><<<blocks, 256, 0, st>>>(
            pw, scales, tensor_scale, nwords, reinterpret_cast<__nv_bfloat16*>(W_hat));
    return launch_status(cudaSuccess);
}

// ------------------------------------------- FP4 block-scaled product
constexpr int kF4MinIters = 4;
constexpr int64_t kF4MaxB = 128;  // activation rows per launch (the MMA's N)

int f4_nt(int64_t B) { return B <= 16 ? 16 : B <= 32 ? 32 : B <= 64 ? 64 : 128; }

SkPlan fp4_plan(int64_t out, int64_t in, int64_t B, int sms) {
    return stream_k_plan(out, in, kF4RT, sms, kF4MinIters, f4_nt(B), kF4ChunkCodes);
}

// Cluster plan of the tcgen05 products (FP4, bf16 reference) for activation
// tiles NT >= 64, whose stream-K final epilogue (an NT x 128 fp32 partial per
// CTA stored, counted and summed by the last arriver) costs the most: the
// largest S <= 8 with row_tiles x S CTAs all resident, each CTA at most 25 %
// longer than the longest stream-K range.  Returns 1 for stream-K.
template <typename Kern>
int tc_cluster_size(Kern kcl, const SkPlan& p, int nt, size_t smem, int64_t pmax) {
    if (nt < 64) return 1;
    const int64_t sk_iters = (p.T + p.P - 1) / p.P;
    for (int S = 8; S >= 2; --S) {
        if (S > p.nchunks || p.row_tiles * S > pmax) continue;
        if ((p.nchunks + S - 1) / S * 4 > sk_iters * 5) return 1;
        if (!set_kernel_attrs(kcl, static_cast<int>(smem), false)) return 1;
        if (max_active_clusters(kcl, S, dim3(kF4Threads), smem) >= p.row_tiles) return S;
    }
    return 1;
}

template <bool NV, int NT>
q4_status run_fp4(const uint8_t* wq, const uint8_t* wsc, const float* wts, int64_t out,
                  int64_t in, const uint8_t* xq, const uint8_t* xsc, const float* xts, int64_t B,
                  void* y, int ydt, void* ws, size_t ws_bytes, cudaStream_t st) {
    constexpr int VS = F4Fmt<NV>::VS;
    constexpr int SFB = F4Fmt<NV>::sf_bytes;
    const int dev = current_device();
    const SkPlan p = fp4_plan(out, in, B, sm_count(dev));
    if (p.row_tiles > static_cast<int64_t>(kWsCounterBytes / 4)) return Q4_ERR_SHAPE;
    if (!ws || ws_bytes < p.ws_bytes) return Q4_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return Q4_ERR_ALIGNMENT;
    const size_t smax = static_cast<size_t>(max_smem_optin(dev));
    int stages = kF4MaxStages;
    F4Geom geo = f4_geom(NT, SFB, stages);
    while (stages > 2 && geo.total > smax) geo = f4_geom(NT, SFB, --stages);
    if (geo.total > smax) return Q4_ERR_UNSUPPORTED;
    CUtensorMap tmap_w, tmap_sw, tmap_x, tmap_sx;
    const uint64_t cb = static_cast<uint64_t>(in / 2), sb = static_cast<uint64_t>(in / VS);
    if (!make_tmap_2d(&tmap_w, wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, static_cast<uint64_t>(out),
                      cb, kF4RT, kF4Box) ||
        !make_tmap_2d(&tmap_sw, wsc, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1,
                      static_cast<uint64_t>(out), sb, kF4RT, SFB, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_tmap_2d(&tmap_x, xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, static_cast<uint64_t>(B), cb,
                      NT, kF4Box) ||
        !make_tmap_2d(&tmap_sx, xsc, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, static_cast<uint64_t>(B),
                      sb, NT, SFB, CU_TENSOR_MAP_SWIZZLE_NONE))
        return Q4_ERR_CUDA;
    const int cluster_s = tc_cluster_size(fp4_gemm_tc_kernel<NV, NT, true>, p, NT, geo.total,
                                          sm_count(dev));
    auto kernel = cluster_s > 1 ? fp4_gemm_tc_kernel<NV, NT, true> : fp4_gemm_tc_kernel<NV, NT, false>;
    const int64_t grid = cluster_s > 1 ? p.row_tiles * cluster_s : p.P;
    if (!set_kernel_attrs(kernel, static_cast<int>(geo.total), false)) return Q4_ERR_CUDA;
    unsigned* status = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&status), g_q4_status) != cudaSuccess)
        return Q4_ERR_CUDA;
    unsigned* ws_count = reinterpret_cast<unsigned*>(ws);
    float* ws_part = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) + kWsCounterBytes);
    return launch_ex(kernel, dim3(static_cast<unsigned>(grid)), dim3(kF4Threads), geo.total,
                     cluster_s, true, st, tmap_w, tmap_sw, tmap_x, tmap_sx, wts, xts, stages,
                     static_cast<int>(B), out, p.nchunks, p.T, y, ydt, ws_part, ws_count, status,
                     cluster_s);
}

SkPlan bf16_plan(int64_t out, int64_t in, int64_t B, int sms) {
    return stream_k_plan(out, in, kF4RT, sms, kF4MinIters, f4_nt(B), TcKind<kKindBF16>::chunk_elems);
}

template <int NT>
q4_status run_bf16_tc(const void* W, int64_t out, int64_t in, const void* x, int64_t B, void* y,
                      void* ws, size_t ws_bytes, cudaStream_t st) {
    const int dev = current_device();
    const SkPlan p = bf16_plan(out, in, B, sm_count(dev));
    if (p.row_tiles > static_cast<int64_t>(kWsCounterBytes / 4)) return Q4_ERR_SHAPE;
    if (ws_bytes < p.ws_bytes) return Q4_ERR_WORKSPACE;
    if (!aligned(ws, 256)) return Q4_ERR_ALIGNMENT;
    const size_t smax = static_cast<size_t>(max_smem_optin(dev));
    int stages = kF4MaxStages;
    F4Geom geo = f4_geom(NT, 0, stages);
    while (stages > 2 && geo.total > smax) geo = f4_geom(NT, 0, --stages);
    if (geo.total > smax) return Q4_ERR_UNSUPPORTED;
    CUtensorMap tmap_w, tmap_x;
    constexpr uint32_t kBoxElems = TcKind<kKindBF16>::box_step;  // 64 bf16 = one 128-byte row
    if (!make_tmap_2d(&tmap_w, W, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, static_cast<uint64_t>(out),
                      static_cast<uint64_t>(in), kF4RT, kBoxElems) ||
        !make_tmap_2d(&tmap_x, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, static_cast<uint64_t>(B),
                      static_cast<uint64_t>(in), NT, kBoxElems))
        return Q4_ERR_CUDA;
    const int cluster_s = tc_cluster_size(bf16_gemm_tc_kernel<NT, true>, p, NT, geo.total,
                                          sm_count(dev));
    auto kernel = cluster_s > 1 ? bf16_gemm_tc_kernel<NT, true> : bf16_gemm_tc_kernel<NT, false>;
    const int64_t grid = cluster_s > 1 ? p.row_tiles * cluster_s : p.P;
    if (!set_kernel_attrs(kernel, static_cast<int>(geo.total), false)) return Q4_ERR_CUDA;
    unsigned* status = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&status), g_q4_status) != cudaSuccess)
        return Q4_ERR_CUDA;
    unsigned* ws_count = reinterpret_cast<unsigned*>(ws);
    float* ws_part = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws) + kWsCounterBytes);
    return launch_ex(kernel, dim3(static_cast<unsigned>(grid)), dim3(kF4Threads), geo.total,
                     cluster_s, true, st, tmap_w, tmap_x, stages, static_cast<int>(B), out,
                     p.nchunks, p.T, y, 1, ws_part, ws_count, status, cluster_s);
}

template <bool NV>
q4_status dispatch_fp4(const uint8_t* wq, const uint8_t* wsc, const float* wts, int64_t out,
                       int64_t in, const uint8_t* xq, const uint8_t* xsc, const float* xts,
                       int64_t B, void* y, int ydt, void* ws, size_t wsb, cudaStream_t st) {
    switch (f4_nt(B)) {
        case 16: return run_fp4<NV, 16>(wq, wsc, wts, out, in, xq, xsc, xts, B, y, ydt, ws, wsb, st);
        case 32: return run_fp4<NV, 32>(wq, wsc, wts, out, in, xq, xsc, xts, B, y, ydt, ws, wsb, st);
        case 64: return run_fp4<NV, 64>(wq, wsc, wts, out, in, xq, xsc, xts, B, y, ydt, ws, wsb, st);
        default:
            return run_fp4<NV, 128>(wq, wsc, wts, out, in, xq, xsc, xts, B, y, ydt, ws, wsb, st);
    }
}
}  // namespace

extern "C" {

const char* q4_version(void) { return "q4-b200 0.1 (sm_100a)"; }

const char* q4_status_string(q4_status s) {
    switch (s) {
        case Q4_OK: return "Q4_OK";
        case Q4_ERR_INVALID_ARG: return "Q4_ERR_INVALID_ARG";
        case Q4_ERR_SHAPE: return "Q4_ERR_SHAPE";
        case Q4_ERR_ALIGNMENT: return "Q4_ERR_ALIGNMENT";
        case Q4_ERR_UNSUPPORTED: return "Q4_ERR_UNSUPPORTED";
        case Q4_ERR_CUDA: return "Q4_ERR_CUDA";
        case Q4_ERR_TIMEOUT: return "Q4_ERR_TIMEOUT";
        case Q4_ERR_WORKSPACE: return "Q4_ERR_WORKSPACE";
    }
    return "Q4_ERR_UNKNOWN";
}

q4_status q4_quantize_pack(const void* W, q4_dtype w_dtype, int64_t out, int64_t in,
                           int32_t group_size, int32_t bits, int32_t symmetric, uint8_t* qweight,
                           void* scales, void* zeros, q4_stream stream) {
    if (w_dtype != Q4_F16 && w_dtype != Q4_BF16) {
        return valid_dtype(w_dtype) ? Q4_ERR_UNSUPPORTED : Q4_ERR_INVALID_ARG;
    }
    if (bits != 4) return Q4_ERR_UNSUPPORTED;
    if (symmetric != 0 && symmetric != 1) return Q4_ERR_INVALID_ARG;
    if (out < 0 || in <= 0 || group_size <= 0) return Q4_ERR_SHAPE;
    if ((group_size & 1) || (in % group_size) != 0 || (in % 8) != 0) return Q4_ERR_SHAPE;
    if (out == 0) return Q4_OK;
    if (!W || !qweight || !scales) return Q4_ERR_INVALID_ARG;
    if (symmetric ? (zeros != nullptr) : (zeros == nullptr)) return Q4_ERR_INVALID_ARG;
    if (!aligned(W, 16) || !aligned(qweight, 4) || !aligned(scales, 2) ||
        (zeros && !aligned(zeros, 2)))
        return Q4_ERR_ALIGNMENT;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    __half* s = reinterpret_cast<__half*>(scales);
    __half* z = reinterpret_cast<__half*>(zeros);
    const bool bf = (w_dtype == Q4_BF16);
    if (symmetric)
        return bf ? run_quantize<true, true>(W, out, in, group_size, qweight, s, z, st)
                  : run_quantize<true, false>(W, out, in, group_size, qweight, s, z, st);
    return bf ? run_quantize<false, true>(W, out, in, group_size, qweight, s, z, st)
              : run_quantize<false, false>(W, out, in, group_size, qweight, s, z, st);
}

q4_status q4_quantize_pack_perm(const void* W, q4_dtype w_dtype, int64_t out, int64_t in,
                                int32_t group_size, int32_t bits, int32_t symmetric,
                                const int32_t* perm, uint8_t* qweight, void* scales, void* zeros,
                                q4_stream stream) {
    if (w_dtype != Q4_F16 && w_dtype != Q4_BF16) {
        return valid_dtype(w_dtype) ? Q4_ERR_UNSUPPORTED : Q4_ERR_INVALID_ARG;
    }
    if (bits != 4) return Q4_ERR_UNSUPPORTED;
    if (symmetric != 0 && symmetric != 1) return Q4_ERR_INVALID_ARG;
    if (out < 0 || in <= 0 || group_size <= 0) return Q4_ERR_SHAPE;
    if ((group_size & 1) || (in % group_size) != 0 || (in % 8) != 0) return Q4_ERR_SHAPE;
    if (out == 0) return Q4_OK;
    if (!W || !qweight || !scales || !perm) return Q4_ERR_INVALID_ARG;
    if (symmetric ? (zeros != nullptr) : (zeros == nullptr)) return Q4_ERR_INVALID_ARG;
    if (!aligned(W, 2) || !aligned(qweight, 4) || !aligned(scales, 2) || !aligned(perm, 4) ||
        (zeros && !aligned(zeros, 2)))
        return Q4_ERR_ALIGNMENT;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    __half* s = reinterpret_cast<__half*>(scales);
    __half* z = reinterpret_cast<__half*>(zeros);
    const bool bf = (w_dtype == Q4_BF16);
    if (symmetric)
        return bf ? run_quantize<true, true>(W, out, in, group_size, qweight, s, z, st, perm)
                  : run_quantize<true, false>(W, out, in, group_size, qweight, s, z, st, perm);
    return bf ? run_quantize<false, true>(W, out, in, group_size, qweight, s, z, st, perm)
              : run_quantize<false, false>(W, out, in, group_size, qweight, s, z, st, perm);
}

q4_status q4_permute_activations(const void* x, q4_dtype x_dtype, int64_t rows, int64_t in,
                                 const int32_t* perm, void* x_perm, q4_stream stream) {
    if (!valid_dtype(x_dtype)) return Q4_ERR_INVALID_ARG;
    if (x_dtype == Q4_F32) return Q4_ERR_UNSUPPORTED;
    if (rows < 0 || in <= 0 || (in % 8) != 0) return Q4_ERR_SHAPE;
    if (rows == 0) return Q4_OK;
    if (!x || !perm || !x_perm) return Q4_ERR_INVALID_ARG;
    if (!aligned(x, 2) || !aligned(perm, 4) || !aligned(x_perm, 16)) return Q4_ERR_ALIGNMENT;
    unsigned* status = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&status), g_q4_status) != cudaSuccess)
        return Q4_ERR_CUDA;
    const int sms = sm_count(current_device());
    const int64_t n8 = rows * in / 8;
    const int64_t want = (n8 + 255) / 256;
    const int blocks = static_cast<int>(want < 4LL * sms ? want : 4LL * sms);
    return launch_ex(permute_columns_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, 1,
                     true, reinterpret_cast<cudaStream_t>(stream),
                     reinterpret_cast<const uint16_t*>(x), rows, in, perm,
                     reinterpret_cast<uint16_t*>(x_perm), status);
}

q4_status q4_quantize_pack_clip(const void* W, q4_dtype w_dtype, int64_t out, int64_t in,
                                int32_t group_size, int32_t n_alpha, uint8_t* qweight,
                                void* scales, q4_stream stream) {
    if (w_dtype != Q4_F16 && w_dtype != Q4_BF16) {
        return valid_dtype(w_dtype) ? Q4_ERR_UNSUPPORTED : Q4_ERR_INVALID_ARG;
    }
    if (n_alpha < 1 || n_alpha > 64) return Q4_ERR_INVALID_ARG;
    if (out < 0 || in <= 0 || group_size <= 0) return Q4_ERR_SHAPE;
    if ((group_size & 1) || (in % group_size) != 0 || (in % 8) != 0) return Q4_ERR_SHAPE;
    if (group_size != 8 && group_size != 16 && group_size != 32 && group_size != 64 &&
        group_size != 128 && group_size != 256)
        return Q4_ERR_UNSUPPORTED;
    if (out == 0) return Q4_OK;
    if (!W || !qweight || !scales) return Q4_ERR_INVALID_ARG;
    if (!aligned(W, 16) || !aligned(qweight, 4) || !aligned(scales, 2)) return Q4_ERR_ALIGNMENT;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    __half* s = reinterpret_cast<__half*>(scales);
    return w_dtype == Q4_BF16
               ? run_quantize_clip<true>(W, out, in, group_size, n_alpha, qweight, s, st)
               : run_quantize_clip<false>(W, out, in, group_size, n_alpha, qweight, s, st);
}

q4_status q4_dequant(const q4_weight* w, void* W_hat, q4_dtype out_dtype, q4_stream stream) {
    q4_status s = validate_weight(w);
    if (s != Q4_OK) return s;
    if (!valid_dtype(out_dtype)) return Q4_ERR_INVALID_ARG;
    if ((w->in % 8) != 0) return Q4_ERR_SHAPE;
    if (w->out == 0) return Q4_OK;
    if (!W_hat) return Q4_ERR_INVALID_ARG;
    if (!aligned(W_hat, 16) || !aligned(w->qweight, 4)) return Q4_ERR_ALIGNMENT;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int dev = current_device();
    const int sms = sm_count(dev);
    const int64_t nwords = w->out * w->in / 8;
    const int64_t want = (nwords + 255) / 256;
    const int blocks = static_cast<int>(want < 8LL * sms ? want : 8LL * sms);
    const uint32_t* qw = reinterpret_cast<const uint32_t*>(w->qweight);
    const __half* sc = reinterpret_cast<const __half*>(w->scales);
    const __half* zc = reinterpret_cast<const __half*>(w->zeros);
    const int g = w->group_size;
    if (out_dtype == Q4_F32) {
        if (w->symmetric)
            dequant_kernel<float, true><<<blocks, 256, 0, st>>>(qw, sc, zc, nwords, w->in, g,
                                                                reinterpret_cast<float*>(W_hat));
        else
            dequant_kernel<float, false><<<blocks, 256, 0, st>>>(qw, sc, zc, nwords, w->in, g,
                                                                 reinterpret_cast<float*>(W_hat));
    } else if (out_dtype == Q4_F16) {
        if (w->symmetric)
            dequant_kernel<__half, true><<<blocks, 256, 0, st>>>(qw, sc, zc, nwords, w->in, g,
                                                                 reinterpret_cast<__half*>(W_hat));
        else
            dequant_kernel<__half, false><<<blocks, 256, 0, st>>>(qw, sc, zc, nwords, w->in, g,
                                                                  reinterpret_cast<__half*>(W_hat));
    } else {
        if (w->symmetric)
            dequant_kernel<__nv_bfloat16, true><<<blocks, 256, 0, st>>>(
                qw, sc, zc, nwords, w->in, g, reinterpret_cast<__nv_bfloat16*>(W_hat));
        else
            dequant_kernel<__nv_bfloat16, false><<<blocks, 256, 0, st>>>(
                qw, sc, zc, nwords, w->in, g, reinterpret_cast<__nv_bfloat16*>(W_hat));
    }
    return launch_status(cudaSuccess);
}

size_t q4_workspace_bytes(int64_t out, int64_t in, int64_t B, int32_t group_size) {
    if (out < 0 || in <= 0 || B < 1 || B > 128 || group_size <= 0) return 0;
    if (out == 0) return 0;
    return product_plan(out, in, B, sm_count(current_device())).ws_bytes;
}

q4_status q4_gemv(const q4_weight* w, const void* x, q4_dtype x_dtype, int64_t B, void* y,
                  q4_dtype y_dtype, void* workspace, size_t workspace_bytes, q4_stream stream) {
    q4_status s = validate_product(w, x, x_dtype, B, y, y_dtype, 8);
    if (s != Q4_OK) return s;
    if (w->out == 0) return Q4_OK;
    if (!workspace) return Q4_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int ydt = y_dtype == Q4_F32 ? 2 : (y_dtype == Q4_BF16 ? 1 : 0);
    return x_dtype == Q4_BF16
               ? dispatch_gemv<true>(w, x, B, y, ydt, workspace, workspace_bytes, st)
               : dispatch_gemv<false>(w, x, B, y, ydt, workspace, workspace_bytes, st);
}

q4_status q4_gemm_skinny(const q4_weight* w, const void* x, q4_dtype x_dtype, int64_t B,
                         void* y, q4_dtype y_dtype, void* workspace, size_t workspace_bytes,
                         q4_stream stream) {
    q4_status s = validate_product(w, x, x_dtype, B, y, y_dtype, 128);
    if (s != Q4_OK) return s;
    if (B <= 8) return q4_gemv(w, x, x_dtype, B, y, y_dtype, workspace, workspace_bytes, stream);
    if (w->out == 0) return Q4_OK;
    if (!workspace) return Q4_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int ydt = y_dtype == Q4_F32 ? 2 : (y_dtype == Q4_BF16 ? 1 : 0);
    return x_dtype == Q4_BF16
               ? dispatch_skinny<true>(w, x, B, y, ydt, workspace, workspace_bytes, st)
               : dispatch_skinny<false>(w, x, B, y, ydt, workspace, workspace_bytes, st);
}

q4_status q4_gemv_grouped(const q4_weight* ws, int32_t n, const void* x, q4_dtype x_dtype,
                          int64_t B, void* const* ys, q4_dtype y_dtype, void* workspace,
                          size_t workspace_bytes, q4_stream stream) {
    if (!ws || !ys || n < 1 || n > Q4_GROUP_MAX) return Q4_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i) {
        q4_status s = validate_product(&ws[i], x, x_dtype, B, ys[i], y_dtype, 128);
        if (s != Q4_OK) return s;
        if (ws[i].in != ws[0].in || ws[i].group_size != ws[0].group_size ||
            ws[i].symmetric != ws[0].symmetric)
            return Q4_ERR_SHAPE;
    }
    if (B > 8) {
        // the tensor-core kernel runs one product per launch
        for (int i = 0; i < n; ++i) {
            q4_status s = q4_gemm_skinny(&ws[i], x, x_dtype, B, ys[i], y_dtype, workspace,
                                         workspace_bytes, stream);
            if (s != Q4_OK) return s;
        }
        return Q4_OK;
    }
    const q4_weight* wv[Q4_GROUP_MAX];
    void* yv[Q4_GROUP_MAX];
    int m = 0;
    for (int i = 0; i < n; ++i) {
        if (ws[i].out == 0) continue;  // nothing to read or write
        wv[m] = &ws[i];
        yv[m] = ys[i];
        ++m;
    }
    if (m == 0) return Q4_OK;
    if (!workspace) return Q4_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int ydt = y_dtype == Q4_F32 ? 2 : (y_dtype == Q4_BF16 ? 1 : 0);
    return x_dtype == Q4_BF16
               ? dispatch_gemv<true>(wv, m, x, B, yv, ydt, workspace, workspace_bytes, st)
               : dispatch_gemv<false>(wv, m, x, B, yv, ydt, workspace, workspace_bytes, st);
}

q4_status q4_gemv_noalloc(const q4_weight* w, const void* x, q4_dtype x_dtype, int64_t B,
                          void* y, q4_dtype y_dtype, q4_stream stream) {
    q4_status s = validate_product(w, x, x_dtype, B, y, y_dtype, 8);
    if (s != Q4_OK) return s;
    if (w->out == 0) return Q4_OK;
    const int dev = current_device();
    if (sk_plan(w->out, w->in, sm_count(dev)).ws_bytes > kNoAllocScratchBytes)
        return Q4_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    void* scratch = nullptr;
    s = noalloc_scratch(dev, st, &scratch);
    if (s != Q4_OK) return s;
    const int ydt = y_dtype == Q4_F32 ? 2 : (y_dtype == Q4_BF16 ? 1 : 0);
    return x_dtype == Q4_BF16
               ? dispatch_gemv<true>(w, x, B, y, ydt, scratch, kNoAllocScratchBytes, st)
               : dispatch_gemv<false>(w, x, B, y, ydt, scratch, kNoAllocScratchBytes, st);
}

size_t bf16_ref_workspace_bytes(int64_t out, int64_t in, int64_t B) {
    if (out <= 0 || in <= 0 || B < 1 || B > 128) return 0;
    return bf16_plan(out, in, B, sm_count(current_device())).ws_bytes;
}

q4_status bf16_gemv_ref_bw(const void* W, int64_t out, int64_t in, const void* x, int64_t B,
                           void* y, void* workspace, size_t workspace_bytes, q4_stream stream) {
    if (out < 0 || in <= 0 || (in % 64) != 0) return Q4_ERR_SHAPE;
    if (B < 1 || B > 128) return Q4_ERR_SHAPE;
    if (out == 0) return Q4_OK;
    if (!W || !x || !y) return Q4_ERR_INVALID_ARG;
    if (!aligned(W, 16) || !aligned(x, 16) || !aligned(y, 16)) return Q4_ERR_ALIGNMENT;
    if (!workspace) return Q4_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    switch (f4_nt(B)) {
        case 16: return run_bf16_tc<16>(W, out, in, x, B, y, workspace, workspace_bytes, st);
        case 32: return run_bf16_tc<32>(W, out, in, x, B, y, workspace, workspace_bytes, st);
        case 64: return run_bf16_tc<64>(W, out, in, x, B, y, workspace, workspace_bytes, st);
        default: return run_bf16_tc<128>(W, out, in, x, B, y, workspace, workspace_bytes, st);
    }
}

// ------------------------------------------------- per-channel INT8 weights

q4_status q8_quantize_per_channel(const void* W, q4_dtype w_dtype, int64_t out, int64_t in,
                                  int8_t* qweight, float* scales, q4_stream stream) {
    if (w_dtype != Q4_F16 && w_dtype != Q4_BF16) {
        return valid_dtype(w_dtype) ? Q4_ERR_UNSUPPORTED : Q4_ERR_INVALID_ARG;
    }
    if (out < 0 || in <= 0 || (in % 16) != 0) return Q4_ERR_SHAPE;
    if (out == 0) return Q4_OK;
    if (!W || !qweight || !scales) return Q4_ERR_INVALID_ARG;
    if (!aligned(W, 16) || !aligned(qweight, 16) || !aligned(scales, 4)) return Q4_ERR_ALIGNMENT;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int sms = sm_count(current_device());
    const int blocks = static_cast<int>(out < 16LL * sms ? out : 16LL * sms);
    if (w_dtype == Q4_BF16)
        q8_quantize_rows_kernel<true><<<blocks, 256, 0, st>>>(W, out, in, qweight, scales);
    else
        q8_quantize_rows_kernel<false><<<blocks, 256, 0, st>>>(W, out, in, qweight, scales);
    return launch_status(cudaSuccess);
}

q4_status q8_dequant(const int8_t* qweight, const float* scales, int64_t out, int64_t in,
                     void* W_hat, q4_dtype out_dtype, q4_stream stream) {
    if (!valid_dtype(out_dtype)) return Q4_ERR_INVALID_ARG;
    if (out < 0 || in <= 0 || (in % 16) != 0) return Q4_ERR_SHAPE;
    if (out == 0) return Q4_OK;
    if (!qweight || !scales || !W_hat) return Q4_ERR_INVALID_ARG;
    if (!aligned(qweight, 16) || !aligned(scales, 4) || !aligned(W_hat, 16))
        return Q4_ERR_ALIGNMENT;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int sms = sm_count(current_device());
    const int64_t nvec = out * in / 8;
    const int64_t want = (nvec + 255) / 256;
    const int blocks = static_cast<int>(want < 8LL * sms ? want : 8LL * sms);
    if (out_dtype == Q4_F32)
        q8_dequant_kernel<float><<<blocks, 256, 0, st>>>(qweight, scales, nvec, in,
                                                         reinterpret_cast<float*>(W_hat));
    else if (out_dtype == Q4_F16)
        q8_dequant_kernel<__half><<<blocks, 256, 0, st>>>(qweight, scales, nvec, in,
                                                          reinterpret_cast<__half*>(W_hat));
    else
        q8_dequant_kernel<__nv_bfloat16><<<blocks, 256, 0, st>>>(
            qweight, scales, nvec, in, reinterpret_cast<__nv_bfloat16*>(W_hat));
    return launch_status(cudaSuccess);
}

size_t q8_workspace_bytes(int64_t out, int64_t in, int64_t B) {
    if (out <= 0 || in <= 0 || B < 1 || B > 8) return 0;
    return q8_plan(out, in, sm_count(current_device())).ws_bytes;
}

q4_status q8_gemv(const int8_t* qweight, const float* scales, int64_t out, int64_t in,
                  const void* x, q4_dtype x_dtype, int64_t B, void* y, q4_dtype y_dtype,
                  void* workspace, size_t workspace_bytes, q4_stream stream) {
    if (!valid_dtype(x_dtype) || !valid_dtype(y_dtype)) return Q4_ERR_INVALID_ARG;
    if (x_dtype == Q4_F32) return Q4_ERR_UNSUPPORTED;
    if (y_dtype != x_dtype && y_dtype != Q4_F32) return Q4_ERR_UNSUPPORTED;
    if (B < 1 || B > 8) return Q4_ERR_SHAPE;
    if (out < 0 || in <= 0 || (in % 16) != 0) return Q4_ERR_SHAPE;
    if (in > (int64_t(1) << 30) || out > int64_t(65535) * kQ8RT) return Q4_ERR_SHAPE;
    if (out == 0) return Q4_OK;
    if (!qweight || !scales || !x || !y) return Q4_ERR_INVALID_ARG;
    if (!aligned(qweight, 16) || !aligned(scales, 4) || !aligned(x, 16) || !aligned(y, 16))
        return Q4_ERR_ALIGNMENT;
    if (!workspace) return Q4_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int ydt = y_dtype == Q4_F32 ? 2 : (y_dtype == Q4_BF16 ? 1 : 0);
    return x_dtype == Q4_BF16 ? run_q8_gemv<true>(qweight, scales, out, in, x, B, y, ydt, workspace,
                                                  workspace_bytes, st)
                              : run_q8_gemv<false>(qweight, scales, out, in, x, B, y, ydt,
                                                   workspace, workspace_bytes, st);
}

// ------------------------------------------------------------- KV cache

q4_status kv_quantize_int8(const void* kv, q4_dtype dtype, int64_t rows, int64_t head_dim,
                           int8_t* codes, void* scales, q4_stream stream) {
    if (dtype != Q4_F16 && dtype != Q4_BF16) {
        return valid_dtype(dtype) ? Q4_ERR_UNSUPPORTED : Q4_ERR_INVALID_ARG;
    }
    if (rows < 0 || head_dim < 8 || head_dim > 512 || (head_dim % 8) != 0) return Q4_ERR_SHAPE;
    if (rows == 0) return Q4_OK;
    if (!kv || !codes || !scales) return Q4_ERR_INVALID_ARG;
    if (!aligned(kv, 16) || !aligned(codes, 16) || !aligned(scales, 2)) return Q4_ERR_ALIGNMENT;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int sms = sm_count(current_device());
    const int d = static_cast<int>(head_dim);
    const int V = d / 8;
    int ts = 1;
    while (ts * 2 < V) ts *= 2;  // smallest power of two with 2 * ts >= V
    const int64_t rpw = 32 / ts;
    const int64_t warps = (rows + rpw - 1) / rpw;
    const int64_t want = (warps + 7) / 8;
    const int blocks = static_cast<int>(want < 16LL * sms ? want : 16LL * sms);
    const uint16_t* in = reinterpret_cast<const uint16_t*>(kv);
    uint16_t* sc = reinterpret_cast<uint16_t*>(scales);
    const bool bf = dtype == Q4_BF16;
    switch (ts) {
#define Q4_KVCASE(TSV)                                                                          \
    case TSV:                                                                                   \
        if (bf)                                                                                 \
            kv_quantize_int8_kernel<true, TSV><<<blocks, 256, 0, st>>>(in, rows, d, codes, sc); \
        else                                                                                    \
            kv_quantize_int8_kernel<false, TSV><<<blocks, 256, 0, st>>>(in, rows, d, codes, sc); \
        break;
        Q4_KVCASE(1) Q4_KVCASE(2) Q4_KVCASE(4) Q4_KVCASE(8) Q4_KVCASE(16) Q4_KVCASE(32)
#undef Q4_KVCASE
        default: return Q4_ERR_SHAPE;
    }
    return launch_status(cudaSuccess);
}

q4_status kv_dequant_int8(const int8_t* codes, const void* scales, q4_dtype dtype, int64_t rows,
                          int64_t head_dim, void* out, q4_stream stream) {
    if (dtype != Q4_F16 && dtype != Q4_BF16) {
        return valid_dtype(dtype) ? Q4_ERR_UNSUPPORTED : Q4_ERR_INVALID_ARG;
    }
    if (rows < 0 || head_dim < 8 || head_dim > 512 || (head_dim % 8) != 0) return Q4_ERR_SHAPE;
    if (rows == 0) return Q4_OK;
    if (!codes || !scales || !out) return Q4_ERR_INVALID_ARG;
    if (!aligned(codes, 16) || !aligned(scales, 2) || !aligned(out, 16)) return Q4_ERR_ALIGNMENT;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int sms = sm_count(current_device());
    const int64_t nvec = rows * head_dim / 8;
    const int64_t want = (nvec + 255) / 256;
    const int blocks = static_cast<int>(want < 8LL * sms ? want : 8LL * sms);
    const uint16_t* sc = reinterpret_cast<const uint16_t*>(scales);
    uint16_t* o = reinterpret_cast<uint16_t*>(out);
    if (dtype == Q4_BF16)
        kv_dequant_int8_kernel<true><<<blocks, 256, 0, st>>>(codes, sc, nvec,
                                                             static_cast<int>(head_dim), o);
    else
        kv_dequant_int8_kernel<false><<<blocks, 256, 0, st>>>(codes, sc, nvec,
                                                              static_cast<int>(head_dim), o);
    return launch_status(cudaSuccess);
}

q4_status kv_quantize_int4(const void* kv, q4_dtype dtype, int64_t rows, int64_t head_dim,
                           int32_t group_size, uint8_t* packed, void* scales, q4_stream stream) {
    if (dtype != Q4_F16 && dtype != Q4_BF16) {
        return valid_dtype(dtype) ? Q4_ERR_UNSUPPORTED : Q4_ERR_INVALID_ARG;
    }
    if (rows < 0 || head_dim <= 0 || (head_dim % 8) != 0 || group_size <= 0) return Q4_ERR_SHAPE;
    if ((group_size & 1) || (head_dim % group_size) != 0) return Q4_ERR_SHAPE;
    if (rows == 0) return Q4_OK;
    if (!kv || !packed || !scales) return Q4_ERR_INVALID_ARG;
    if (!aligned(kv, 16) || !aligned(packed, 4) || !aligned(scales, 2)) return Q4_ERR_ALIGNMENT;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    __half* s = reinterpret_cast<__half*>(scales);
    return dtype == Q4_BF16
               ? run_quantize<true, true>(kv, rows, head_dim, group_size, packed, s, nullptr, st)
               : run_quantize<true, false>(kv, rows, head_dim, group_size, packed, s, nullptr, st);
}

q4_status kv_dequant_int4(const uint8_t* packed, const void* scales, int64_t rows,
                          int64_t head_dim, int32_t group_size, void* out, q4_dtype out_dtype,
                          q4_stream stream) {
    if (rows < 0 || head_dim <= 0) return Q4_ERR_SHAPE;
    q4_weight w{};
    w.qweight = packed;
    w.scales = scales;
    w.zeros = nullptr;
    w.out = rows;
    w.in = head_dim;
    w.group_size = group_size;
    w.bits = 4;
    w.symmetric = 1;
    return q4_dequant(&w, out, out_dtype, stream);
}

// ------------------------------------------------------ FP4 microscaling

q4_status mxfp4_quantize(const void* W, q4_dtype w_dtype, int64_t out, int64_t in,
                         uint8_t* packed, uint8_t* scales, q4_stream stream) {
    q4_status s = fp4_check_quant(W, w_dtype, out, in, 32, packed, scales);
    if (s != Q4_OK || out == 0) return s;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int64_t nchunks = out * in / 8;
    const int blocks = fp4_blocks(nchunks, sm_count(current_device()));
    uint32_t* pw = reinterpret_cast<uint32_t*>(packed);
    if (w_dtype == Q4_BF16)
        mxfp4_quantize_kernel<true><<<blocks, 256, 0, st>>>(W, nchunks, pw, scales);
    else
        mxfp4_quantize_kernel<false><<<blocks, 256, 0, st>>>(W, nchunks, pw, scales);
    return launch_status(cudaSuccess);
}

q4_status mxfp4_dequant(const uint8_t* packed, const uint8_t* scales, int64_t out, int64_t in,
                        void* W_hat, q4_dtype out_dtype, q4_stream stream) {
    if (!valid_dtype(out_dtype)) return Q4_ERR_INVALID_ARG;
    if (out < 0 || in <= 0 || (in % 32) != 0) return Q4_ERR_SHAPE;
    if (out == 0) return Q4_OK;
    if (!packed || !scales || !W_hat) return Q4_ERR_INVALID_ARG;
    if (!aligned(packed, 4) || !aligned(W_hat, 16)) return Q4_ERR_ALIGNMENT;
    return fp4_dequant<false>(packed, scales, nullptr, out, in, W_hat, out_dtype,
                              reinterpret_cast<cudaStream_t>(stream));
}

q4_status nvfp4_quantize(const void* W, q4_dtype w_dtype, int64_t out, int64_t in,
                         uint8_t* packed, uint8_t* scales, float* tensor_scale,
                         q4_stream stream) {
    q4_status s = fp4_check_quant(W, w_dtype, out, in, 16, packed, scales);
    if (s != Q4_OK || out == 0) return s;
    if (!tensor_scale) return Q4_ERR_INVALID_ARG;
    if (!aligned(tensor_scale, 4)) return Q4_ERR_ALIGNMENT;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int64_t nchunks = out * in / 8;
    const int sms = sm_count(current_device());
    const int blocks = fp4_blocks(nchunks, sms);
    unsigned* amax = reinterpret_cast<unsigned*>(tensor_scale);
    if (cudaMemsetAsync(amax, 0, sizeof(unsigned), st) != cudaSuccess) return Q4_ERR_CUDA;
    uint32_t* pw = reinterpret_cast<uint32_t*>(packed);
    if (w_dtype == Q4_BF16) {
        tensor_amax_kernel<true><<<blocks, 256, 0, st>>>(W, nchunks, amax);
        nvfp4_quantize_kernel<true><<<blocks, 256, 0, st>>>(W, nchunks, amax, pw, scales);
    } else {
        tensor_amax_kernel<false><<<blocks, 256, 0, st>>>(W, nchunks, amax);
        nvfp4_quantize_kernel<false><<<blocks, 256, 0, st>>>(W, nchunks, amax, pw, scales);
    }
    nvfp4_finalize_kernel<<<1, 32, 0, st>>>(amax);
    return launch_status(cudaSuccess);
}

q4_status nvfp4_dequant(const uint8_t* packed, const uint8_t* scales, const float* tensor_scale,
                        int64_t out, int64_t in, void* W_hat, q4_dtype out_dtype,
                        q4_stream stream) {
    if (!valid_dtype(out_dtype)) return Q4_ERR_INVALID_ARG;
    if (out < 0 || in <= 0 || (in % 16) != 0) return Q4_ERR_SHAPE;
    if (out == 0) return Q4_OK;
    if (!packed || !scales || !tensor_scale || !W_hat) return Q4_ERR_INVALID_ARG;
    if (!aligned(packed, 4) || !aligned(W_hat, 16) || !aligned(tensor_scale, 4))
        return Q4_ERR_ALIGNMENT;
    return fp4_dequant<true>(packed, scales, tensor_scale, out, in, W_hat, out_dtype,
                             reinterpret_cast<cudaStream_t>(stream));
}

size_t fp4_gemm_workspace_bytes(int32_t format, int64_t out, int64_t in, int64_t B) {
    if ((format != Q4_FP4_MXFP4 && format != Q4_FP4_NVFP4) || out <= 0 || in <= 0 || B < 1)
        return 0;
    return fp4_plan(out, in, B < kF4MaxB ? B : kF4MaxB, sm_count(current_device())).ws_bytes;
}

q4_status fp4_gemm(int32_t format, const uint8_t* w_packed, const uint8_t* w_scales,
                   const float* w_tensor_scale, int64_t out, int64_t in, const uint8_t* x_packed,
                   const uint8_t* x_scales, const float* x_tensor_scale, int64_t B, void* y,
                   q4_dtype y_dtype, void* workspace, size_t workspace_bytes, q4_stream stream) {
    if (format != Q4_FP4_MXFP4 && format != Q4_FP4_NVFP4) return Q4_ERR_INVALID_ARG;
    if (!valid_dtype(y_dtype)) return Q4_ERR_INVALID_ARG;
    const bool nv = format == Q4_FP4_NVFP4;
    if (out < 0 || in <= 0 || B < 1 || (in % (nv ? 256 : 512)) != 0) return Q4_ERR_SHAPE;
    if (out == 0) return Q4_OK;
    if (!w_packed || !w_scales || !x_packed || !x_scales || !y) return Q4_ERR_INVALID_ARG;
    if (nv && (!w_tensor_scale || !x_tensor_scale)) return Q4_ERR_INVALID_ARG;
    const int ysz = y_dtype == Q4_F32 ? 4 : 2;
    if (!aligned(w_packed, 16) || !aligned(w_scales, 16) || !aligned(x_packed, 16) ||
        !aligned(x_scales, 16) || !aligned(y, ysz) ||
        (nv && (!aligned(w_tensor_scale, 4) || !aligned(x_tensor_scale, 4))))
        return Q4_ERR_ALIGNMENT;
    if (!workspace) return Q4_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int ydt = y_dtype == Q4_F32 ? 2 : (y_dtype == Q4_BF16 ? 1 : 0);
    const int64_t vs = nv ? 16 : 32;
    // batches beyond the MMA's N run as slices of 128 activation rows
    for (int64_t b0 = 0; b0 < B; b0 += kF4MaxB) {
        const int64_t nb = B - b0 < kF4MaxB ? B - b0 : kF4MaxB;
        const uint8_t* xq = x_packed + b0 * (in / 2);
        const uint8_t* xs = x_scales + b0 * (in / vs);
        void* yb = reinterpret_cast<uint8_t*>(y) + b0 * out * ysz;
        const q4_status s =
            nv ? dispatch_fp4<true>(w_packed, w_scales, w_tensor_scale, out, in, xq, xs,
                                    x_tensor_scale, nb, yb, ydt, workspace, workspace_bytes, st)
               : dispatch_fp4<false>(w_packed, w_scales, nullptr, out, in, xq, xs, nullptr, nb, yb,
                                     ydt, workspace, workspace_bytes, st);
        if (s != Q4_OK) return s;
    }
    return Q4_OK;
}

q4_status q4_selftest_wait_timeout(int64_t limit_ns, q4_stream stream) {
    if (limit_ns < 1 || limit_ns > 1000000000LL) return Q4_ERR_INVALID_ARG;
    selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        static_cast<uint64_t>(limit_ns));
    return launch_status(cudaSuccess);
}

q4_status q4_sync_status(q4_stream stream) {
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return Q4_ERR_CUDA;
    unsigned h = 0;
    if (cudaMemcpyFromSymbol(&h, g_q4_status, sizeof(h)) != cudaSuccess) return Q4_ERR_CUDA;
    if (h != 0) {
        const unsigned zero = 0;
        if (cudaMemcpyToSymbol(g_q4_status, &zero, sizeof(zero)) != cudaSuccess)
            return Q4_ERR_CUDA;
        if (h & kStatusTimeout) {
            noalloc_mark_reclear();
            return Q4_ERR_TIMEOUT;
        }
        if (h & (kStatusBadIndex | kStatusRange)) return Q4_ERR_INVALID_ARG;
    }
    return cudaGetLastError() == cudaSuccess ? Q4_OK : Q4_ERR_CUDA;
}

}  // extern "C"
