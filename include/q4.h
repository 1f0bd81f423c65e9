/*
 * q4.h -- C ABI of the group-wise INT4 weight quantization and W4A16 decode
 * library for NVIDIA B200 (sm_100a).
 *
 * The operations are those of the pages this library follows:
 *
 *   affine quantization  q = clamp(round(w / s) + z, qmin, qmax),
 *   dequantization       w_hat = s * (q - z),
 *     -- "LLM 后训练量化深度实战" (ybb.press), section 二, first equation;
 *        arganzheng.life post-training-quantization-gptq-awq-and-rotation,
 *        section 二.2 (基本形式与粒度);
 *   symmetric scale s = max|w| / 7 (z = 0, codes in [-8, 7]) and asymmetric
 *   scale s = (max - min) / 15 with integer zero point z (codes in [0, 15]),
 *     -- arganzheng.life section 二.2; ybb.press section 二
 *        (quantize_per_group: groups of group_size along in_features);
 *   the decode product of W4A16: packed INT4 weights plus per-group scale /
 *   zero are read from HBM, dequantised on chip and multiplied with 16-bit
 *   activations, y = x W_hat^T,
 *     -- arganzheng.life section 二.1 (decode GEMM [B, k] x [k, n]) and
 *        section 二.3 (W4A16 dataflow: shift, mask, x s, + z on chip).
 *
 * Beside the INT4 path: the per-group range (clipping) search and act order
 * of the INT4 quantizer (arganzheng.life sections 三.2, 五.3, 九.2);
 * per-output-channel INT8 weights and their W8A16 product
 * ("量化：PTQ、GPTQ、AWQ 与 SmoothQuant" (charles2530.github.io) section 13);
 * INT8 and INT4 KV-cache quantization ("压缩算法" (cs-knowledge-wiki)
 * sections 7.4.1.1-7.4.1.2); and the FP4 microscaling formats MXFP4 and
 * NVFP4 (arganzheng.life sections 九.1-九.2).  Each is documented at its
 * declaration below.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every pointer argument is a DEVICE pointer (except `w`, the q4_weight
 *    descriptor, which is a host struct passed by pointer and read during the
 *    call only).  The caller owns all memory.  The library never allocates,
 *    frees or synchronizes (except q4_sync_status and the first
 *    q4_gemv_noalloc call per device) and enqueues all of its work on
 *    `stream` (a cudaStream_t; NULL = the legacy default stream).
 *  - Tensors are dense and row-major.  W and W_hat are [out, in]; x is
 *    [B, in]; y is [B, out]; scales and zeros are [out, in / group_size].
 *  - Packed codes: qweight is [out, in / 2] bytes; byte j of a row holds
 *    element 2j in its low nibble and element 2j+1 in its high nibble.
 *    Symmetric codes are stored as 4-bit two's complement (q & 0xF);
 *    asymmetric codes as unsigned 4-bit integers.
 *  - INT4 scales are fp16.  Zero points are fp16 holding integers in
 *    [0, 15]; zeros == NULL if and only if symmetric.  (INT8 weights carry
 *    fp32 row scales, KV caches scales in their own 16-bit type, FP4 formats
 *    E8M0 / E4M3 scale bytes: see their declarations.)
 *  - Argument errors are returned synchronously and nothing is launched.
 *    Errors that happen on the device after a successful return (a bounded
 *    wait that ran out) are reported by q4_sync_status.  A CUDA launch error
 *    is returned as Q4_ERR_CUDA.
 *  - Weights or activations holding Inf / NaN give unspecified values but no
 *    fault.
 */
#ifndef Q4_H
#define Q4_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define Q4_API __attribute__((visibility("default")))
#else
#define Q4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    Q4_OK = 0,
    Q4_ERR_INVALID_ARG = 1,  /* NULL pointer, bad enum value, negative size */
    Q4_ERR_SHAPE = 2,        /* group_size does not divide in, odd sizes, B out of range */
    Q4_ERR_ALIGNMENT = 3,    /* a pointer is not aligned as the call requires */
    Q4_ERR_UNSUPPORTED = 4,  /* bits != 4, a group size or dtype this call does not take */
    Q4_ERR_CUDA = 5,         /* a CUDA runtime or launch error */
    Q4_ERR_TIMEOUT = 6,      /* a kernel's bounded wait ran out (see q4_sync_status) */
    Q4_ERR_WORKSPACE = 7     /* workspace NULL or smaller than q4_workspace_bytes() */
} q4_status;

typedef enum { Q4_F16 = 0, Q4_BF16 = 1, Q4_F32 = 2 } q4_dtype;

/* A cudaStream_t, passed as an opaque pointer so that this header needs no
 * CUDA include. */
typedef void* q4_stream;

/* A quantized weight matrix, as q4_quantize_pack writes it. */
typedef struct q4_weight {
    const uint8_t* qweight;  /* [out, in/2] packed codes, 16-byte aligned */
    const void* scales;      /* [out, in/group_size] fp16, 2-byte aligned */
    const void* zeros;       /* [out, in/group_size] fp16 integers, NULL iff symmetric */
    int64_t out;             /* rows (output features), >= 0 */
    int64_t in;              /* columns (input features, the reduction dim), > 0 */
    int32_t group_size;      /* codes sharing one scale along `in` */
    int32_t bits;            /* must be 4 */
    int32_t symmetric;       /* 1: codes in [-8, 7], z = 0;  0: codes in [0, 15] */
} q4_weight;

/*
 * Group-wise INT4 round-to-nearest quantization and packing of W [out, in].
 *
 * For each row r and group j (elements k in [j*g, (j+1)*g)), in fp32:
 *   symmetric:  s = fp16(max|w| / 7);          q = clamp(rne(w / s), -8, 7)
 *   asymmetric: s = fp16((max - min) / 15);   z = clamp(rne(-min / s), 0, 15)
 *               q = clamp(rne(w / s) + z, 0, 15)
 * where rne rounds half to even, the divisions are IEEE fp32 divisions, and
 * the stored fp16 scale is the one used to compute the codes.  A group whose
 * stored scale is 0 gets codes 0 (and z = 0).  (Sources: ybb.press section
 * 二 quantize_per_group; arganzheng.life section 二.2; "压缩算法"
 * (cs-knowledge-wiki) section 7.4.1.2, pack_int4.)
 *
 *   W          [out, in] fp16 or bf16 (w_dtype), 16-byte aligned
 *   group_size even, divides `in`; any even value is accepted
 *   bits       must be 4, else Q4_ERR_UNSUPPORTED
 *   qweight    [out, in/2] output, 4-byte aligned
 *   scales     [out, in/group_size] fp16 output, 2-byte aligned
 *   zeros      [out, in/group_size] fp16 output; NULL iff symmetric
 * `in` must be a multiple of 8.  Results are bit-identical to the CPU oracle.
 */
Q4_API q4_status q4_quantize_pack(const void* W, q4_dtype w_dtype, int64_t out, int64_t in,
                           int32_t group_size, int32_t bits, int32_t symmetric,
                           uint8_t* qweight, void* scales, void* zeros, q4_stream stream);

/*
 * Act-order quantization ("post-training-quantization-gptq-awq-and-rotation"
 * (arganzheng.life) section 五.3: GPTQ's desc_act quantizes the columns in the
 * order of decreasing input-channel variance, and kernels then need the
 * reorder index g_idx).  The columns are taken in the order perm[0],
 * perm[1], ...: groups are g consecutive positions of that order and codes,
 * scales (and zeros) are stored in it, i.e. this is q4_quantize_pack of
 * W[:, perm]; g_idx[perm[j]] = j / g.  The product of such a weight with x
 * is the product of the stored weight with x[:, perm]
 * (q4_permute_activations, then q4_gemv / q4_gemm_skinny).
 *   perm  int32 [in], a permutation of [0, in), 4-byte aligned; an entry
 *         outside [0, in) is clamped and the next q4_sync_status returns
 *         Q4_ERR_INVALID_ARG (nothing is read out of bounds).
 *   W may be 2-byte aligned; other arguments and errors as q4_quantize_pack.
 */
Q4_API q4_status q4_quantize_pack_perm(const void* W, q4_dtype w_dtype, int64_t out, int64_t in,
                                       int32_t group_size, int32_t bits, int32_t symmetric,
                                       const int32_t* perm, uint8_t* qweight, void* scales,
                                       void* zeros, q4_stream stream);

/*
 * The gather of act order (arganzheng.life section 九.2: the g_idx reorder is
 * a gather): x_perm[b, j] = x[b, perm[j]] for a [rows, in] fp16 or bf16
 * matrix.  x 2-byte aligned, x_perm 16-byte aligned, `in` a multiple of 8;
 * perm as for q4_quantize_pack_perm (out-of-range entries clamped and
 * reported by q4_sync_status as Q4_ERR_INVALID_ARG).
 */
Q4_API q4_status q4_permute_activations(const void* x, q4_dtype x_dtype, int64_t rows, int64_t in,
                                        const int32_t* perm, void* x_perm, q4_stream stream);

/*
 * Symmetric group-wise INT4 quantization with a per-group range (clipping)
 * search ("post-training-quantization-gptq-awq-and-rotation" (arganzheng.life)
 * section 三.2, 裁剪与舍入的权衡: scan ranges alpha from 0.8 to 1.0 of max|w|
 * and keep the one with the smallest error).  Candidates
 *   alpha_j = amax (K - j) / K,   j = 0 .. n_alpha-1,   K = 5 (n_alpha - 1),
 *   s_j = fp16(amax (K - j) / (7 K))   (IEEE fp32 division),
 *   q = clamp(rne(w / s_j), -7, 7)     (the section's symmetric grid),
 *   E_j = sum over the group of (w - s_j q)^2 in fp64;
 * candidate j replaces the best only if E_j < E_best (1 - 1e-12) (ties keep
 * the wider range).  n_alpha = 1 is q4_quantize_pack's symmetric RTN exactly.
 *   W        [out, in] fp16 or bf16, 16-byte aligned; `in` a multiple of 8
 *   group_size one of 8, 16, 32, 64, 128, 256 (else Q4_ERR_UNSUPPORTED),
 *            dividing `in` (else Q4_ERR_SHAPE)
 *   n_alpha  1 .. 64 (else Q4_ERR_INVALID_ARG)
 *   qweight  [out, in/2] uint8, 4-byte aligned; scales [out, in/g] fp16.
 * The output is a symmetric q4_weight for q4_dequant / q4_gemv / q4_gemm_skinny.
 * Errors of the summation order are below the tie margin, so the chosen
 * range matches the CPU reference except on ties within 1e-12.
 */
Q4_API q4_status q4_quantize_pack_clip(const void* W, q4_dtype w_dtype, int64_t out, int64_t in,
                                       int32_t group_size, int32_t n_alpha, uint8_t* qweight,
                                       void* scales, q4_stream stream);

/*
 * Dequantization W_hat = s * (q - z), [out, in], in fp16, bf16 or fp32.
 * s * (q - z) is exact in fp32; fp16 / bf16 outputs are that value rounded
 * to nearest even.  (ybb.press section 二; arganzheng.life section 二.2.)
 * Any even group size dividing `in`; `in` a multiple of 8; W_hat 16-byte
 * aligned.
 */
Q4_API q4_status q4_dequant(const q4_weight* w, void* W_hat, q4_dtype out_dtype, q4_stream stream);

/*
 * Bytes of device workspace that q4_gemv / q4_gemm_skinny need for a weight
 * of this shape and a batch B, on the current device (an upper bound that
 * depends on the device's SM count and on B).  0 for invalid arguments.
 * Layout, the same for every shape, batch and kernel: 256 KiB of per-row-tile
 * counters, then fp32 partial sums.
 */
Q4_API size_t q4_workspace_bytes(int64_t out, int64_t in, int64_t B, int32_t group_size);

/*
 * Fused W4A16 decode product for small batches:
 *   y[b, r] = sum_k x[b, k] * s[r, k/g] * (q[r, k] - z[r, k/g]),   1 <= B <= 8.
 * The packed weights are streamed from HBM once; codes are unpacked to exact
 * 16-bit integers in registers, multiplied with x on the tensor cores with
 * fp32 accumulation per group, and each group's partial sum is scaled by its
 * fp32 scale (arganzheng.life section 二.2: per-group scales must be applied
 * inside the K accumulation; section 二.3: on-chip dequantization).
 *
 *   x      [B, in] bf16 or fp16 (x_dtype), 16-byte aligned
 *   y      [B, out] in y_dtype (= x_dtype or Q4_F32), 16-byte aligned
 *   group_size 32, 64 or 128 (else Q4_ERR_UNSUPPORTED); `in` a multiple of 32
 *   qweight 16-byte aligned.
 *   workspace  device scratch of at least q4_workspace_bytes(out, in, B,
 *              group_size) bytes, 256-byte aligned, ZERO-FILLED before its
 *              first use.  It holds per-row-tile counters, which every call
 *              that completes leaves at zero, and partial sums, which need no
 *              clearing; its layout is the same for every shape, so one
 *              buffer (sized for the largest shape) serves any number of calls
 *              of any shape in stream order.  Calls that may overlap on the
 *              GPU need separate buffers.  After a call that ends in
 *              Q4_ERR_TIMEOUT, re-zero it.
 * Small products (row tiles x S CTAs fit the device, S <= 8) split each
 * 128-row tile's K range over a thread-block cluster of S CTAs that add
 * their partials through distributed shared memory; those launches leave the
 * workspace untouched.  The plan depends only on the shape and the device.
 * The K reduction order is fixed, so results are bit-for-bit reproducible.
 * Summation order differs from the fp64 oracle; results agree within
 * |y - y_ref| <= 4e-3 * (|y_ref| + rms(y_ref)) (the bf16 output rounding
 * included).
 */
Q4_API q4_status q4_gemv(const q4_weight* w, const void* x, q4_dtype x_dtype, int64_t B, void* y,
                         q4_dtype y_dtype, void* workspace, size_t workspace_bytes,
                         q4_stream stream);

/*
 * The same product for batches 1 <= B <= 128 (the skinny-GEMM regime of
 * arganzheng.life section 二.4, where W4A16 turns compute-bound near
 * B = ridge / 4).  B <= 8 runs the q4_gemv kernel; 9 <= B <= 64 runs on the
 * tcgen05 tensor cores: codes unpacked to exact 16-bit integers in tensor
 * memory, activations padded to 16/32/64 columns, fp32 accumulation per
 * group, group partials scaled in fp32.  65 <= B <= 128 runs on the tcgen05
 * tensor cores with the group scale applied while unpacking: each weight
 * becomes fp16(s * (q - z)) (one fp16 rounding, relative error <= 2^-11),
 * the activations are taken in fp16 (bf16 ones are converted first, into the
 * workspace), and one fp32 accumulator spans the whole K range; an
 * activation of magnitude above 65504 (fp16's largest finite value) is then
 * reported by q4_sync_status as Q4_ERR_INVALID_ARG.  Same arguments and
 * requirements as q4_gemv (the workspace of q4_workspace_bytes for this B,
 * which for B > 64 includes room for the fp16 activations), same tolerance,
 * bit-for-bit reproducible.
 */
Q4_API q4_status q4_gemm_skinny(const q4_weight* w, const void* x, q4_dtype x_dtype, int64_t B,
                                void* y, q4_dtype y_dtype, void* workspace,
                                size_t workspace_bytes, q4_stream stream);

/*
 * Several products that share their activations -- the q, k and v
 * projections of a decoder layer, or its gate and up projections -- in one
 * call: y_i = x W_i^T for i < n, the products a decode step runs back to back
 * on one activation (arganzheng.life section 二.1: the decode step streams
 * every weight once; ybb.press section 一: the bottleneck is the HBM read).
 *   ws  n quantized weights, 1 <= n <= Q4_GROUP_MAX, all with the same `in`,
 *       group_size and symmetric flag (else Q4_ERR_SHAPE); each as in q4_gemv;
 *   x   [B, in], 1 <= B <= 128;  ys[i]  [B, ws[i].out] of y_dtype, not
 *       overlapping one another;
 *   workspace  q4_workspace_bytes(out, in, B, group_size) bytes (the size does
 *       not depend on `out` for B <= 8).
 * For B <= 8 it is one launch of the q4_gemv kernel whose stream-K range runs
 * over the products' row tiles one after another (at most 65536 tiles of 128
 * rows in all, else Q4_ERR_SHAPE), so no product pays its own launch, ramp-up
 * and tail.  The result is deterministic and within q4_gemv's tolerance; it
 * may differ from q4_gemv's in the last bits, because the split of a row
 * tile's K range between CTAs differs.  For B > 8 it runs q4_gemm_skinny once
 * per product, in order.
 */
#define Q4_GROUP_MAX 4
Q4_API q4_status q4_gemv_grouped(const q4_weight* ws, int32_t n, const void* x, q4_dtype x_dtype,
                                 int64_t B, void* const* ys, q4_dtype y_dtype, void* workspace,
                                 size_t workspace_bytes, q4_stream stream);

/*
 * Size of the static device scratch that q4_gemv_noalloc uses (3 MiB): it
 * covers every shape q4_gemv accepts on a GPU with up to 176 SMs.
 */
#define Q4_NOALLOC_SCRATCH_BYTES (3u << 20)

/*
 * q4_gemv without a caller workspace and without any allocation.  The
 * method's papers have no counterpart to this entry point: it is a
 * deployment variant for callers that cannot allocate device memory at call
 * time -- a serving engine that reserved nearly all free HBM for its KV cache
 * at start-up (a later cudaMalloc fails), a caller that must not pay the
 * device-wide synchronisation that cudaFree implies inside a decode loop,
 * and plain C hosts with no allocator to hand the library.
 *
 * Arguments, layouts, result and tolerance are those of q4_gemv (1 <= B <= 8).
 * The stream-K scratch (partial sums and per-row-tile counters) lives in a
 * static __device__ array of Q4_NOALLOC_SCRATCH_BYTES inside the library;
 * a shape whose scratch (q4_workspace_bytes) exceeds that returns
 * Q4_ERR_WORKSPACE before anything is launched.  No device memory is
 * allocated or freed, by the library or by anything it calls.
 *
 * Every call looks up the scratch address with the current device (a
 * failure returns Q4_ERR_CUDA).  The first call on each device -- and the
 * first after the device's context was destroyed and created again, which
 * gives the array a new address -- does setup: it zero-fills the scratch on
 * `stream` and waits for that stream.  Make that call before any stream
 * capture.  Completed calls leave the counters at zero;
 * after q4_sync_status has reported Q4_ERR_TIMEOUT the next call zero-fills
 * the scratch again on its stream before launching.
 *
 * All calls on one device share the one scratch: calls that may overlap on
 * the GPU (different streams, or different host threads without ordering)
 * race on it and give wrong results.  Issue them in one stream order.
 */
Q4_API q4_status q4_gemv_noalloc(const q4_weight* w, const void* x, q4_dtype x_dtype, int64_t B,
                                 void* y, q4_dtype y_dtype, q4_stream stream);

/*
 * The unquantised bf16 product y = x W^T with fp32 accumulation, a
 * baseline the INT4 path is compared against and the probe of the bandwidth
 * a weight stream reaches (ybb.press section 一, roofline_bound; arganzheng.
 * life section 二.4, BF16 vs W4A16 batch table).  W and x tiles go by TMA to
 * shared memory and straight into the tcgen05 tensor cores (fp32 accumulator
 * in tensor memory), split over a persistent grid like the INT4 products.
 *   W [out, in] bf16, x [B, in] bf16, y [B, out] bf16; `in` a multiple of 64;
 *   W, x, y 16-byte aligned; 1 <= B <= 128 (else Q4_ERR_SHAPE).
 *   workspace  at least bf16_ref_workspace_bytes(out, in, B) bytes, 256-byte
 *              aligned, zero-filled before its first use (the kernel leaves
 *              its counters zero again); the same layout as the INT4
 *              products' workspace, so one buffer serves both.
 * Deterministic: split tiles add their partials in a fixed order (through the
 * workspace, or, for B > 32 when the row tiles x S CTAs fit the device,
 * through distributed shared memory inside clusters of S CTAs).
 */
Q4_API size_t bf16_ref_workspace_bytes(int64_t out, int64_t in, int64_t B);
Q4_API q4_status bf16_gemv_ref_bw(const void* W, int64_t out, int64_t in, const void* x, int64_t B,
                                  void* y, void* workspace, size_t workspace_bytes,
                                  q4_stream stream);

/* ------------------------------------------------ per-channel INT8 weights
 *
 * "量化：PTQ、GPTQ、AWQ 与 SmoothQuant" (charles2530.github.io), section 13
 * (快速代码示例, per_channel_int8_quant): one scale per output row of
 * W [out, in], in fp32 with IEEE divisions and round-half-to-even,
 *   s[r] = max(max_k |W[r, k]|, 1e-6) / 127,   q = clamp(rne(W / s), -127, 127),
 * and w_hat = q * s.
 *
 *   W        [out, in] fp16 or bf16 (fp32: Q4_ERR_UNSUPPORTED), 16-byte aligned
 *   qweight  [out, in] int8, row-major, 16-byte aligned (written)
 *   scales   [out] fp32, 4-byte aligned (written)
 *   in       a multiple of 16 (else Q4_ERR_SHAPE); out == 0 is a no-op
 * The caller owns every buffer.  Asynchronous on `stream`.
 */
Q4_API q4_status q8_quantize_per_channel(const void* W, q4_dtype w_dtype, int64_t out, int64_t in,
                                         int8_t* qweight, float* scales, q4_stream stream);

/* W_hat[r, k] = q[r, k] * s[r] (one fp32 product), written as out_dtype
 * (rounded to nearest even for fp16 / bf16).  W_hat [out, in], 16-byte
 * aligned; same shape rules as q8_quantize_per_channel. */
Q4_API q4_status q8_dequant(const int8_t* qweight, const float* scales, int64_t out, int64_t in,
                            void* W_hat, q4_dtype out_dtype, q4_stream stream);

/* Workspace bytes q8_gemv needs for this shape (0 for invalid arguments).
 * The layout is that of q4_gemv's workspace (a zeroed counter region, then
 * partial slots), so one buffer of the larger size serves both. */
Q4_API size_t q8_workspace_bytes(int64_t out, int64_t in, int64_t B);

/*
 * W8A16 decode product y[b, r] = s[r] * sum_k q[r, k] * x[b, k] for
 * 1 <= B <= 8 (else Q4_ERR_SHAPE): a persistent stream-K kernel on 16-bit
 * tensor cores with the codes converted exactly on chip and fp32
 * accumulation; the row scale multiplies the finished sum.
 *   x   [B, in] fp16 or bf16, 16-byte aligned
 *   y   [B, out] x_dtype or fp32, 16-byte aligned
 *   in  a multiple of 16, at most 2^30; out at most 65535 * 128
 *   workspace  >= q8_workspace_bytes(out, in, B) bytes, 256-byte aligned,
 *              zero-filled once before first use (the kernel leaves it so)
 * Deterministic: the result does not depend on timing.  A bounded wait that
 * runs out is reported by q4_sync_status as Q4_ERR_TIMEOUT.
 */
Q4_API q4_status q8_gemv(const int8_t* qweight, const float* scales, int64_t out, int64_t in,
                         const void* x, q4_dtype x_dtype, int64_t B, void* y, q4_dtype y_dtype,
                         void* workspace, size_t workspace_bytes, q4_stream stream);

/* ------------------------------------------------------ FP4 microscaling
 *
 * "post-training-quantization-gptq-awq-and-rotation" (arganzheng.life),
 * sections 九.1 and 九.2: E2M1 elements {0, 0.5, 1, 1.5, 2, 3, 4, 6} x sign
 * with a small-block scale.  Codes are packed two per byte, the even element
 * in the low nibble; a code is sign << 3 | magnitude index; rounding is to
 * the nearest E2M1 value with ties to the even magnitude index, saturating at
 * 6 and keeping the sign (-0 is code 8).
 *
 * MXFP4 (one E8M0 power-of-two scale per 32 elements, the OCP rule):
 *   e = clamp(floor(log2(max |v|)) - 2, -127, 127), scale byte e + 127,
 *   q = e2m1(v * 2^-e); an all-zero block gets scale byte 0 and codes +0.
 *   W       [out, in] fp16 or bf16, 16-byte aligned; in a multiple of 32
 *   packed  [out, in/2] uint8, 4-byte aligned (written)
 *   scales  [out, in/32] E8M0 bytes (written)
 */
Q4_API q4_status mxfp4_quantize(const void* W, q4_dtype w_dtype, int64_t out, int64_t in,
                                uint8_t* packed, uint8_t* scales, q4_stream stream);

/* w_hat = e2m1(q) * 2^(scale - 127), exact in fp32, written as out_dtype
 * (W_hat [out, in], 16-byte aligned). */
Q4_API q4_status mxfp4_dequant(const uint8_t* packed, const uint8_t* scales, int64_t out,
                               int64_t in, void* W_hat, q4_dtype out_dtype, q4_stream stream);

/* NVFP4 (one E4M3 scale per 16 elements and one fp32 scale per tensor):
 *   s_t = A / 2688 (A = max |W| over the tensor; 2688 = 6 * 448; 1 if A = 0),
 *   c_b = e4m3(fp32(amax_b / 6) / s_t) rounded to nearest even, saturating
 *   at 448; S_b = fp32(e4m3(c_b) * s_t); q = e2m1(v / S_b) (IEEE fp32
 *   division), codes 0 where S_b = 0.
 *   W             [out, in] fp16 or bf16, 16-byte aligned; in a multiple of 16
 *   packed        [out, in/2] uint8, 4-byte aligned (written)
 *   scales        [out, in/16] E4M3 bytes (written)
 *   tensor_scale  one fp32 in device memory, 4-byte aligned (written; used as
 *                 scratch for the tensor maximum while the call runs)
 */
Q4_API q4_status nvfp4_quantize(const void* W, q4_dtype w_dtype, int64_t out, int64_t in,
                                uint8_t* packed, uint8_t* scales, float* tensor_scale,
                                q4_stream stream);

/* w_hat = fp32(e2m1(q) * S_b) with S_b = fp32(e4m3(c_b) * s_t), written as
 * out_dtype (W_hat [out, in], 16-byte aligned; tensor_scale a device pointer). */
Q4_API q4_status nvfp4_dequant(const uint8_t* packed, const uint8_t* scales,
                               const float* tensor_scale, int64_t out, int64_t in, void* W_hat,
                               q4_dtype out_dtype, q4_stream stream);

/* W4A4 product of two FP4 operands of the same format on the block-scaled
 * tensor cores ("post-training-quantization-gptq-awq-and-rotation"
 * (arganzheng.life), section 九.2: Blackwell multiplies microscaled FP4
 * operands natively, the block scales applied inside the MMA):
 *
 *   y[b, r] = g * sum_k e2m1(wq[r, k]) * S_w[r, k / VS] * e2m1(xq[b, k]) * S_x[b, k / VS]
 *
 *   MXFP4 (format Q4_FP4_MXFP4): VS = 32, S = 2^(byte - 127), g = 1;
 *   NVFP4 (format Q4_FP4_NVFP4): VS = 16, S = e4m3(byte),
 *                                g = w_tensor_scale * x_tensor_scale.
 *
 * Both operands are laid out as mxfp4_quantize / nvfp4_quantize write them
 * (the activations are quantized as a [B, in] matrix by the same calls):
 *   w_packed        [out, in/2] codes, 16-byte aligned
 *   w_scales        [out, in/VS] scale bytes, 16-byte aligned
 *   w_tensor_scale  one fp32 on the device (NVFP4; ignored for MXFP4)
 *   x_packed        [B, in/2] codes, 16-byte aligned
 *   x_scales        [B, in/VS] scale bytes, 16-byte aligned
 *   x_tensor_scale  one fp32 on the device (NVFP4; ignored for MXFP4)
 *   y               [B, out] in y_dtype (f16, bf16 or f32), written
 *   in              a multiple of 256 (NVFP4) or 512 (MXFP4): the scale rows
 *                   are read by TMA, whose row strides are multiples of 16 B
 *   workspace       at least fp4_gemm_workspace_bytes(format, out, in, B)
 *                   bytes, 256-byte aligned, zero-filled once before its
 *                   first use (the kernels leave it zeroed again); one call
 *                   at a time per workspace
 * Accumulation is fp32 inside the tensor core; the result is deterministic
 * (split tiles add their partials in a fixed order: through the workspace,
 * or, for B > 32 when the row tiles x S CTAs fit the device, through
 * distributed shared memory inside clusters of S CTAs).  B > 128 runs as slices
 * of 128 activation rows.  Errors: Q4_ERR_INVALID_ARG (format, dtype, null
 * pointer), Q4_ERR_SHAPE, Q4_ERR_ALIGNMENT, Q4_ERR_WORKSPACE; a device-side
 * wait that runs out sets Q4_ERR_TIMEOUT for q4_sync_status.
 */
#define Q4_FP4_MXFP4 0
#define Q4_FP4_NVFP4 1
Q4_API size_t fp4_gemm_workspace_bytes(int32_t format, int64_t out, int64_t in, int64_t B);
Q4_API q4_status fp4_gemm(int32_t format, const uint8_t* w_packed, const uint8_t* w_scales,
                          const float* w_tensor_scale, int64_t out, int64_t in,
                          const uint8_t* x_packed, const uint8_t* x_scales,
                          const float* x_tensor_scale, int64_t B, void* y, q4_dtype y_dtype,
                          void* workspace, size_t workspace_bytes, q4_stream stream);

/* --------------------------------------------------------------- KV cache
 *
 * A KV cache [batch, heads, seq, head_dim] in fp16 or bf16 is passed as
 * rows = batch * heads * seq contiguous rows of head_dim values.
 *
 * INT8 ("压缩算法" (cs-knowledge-wiki), section 7.4.1.1,
 * quantize_kv_cache_int8 / dequantize_kv_cache_int8 along the last axis):
 * one scale per row, stored in the cache's own type,
 *   s = cache_type(max |x| / 127),   q = clamp(rne(x / s), -128, 127),
 * in fp32 with the stored scale; a row whose stored scale is 0 gets codes 0.
 *   kv      [rows, head_dim], 16-byte aligned
 *   codes   [rows, head_dim] int8, 16-byte aligned (written)
 *   scales  [rows] in the cache type, 2-byte aligned (written)
 *   head_dim a multiple of 8 in [8, 512] (else Q4_ERR_SHAPE)
 */
Q4_API q4_status kv_quantize_int8(const void* kv, q4_dtype dtype, int64_t rows, int64_t head_dim,
                                  int8_t* codes, void* scales, q4_stream stream);

/* out[r, k] = cache_type(q[r, k] * s[r]), one rounding of the exact product;
 * out [rows, head_dim] 16-byte aligned, shape rules of kv_quantize_int8. */
Q4_API q4_status kv_dequant_int8(const int8_t* codes, const void* scales, q4_dtype dtype,
                                 int64_t rows, int64_t head_dim, void* out, q4_stream stream);

/* INT4 ("压缩算法" section 7.4.1.2, quantize_kv_cache_int4): the symmetric
 * group quantizer of q4_quantize_pack (s = fp16(amax / 7), codes in [-8, 7],
 * two codes per byte, even element in the low nibble) over groups of
 * group_size values along head_dim.
 *   packed  [rows, head_dim / 2], 4-byte aligned (written)
 *   scales  [rows, head_dim / group_size] fp16, 2-byte aligned (written)
 *   head_dim a multiple of 8; group_size even and dividing head_dim */
Q4_API q4_status kv_quantize_int4(const void* kv, q4_dtype dtype, int64_t rows, int64_t head_dim,
                                  int32_t group_size, uint8_t* packed, void* scales,
                                  q4_stream stream);

/* The dequantization s * q of kv_quantize_int4's output as out_dtype (the
 * rules of q4_dequant; packed 16-byte aligned). */
Q4_API q4_status kv_dequant_int4(const uint8_t* packed, const void* scales, int64_t rows,
                                 int64_t head_dim, int32_t group_size, void* out,
                                 q4_dtype out_dtype, q4_stream stream);

/*
 * Waits for `stream`, then reports the first device-side error recorded
 * since the previous call (Q4_ERR_TIMEOUT when a kernel's bounded wait ran
 * out, Q4_ERR_INVALID_ARG when a permutation entry was out of range) or a
 * pending CUDA error (Q4_ERR_CUDA), and clears the record.
 */
Q4_API q4_status q4_sync_status(q4_stream stream);

/*
 * Self-test of the bounded-wait machinery every pipelined kernel uses: one
 * CTA waits on a shared-memory barrier that nothing ever arrives on, gives up
 * after limit_ns nanoseconds (1 <= limit_ns <= 1e9, else Q4_ERR_INVALID_ARG)
 * and records the timeout; a following q4_sync_status returns
 * Q4_ERR_TIMEOUT and clears it.  No memory is touched, nothing faults, and
 * the context stays usable.  (The pages have no counterpart; this checks the
 * library's failure path without a GPU fault.)
 */
Q4_API q4_status q4_selftest_wait_timeout(int64_t limit_ns, q4_stream stream);

/* Human-readable name of a status code (static storage). */
Q4_API const char* q4_status_string(q4_status s);

/* Library version string (static storage). */
Q4_API const char* q4_version(void);

#ifdef __cplusplus
}
#endif

#endif /* Q4_H */
