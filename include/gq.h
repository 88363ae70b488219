/*
 * gq.h -- libgq: per-row / per-tensor int6 and int8 weight quantization on
 * NVIDIA B200 (sm_100a).  C ABI: plain pointers and sizes only.
 *
 * What the library computes follows the parameter-golf pages:
 *  - "SubSixteen v2: Int6 QAT + MLP 3x + SWA + Sliding Window" (PR #69),
 *    "Training Techniques / Quantization" (STE QAT, bits 6) and "Other"
 *    (straight-through estimator fake quantization in the forward pass,
 *    quant_range [-31, 31]);
 *  - "Swiglu gating_ QAT_Residual Attention Scalin _EMA- Sliding window_
 *    Optimizations for 10min/16MB Track" (PR #2159), "Key Explored
 *    Modifications" 1 (STE fake quantization), 13 (int8 export), 14 (per-row
 *    / per-tensor quantization), 15 (percentile clipping for the export),
 *    16 (small-tensor FP16 passthrough), and "Final Observed Results" (int8
 *    export validation: dequantize what was exported);
 *  - "Record: Unified Attention + FA3 + Legal TTT" (PR #1202),
 *    "Quantization" (int8 embeddings, int6 STE QAT on all weights);
 *  - "Add non-record submission: 12L 24min Vocab1792 ... Int6AWQ MixedBits"
 *    (PR #1495), "Mixed-bit quantization details" (int6 by default, tensors
 *    named in QUANT_INT8_NAME_PATTERNS promoted to int8; default list
 *    tok_emb.weight, lm_head.weight).
 *
 * The pages give no formulas.  The definitions used throughout (they are the
 * plainest readings of the pages):
 *   group    one row (GQ_PER_ROW) or the whole tensor (GQ_PER_TENSOR),
 *            n elements;
 *   k        min(n, max(1, ceil(p * n))), p * n one IEEE double multiply,
 *            p in (0, 1];
 *   clip c   the k-th smallest |w| of the group (1-indexed order statistic;
 *            p = 1 gives max |w|);
 *   qmax     31 for int6, 127 for int8 (symmetric; -32 / -128 never occur);
 *   scale    s32 = c / qmax (binary32 division).  Export mode stores
 *            h = binary16(s32) (round to nearest even) and uses s = (float)h to
 *            quantize and to dequantize; training mode uses s = s32;
 *   code     q = clamp(round_half_even(clip(w, -c, c) / s), -qmax, qmax),
 *            binary32 division; s = 0 gives q = 0;
 *   w_hat    (float)q * s (binary32 multiply; q = 0 gives +0.0); bf16 tensors
 *            are widened exactly, computed in binary32, and w_hat is rounded
 *            to bf16 (nearest even);
 *   packing  int6: 4 codes in 3 bytes, 6-bit two's complement fields, first
 *            code in the least significant bits of a little-endian 24-bit
 *            group, last group of a row zero-padded, row stride
 *            3 * ceil(cols / 4) bytes; int8: the code bytes.
 * Every output is bit-exact to that definition.
 *
 * Conventions for every entry point:
 *  - All pointers named d_* or held in gq_tensor are DEVICE pointers owned by
 *    the caller; the gq_tensor array itself is HOST memory, read during the
 *    call only.  The library allocates no memory and keeps no state beyond a
 *    cached per-device property query.
 *  - Calls are asynchronous on `stream` and never synchronize.
 *  - Argument errors are returned before anything is launched (nothing is
 *    written).  A failed launch returns GQ_ERR_CUDA.
 *  - Conditions found on the device (non-finite input, a binary16 scale
 *    overflow) are OR-ed into d_status[i] (one int32 per descriptor, nullable)
 *    as GQ_STATUS_* bits; the call clears d_status[0..n) on the stream first.
 *    The outputs of a descriptor whose status is non-zero are unspecified.
 *  - Outputs are dense row-major [rows, cols] (packed: [rows, packed row
 *    bytes]); the input may be strided (ld >= cols elements).
 *  - A tensor with rows == 0 or cols == 0 is a no-op; its pointers may be NULL.
 *  - No call synchronizes with the host, traps or asserts on the device.  The
 *    only waits on the device are the fused row kernel's waits for its own
 *    bulk copies into shared memory (and its consumers' waits for one
 *    another); each gives up after about 4 s of %globaltimer, drains the
 *    copies still in flight (again bounded), sets GQ_STATUS_TIMEOUT in the
 *    descriptor's status word and lets the launch end.
 */
#ifndef GQ_H
#define GQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported entry points (the library is built with hidden default visibility). */
#if defined(__GNUC__)
#define GQ_API __attribute__((visibility("default")))
#else
#define GQ_API
#endif

/* Same type as the CUDA runtime's cudaStream_t (NULL = legacy default stream). */
typedef struct CUstream_st* cudaStream_t;

typedef enum gq_status {
    GQ_OK = 0,
    GQ_ERR_INVALID_ARG = 1,   /* null required pointer, bad enum, p, ld, n */
    GQ_ERR_UNSUPPORTED = 2,   /* valid request this build does not serve */
    GQ_ERR_MISALIGNED = 3,    /* a pointer violates its stated alignment */
    GQ_ERR_WORKSPACE = 4,     /* workspace missing or smaller than required */
    GQ_ERR_RANGE = 5,         /* reserved (device-side: GQ_STATUS_RANGE) */
    GQ_ERR_NONFINITE = 6,     /* reserved (device-side: GQ_STATUS_NONFINITE) */
    GQ_ERR_CUDA = 7,          /* a CUDA runtime call or launch failed */
    GQ_ERR_TIMEOUT = 8        /* reserved (device-side: GQ_STATUS_TIMEOUT) */
} gq_status;

typedef enum gq_dtype { GQ_F32 = 0, GQ_BF16 = 1 } gq_dtype;
typedef enum gq_gran { GQ_PER_ROW = 0, GQ_PER_TENSOR = 1 } gq_gran;
typedef enum gq_scale_mode {
    GQ_SCALE_F32 = 0,         /* training: s = c / qmax in binary32 */
    GQ_SCALE_F16 = 1          /* export: s = (float)binary16(c / qmax) */
} gq_scale_mode;

/* Bits OR-ed into d_status[i]. */
#define GQ_STATUS_NONFINITE 0x1  /* a NaN or +-inf in the tensor */
#define GQ_STATUS_RANGE     0x2  /* binary16(c / qmax) overflowed to inf */
#define GQ_STATUS_TIMEOUT   0x4  /* a bounded wait on the device gave up */

/* Kinds returned by gq_plan_kind. */
#define GQ_KIND_RAW  0  /* not floating point: stored as is */
#define GQ_KIND_FP16 1  /* small tensor: binary16 passthrough */
#define GQ_KIND_INT8 2  /* name matched a promotion pattern: int8 per row */
#define GQ_KIND_INT6 3  /* default: int6 per row */

/*
 * One tensor of a batch.  w and every output are device pointers.
 *   w          input, row-major [rows, ld] of dtype, first cols used
 *   dtype      GQ_F32 or GQ_BF16
 *   qbits      6 or 8; 16 means binary16 passthrough (gq_export_pack only)
 *   gran       GQ_PER_ROW or GQ_PER_TENSOR
 *   p          percentile in (0, 1]; 1 = absolute maximum
 *   dq         nullable: w_hat [rows, cols], same dtype as w
 *   codes      nullable: int8 codes [rows, cols]
 *   packed     nullable: [rows, gq_packed_row_bytes(cols, qbits)] bytes;
 *              for qbits 16 it receives binary16 [rows, cols]
 *   scale_f16  nullable: binary16 scales [groups] (export mode only)
 *   scale_f32  nullable: the binary32 scale used, [groups]
 *   clip       nullable: the clip value c, [groups]
 * groups = rows for GQ_PER_ROW, 1 for GQ_PER_TENSOR.
 * Alignment: element pointers must be aligned to their element size; 16-byte
 * aligned rows take the vectorised path.
 */
typedef struct gq_tensor {
    const void* w;
    int32_t dtype;
    int32_t qbits;
    int32_t gran;
    int32_t reserved;         /* must be 0 */
    int64_t rows;
    int64_t cols;
    int64_t ld;
    double p;
    void* dq;
    int8_t* codes;
    uint8_t* packed;
    uint16_t* scale_f16;
    float* scale_f32;
    float* clip;
    /* AWQ column scaling, nullable: binary32 [cols] per-column scales t.
     * When given, the group quantized is the column-scaled weight
     * w'[r, c] = RN_dtype(w[r, c] * t[c]) (one binary32 multiply; a bf16
     * weight is then rounded to nearest even bf16), and clip, scales, codes,
     * packed and dq are those of w'.  Per-row groups of gq_row_clip_select,
     * gq_fakequant_fwd, gq_fakequant_average and gq_export_pack only
     * (GQ_ERR_UNSUPPORTED with GQ_PER_TENSOR or qbits 16); 4-byte aligned.
     * The pages give no rule from activation statistics to t, so t is the
     * caller's; the activations are divided by t at inference.  Source:
     * "... Int6AWQ MixedBits" (PR #1495): "mixed-bit int6 AWQ" export and,
     * in its Community Review, activation statistics collected for AWQ
     * column scaling before post-training quantization. */
    const float* col_scale;
} gq_tensor;

/*
 * Percentile clip selection alone: writes t[i].clip (required) and, when
 * given, nothing else.  Per-tensor descriptors need workspace
 * (gq_workspace_size).  Source: percentile clipping, "Swiglu gating_ QAT_..."
 * page, Key Explored Modifications 15; per-row / per-tensor, item 14.
 */
GQ_API gq_status gq_row_clip_select(const gq_tensor* t, int n, void* d_ws,
                             size_t ws_bytes, int32_t* d_status,
                             cudaStream_t stream);

/*
 * STE fake-quant forward: clip, scale, round, clamp, dequantize.  t[i].dq is
 * required; codes, clip, scale_f32 (and scale_f16 in GQ_SCALE_F16 mode) are
 * optional extra outputs; packed must be NULL; qbits 6 or 8.  Source: "STE
 * QAT bits 6" and quant_range [-31, 31] ("SubSixteen v2", sections
 * "Quantization" and "Other"); "STE QAT bits 6 scope all" (PR #1202).
 */
GQ_API gq_status gq_fakequant_fwd(const gq_tensor* t, int n, gq_scale_mode mode,
                           void* d_ws, size_t ws_bytes, int32_t* d_status,
                           cudaStream_t stream);

/*
 * Averaging of quantize-dequantize snapshots (weight averaging of the
 * fake-quant weights): one binary32 running average per tensor, updated in
 * the same pass that fake-quantizes the tensor.  The snapshot x is the
 * fake-quant output w_hat as the model holds it (bf16 w_hat widened
 * exactly), as gq_fakequant_fwd would write it in the same mode.
 *   avg    device binary32 [rows, cols], dense, at least 4-byte aligned
 *          (16-byte aligned rows take the vector path); read and written
 *   kind   GQ_AVG_MEAN: a' = RN(a + RN(RN(x - a) * t)), t = RN(1 / (count + 1)),
 *          and count == 0 sets a' = x (the first snapshot);
 *          GQ_AVG_EMA:  a' = RN(RN(decay * a) + RN(c * x)), c = RN(1 - decay)
 *   decay  EMA factor in [0, 1]
 *   count  GQ_AVG_MEAN: snapshots already in avg, 0 <= count < 2^24
 * Sources: stochastic quantized weight averaging of quantize-dequantize
 * snapshots ("Record: Unified Attention + FA3 + Legal TTT" page, Novel
 * Contributions); EMA decay 0.997 and SWA every 50 steps ("SubSixteen v2"
 * page, Weight Averaging).
 */
typedef enum gq_avg_kind { GQ_AVG_MEAN = 0, GQ_AVG_EMA = 1 } gq_avg_kind;

typedef struct gq_avg {
    float* avg;
    int32_t kind;
    float decay;
    int64_t count;
} gq_avg;

/*
 * Fake-quant forward fused with the snapshot average a[i] of t[i]: t[i].dq
 * is optional (w_hat is written when given); clip, scale_f32 (and scale_f16
 * in GQ_SCALE_F16 mode) are optional; codes and packed must be NULL.
 * Argument errors as gq_fakequant_fwd, plus GQ_ERR_INVALID_ARG for a NULL
 * average of a non-empty tensor, an unknown kind, decay outside [0, 1] or
 * count outside [0, 2^24), and GQ_ERR_MISALIGNED for an average that is
 * not 4-byte aligned.
 */
GQ_API gq_status gq_fakequant_average(const gq_tensor* t, const gq_avg* a, int n,
                                      gq_scale_mode mode, void* d_ws, size_t ws_bytes,
                                      int32_t* d_status, cudaStream_t stream);

/*
 * Straight-through backward: g_w = g_out (accumulate = 0, bitwise copy) or
 * g_w = g_w + g_out (accumulate = 1, one binary32 add, rounded back to bf16
 * for GQ_BF16).  numel elements, dense.  Source: the straight-through
 * estimator of "SubSixteen v2", section "Other": the fake-quant step is
 * treated as the identity in the backward pass.
 */
GQ_API gq_status gq_ste_bwd(const void* d_g_out, void* d_g_w, gq_dtype dtype,
                     int64_t numel, int accumulate, cudaStream_t stream);

/*
 * Export: export-mode (binary16 scale) quantization with packed output.
 * qbits 6/8: packed and scale_f16 are required; dq, codes, clip, scale_f32
 * optional.  qbits 16: binary16 passthrough of w into packed (read as
 * uint16 [rows, cols]); no other output.  Source: int8 + zlib export,
 * per-row / per-tensor, percentile clipping and FP16 passthrough ("Swiglu
 * gating_ QAT_..." page, items 13-16); int6 export ("SubSixteen v2"); mixed
 * int6 / int8 export ("... Int6AWQ MixedBits", Mixed-bit quantization
 * details).
 */
GQ_API gq_status gq_export_pack(const gq_tensor* t, int n, void* d_ws,
                         size_t ws_bytes, int32_t* d_status,
                         cudaStream_t stream);

/*
 * Export without any caller-provided device memory.  The paper has no
 * counterpart: this is a convenience of this library.
 *
 * Same computation, arguments and outputs as gq_export_pack, but the scratch
 * that per-tensor groups need comes from a fixed array inside the library
 * (GQ_NOALLOC_SCRATCH_BYTES per GPU, held by every GPU that loads the library
 * until the process exits) instead of a workspace.  It is meant for callers
 * that cannot allocate device memory for a workspace: runtimes that own a
 * fixed device-memory budget and hand out only the tensors themselves, code
 * that must not trigger cudaMalloc's implicit device-wide synchronization,
 * and plain C hosts with no allocator at hand.  It calls no cudaMalloc,
 * cudaFree or other allocating routine.
 *
 *  - At most GQ_NOALLOC_MAX_PER_TENSOR per-tensor descriptors per call; a
 *    larger batch returns GQ_ERR_WORKSPACE before anything is launched.
 *  - Every call looks up the array's device address in the current context
 *    (cudaGetSymbolAddress, no allocation), so it stays valid after a
 *    cudaDeviceReset reloads the library's device code.
 *  - All calls on a device share the one array and each call clears the part
 *    it uses; calls whose work overlaps on the GPU (different streams, or
 *    different host threads without ordering) race on it.
 */
#define GQ_NOALLOC_MAX_PER_TENSOR 64
#define GQ_NOALLOC_SCRATCH_BYTES (64 * 8448)
GQ_API gq_status gq_export_pack_noalloc(const gq_tensor* t, int n,
                                        int32_t* d_status, cudaStream_t stream);

/*
 * Dequant on load: out[r, c] = (float)q[r, c] * (float)scale_f16[r] (or
 * scale_f16[0] for GQ_PER_TENSOR), codes read from packed rows of
 * gq_packed_row_bytes(cols, qbits) bytes; bitwise equal to the w_hat of the
 * export call that produced them.  Source: "Successful int8 + zlib export
 * validation" ("Swiglu gating_ QAT_..." page, Final Observed Results).
 */
GQ_API gq_status gq_dequant(const uint8_t* d_packed, const uint16_t* d_scale_f16,
                     int qbits, gq_gran gran, int64_t rows, int64_t cols,
                     void* d_out, gq_dtype out_dtype, cudaStream_t stream);

/*
 * The consuming GEMM with the dequant in its weight load:
 *   Y[m, n] = sum_k X[m, k] * W_hat[n, k],  W_hat[n, k] = bf16(RN(q[n, k] * s[n]))
 * with q the int6 / int8 codes of row n in d_packed (rows of
 * gq_packed_row_bytes(K, qbits) bytes, as gq_export_pack writes them for a
 * weight [N, K] exported per row) and s[n] = (float)scale_f16[n].  W_hat is
 * the bf16 fake-quant weight the forward pass would multiply by; it is
 * rebuilt tile by tile in tensor memory (the MMA's A operand) and never
 * written out.  Decode-sized batches (M <= 16) whose packed rows are a
 * multiple of 16 bytes long run on a register-level kernel instead: each
 * warp streams its weight rows by TMA and dequantizes them straight into
 * mma.sync fragments (the same W_hat, the same bound).
 *   d_x      bf16 [M, ldx] activations, row-major, 16-byte aligned, ldx % 8 == 0
 *   d_packed [N, gq_packed_row_bytes(K, qbits)] bytes, 16-byte aligned (4-byte
 *            aligned when the row length is not a multiple of 16 bytes)
 *   d_scale_f16 [N] binary16 bit patterns, 2-byte aligned
 *   d_y      fp32 [M, ldy] output, overwritten; 4-byte aligned, ldy >= N
 *   d_status nullable: set to 0 on the stream, then GQ_STATUS_TIMEOUT if a
 *            bounded wait on the device gave up (Y is then not valid)
 * All buffers are the caller's; the call allocates nothing, checks its
 * arguments on the host before launching, and runs asynchronously on
 * `stream` (one kernel launch, plus a memset of Y when the batch has few
 * tiles and their K ranges are split over blocks, and always on the
 * decode-sized path).
 * Products are exact (bf16 x bf16) and accumulate in binary32 in the tensor
 * cores' order (two accumulators for small batches, partial sums of split K
 * ranges added into Y), so Y is not bitwise reproducible against a sequential
 * sum: |Y - exact| <= (K/8 + 16) * 2^-24 * sum_k |X[m, k] * W_hat[n, k]|.
 * Any K: the last 64-wide stage is zero-filled.  Packed rows must be 4-byte
 * aligned in length (int6: K % 16 == 0; int8: K % 4 == 0), else
 * GQ_ERR_UNSUPPORTED; rows whose length is a multiple of 16 bytes arrive by
 * TMA, others by 4-byte copies.  Source: STE
 * fake quantization in the forward pass whose weights feed the layer's
 * matmuls ("SubSixteen v2" page, Other; PR #1202, Quantization), with the
 * int6 / int8 storage of the export (PR #1495, Mixed-bit quantization).
 */
GQ_API gq_status gq_gemm_dequant(const void* d_x, int64_t M, int64_t K, int64_t ldx, const uint8_t* d_packed,
                                 const uint16_t* d_scale_f16, int qbits, int64_t N, float* d_y, int64_t ldy,
                                 int32_t* d_status, cudaStream_t stream);

/*
 * TEST HOOK, not for production use: exercises the timeout path of the bounded
 * waits of the pipelined row kernel (the kernel behind gq_row_clip_select,
 * gq_fakequant_fwd, gq_fakequant_average and gq_export_pack for rows that
 * are 16-byte aligned with a pitch that is a multiple of 16 bytes).  The next
 * launch of that kernel from the calling host thread (and only that one)
 * gives its tile number `tile` (counted over the launch's descriptors, in
 * order) a copy that announces 16 bytes more than it transfers, so that
 * tile's barrier never completes although every issued copy does, and gives
 * up every wait after wait_ns nanoseconds (1e6 .. 4e9).  The launch then sets
 * GQ_STATUS_TIMEOUT in the status word of the descriptor that owns the tile
 * it was on, ends, and leaves the library usable; outputs of that call are
 * unspecified.  If no such launch follows, the hook stays armed.
 * GQ_ERR_INVALID_ARG for tile < 0 or wait_ns outside that range.
 * The pages have no counterpart: this is a test of the library's own
 * failure handling.
 */
GQ_API gq_status gq_test_arm_wait_expiry(int64_t tile, uint64_t wait_ns);

/*
 * GPTQ-lite: int6 / int8 export of one weight W [rows, cols] (rows = output
 * features, cols = inputs) in which each column's codes absorb the rounding
 * error of the columns before it, weighted by the Hessian H of the layer's
 * inputs.  Source: "Record: Unified Attention + FA3 + Legal TTT" (PR #1202),
 * section Quantization: "GPTQ-lite", bits 6, scope weights.  The page gives no
 * algorithm; this is the published GPTQ algorithm (Frantar et al., 2022,
 * Algorithm 1) on the export's per-row grid:
 *   - scales: exactly those of gq_export_pack on W (percentile clip of each
 *     ORIGINAL row, s = binary16(c / qmax)); GPTQ changes only the codes;
 *   - inputs whose diagonal H[j, j] is 0 are dead: H[j, j] is taken as 1 and
 *     column j of W as 0; then lambda = percdamp * mean(diag H) is added to
 *     the diagonal (the usual percdamp is 0.01);
 *   - columns are quantized left to right; column j is rounded from
 *     w~_j = w_j + sum_{i<j} (w_i - q_i s) V[i, j] / V[j, j], where V is the
 *     upper-triangular factor with H = V V^T (V^-1 is the upper Cholesky factor
 *     of H^-1 that the algorithm feeds its errors through), by the export's
 *     quantizer: clip to +-c, divide by s, round half to even, clamp;
 *   - all of it in binary64.
 * Arguments:
 *   t        one descriptor: GQ_PER_ROW, qbits 6 or 8, no col_scale, cols at
 *            most 5800; packed and scale_f16 required; dq (q * s in w's
 *            dtype), codes and clip optional; scale_f32 ignored
 *   d_H      device binary64 [cols, cols], symmetric (e.g. from
 *            gq_gptq_hessian), read only
 *   percdamp damping fraction, >= 0
 *   d_ws     device workspace of gq_gptq_workspace_size(rows, cols) bytes,
 *            256-byte aligned (clip per row, dead flags, the Cholesky factor)
 *   d_status nullable, one int32: cleared, then GQ_STATUS_NONFINITE for a
 *            non-finite weight or a Hessian that is not positive definite
 *            after damping, GQ_STATUS_RANGE for a binary16 scale overflow
 * Asynchronous on `stream`; about 2 * cols / 64 + 5 kernel launches.
 */
GQ_API size_t gq_gptq_workspace_size(int64_t rows, int64_t cols);
GQ_API gq_status gq_gptq_quantize(const gq_tensor* t, const double* d_H, double percdamp, void* d_ws,
                                  size_t ws_bytes, int32_t* d_status, cudaStream_t stream);

/*
 * GPTQ-lite of n weights in one call: the same computation and outputs as n
 * calls of gq_gptq_quantize (bitwise), but every step runs once for all the
 * weights (their chains are independent), so the launches are about
 * 2 * max(cols) / 64 + 5 per group of 64 weights instead of per weight.
 *
 *   t       [n] host array of descriptors, each as for gq_gptq_quantize
 *   d_H     [n] host array of device pointers: d_H[i] is the fp64 [cols_i,
 *           cols_i] Hessian of weight i (unused for an empty weight)
 *   d_ws    device workspace of at least gq_gptq_batch_workspace_size(t, n)
 *           bytes, 256-byte aligned; weight i takes the
 *           gq_gptq_workspace_size(rows_i, cols_i) bytes after those of the
 *           weights before it
 *   d_status  nullable, [n] int32: d_status[i] reports weight i
 * Errors as gq_gptq_quantize, checked for every weight before any launch.
 */
GQ_API size_t gq_gptq_batch_workspace_size(const gq_tensor* t, int n);
GQ_API gq_status gq_gptq_quantize_batch(const gq_tensor* t, int n, const double* const* d_H, double percdamp,
                                        void* d_ws, size_t ws_bytes, int32_t* d_status, cudaStream_t stream);

/*
 * The Hessian of GPTQ-lite from calibration inputs: H = 2 X^T X (accumulate =
 * 0) or H += 2 X^T X (accumulate = 1), binary64 [cols, cols], full symmetric.
 * d_x is fp32 or bf16 (dtype) [n, ldx] row-major, one row per token, widened
 * exactly; the products and sums are binary64.  The scale of H does not
 * change the result of gq_gptq_quantize (its damping is relative).
 */
GQ_API gq_status gq_gptq_hessian(const void* d_x, int32_t dtype, int64_t n, int64_t cols, int64_t ldx,
                                 double* d_H, int accumulate, cudaStream_t stream);

/*
 * The consuming GEMM of quantization-aware training, with the fake-quant in
 * its weight load:
 *   Y[m, n] = sum_k X[m, k] * W_hat[n, k],  W_hat[n, k] = bf16(RN(q[n, k] * s[n])),
 *   q = clamp(round_half_even(clip(w[n, k], -c[n], c[n]) / s[n]), -qmax, qmax),
 *   s[n] = c[n] / qmax (GQ_SCALE_F32) or binary16(c[n] / qmax) (GQ_SCALE_F16),
 * i.e. exactly the w_hat that gq_fakequant_fwd writes for the same weight and
 * clips (for fp32 weights, that w_hat rounded once to bf16 for the tensor
 * cores), rebuilt tile by tile in tensor memory and never written out.
 *   d_x      bf16 [M, ldx], 16-byte aligned, ldx % 8 == 0
 *   d_w      w_dtype (GQ_F32 / GQ_BF16) [N, ldw] row-major, 16-byte aligned,
 *            ldw * element size a multiple of 16
 *   d_clip   binary32 [N] row clips c, e.g. from gq_row_clip_select
 *   d_y, ldy, d_status, accumulation and error bound as gq_gemm_dequant;
 *   any K.  d_status also receives GQ_STATUS_RANGE for a binary16 scale
 *   overflow (GQ_SCALE_F16).
 * Source: STE fake quantization in the forward pass ("SubSixteen v2", Other;
 * PR #1202, Quantization: STE QAT, bits 6, scope all).
 */
GQ_API gq_status gq_gemm_fakequant(const void* d_x, int64_t M, int64_t K, int64_t ldx, const void* d_w,
                                   int32_t w_dtype, int64_t ldw, const float* d_clip, int qbits,
                                   gq_scale_mode mode, int64_t N, float* d_y, int64_t ldy, int32_t* d_status,
                                   cudaStream_t stream);

/* Device workspace bytes a batch needs (0 when it has no per-tensor group). */
GQ_API size_t gq_workspace_size(const gq_tensor* t, int n);

/* Bytes of one packed row: 3*ceil(cols/4) (qbits 6), cols (8), 2*cols (16);
 * -1 for another qbits or cols < 0. */
GQ_API int64_t gq_packed_row_bytes(int64_t cols, int qbits);

/* k = min(n, max(1, ceil(p * n))) in IEEE double; -1 if n < 1 or p not in (0, 1]. */
GQ_API int64_t gq_k_from_p(int64_t n, double p);

/*
 * Export plan for one named tensor (host only): GQ_KIND_RAW if not floating
 * point, GQ_KIND_FP16 if numel < small_numel, GQ_KIND_INT8 if any
 * comma-separated pattern (NULL: "tok_emb.weight,lm_head.weight") is a
 * substring of name, else GQ_KIND_INT6.  -1 on a bad argument.  Source:
 * "... Int6AWQ MixedBits" (Mixed-bit quantization details) and FP16
 * passthrough ("Swiglu gating_ QAT_..." item 16).
 */
GQ_API int gq_plan_kind(const char* name, const int64_t* shape, int ndim,
                 int is_float, const char* patterns, int64_t small_numel);

/* The CUDA runtime error code (cudaError_t value) behind the calling
 * thread's most recent GQ_ERR_CUDA, or 0; and its text from the runtime. */
GQ_API int gq_last_cuda_error(void);
GQ_API const char* gq_last_cuda_error_string(void);

/* Static text for a status code. */
GQ_API const char* gq_status_string(gq_status s);

#ifdef __cplusplus
}
#endif

#endif /* GQ_H */
