/*
 * awq.h - C ABI of the B200 (sm_100a) AWQ group-wise W4A16 library.
 *
 * The operations are the per-layer core of activation-aware weight quantisation
 * (AWQ) as the pages describe it:
 *   - "AI-Research-SKILLs AWQ advanced usage guide" (lshu.cn), section 算法原理:
 *     the objective L(s) = || Q(W*s)(s^-1*X) - W*X || over a per-input-channel
 *     scale s derived from activation statistics; salient channels are protected
 *     by scaling, with no mixed precision;
 *   - same page, section 量化超参数调优 (group size and zero-point choices) and
 *     section "WQLinear kernels" (GEMM for batches, GEMV for a single token);
 *   - "Optimization Awq" (skillsdirectory.com), the quant_config block
 *     {"zero_point", "q_group_size", "w_bit": 4, "version": "GEMM" | "GEMV"}.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Types.    fp16 tensors are passed as `uint16_t*` holding IEEE binary16 bit
 *           patterns; packed codes as `uint32_t*`.  No CUDA or framework type
 *           appears in a signature: `stream` is a `cudaStream_t` passed as
 *           `void*` (NULL = the legacy default stream).
 * Memory.   Every tensor pointer is DEVICE memory owned by the caller unless the
 *           argument says "host".  The library never allocates, frees or keeps a
 *           pointer after the call returns; scratch space comes from the caller
 *           through (ws, ws_bytes), sized by awq_workspace_bytes().
 * Layout.   Row-major, innermost index contiguous:
 *             W       [N][K] fp16      (out_features x in_features; y = X W^T)
 *             X, Y    [M][K] / [M][N] fp16
 *             qweight [N][K/8] uint32: the 4-bit code of (n, k) sits in bits
 *                     4*(k%8) .. 4*(k%8)+3 of word k/8 (little-endian nibbles)
 *             scales  [N][K/G] fp16
 *             qzeros  [N][ceil((K/G)/8)] uint32, same nibble order, unused
 *                     nibbles 0; NULL when zero_point is 0 (implicit zero 8)
 *           Every pointer must be 16-byte aligned; K must be a multiple of G.
 * Async.    Calls enqueue work on `stream` and return without synchronising.
 * Errors.   Argument errors are detected on the host, before anything is
 *           launched, and return AWQ_ERR_INVALID_ARG / AWQ_ERR_UNSUPPORTED /
 *           AWQ_ERR_WORKSPACE.  A failed launch returns AWQ_ERR_CUDA.  Device-side
 *           waits are bounded: a wait that runs out sets a device error word
 *           and the kernel returns; awq_device_error() reports it as
 *           AWQ_ERR_TIMEOUT (or AWQ_ERR_RANGE for the fp16 limit of
 *           awq_linear_gemm).  NaN or Inf in W or X propagate into the outputs.
 */
#ifndef AWQ_B200_H
#define AWQ_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* quant_config of the pages: w_bit must be 4, q_group_size one of 32/64/128/256,
 * zero_point 1 = asymmetric (per-group zero), 0 = symmetric (implicit zero 8). */
typedef struct awq_quant_config {
    int32_t w_bit;
    int32_t q_group_size;
    int32_t zero_point;
} awq_quant_config;

typedef enum awq_status {
    AWQ_OK = 0,
    AWQ_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size */
    AWQ_ERR_UNSUPPORTED = 2,   /* valid but not handled (w_bit != 4, group size, M too large for GEMV) */
    AWQ_ERR_WORKSPACE = 3,     /* ws too small (see awq_workspace_bytes) */
    AWQ_ERR_CUDA = 4,          /* a CUDA runtime/driver call or launch failed */
    AWQ_ERR_TIMEOUT = 5,       /* a bounded device wait ran out (see awq_device_error) */
    AWQ_ERR_RANGE = 6          /* awq_linear_gemm met a group whose fp16 dequantised weights
                                  overflow (see awq_linear_gemm; reported by awq_device_error) */
} awq_status;

/* Operation ids for awq_workspace_bytes. */
enum {
    AWQ_OP_QUANTIZE_PACK = 0,
    AWQ_OP_SCALE_SEARCH = 1,
    AWQ_OP_GEMV = 2,
    AWQ_OP_GEMM = 3
};

/* Static string for a status code; never NULL. */
const char* awq_status_string(awq_status status);

/* ABI version of this header (increases on incompatible change). */
int32_t awq_abi_version(void);

/*
 * Group-wise 4-bit quantisation and packing of ws = W * diag(s).
 * Source: lshu.cn guide, 量化超参数调优 (group size, zero-point); quant_config
 * block of "Optimization Awq".  Per row n and group g of G input channels, in
 * IEEE fp32 with round-half-even rint:
 *   zero_point=1: scale = max((max-min)/15, 1e-5) rounded to fp16 (scale16),
 *                 zero  = clamp(rint(-min/scale16), 0, 15),
 *                 q     = clamp(rint(ws/scale16) + zero, 0, 15)
 *   zero_point=0: scale = max(max|ws|/7, 1e-5) rounded to fp16,
 *                 q     = clamp(rint(ws/scale16), -8, 7) + 8
 * ws = fp32(W)*fp32(s) is exact.  s may be NULL (s = 1: plain round-to-nearest).
 * W [N][K], s [K] -> qweight [N][K/8], scales [N][K/G], qzeros (zero_point=1 only).
 * Needs no workspace.  N, K > 0.  Ends with an ordering kernel on `stream`, so an
 * awq_linear_gemv may directly follow it (see the ordering note there).
 */
awq_status awq_quantize_pack(const uint16_t* W, const uint16_t* s, int32_t N, int32_t K,
                             awq_quant_config cfg, uint32_t* qweight, uint16_t* scales,
                             uint32_t* qzeros, void* stream);

/*
 * Activation-aware scale search (lshu.cn guide, 算法原理): for alpha_i = i/n_grid,
 * i = 0 .. n_grid-1, with m_k = mean_t |X[t][k]| (exact, fp64) and
 * s_i = fp16(max(pow(m_k, alpha_i), 2^-14)), evaluate
 *   loss_i = mean_{t,n} ( sum_k X[t][k] * (Q(W s_i)/s_i - W)[n][k] )^2
 * where Q is the group quantiser of awq_quantize_pack with the same cfg, and keep
 * the smallest (ties to the smaller alpha).  Writes s_out [K] fp16 = s of the
 * best alpha; losses_out [n_grid] fp64 and best_index_out [1] int32 are DEVICE
 * pointers and may be NULL.  alpha* = best_index / n_grid.
 * X [M][K] are the calibration activations (M >= 1 tokens), W [N][K].
 * 1 <= n_grid <= 64.  ws_bytes >= awq_workspace_bytes(AWQ_OP_SCALE_SEARCH, M, N, K, cfg)
 * (a few MB: statistics, the s table, per-tile partial sums; Q(Ws)/s - W is built
 * tile by tile in shared memory and never stored).
 * Every fp32 product of the loss uses X exactly and Q(Ws)/s - W (scaled by a power of
 * two per alpha) split into two fp16 terms (22-bit significand), accumulated in fp32
 * on the tensor cores and summed in fp64.
 * Results stay on the device and the call is asynchronous like the others (the host
 * reads best_index_out when it needs alpha; nothing here synchronises the stream).
 */
awq_status awq_scale_search(const uint16_t* X, int32_t M, const uint16_t* W, int32_t N,
                            int32_t K, awq_quant_config cfg, int32_t n_grid, uint16_t* s_out,
                            double* losses_out, int32_t* best_index_out, void* ws,
                            size_t ws_bytes, void* stream);

/*
 * The scale search with duo scaling (lshu.cn guide, 校准参数全景: duo_scaling, "scale
 * weights and activations"): the same grid, loss, tie rule, outputs and workspace as
 * awq_scale_search, with the scale of alpha_i taken from both statistics,
 *   s_i = fp16(min(max(max(pow(m_k, alpha_i), 2^-14) / max(pow(w_k, 1 - alpha_i), 2^-14),
 *                      2^-14), 65504)),   w_k = mean_n |W[n][k]| (fp64),
 * all in fp64 with one rounding to fp16 (with w = 1 it is the plain search's s).
 */
awq_status awq_scale_search_duo(const uint16_t* X, int32_t M, const uint16_t* W, int32_t N,
                                int32_t K, awq_quant_config cfg, int32_t n_grid, uint16_t* s_out,
                                double* losses_out, int32_t* best_index_out, void* ws,
                                size_t ws_bytes, void* stream);

/*
 * Weight clipping chosen by the output error (lshu.cn guide, 校准参数全景: apply_clip,
 * clip the weights to further reduce the effect of outliers on the quantisation error),
 * then group quantisation and packing of the clipped weights.  With ws = W * diag(s)
 * (s from the scale search; NULL = 1), for every output channel n, group g and clip ratio
 * r_j = fl32(1 - j/n_grid), j = 0 .. n_clip-1:
 *   c_j = fl32(r_j * max|ws| over the group),  Q_j = the quantiser of awq_quantize_pack
 *   applied to clamp(ws, -c_j, c_j),
 *   err_j = sum_t ( sum_{k in g} X[t][k] * (Q_j/s - W)[n][k] )^2
 * (the objective's share of that group; X the calibration activations as given to the
 * search).  Each group keeps the j with the smallest err_j (ties to the smaller j, i.e.
 * less clipping) and is written into qweight/scales/qzeros clipped at it, in the layout of
 * awq_quantize_pack; clip_index_out [N][K/G] uint8 (DEVICE, may be NULL) receives j and
 * err_out [N][K/G][n_clip] fp64 (DEVICE, may be NULL) every err_j.
 * 1 <= n_clip <= min(n_grid, 32).  ws_bytes >= awq_apply_clip_workspace_bytes(...).
 * err_j is evaluated on the tensor cores: Q_j/s - W split into two fp16 terms (22-bit
 * significand), X exact, fp32 accumulation over the group, squares summed in fp32 per 16
 * tokens and in fp64 beyond.  Ends with an ordering kernel (see awq_linear_gemv).
 */
awq_status awq_apply_clip(const uint16_t* X, int32_t M, const uint16_t* W, const uint16_t* s,
                          int32_t N, int32_t K, awq_quant_config cfg, int32_t n_grid,
                          int32_t n_clip, uint32_t* qweight, uint16_t* scales, uint32_t* qzeros,
                          uint8_t* clip_index_out, double* err_out, void* ws, size_t ws_bytes,
                          void* stream);

/* Workspace bytes of awq_apply_clip (0 for invalid sizes). */
size_t awq_apply_clip_workspace_bytes(int32_t M, int32_t N, int32_t K, awq_quant_config cfg,
                                      int32_t n_clip);

/*
 * Activation side of the scaling (lshu.cn guide, 算法原理: "s^-1 * X"):
 * X_out[m][k] = fp16(fp32(X[m][k]) / fp32(s[k])), IEEE division, round to nearest.
 * The linear entry points take activations already divided this way (in a model
 * the division folds into the preceding normalisation).  X_out may equal X.
 */
awq_status awq_fold_inverse_scale(const uint16_t* X, const uint16_t* s, int32_t M, int32_t K,
                                  uint16_t* X_out, void* stream);

/*
 * Fused dequantising linear, single-token / small-batch form ("GEMV", the pages'
 * WQLinear_GEMV: batch 1 decode).  Y[m][n] = fp16( sum_k X[m][k] *
 * (q[n][k] - zero[n][k/G]) * scale16[n][k/G] ), products exact, fp32 accumulation.
 * 1 <= M <= 8: the batch is the n = 8 side of the m16n8k16 tensor-core fragment the
 * kernel multiplies with, so M up to 8 costs the same weight traffic as M = 1; larger
 * batches belong to awq_linear_gemm (M > 8 returns AWQ_ERR_UNSUPPORTED).  The M rows
 * of X are staged in shared memory; when M * K * 2 bytes do not fit (e.g. 8 x 14336) the
 * batch is processed in parts, one launch each, each streaming the weights once.
 * Needs no workspace (ws may be NULL).
 * Ordering: the kernel is launched as a programmatic dependent of the previous kernel
 * on `stream` and starts streaming qweight/scales/qzeros before that kernel has
 * completed; it reads X only after it.  So the kernel immediately before it on the
 * stream must not write the weights.  awq_quantize_pack ends with an ordering kernel
 * of its own, so a GEMV may follow it directly; any other writer of the weights must
 * be followed by some other stream work (a kernel, a copy, an event wait) first.
 */
awq_status awq_linear_gemv(const uint16_t* X, int32_t M, const uint32_t* qweight,
                           const uint16_t* scales, const uint32_t* qzeros, int32_t N, int32_t K,
                           awq_quant_config cfg, uint16_t* Y, void* ws, size_t ws_bytes,
                           void* stream);

/*
 * Fused dequantising linear, batched / prefill form ("GEMM", the pages'
 * WQLinear_GEMM, the default for batch > 1).  Same result definition as
 * awq_linear_gemv; the weight tile is dequantised to fp16 ((q-zero)*scale16,
 * one rounding) in shared memory and multiplied on the tcgen05 tensor cores with
 * fp32 accumulation in tensor memory.  Any M >= 1.
 * Workspace: when the batch gives fewer 128-channel tiles than the GPU has SMs, the
 * kernel splits K into up to awq_workspace_bytes(AWQ_OP_GEMM, ...) / (4 M N) parts whose
 * fp32 partial sums go to ws and are added in a fixed order into Y (one fp16 rounding);
 * ws may be NULL (or small), which only disables the split.  ws must not be used by two
 * calls at once.
 * Range: each dequantised weight is rounded once to fp16, so it must be finite there:
 * max|q - zero| * scale16 < 65520 for every group (max|q - zero| is max(zero, 15 - zero),
 * or 8 without zero point).  awq_quantize_pack gives that whenever the group's scaled
 * weights stay within about +-61000.  A group beyond it sets the device error word and
 * the next awq_device_error() returns AWQ_ERR_RANGE (Y is then not meaningful);
 * awq_linear_gemv has no such limit (it applies scales in fp32).
 */
awq_status awq_linear_gemm(const uint16_t* X, int32_t M, const uint32_t* qweight,
                           const uint16_t* scales, const uint32_t* qzeros, int32_t N, int32_t K,
                           awq_quant_config cfg, uint16_t* Y, void* ws, size_t ws_bytes,
                           void* stream);

/*
 * awq_scale_search without a workspace argument, for callers that cannot allocate
 * device memory when they quantise (an allocator-less runtime, a memory pool that
 * is already fully carved up, a process that must not grow after start-up).  The
 * pages have no counterpart: this is a property of this library, not of the method.
 *
 * Scratch lives in a fixed 12 MiB device array inside the library; every device
 * that loads the library holds it until the process exits.  The result is the one
 * awq_scale_search defines; only the order in which the loss is summed differs
 * (one alpha and one chunk of output channels at a time), so losses agree to
 * rounding.  Limits: K <= 16384 and M <= 2^20 (larger sizes return
 * AWQ_ERR_UNSUPPORTED before anything is launched); any N.
 * The first call on a device looks up the array's device address (with that device
 * current); make that first call before any stream capture.  All calls on a
 * device share the array and it keeps the last call's contents: calls that can
 * overlap on the GPU (different streams, no ordering) race and must not be made.
 * Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 */
awq_status awq_scale_search_noalloc(const uint16_t* X, int32_t M, const uint16_t* W, int32_t N, int32_t K,
                                    awq_quant_config cfg, int32_t n_grid, uint16_t* s_out, double* losses_out,
                                    int32_t* best_index_out, void* stream);

/* Workspace bytes an operation needs for the given sizes (0 = none). */
size_t awq_workspace_bytes(int32_t op, int32_t M, int32_t N, int32_t K, awq_quant_config cfg);

/*
 * Synchronises `stream`, then reads and clears the device error word of the
 * current device: AWQ_ERR_TIMEOUT if a bounded device wait ran out since the
 * last call, else AWQ_ERR_RANGE if awq_linear_gemm met a group outside its fp16
 * range, AWQ_ERR_CUDA if the synchronisation itself failed, else AWQ_OK.
 * The library keeps per-device state (launch plans, tensor maps, the address of the
 * fixed scratch array): after cudaDeviceReset on a device, reload the library
 * before calling it again on that device.
 */
awq_status awq_device_error(void* stream);

/*
 * Diagnostic of the bounded device waits: enqueues on `stream` one small kernel whose
 * mbarrier wait can never complete (nothing arrives on the barrier).  The wait gives
 * up after the library's limit (2 s), the kernel sets the device error word and
 * returns, so the next awq_device_error() reports AWQ_ERR_TIMEOUT and the context
 * stays usable.  Lets a caller check, on its GPU, that a stalled pipeline of this
 * library ends with an error status instead of a hang.  No counterpart in the pages.
 * Returns AWQ_OK once enqueued, AWQ_ERR_CUDA if the launch fails.
 */
awq_status awq_check_bounded_wait(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* AWQ_B200_H */
