/*
 * binattn.h — C ABI of the BinaryAttention forward pass (and its backward) for
 * NVIDIA B200 (sm_100a).
 *
 * The method ("BinaryAttention: One-Bit QK-Attention for Vision and Diffusion
 * Transformers", technical summaries, §2 Methodology) replaces the query/key
 * dot product of softmax attention by a 1-bit one:
 *
 *   s_i = alpha_q_i * sign(q_i),  t_j = alpha_k_j * sign(k_j)
 *       (§2 "scaled binary representations"; alpha = per-token mean |x|)
 *   S_ij = <sign q_i, sign k_j> = d - 2 * popcount(q_bits_i XOR k_bits_j)
 *       (§2: similarity through XNOR and popcount instead of float multiplies)
 *   logit_ij = softmax_scale * alpha_q_i * alpha_k_j * S_ij + bias[h, i, j]
 *       (§2 "bias enhancement": a learnable dense additive bias b_ij)
 *   O_i = sum_j softmax_j(logit_i.) * V_j
 *       (§2 hardware implementation: FlashAttention2-style tiling, so the N x N
 *        matrix is never written out)
 *
 * Conventions for every call:
 *  - All tensor pointers are DEVICE pointers (cudaMalloc / torch CUDA memory)
 *    owned by the caller. The library never allocates device memory in these
 *    calls and never frees caller memory.
 *  - Layouts are row-major and contiguous, last index fastest.
 *  - bf16 tensors are passed as uint16_t bit patterns.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream). Work is
 *    enqueued asynchronously; results are valid after the stream is synchronized.
 *  - Kernels launch on the calling thread's current device (cudaSetDevice).
 *    Every pointer and the stream must belong to that device; one-time kernel
 *    set-up is done once per device.
 *  - Every call returns a binattn_status. Arguments are validated on the host
 *    before anything is launched; on any error nothing is launched and the
 *    outputs are untouched. No exception or abort crosses the ABI.
 *    binattn_last_error_message() gives a one-line detail for the calling thread.
 *  - Sizes: B, H, N >= 1; 1 <= d <= 128; B*H <= 65535; N <= 65535.
 *    All pointers must be 16-byte aligned.
 *  - Inputs containing NaN or Inf are outside the contract.
 */
#ifndef BINATTN_H
#define BINATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define BINATTN_ABI_VERSION 1

typedef enum {
    BINATTN_OK = 0,
    BINATTN_ERR_NULL = 1,        /* a required pointer is NULL                         */
    BINATTN_ERR_SHAPE = 2,       /* B, H, N or d out of range                          */
    BINATTN_ERR_DTYPE = 3,       /* unknown dtype code                                 */
    BINATTN_ERR_ALIGN = 4,       /* a pointer is not 16-byte aligned                   */
    BINATTN_ERR_UNSUPPORTED = 5, /* valid request this build cannot serve (engine/d)   */
    BINATTN_ERR_CUDA = 6,        /* a CUDA call failed (detail in last_error_message)  */
    BINATTN_ERR_TIMEOUT = 7,     /* a kernel gave up a bounded wait (device status)    */
    BINATTN_ERR_ARG = 8          /* other invalid argument (non-finite scale, engine)  */
} binattn_status;

typedef enum {
    BINATTN_F32 = 0,
    BINATTN_BF16 = 1
} binattn_dtype;

/*
 * Score engines. All give identical integer scores S_ij; they differ in the
 * hardware unit that evaluates them.
 *   AUTO      — the fastest engine for the shape (TC where supported, else SIMT).
 *   SIMT      — CUDA cores only: __popc over uint32 words for S, fp32 softmax,
 *               fp32 P.V. Any d in [1, 128]. Reference-grade GPU path.
 *   POPC_TC   — S by __popc over uint32 words in the softmax threads; P.V as a
 *               bf16 tcgen05 MMA with the accumulator in tensor memory.
 *               Needs d % 8 == 0.
 *   TC        — S by a tcgen05 MMA on +-1 operands expanded from the sign bits in
 *               shared memory (exact integer scores in an fp32 accumulator);
 *               P.V as a bf16 tcgen05 MMA. Needs d % 8 == 0. For d <= 80 (and,
 *               with a bias, N % 8 == 0) the operands are e4m3 +-1.0 and the
 *               inputs arrive by TMA; other shapes use bf16 +-1 operands.
 * (A warp-level mma.sync .b1 XOR-popc engine was measured on sm_100a and runs
 *  below __popc throughput; it is not built.)
 */
typedef enum {
    BINATTN_ENGINE_AUTO = 0,
    BINATTN_ENGINE_SIMT = 1,
    BINATTN_ENGINE_POPC_TC = 2,
    BINATTN_ENGINE_TC = 3,
    /* binattn_scores_debug only: the scores of the TC engine as a forward
     * with a bias computes them. With and without a bias the TC forward now
     * runs the same kernel, so this gives the same scores as
     * BINATTN_ENGINE_TC; the code is kept so that callers that name it still
     * work. */
    BINATTN_ENGINE_TC_BIASED = 4
} binattn_engine;

/*
 * binattn_pack — sign bits and per-token scale of Q or K (one call per tensor).
 *
 * Source: §2 scaled binary representations, s_i = mu * sign(q_i); mu read as
 * the per-token mean of |x| over the d channels (the closed-form minimiser of
 * ||x - mu * sign(x)||_2).
 *
 *   x      [B, H, N, d]  dtype `dtype` (BINATTN_F32 or BINATTN_BF16), device.
 *   bits   [B, H, N, W]  uint32, W = ceil(d / 32), device, written.
 *          Channel c of a token is bit (c % 32) of word (c / 32); the bit is 1
 *          exactly when x >= 0 (so +0.0 and -0.0 give 1). Bits for c >= d are 0.
 *          This bit format is part of the ABI.
 *   alpha  [B, H, N]     fp32, device, written: (1/d) * sum_c |x_c|, summed in
 *          fp32 (order of summation unspecified; relative error ~1e-6).
 */
int binattn_pack(const void *x, int dtype, int B, int H, int N, int d,
                 uint32_t *bits, float *alpha, void *stream);

/*
 * binattn_forward — O = softmax(logits) V with binary scores (engine AUTO).
 *
 * Source: §2 (all four bullets above) and the FlashAttention2-style kernel of
 * §2 hardware-aware implementation.
 *
 *   q_bits, k_bits    [B, H, N, W] uint32 from binattn_pack, device, read.
 *   alpha_q, alpha_k  [B, H, N] fp32 from binattn_pack, device, read.
 *   bias              [H, N, N] bf16 or NULL (= zero), device, read. Shared by
 *                     every batch index b. Added after scaling; not scaled.
 *   v                 [B, H, N, d] bf16, device, read.
 *   softmax_scale     finite float (usually 1/sqrt(d)).
 *   out               [B, H, N, d] bf16, device, written (round to nearest even
 *                     of the fp32 result). Must not overlap any input.
 * Numerics: S exact (integer); logits and softmax in fp32; P rounded to bf16
 * before a bf16 x bf16 -> fp32 P.V on the tensor-core engines (fp32 P on SIMT);
 * normalisation by the fp32 row sum in the epilogue.
 * No mask: every query attends to all N keys (vision / diffusion self-attention).
 * Speed: for d % 8 == 0, d <= 80 this runs the TMA-fed tensor-core pipeline,
 * except with a bias whose rows are not a multiple of 8 elements (N % 8 != 0,
 * e.g. N = 197 or 577): TMA cannot read such rows, so that call reads the bias
 * with plain loads at a few per cent of the roofline. Give such a bias a
 * workspace (binattn_forward_ws pads it per call) or store it once with padded
 * rows (binattn_forward_bias_ld_ws).
 */
int binattn_forward(const uint32_t *q_bits, const uint32_t *k_bits,
                    const float *alpha_q, const float *alpha_k,
                    const uint16_t *bias, const uint16_t *v, float softmax_scale,
                    int B, int H, int N, int d, uint16_t *out, void *stream);

/*
 * binattn_forward_workspace_bytes — device workspace that binattn_forward_ws
 * needs for this shape on the current device; 0 when binattn_forward_ws would
 * simply run binattn_forward. For the TMA-fed pipeline (d % 8 == 0, d <= 80)
 * it holds (a) a copy of the bias with rows padded to roundup(N, 8) elements
 * when N % 8 != 0 (H * N * roundup(N, 8) * 2 bytes, rounded up to 256), and
 * (b) when the 256-row pairs of the call leave a last wave at most half full
 * of the device's SMs, fp32 partial results of those R pairs, whose key tiles
 * are then split over two CTAs each (R * 512 * 2 * (d + 2) * 4 bytes). Never
 * fails; a call with no CUDA device to query gets no part (b).
 */
size_t binattn_forward_workspace_bytes(int B, int H, int N, int d, int has_bias);

/*
 * binattn_forward_ws — binattn_forward (engine AUTO) with a caller-owned
 * device workspace of binattn_forward_workspace_bytes(...) bytes: biases with
 * N % 8 != 0 run on the TMA-fed pipeline from a padded copy, and a short last
 * wave of row pairs is split by key halves (each half writes unnormalised O,
 * its row max m and row sum l; a combine kernel joins them: O = (w0 O0 +
 * w1 O1) / (w0 l0 + w1 l1), w_h = exp(m_h - max(m0, m1))). Same result as
 * binattn_forward up to fp32 rounding.
 *   workspace        device, 16-byte aligned, at least
 *                    binattn_forward_workspace_bytes(...) bytes, overwritten;
 *                    may be NULL when that size is 0.
 *   workspace_bytes  its size.
 * Errors: BINATTN_ERR_NULL / ERR_ALIGN for the workspace, BINATTN_ERR_ARG when
 * it is smaller than needed; otherwise as binattn_forward. Asynchronous on
 * `stream`; the workspace must not be reused before the call completes.
 */
int binattn_forward_ws(const uint32_t *q_bits, const uint32_t *k_bits,
                       const float *alpha_q, const float *alpha_k,
                       const uint16_t *bias, const uint16_t *v, float softmax_scale,
                       int B, int H, int N, int d, uint16_t *out,
                       void *workspace, size_t workspace_bytes, void *stream);

/*
 * binattn_forward_bias_ld_ws — binattn_forward_ws with the bias rows
 * bias_ld >= N elements apart: element (h, i, j) of the bias is
 * bias[(h * N + i) * bias_ld + j] (bf16, device, 16-byte aligned, not NULL).
 * The bias is a learned parameter, fixed across calls: a caller that stores it
 * once with bias_ld a multiple of 8 (binattn_padded_bias_ld(N)) lets the
 * TMA-fed pipeline read it as it is, so no call pads it again; with any other
 * bias_ld the rows are copied into the workspace as in binattn_forward_ws.
 * Needs d % 8 == 0 and d <= 80 when bias_ld != N (BINATTN_ERR_UNSUPPORTED
 * otherwise); bias_ld == N is binattn_forward_ws itself. Same result as
 * binattn_forward_ws on the same bias values.
 *   workspace  at least binattn_forward_bias_ld_workspace_bytes(...) bytes.
 * Source: §2 methodology, the learnable bias b_ij added before the softmax.
 */
size_t binattn_forward_bias_ld_workspace_bytes(int B, int H, int N, int d, int bias_ld);
int binattn_padded_bias_ld(int N);
int binattn_forward_bias_ld_ws(const uint32_t *q_bits, const uint32_t *k_bits,
                               const float *alpha_q, const float *alpha_k,
                               const uint16_t *bias, int bias_ld, const uint16_t *v,
                               float softmax_scale, int B, int H, int N, int d, uint16_t *out,
                               void *workspace, size_t workspace_bytes, void *stream);

/*
 * binattn_forward_static_ws — binattn_forward_ws for callers that cannot
 * allocate device memory: a plug-in or hook that is handed its buffers by a
 * host framework whose caching allocator owns the device's memory, or a
 * latency-bound loop where a cudaMalloc, which can synchronise the device,
 * is not allowed. The paper has no counterpart of this call; it is a
 * convenience of this library.
 *
 * The scratch is a file-scope __device__ array of 32 MiB (256-byte aligned)
 * inside the library, which every GPU that loads the library holds until the
 * process exits. The caller still passes every input and the output, as for
 * binattn_forward_ws. The call allocates and frees nothing, through CUDA or
 * any library.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current) and keeps it; make that
 *    first call before any stream capture that includes this call. The kept
 *    address belongs to the device's current context: after cudaDeviceReset
 *    on a device that this call has used, the library's kernel set-up and
 *    this address are stale, and the library must not be used on that device
 *    again in the same process.
 *  - Shapes whose binattn_forward_workspace_bytes exceeds 32 MiB return
 *    BINATTN_ERR_UNSUPPORTED before anything is launched (for example a bias
 *    with N % 8 != 0 and H * N * roundup(N, 8) * 2 > 32 MiB).
 *  - Every call in the process shares the one array, which keeps the last
 *    call's contents. Nothing in it needs to start at zero (each call writes
 *    what it reads), but calls whose kernels overlap on the GPU (other
 *    streams, other host threads) race on it and corrupt each other's
 *    results: serialise them (one stream, or synchronise between calls).
 * Other errors are those of binattn_forward_ws.
 */
int binattn_forward_static_ws(const uint32_t *q_bits, const uint32_t *k_bits,
                              const float *alpha_q, const float *alpha_k,
                              const uint16_t *bias, const uint16_t *v, float softmax_scale,
                              int B, int H, int N, int d, uint16_t *out, void *stream);

/*
 * binattn_forward_fused_workspace_bytes — device workspace that
 * binattn_forward_fused_ws needs for this shape and Q dtype on the current
 * device (0 when it needs none). For bf16 Q on the TMA-fed pipeline (d % 8 == 0,
 * d <= 80) it equals binattn_forward_workspace_bytes; otherwise it adds room for
 * Q's sign words and alpha_q (each part rounded up to 256 bytes).
 */
size_t binattn_forward_fused_workspace_bytes(int B, int H, int N, int d, int q_dtype, int has_bias);

/*
 * binattn_forward_fused_ws — binattn_pack of Q and binattn_forward_ws in one
 * call, with Q's binarisation done by the forward kernel itself where it can.
 *
 * Source: §2 (scaled binary representations; the forward as for
 * binattn_forward). The result is the same computation: for bf16 Q with
 * d % 8 == 0 and d <= 80, the forward kernel derives each query row's sign
 * words and alpha_q with the same device code and summation order as
 * binattn_pack, so O is bit-identical to binattn_pack followed by
 * binattn_forward_ws. Other shapes and fp32 Q run binattn_pack into the
 * workspace, then binattn_forward_ws.
 *
 *   q                 [B, H, N, d] dtype `q_dtype` (BINATTN_F32 or BINATTN_BF16),
 *                     device, read.
 *   k_bits, alpha_k   from binattn_pack of K, device, read.
 *   bias, v, softmax_scale, out: as binattn_forward.
 *   workspace         device, 16-byte aligned, at least
 *                     binattn_forward_fused_workspace_bytes(...) bytes,
 *                     overwritten; may be NULL when that size is 0.
 *   workspace_bytes   its size.
 * Errors: as binattn_forward_ws, and BINATTN_ERR_DTYPE for an unknown q_dtype.
 */
int binattn_forward_fused_ws(const void *q, int q_dtype, const uint32_t *k_bits, const float *alpha_k,
                             const uint16_t *bias, const uint16_t *v, float softmax_scale,
                             int B, int H, int N, int d, uint16_t *out,
                             void *workspace, size_t workspace_bytes, void *stream);

/* binattn_forward with an explicit score engine (binattn_engine). Returns
 * BINATTN_ERR_UNSUPPORTED when the engine cannot serve the shape. */
int binattn_forward_engine(const uint32_t *q_bits, const uint32_t *k_bits,
                           const float *alpha_q, const float *alpha_k,
                           const uint16_t *bias, const uint16_t *v, float softmax_scale,
                           int B, int H, int N, int d, uint16_t *out, int engine,
                           void *stream);

/*
 * binattn_quantize_v — the per-channel 8-bit code of V that the 8-bit P.V
 * forward multiplies by: for each (b, h, channel c),
 * scale[b,h,c] = max_j |V[b,h,j,c]| / 127 and
 * vq[b,h,j,c] = rint(V[b,h,j,c] / scale[b,h,c]) (ties to even, clamped to
 * [-127, 127]; 0 when the scale is 0), in fp32.
 *   v      [B, H, N, d] bf16, device; d % 8 == 0 (else BINATTN_ERR_UNSUPPORTED).
 *   vq     [B, H, N, d] int8, device, written.
 *   scale  [B, H, d] fp32, device, written.
 * Source: §2 hybrid quantisation (values in a per-channel 8-bit code).
 */
int binattn_quantize_v(const uint16_t *v, int B, int H, int N, int d, int8_t *vq, float *scale,
                       void *stream);

/*
 * binattn_forward_int8 — the forward with an 8-bit P.V, the pages' hybrid
 * variant: the scores, scale and bias as in binattn_forward; then
 * u_ij = rint(255 * exp(logit_ij - max_j logit_ij)) (attention coefficients on
 * [0, 1] in a static unsigned 8-bit code), V in its per-channel 8-bit code
 * (binattn_quantize_v), and O[b,h,i,c] = scale[b,h,c] * sum_j u_ij vq_jc /
 * sum_j u_ij, the products and sums exact in 32-bit integers
 * (tcgen05.mma kind::i8, the successor of mma.s32.u8.s8.s32). Two passes over
 * the keys: the first finds each row's exact max, so that no u exceeds 255
 * and no integer sum is ever rescaled. Needs d % 8 == 0 and d <= 80
 * (BINATTN_ERR_UNSUPPORTED otherwise); any N; bias [H, N, N] or NULL.
 *   workspace  device, 16-byte aligned, at least
 *              binattn_forward_int8_workspace_bytes(...) bytes (V's tiled
 *              8-bit code, its scales, the row maxima and, for N % 8 != 0, a
 *              padded copy of the bias), overwritten.
 * Source: §2 hybrid quantisation; §2 hardware-aware implementation
 * (mma.s32.u8.s8.s32).
 */
size_t binattn_forward_int8_workspace_bytes(int B, int H, int N, int d, int has_bias);
int binattn_forward_int8(const uint32_t *q_bits, const uint32_t *k_bits,
                         const float *alpha_q, const float *alpha_k,
                         const uint16_t *bias, const uint16_t *v, float softmax_scale,
                         int B, int H, int N, int d, uint16_t *out,
                         void *workspace, size_t workspace_bytes, void *stream);

/*
 * binattn_forward_sample_bias_ws — binattn_forward_ws with one bias per batch
 * entry: bias bf16 [B, H, N, bias_ld] (device, 16-byte aligned, not NULL),
 * element (b, h, i, j) at bias[((b * H + h) * N + i) * bias_ld + j], bias_ld
 * >= N. This is the context-aware form of the learnable bias: a bias computed
 * from each sample's own content differs from sample to sample, so the
 * forward takes the result of that computation, whatever it is, as a dense
 * bias per batch entry. The logit of row (b, h, i), key j is
 * softmax_scale * alpha_q * alpha_k * S_ij + bias[b, h, i, j].
 * With bias_ld % 8 == 0 the kernel reads the rows as they are; otherwise they
 * are first copied into the workspace with rows padded to 8 elements.
 *   workspace  at least binattn_forward_sample_bias_workspace_bytes(...) bytes
 *              (the padded copy, B * H * N * roundup(N, 8) * 2 bytes when
 *              bias_ld % 8 != 0, and the split tail's partials); may be NULL
 *              when that size is 0.
 * Needs d % 8 == 0 and d <= 80 (BINATTN_ERR_UNSUPPORTED otherwise);
 * BINATTN_ERR_ARG when bias_ld < N or the workspace is too small; otherwise
 * errors as binattn_forward. With the same bias in every batch entry the
 * result equals binattn_forward_ws on that bias, bit for bit.
 * Source: §2 bias enhancement (dense, position-sensitive and context-aware
 * forms of the bias are named).
 */
size_t binattn_forward_sample_bias_workspace_bytes(int B, int H, int N, int d, int bias_ld);
int binattn_forward_sample_bias_ws(const uint32_t *q_bits, const uint32_t *k_bits,
                                   const float *alpha_q, const float *alpha_k,
                                   const uint16_t *bias, int bias_ld, const uint16_t *v,
                                   float softmax_scale, int B, int H, int N, int d,
                                   uint16_t *out, void *workspace, size_t workspace_bytes,
                                   void *stream);

/*
 * binattn_forward_relpos — binattn_forward with the position-sensitive form of
 * the learnable bias instead of a dense [H, N, N] one: a relative-position
 * table. The N tokens are n_cls (0 or 1) class tokens followed by the patches
 * of a gh x gw grid in row-major order (N = n_cls + gh * gw, else
 * BINATTN_ERR_SHAPE). With R0 = (2 gh - 1)(2 gw - 1), the bias of patch query
 * i and patch key j is table[h, (y_i - y_j + gh - 1)(2 gw - 1) + x_i - x_j +
 * gw - 1]; a class query with a patch key takes table[h, R0], a patch query
 * with a class key table[h, R0 + 1], class with class table[h, R0 + 2].
 *   table      bf16 [H, R0 + 3 n_cls], device, 16-byte aligned; at most
 *              20480 entries per head (BINATTN_ERR_UNSUPPORTED beyond).
 *   workspace  at least binattn_forward_relpos_workspace_bytes(...) bytes
 *              (the split tail's partials; may be NULL when that is 0).
 * Needs d % 8 == 0 and d <= 80. The result equals binattn_forward_ws with the
 * dense bias that the table expands to, bit for bit; the table replaces the
 * dense read of H N^2 bias elements by one of H R entries per CTA.
 * Source: §2 bias enhancement (dense, position-sensitive and context-aware
 * forms of the bias are named).
 */
size_t binattn_forward_relpos_workspace_bytes(int B, int H, int N, int d);
int binattn_forward_relpos(const uint32_t *q_bits, const uint32_t *k_bits,
                           const float *alpha_q, const float *alpha_k,
                           const uint16_t *table, int gh, int gw, int n_cls,
                           const uint16_t *v, float softmax_scale, int B, int H, int N, int d,
                           uint16_t *out, void *workspace, size_t workspace_bytes, void *stream);

/*
 * binattn_backward — the gradients of the forward (binattn_forward's result,
 * with exact fp32 softmax weights) for an upstream gradient dO = dLoss/dO.
 * With c = softmax_scale, s_i = alpha_q_i * sign(q_i) and t_j = alpha_k_j *
 * sign(k_j) (the scaled binary Q and K), logit_ij = c <s_i, t_j> + bias[h,i,j]
 * and P = softmax_j(logit):
 *   dV_j = sum_i P_ij dO_i
 *   dlogit_ij = P_ij (<dO_i, V_j> - D_i),  D_i = sum_j P_ij <dO_i, V_j>
 *   ds_i = c sum_j dlogit_ij t_j,  dt_j = c sum_i dlogit_ij s_i
 *   dbias[h, i, j] = sum_b dlogit_bhij
 * The gradient stops at s and t: how it reaches q and k through sign and the
 * mean (the estimator of quantisation-aware training) is the caller's choice;
 * with the straight-through estimator dq = ds and dk = dt.
 *   q_bits, k_bits, alpha_q, alpha_k, bias, v   as binattn_forward.
 *   dO     bf16 [B, H, N, d], device.
 *   dV, ds, dt   fp32 [B, H, N, d], device, written.
 *   dbias  fp32 [H, N, N], device, written (the gradient of a zero bias when
 *          bias is NULL); NULL skips it. The sum over b runs in order b, so
 *          the result does not depend on scheduling.
 *   workspace  device, 16-byte aligned, at least
 *          binattn_backward_workspace_bytes(B, H, N, d) bytes (the row
 *          log-sum-exp and D, one float each per query row).
 * Any d in 1..128. Runs on CUDA cores. Errors as binattn_forward, plus
 * BINATTN_ERR_ARG for a workspace that is too small. Asynchronous on stream.
 * Source: §2 methodology (the forward's steps) and its training bullet
 * (quantisation-aware training with self-distillation, which needs them).
 */
size_t binattn_backward_workspace_bytes(int B, int H, int N, int d);
int binattn_backward(const uint32_t *q_bits, const uint32_t *k_bits,
                     const float *alpha_q, const float *alpha_k,
                     const uint16_t *bias, const uint16_t *v, const uint16_t *dO,
                     float softmax_scale, int B, int H, int N, int d,
                     float *dV, float *ds, float *dt, float *dbias,
                     void *workspace, size_t workspace_bytes, void *stream);

/*
 * binattn_scores_debug — writes the integer scores S [B, H, N, N] (int32,
 * device) that engine `engine` computes inside the forward pass, using the same
 * kernel and score routine. For testing only: it materialises the N x N matrix.
 * BINATTN_ENGINE_TC and BINATTN_ENGINE_TC_BIASED give the scores of the
 * kernel the TC forward runs for this shape (the TMA-fed 64-key pipeline for
 * d % 8 == 0, d <= 80; else the load-mode one).
 * Source: §2, S_ij = d - 2 * popcount(q_i XOR k_j) (identical pad bits add 0).
 */
int binattn_scores_debug(const uint32_t *q_bits, const uint32_t *k_bits,
                         int B, int H, int N, int d, int32_t *S, int engine,
                         void *stream);

/*
 * binattn_ref_bf16_forward — full-precision softmax attention on the same
 * shapes, the speed reference the binary kernel is compared against:
 * O = softmax(softmax_scale * Q K^T + bias) V with bf16 Q, K, V, bias (NULL =
 * zero), fp32 accumulation and softmax, bf16 output. Needs d % 8 == 0.
 */
int binattn_ref_bf16_forward(const uint16_t *q, const uint16_t *k,
                             const uint16_t *bias, const uint16_t *v,
                             float softmax_scale, int B, int H, int N, int d,
                             uint16_t *out, void *stream);

/*
 * binattn_ref_bf16_forward_ws — the same reference with the long-sequence
 * launch plan of binattn_forward_ws: where a short last wave of 256-row
 * pairs would leave SMs idle, those pairs run as two key halves each, joined
 * by a combine kernel, so that the reference and the binary forward are
 * timed with the same plan. Arguments as binattn_ref_bf16_forward, plus:
 *   workspace        device, caller-owned, 16-byte aligned, at least
 *                    binattn_ref_bf16_forward_workspace_bytes(B, H, N, d,
 *                    bias != NULL) bytes (it holds the halves' partial
 *                    results); may be NULL when that is 0. Contents need no
 *                    initialisation and are overwritten.
 *   workspace_bytes  its size.
 * Errors: as binattn_ref_bf16_forward; BINATTN_ERR_NULL / _ALIGN / _ARG for a
 * missing, misaligned or short workspace.
 */
size_t binattn_ref_bf16_forward_workspace_bytes(int B, int H, int N, int d, int has_bias);
int binattn_ref_bf16_forward_ws(const uint16_t *q, const uint16_t *k,
                                const uint16_t *bias, const uint16_t *v,
                                float softmax_scale, int B, int H, int N, int d,
                                uint16_t *out, void *workspace,
                                size_t workspace_bytes, void *stream);

/*
 * binattn_test_wait_timeout — test only: the binary forward on the 64-key
 * pipeline (d % 8 == 0, d <= 80; with a bias, N % 8 == 0), arguments as for
 * binattn_forward, except that its TMA producer issues nothing from key tile
 * stall_after (>= 0) on. The consumers of that stage then wait for data that
 * never comes, until their bounded waits run out (about 2 s of SM clock):
 * each CTA records BINATTN_ERR_TIMEOUT in the device status word, waits
 * (bounded) for its own tensor-core work, frees its tensor memory and
 * returns; `out` is undefined. binattn_device_status(stream) then returns
 * BINATTN_ERR_TIMEOUT and the context stays usable. The pages have no
 * counterpart of this call; it exists to test the failure path.
 */
int binattn_test_wait_timeout(const uint32_t *q_bits, const uint32_t *k_bits,
                              const float *alpha_q, const float *alpha_k,
                              const uint16_t *bias, const uint16_t *v, float softmax_scale,
                              int B, int H, int N, int d, uint16_t *out,
                              int stall_after, void *stream);

/*
 * binattn_device_status — synchronizes `stream`, then reads and clears the
 * library's device status word. Returns BINATTN_OK, or BINATTN_ERR_TIMEOUT when
 * a kernel abandoned a bounded wait (its outputs are then undefined), or
 * BINATTN_ERR_CUDA when the synchronize itself failed.
 */
int binattn_device_status(void *stream);

/* Static description of a status code. Never NULL. */
const char *binattn_strerror(int status);

/* One-line detail of the calling thread's last failed call ("" if none). */
const char *binattn_last_error_message(void);

/* BINATTN_ABI_VERSION of the loaded library. */
int binattn_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BINATTN_H */
