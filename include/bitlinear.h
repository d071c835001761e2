/*
 * bitlinear.h -- C ABI of the B200 (sm_100a) BitLinear library.
 *
 * The library computes the forward pass of a BitNet a4.8 BitLinear layer:
 * ternary {-1, 0, +1} weights stored at 2 bits, multiplied by per-token
 * quantised activations. Sources (web pages on the method):
 *   [R] "BitNet a4.8: 4-bit Activations for 1-bit LLMs", Telegram review
 *       (t.center/ru/toshoseti/992), sections "Метод" and "Эксперименты".
 *   [A] "BitNet a4.8: 4-bit Activations for 1-bit LLMs", arXiv 2411.04965
 *       summary page, section "摘要（原文）" (English abstract).
 *
 * Conventions (all entry points):
 *   - Return value: BITLINEAR_OK (0) or a negative BITLINEAR_ERR_* code.
 *     bitlinear_last_error() gives a message for the calling thread.
 *   - Argument errors are found on the host and returned before any launch.
 *   - "device" pointers are CUDA global memory owned by the caller; the
 *     library never allocates, frees or keeps them. Work is asynchronous on
 *     the given stream (NULL = legacy default stream).
 *   - bf16 values are passed as their 16-bit patterns (uint16_t).
 *   - Matrices are row-major. X is M x K (one row per token); weights are
 *     described as W [K x N] (in x out) and stored transposed and packed.
 *   - M == 0 is a valid empty call: nothing is launched.
 *   - Device pointers to TMA-read operands must be 16-byte aligned.
 *   - Launches go to the device current on the calling thread. Each kernel's
 *     shared-memory limit is raised once per device (thread-safe), so one
 *     process may drive several GPUs.
 *   - dev_status (nullable, device int): a kernel that gives up a bounded
 *     wait ORs BITLINEAR_STATUS_TIMEOUT into it and returns early; the
 *     output is then undefined. The caller zeroes it; read it with
 *     bitlinear_check_status().
 */
#ifndef BITLINEAR_H
#define BITLINEAR_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* bitlinear_stream_t; /* same type as cudaStream_t */

enum {
  BITLINEAR_OK = 0,
  BITLINEAR_ERR_INVALID_ARG = -1,
  BITLINEAR_ERR_ALIGNMENT = -2,
  BITLINEAR_ERR_UNSUPPORTED = -3,
  BITLINEAR_ERR_CUDA = -4,
  BITLINEAR_ERR_TIMEOUT = -5
};

enum { BITLINEAR_MODE_INT8 = 0, BITLINEAR_MODE_INT4 = 1, BITLINEAR_MODE_FP4 = 2 };

enum { BITLINEAR_STATUS_TIMEOUT = 1 };

/* Message for the last error returned on this thread ("" if none). */
const char* bitlinear_last_error(void);

/* Library ABI version (major * 100 + minor). */
int bitlinear_version(void);

/*
 * Offline weight preparation (HOST memory, synchronous, no GPU needed).
 * Ternary weights: [R] "Метод". The pages give no scale or rounding rule;
 * this library uses absmean per column group g:
 *   gamma_g = max((float)(sum |W[k,n]| over the group, fp64, row-major order
 *             / count), 1e-5f)
 *   W_t[k,n] = clamp(round_half_even(W[k,n] / gamma_g), -1, 1)   (fp32 divide)
 * and packs code c = W_t + 1 in {0,1,2} at 2 bits: row n of Wp holds K/4
 * bytes; the little-endian 32-bit word j covers k = 16j .. 16j+15 and holds
 * element 16j + 8h + i (h in {0,1}, i in 0..7) in bits [4i+2h, 4i+2h+2).
 *   W          fp32 [K x N] row-major (host)
 *   group_ends G increasing column ends, group_ends[G-1] == N (host); G in 1..8
 *   Wp         uint8 [N x K/4] (host, written)
 *   gamma      fp32 [G] (host, written)
 * Requires K % 16 == 0, N >= 1.
 */
int bitlinear_ternarize_pack(const float* W, int64_t K, int64_t N, const int64_t* group_ends,
                             int G, uint8_t* Wp, float* gamma);

/*
 * Per-token activation quantiser ([A] abstract: 4-bit activations on the
 * inputs of attention and FFN; [R] "Метод": INT4 or FP4, absmax INT8).
 * Per row m, in fp32: a' = max(max_k |h[m,k]|, 1e-5f), then
 *   INT8 / INT4 (Q = 127 / 7): q = clamp(rne(h * (Q / a')), -Q-1, Q) as int8
 *   FP4: v = h * (6 / a') rounded to e2m1 (nearest, ties to even, saturating
 *        at 6, sign of v kept), two per byte, even k in the low nibble
 *   xs[m] = a' / Q   (Q = 6 for FP4): the dequantisation multiplier.
 * h = x, or when up != NULL the ReLU^2-gated product ([R] "Метод": ReLU^2 in
 * the FFN gate) h = (r * r) * up with r = (x > 0 ? x : 0), all in fp32.
 *   x, up   device bf16 [M x ldx] (row stride ldx elements); up nullable
 *   q_out   device int8 [M x K] for INT8/INT4, uint8 [M x K/2] for FP4
 *   xs_out  device fp32 [M]
 * Requires K % 16 == 0, K <= 49152, ldx >= K, ldx % 8 == 0.
 */
int bitlinear_quant_act(const uint16_t* x, const uint16_t* up, int64_t M, int64_t K, int64_t ldx,
                        int mode, void* q_out, float* xs_out, bitlinear_stream_t stream);

/*
 * Top-k sparsification then INT8 ([R] "Метод": top-k with 50% sparsity on
 * the out_proj input; [A] abstract: sparsified intermediate states then
 * 8-bit quantisation). Per row: keep the k largest |x| (compared as bf16
 * magnitude bits; equal magnitudes kept lowest column first), zero the rest,
 * then the INT8 quantiser above on the sparsified row.
 *   k        0 selects ceil(K/2); values above K keep the whole row
 *   q_out    device int8 [M x K]; xs_out device fp32 [M]
 *   mask_out nullable device uint8 [M x K/8]: bit (k % 8) of byte k/8 = kept
 * Requires K % 16 == 0, K <= 16384, ldx >= K, ldx % 8 == 0.
 */
int bitlinear_topk_sparsify_i8(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, int64_t k,
                               int8_t* q_out, float* xs_out, uint8_t* mask_out,
                               bitlinear_stream_t stream);

/*
 * BitLinear GEMM, ternary weights x 8-bit integer activation codes
 * ([A] abstract; [R] "Метод"), on tcgen05 tensor cores:
 *   acc[m,n] = sum_k xq[m,k] * W_t[k,n]                (exact int32)
 *   y[m,n]   = bf16_rne((float)acc * (xs[m] * gamma[g(n)]))  (fp32 multiplies)
 *   xq         device int8 [M x K], row stride K
 *   xs         device fp32 [M]
 *   Wp         device uint8 [N x K/4] from bitlinear_ternarize_pack
 *   gamma      device fp32 [G];  group_ends HOST int64 [G] (as for the pack)
 *   y          device bf16 [M x ldy]
 * Requires K % 64 == 0, K <= 32768 (|acc| < 2^22, converted exactly to fp32),
 * N % 16 == 0, ldy >= N, ldy % 8 == 0, G in 1..8.
 * The w2a4 entry point takes INT4 codes ([-8, 7]) in int8 containers: sm_100
 * tensor cores have no 4-bit integer kind, so both run the s8 MMA.
 */
int bitlinear_gemm_w2a8(const int8_t* xq, const float* xs, const uint8_t* Wp, const float* gamma,
                        const int64_t* group_ends, int G, int64_t M, int64_t N, int64_t K,
                        uint16_t* y, int64_t ldy, int* dev_status, bitlinear_stream_t stream);
int bitlinear_gemm_w2a4(const int8_t* xq, const float* xs, const uint8_t* Wp, const float* gamma,
                        const int64_t* group_ends, int G, int64_t M, int64_t N, int64_t K,
                        uint16_t* y, int64_t ldy, int* dev_status, bitlinear_stream_t stream);

/*
 * BitLinear GEMM, ternary weights x FP4 (e2m1) activations ([R] "Метод":
 * FP4 variant; [A] abstract: INT4/FP4 kernels). acc = sum of e2m1 values x
 * W_t in fp32 (exact: multiples of 0.5 below 2^24), same epilogue as above.
 *   xf4  device uint8 [M x K/2] packed e2m1 from bitlinear_quant_act(FP4)
 * Requires K % 128 == 0 and the w2a8 requirements.
 */
int bitlinear_gemm_w2fp4(const uint8_t* xf4, const float* xs, const uint8_t* Wp,
                         const float* gamma, const int64_t* group_ends, int G, int64_t M,
                         int64_t N, int64_t K, uint16_t* y, int64_t ldy, int* dev_status,
                         bitlinear_stream_t stream);

/* The same GEMMs writing the raw accumulators instead of bf16 (for checking
 * the contraction alone): acc device int32 / fp32 [M x N], row stride N. */
int bitlinear_gemm_w2a8_acc(const int8_t* xq, const uint8_t* Wp, int64_t M, int64_t N, int64_t K,
                            int32_t* acc, int* dev_status, bitlinear_stream_t stream);
int bitlinear_gemm_w2fp4_acc(const uint8_t* xf4, const uint8_t* Wp, int64_t M, int64_t N,
                             int64_t K, float* acc, int* dev_status, bitlinear_stream_t stream);

/*
 * Decode-time BitLinear (few tokens): same inputs and result as
 * bitlinear_gemm_w2a8 for 1 <= M <= 64, with weights streamed once from HBM.
 * Requires K % 128 == 0, N % 128 == 0 and the w2a8 requirements.
 */
int bitlinear_gemv_w2(const int8_t* xq, const float* xs, const uint8_t* Wp, const float* gamma,
                      const int64_t* group_ends, int G, int64_t M, int64_t N, int64_t K,
                      uint16_t* y, int64_t ldy, int* dev_status, bitlinear_stream_t stream);

/*
 * Decode-time BitLinear with the activation quantiser fused in: the same
 * result, bit for bit, as bitlinear_quant_act(x, up, M, K, ldx, mode) followed
 * by bitlinear_gemv_w2 on its codes ([R] "Метод": INT4 codes on the q/k/v and
 * gate/up inputs, ReLU^2 gate then INT8 on the down_proj input; [A] abstract:
 * 4-bit activations), without the codes ever reaching HBM: every CTA
 * quantises the few token rows itself.
 *   x, up   device bf16 [M x ldx]; up nullable (ReLU^2 gate when given)
 *   mode    BITLINEAR_MODE_INT8 or BITLINEAR_MODE_INT4
 *   other arguments as bitlinear_gemv_w2
 * Requires 1 <= M <= 8 (BITLINEAR_ERR_UNSUPPORTED above), ldx >= K,
 * ldx % 8 == 0, x and up 16-byte aligned, and the bitlinear_gemv_w2
 * requirements.
 */
int bitlinear_gemv_w2_quant(const uint16_t* x, const uint16_t* up, int64_t ldx, int mode,
                            const uint8_t* Wp, const float* gamma, const int64_t* group_ends, int G,
                            int64_t M, int64_t N, int64_t K, uint16_t* y, int64_t ldy,
                            int* dev_status, bitlinear_stream_t stream);

/*
 * KV-cache quantiser ([R] "Эксперименты": 3-bit KV cache, the <bos> and
 * <eos> tokens kept at 4 bits). Per (token t, head h) over the head dim:
 *   a' = max(max_d |x|, 1e-5f); tokens listed in keep4_pos: Q = 7, codes in
 *   [-8, 7]; others: Q = 3, codes in [-4, 3]; code = clamp(rne(x * (Q / a')))
 *   scale[t,h] = a' / Q
 * Storage: codes3 row (t,h) = 3D/8 bytes, code + 4 as a little-endian 3-bit
 * stream (code d in bits [3d, 3d+3)); all zero for 4-bit tokens.
 * codes4 row (j,h) for the j-th listed token = D/2 bytes, code + 8, low
 * nibble first.
 *   kv         device bf16 [T x H x D]
 *   keep4_pos  device int32 [n_keep4], strictly increasing positions < T
 *              (nullable iff n_keep4 == 0)
 *   codes3     device uint8 [T x H x 3D/8]
 *   codes4     device uint8 [n_keep4 x H x D/2] (nullable iff n_keep4 == 0)
 *   scale      device fp32 [T x H]
 * Requires D in {64, 128, 256}.
 */
int kv_quant_3bit(const uint16_t* kv, int64_t T, int64_t H, int64_t D, const int32_t* keep4_pos,
                  int64_t n_keep4, uint8_t* codes3, uint8_t* codes4, float* scale,
                  bitlinear_stream_t stream);

/*
 * The same quantiser ([R] "Эксперименты") applied to the K and the V cache
 * of a layer in one launch: k_* are written exactly as kv_quant_3bit(k, ...)
 * would write them, v_* as kv_quant_3bit(v, ...), with one keep4_pos list
 * for both. Saves the second launch's ramp when both are quantised
 * together, as in a decoder layer. Same requirements, per tensor, as
 * kv_quant_3bit; the two tensors may not overlap their outputs.
 */
int kv_quant_3bit_kv(const uint16_t* k, const uint16_t* v, int64_t T, int64_t H, int64_t D,
                     const int32_t* keep4_pos, int64_t n_keep4, uint8_t* k_codes3, uint8_t* k_codes4,
                     float* k_scale, uint8_t* v_codes3, uint8_t* v_codes4, float* v_scale,
                     bitlinear_stream_t stream);

/*
 * The positions kept at 4 bits, from the token ids ([R] "Эксперименты": the
 * <bos> and <eos> tokens stay at 4 bits): every t < T whose token_ids[t]
 * equals one of special_ids, in increasing order; the list kv_quant_3bit and
 * kv_attention_3bit take.
 *   token_ids    device int32 [T]
 *   special_ids  host int32 [n_special], 1 <= n_special <= 8 (e.g. the bos
 *                and eos ids)
 *   pos_out      device int32 [T]; the first *count_out entries are written
 *   count_out    device int32 [1]
 * Runs as one block on the stream (the count is device memory: read it back
 * to size the list on the host).
 */
int kv_keep4_positions(const int32_t* token_ids, int64_t T, const int32_t* special_ids,
                       int n_special, int32_t* pos_out, int32_t* count_out,
                       bitlinear_stream_t stream);

/*
 * Decode attention over that cache ([R] "Эксперименты": the 3-bit KV cache
 * with <bos>/<eos> at 4 bits is what attention reads at inference). For
 * every query (b, h) and every cached token t < T of head h:
 *   s_t = (q[b,h] . k[t,h]) / sqrt(D),  p = softmax_t(s),
 *   out[b,h] = bf16_rne(sum_t p_t v[t,h])
 * with k, v dequantised from the kv_quant_3bit storage ((code) * scale), in
 * fp32 with an online softmax. Agrees with the fp64 result within one bf16
 * ulp plus 2^-16 (sum_t p_t |v_t| + |out|) per element (fp32 rounding of
 * the D-term scores and of the weighted sums).
 *   q          device bf16 [B x H x D]
 *   k_*, v_*   codes3 / codes4 / scale of K and V as written by kv_quant_3bit
 *              with the same keep4_pos list (codes4 nullable iff n_keep4 == 0)
 *   keep4_pos  device int32 [n_keep4], strictly increasing, n_keep4 <= 1024
 *   out        device bf16 [B x H x D]
 *   dev_status as for the GEMMs (bounded waits on the cache tiles)
 * Requires D in {128, 256}, H % 4 == 0, T >= 1, every pointer but keep4_pos
 * 16-byte aligned (codes4 only when n_keep4 > 0); B == 0 launches nothing.
 */
int kv_attention_3bit(const uint16_t* q, int64_t B, int64_t H, int64_t D, int64_t T,
                      const uint8_t* k_codes3, const uint8_t* k_codes4, const float* k_scale,
                      const uint8_t* v_codes3, const uint8_t* v_codes4, const float* v_scale,
                      const int32_t* keep4_pos, int64_t n_keep4, uint16_t* out, int* dev_status,
                      bitlinear_stream_t stream);

/*
 * Measurement helper (not part of the method): the dense tensor-pipe rate of
 * this GPU in the MMA shapes the GEMMs issue, for roofline denominators.
 * Launches one CTA pair per two SMs (kind 0, 1) or one CTA per SM (kind 2);
 * each issues 4 * iters back-to-back tcgen05 MMAs on operands resident in
 * shared memory (no unpack, no global reads) and writes the device time of
 * its stream, in ns, to ns_out[unit].
 *   kind 0: kind::i8, CTA pair, M = 256, N = 256, K = 32 (2 M N K ops each)
 *   kind 1: kind::mxf4, CTA pair, M = 256, N = 256, K = 64, unit scales
 *   kind 2: kind::i8, one CTA, M = 128, N = 256, K = 32
 *   ns_out     device uint64 [SM count] (the first *units_out entries written)
 *   units_out  host int: CTA pairs (kind 0, 1) or CTAs (kind 2) launched
 * Rate = units * 4 * iters * 2 M N K / max(ns_out).
 */
int bitlinear_tensor_peak(int kind, int iters, uint64_t* ns_out, int* units_out, int* dev_status,
                          bitlinear_stream_t stream);

/* Synchronise the stream and read *dev_status: BITLINEAR_OK, or
 * BITLINEAR_ERR_TIMEOUT if a kernel gave up a bounded wait. */
int bitlinear_check_status(const int* dev_status, bitlinear_stream_t stream);

/*
 * Launch overlap (programmatic dependent launch), process-wide, default off.
 * When enabled, later launches may start while the previous kernel in the
 * same stream is still running: each kernel first does the work that needs
 * only the weights (Wp, gamma: loads into shared memory, barrier and tensor
 * memory set-up) and waits for that previous kernel to complete before it
 * reads activation codes, inputs or scales, or writes any output. Enable it
 * only when no call's Wp or gamma is written by the kernel just before it in
 * its stream. A CUDA graph keeps the setting in force when it was captured.
 */
int bitlinear_set_launch_overlap(int enable);

/* Limit (ns) on every in-kernel wait of later launches; default 2e9. */
int bitlinear_set_wait_timeout_ns(int64_t ns);

/* Launch one block that waits on an mbarrier nothing arrives on, bounded by
 * timeout_ns, then reports BITLINEAR_STATUS_TIMEOUT into dev_status: checks
 * the bounded-wait path without any real fault. */
int bitlinear_debug_wait_timeout(int* dev_status, int64_t timeout_ns, bitlinear_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* BITLINEAR_H */
