// C ABI entry points: argument validation on the host, then one launch on
// the caller's stream. The library allocates no device memory.
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>
#include <vector>

#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace {

thread_local char g_err[512] = "";
std::atomic<int64_t> g_timeout_ns{2000000000LL};
std::atomic<bool> g_overlap{false};

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

int ok() {
  g_err[0] = '\0';
  return BITLINEAR_OK;
}

int cuda_fail(cudaError_t e, const char* what, const char* why = nullptr) {
  return fail(BITLINEAR_ERR_CUDA, "%s: %s%s%s", what, cudaGetErrorString(e), why ? " (" : "",
              why ? why : "");
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Common checks of the GEMM family. Fills the group table.
int check_gemm(const char* fn, const void* xq, const void* xs, const uint8_t* Wp,
               const float* gamma, const int64_t* group_ends, int G, int64_t M, int64_t N,
               int64_t K, const void* y, int64_t ldy, bool need_scales, blt::GemmArgs* a) {
  if (M < 0 || N <= 0 || K <= 0) return fail(BITLINEAR_ERR_INVALID_ARG, "%s: bad sizes M=%lld N=%lld K=%lld", fn, (long long)M, (long long)N, (long long)K);
  if (K % 64 != 0) return fail(BITLINEAR_ERR_INVALID_ARG, "%s: K=%lld must be a multiple of 64", fn, (long long)K);
  if (N % 16 != 0) return fail(BITLINEAR_ERR_INVALID_ARG, "%s: N=%lld must be a multiple of 16", fn, (long long)N);
  if (M > (1LL << 30) || N > (1LL << 30) || K > 32768)
    return fail(BITLINEAR_ERR_UNSUPPORTED, "%s: sizes beyond the supported range", fn);
  if (M == 0) return BITLINEAR_OK;  // empty call: pointers may be null, nothing is launched
  if (!xq || !Wp || !y) return fail(BITLINEAR_ERR_INVALID_ARG, "%s: null operand pointer", fn);
  if (!aligned16(xq) || !aligned16(Wp) || !aligned16(y))
    return fail(BITLINEAR_ERR_ALIGNMENT, "%s: operands must be 16-byte aligned", fn);
  if (ldy < N || ldy % 8 != 0) return fail(BITLINEAR_ERR_INVALID_ARG, "%s: ldy=%lld must be >= N and a multiple of 8", fn, (long long)ldy);
  a->G = 1;
  for (int i = 0; i < 8; ++i) a->group_end[i] = static_cast<int>(N);
  if (need_scales) {
    if (!xs || !gamma) return fail(BITLINEAR_ERR_INVALID_ARG, "%s: null scale pointer", fn);
    if (!group_ends || G < 1 || G > 8) return fail(BITLINEAR_ERR_INVALID_ARG, "%s: need 1..8 column groups", fn);
    int64_t prev = 0;
    for (int i = 0; i < G; ++i) {
      if (group_ends[i] <= prev) return fail(BITLINEAR_ERR_INVALID_ARG, "%s: group_ends must increase", fn);
      prev = group_ends[i];
      a->group_end[i] = static_cast<int>(group_ends[i]);
    }
    if (prev != N) return fail(BITLINEAR_ERR_INVALID_ARG, "%s: last group end must equal N", fn);
    a->G = G;
  }
  a->xq = xq;
  a->xs = static_cast<const float*>(xs);
  a->Wp = Wp;
  a->gamma = gamma;
  a->M = M;
  a->N = N;
  a->K = K;
  a->timeout_ns = static_cast<uint64_t>(g_timeout_ns.load(std::memory_order_relaxed));
  return BITLINEAR_OK;
}

__global__ void wait_probe_kernel(int* status, uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    blt::mbar_init(&bar, 1);
    blt::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // nothing ever arrives on this barrier: the bounded wait must give up
    if (!blt::mbar_wait(&bar, 0, timeout_ns, nullptr)) blt::report_status(status, BITLINEAR_STATUS_TIMEOUT);
    blt::mbar_arrive(&bar);  // complete the phase so the barrier is left quiescent
  }
}

}  // namespace

namespace blt {

EncodeTiledFn get_encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

int num_sms() {
  static int cache[64] = {0};
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  if (dev >= 0 && dev < 64 && cache[dev] > 0) return cache[dev];
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) return 1;
  if (dev >= 0 && dev < 64) cache[dev] = n;
  return n;
}

bool launch_overlap() { return g_overlap.load(std::memory_order_relaxed); }

cudaError_t set_smem_limit(const void* kern, int bytes, bool max_carveout) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static std::mutex mu;
  static std::map<std::pair<int, const void*>, int> raised;  // (device, kernel) -> limit set
  std::lock_guard<std::mutex> lock(mu);
  int& have = raised[std::make_pair(dev, kern)];
  if (bytes <= have) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && max_carveout)
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess) have = bytes;
  return e;
}

cudaError_t launch_wait_probe(int* status, uint64_t timeout_ns, cudaStream_t s) {
  wait_probe_kernel<<<1, 32, 0, s>>>(status, timeout_ns);
  return cudaGetLastError();
}

}  // namespace blt

extern "C" {

const char* bitlinear_last_error(void) { return g_err; }

int bitlinear_version(void) { return 106; }

int bitlinear_set_launch_overlap(int enable) {
  g_overlap.store(enable != 0);
  return ok();
}

int bitlinear_set_wait_timeout_ns(int64_t ns) {
  if (ns <= 0) return fail(BITLINEAR_ERR_INVALID_ARG, "timeout must be positive");
  g_timeout_ns.store(ns, std::memory_order_relaxed);
  return ok();
}

int bitlinear_ternarize_pack(const float* W, int64_t K, int64_t N, const int64_t* group_ends, int G,
                             uint8_t* Wp, float* gamma) {
  if (!W || !Wp || !gamma || !group_ends) return fail(BITLINEAR_ERR_INVALID_ARG, "ternarize_pack: null pointer");
  if (K <= 0 || N <= 0 || K % 16 != 0) return fail(BITLINEAR_ERR_INVALID_ARG, "ternarize_pack: K must be a positive multiple of 16");
  if (G < 1 || G > 8) return fail(BITLINEAR_ERR_INVALID_ARG, "ternarize_pack: need 1..8 column groups");
  int64_t prev = 0;
  for (int i = 0; i < G; ++i) {
    if (group_ends[i] <= prev) return fail(BITLINEAR_ERR_INVALID_ARG, "ternarize_pack: group_ends must increase");
    prev = group_ends[i];
  }
  if (prev != N) return fail(BITLINEAR_ERR_INVALID_ARG, "ternarize_pack: last group end must equal N");

  std::vector<float> g(G);
  int64_t start = 0;
  for (int gi = 0; gi < G; ++gi) {
    const int64_t end = group_ends[gi];
    double sum = 0.0;  // sequential, row-major over the group's block
    for (int64_t k = 0; k < K; ++k)
      for (int64_t n = start; n < end; ++n) sum += std::fabs(static_cast<double>(W[k * N + n]));
    float gm = static_cast<float>(sum / static_cast<double>(K * (end - start)));
    g[gi] = gm > 1e-5f ? gm : 1e-5f;
    gamma[gi] = g[gi];
    start = end;
  }
  std::memset(Wp, 0, static_cast<size_t>(N) * static_cast<size_t>(K / 4));
  start = 0;
  for (int gi = 0; gi < G; ++gi) {
    const int64_t end = group_ends[gi];
    const float gm = g[gi];
    for (int64_t k = 0; k < K; ++k) {
      const int64_t word = k >> 4, e = k & 15;
      const int shift = 4 * (e & 7) + 2 * (e >> 3);
      for (int64_t n = start; n < end; ++n) {
        volatile float q = W[k * N + n] / gm;  // IEEE fp32 division
        float r = std::nearbyint(q);             // round half to even (default mode)
        r = r > 1.f ? 1.f : (r < -1.f ? -1.f : r);
        const uint32_t code = static_cast<uint32_t>(static_cast<int>(r) + 1);
        uint8_t* wrow = Wp + n * (K / 4) + word * 4;
        wrow[shift >> 3] |= static_cast<uint8_t>(code << (shift & 7));
      }
    }
    start = end;
  }
  return ok();
}

int bitlinear_quant_act(const uint16_t* x, const uint16_t* up, int64_t M, int64_t K, int64_t ldx,
                        int mode, void* q_out, float* xs_out, bitlinear_stream_t stream) {
  if (mode != BITLINEAR_MODE_INT8 && mode != BITLINEAR_MODE_INT4 && mode != BITLINEAR_MODE_FP4)
    return fail(BITLINEAR_ERR_INVALID_ARG, "quant_act: unknown mode %d", mode);
  if (M < 0 || K <= 0 || K % 16 != 0) return fail(BITLINEAR_ERR_INVALID_ARG, "quant_act: K must be a positive multiple of 16");
  if (K > 49152) return fail(BITLINEAR_ERR_UNSUPPORTED, "quant_act: K above 49152");
  if (M > 0x7FFFFFFF) return fail(BITLINEAR_ERR_UNSUPPORTED, "quant_act: too many rows");
  if (ldx < K || ldx % 8 != 0) return fail(BITLINEAR_ERR_INVALID_ARG, "quant_act: ldx must be >= K and a multiple of 8");
  if (M == 0) return ok();
  if (!x || !q_out || !xs_out) return fail(BITLINEAR_ERR_INVALID_ARG, "quant_act: null pointer");
  if (!aligned16(x) || (up && !aligned16(up)) || !aligned16(q_out))
    return fail(BITLINEAR_ERR_ALIGNMENT, "quant_act: pointers must be 16-byte aligned");
  if (M == 0) return ok();
  cudaError_t e = blt::launch_quant_act(x, up, M, K, ldx, mode, q_out, xs_out, stream);
  return e == cudaSuccess ? ok() : cuda_fail(e, "quant_act launch");
}

int bitlinear_topk_sparsify_i8(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, int64_t k,
                               int8_t* q_out, float* xs_out, uint8_t* mask_out,
                               bitlinear_stream_t stream) {
  if (M < 0 || K <= 0 || K % 16 != 0) return fail(BITLINEAR_ERR_INVALID_ARG, "topk: K must be a positive multiple of 16");
  if (K > 16384) return fail(BITLINEAR_ERR_UNSUPPORTED, "topk: K above 16384");
  if (M > 0x7FFFFFFF) return fail(BITLINEAR_ERR_UNSUPPORTED, "topk: too many rows");
  if (k < 0) return fail(BITLINEAR_ERR_INVALID_ARG, "topk: k must be >= 0");
  if (ldx < K || ldx % 8 != 0) return fail(BITLINEAR_ERR_INVALID_ARG, "topk: ldx must be >= K and a multiple of 8");
  if (M == 0) return ok();
  if (!x || !q_out || !xs_out) return fail(BITLINEAR_ERR_INVALID_ARG, "topk: null pointer");
  if (!aligned16(x) || !aligned16(q_out)) return fail(BITLINEAR_ERR_ALIGNMENT, "topk: pointers must be 16-byte aligned");
  if (k == 0) k = (K + 1) / 2;
  if (k > K) k = K;
  if (M == 0) return ok();
  cudaError_t e = blt::launch_topk_i8(x, M, K, ldx, k, q_out, xs_out, mask_out, stream);
  return e == cudaSuccess ? ok() : cuda_fail(e, "topk launch");
}

static int gemm_common(const char* fn, const void* xq, const float* xs, const uint8_t* Wp,
                       const float* gamma, const int64_t* group_ends, int G, int64_t M, int64_t N,
                       int64_t K, void* out, int64_t ldo, int out_mode, int* dev_status, bool fp4,
                       bitlinear_stream_t stream) {
  blt::GemmArgs a{};
  if (fp4 && K % 128 != 0) return fail(BITLINEAR_ERR_INVALID_ARG, "%s: K must be a multiple of 128", fn);
  const int rc = check_gemm(fn, xq, xs, Wp, gamma, group_ends, G, M, N, K, out, ldo,
                            out_mode == blt::kOutBf16, &a);
  if (rc != BITLINEAR_OK) return rc;
  if (M == 0) return ok();
  a.out = out;
  a.ldo = ldo;
  a.out_mode = out_mode;
  a.status = dev_status;
  const char* why = nullptr;
  cudaError_t e = blt::launch_gemm(a, fp4, stream, &why);
  return e == cudaSuccess ? ok() : cuda_fail(e, fn, why);
}

int bitlinear_gemm_w2a8(const int8_t* xq, const float* xs, const uint8_t* Wp, const float* gamma,
                        const int64_t* group_ends, int G, int64_t M, int64_t N, int64_t K,
                        uint16_t* y, int64_t ldy, int* dev_status, bitlinear_stream_t stream) {
  return gemm_common("gemm_w2a8", xq, xs, Wp, gamma, group_ends, G, M, N, K, y, ldy,
                     blt::kOutBf16, dev_status, false, stream);
}

int bitlinear_gemm_w2a4(const int8_t* xq, const float* xs, const uint8_t* Wp, const float* gamma,
                        const int64_t* group_ends, int G, int64_t M, int64_t N, int64_t K,
                        uint16_t* y, int64_t ldy, int* dev_status, bitlinear_stream_t stream) {
  return gemm_common("gemm_w2a4", xq, xs, Wp, gamma, group_ends, G, M, N, K, y, ldy,
                     blt::kOutBf16, dev_status, false, stream);
}

int bitlinear_gemm_w2fp4(const uint8_t* xf4, const float* xs, const uint8_t* Wp,
                         const float* gamma, const int64_t* group_ends, int G, int64_t M,
                         int64_t N, int64_t K, uint16_t* y, int64_t ldy, int* dev_status,
                         bitlinear_stream_t stream) {
  return gemm_common("gemm_w2fp4", xf4, xs, Wp, gamma, group_ends, G, M, N, K, y, ldy,
                     blt::kOutBf16, dev_status, true, stream);
}

int bitlinear_gemm_w2a8_acc(const int8_t* xq, const uint8_t* Wp, int64_t M, int64_t N, int64_t K,
                            int32_t* acc, int* dev_status, bitlinear_stream_t stream) {
  return gemm_common("gemm_w2a8_acc", xq, nullptr, Wp, nullptr, nullptr, 0, M, N, K, acc, N,
                     blt::kOutRaw, dev_status, false, stream);
}

int bitlinear_gemm_w2fp4_acc(const uint8_t* xf4, const uint8_t* Wp, int64_t M, int64_t N,
                             int64_t K, float* acc, int* dev_status, bitlinear_stream_t stream) {
  return gemm_common("gemm_w2fp4_acc", xf4, nullptr, Wp, nullptr, nullptr, 0, M, N, K, acc, N,
                     blt::kOutRaw, dev_status, true, stream);
}

int bitlinear_gemv_w2(const int8_t* xq, const float* xs, const uint8_t* Wp, const float* gamma,
                      const int64_t* group_ends, int G, int64_t M, int64_t N, int64_t K,
                      uint16_t* y, int64_t ldy, int* dev_status, bitlinear_stream_t stream) {
  blt::GemmArgs a{};
  if (M > 64) return fail(BITLINEAR_ERR_INVALID_ARG, "gemv_w2: M=%lld above 64 (use a GEMM)", (long long)M);
  if (K % 128 != 0 || N % 128 != 0) return fail(BITLINEAR_ERR_INVALID_ARG, "gemv_w2: K and N must be multiples of 128");
  const int rc = check_gemm("gemv_w2", xq, xs, Wp, gamma, group_ends, G, M, N, K, y, ldy, true, &a);
  if (rc != BITLINEAR_OK) return rc;
  if (M == 0) return ok();
  a.out = y;
  a.ldo = ldy;
  a.out_mode = blt::kOutBf16;
  a.status = dev_status;
  const char* why = nullptr;
  // one token: CUDA-core dp4a on the packed codes; 2..8: warp-level MMAs;
  // more: the tcgen05 GEMV (measured crossovers on the decode layer shapes)
  if (M == 1 && blt::gemv_dp4a_supported(M, K)) {
    cudaError_t e = blt::launch_gemv_dp4a(a, stream);
    return e == cudaSuccess ? ok() : cuda_fail(e, "gemv_w2 (dp4a)");
  }
  if (blt::gemv_mma_supported(M, N, K)) {
    cudaError_t e = blt::launch_gemv_mma(a, stream, &why);
    return e == cudaSuccess ? ok() : cuda_fail(e, "gemv_w2 (warp MMA)", why);
  }
  cudaError_t e = blt::launch_gemv(a, stream, &why);
  return e == cudaSuccess ? ok() : cuda_fail(e, "gemv_w2", why);
}

int bitlinear_gemv_w2_quant(const uint16_t* x, const uint16_t* up, int64_t ldx, int mode,
                            const uint8_t* Wp, const float* gamma, const int64_t* group_ends, int G,
                            int64_t M, int64_t N, int64_t K, uint16_t* y, int64_t ldy,
                            int* dev_status, bitlinear_stream_t stream) {
  blt::GemmArgs a{};
  if (mode != BITLINEAR_MODE_INT8 && mode != BITLINEAR_MODE_INT4)
    return fail(BITLINEAR_ERR_INVALID_ARG, "gemv_w2_quant: mode must be INT8 or INT4");
  if (M > blt::kGemvDp4aMaxTokens)
    return fail(BITLINEAR_ERR_UNSUPPORTED, "gemv_w2_quant: M=%lld above %d", (long long)M, blt::kGemvDp4aMaxTokens);
  if (K % 128 != 0 || N % 128 != 0) return fail(BITLINEAR_ERR_INVALID_ARG, "gemv_w2_quant: K and N must be multiples of 128");
  // the codes pointer checks apply to x; xs is not used (the kernel computes it)
  const int rc = check_gemm("gemv_w2_quant", x, x, Wp, gamma, group_ends, G, M, N, K, y, ldy, true, &a);
  if (rc != BITLINEAR_OK) return rc;
  if (M == 0) return ok();
  if (ldx < K || ldx % 8 != 0) return fail(BITLINEAR_ERR_INVALID_ARG, "gemv_w2_quant: ldx must be >= K and a multiple of 8");
  if (up && !aligned16(up)) return fail(BITLINEAR_ERR_ALIGNMENT, "gemv_w2_quant: up must be 16-byte aligned");
  if (!blt::gemv_dp4a_supported(M, K))
    return fail(BITLINEAR_ERR_UNSUPPORTED, "gemv_w2_quant: K=%lld too large for %lld tokens", (long long)K, (long long)M);
  a.out = y;
  a.ldo = ldy;
  a.out_mode = blt::kOutBf16;
  a.status = dev_status;
  cudaError_t e = blt::launch_gemv_dp4a_quant(a, x, up, ldx, mode, stream);
  return e == cudaSuccess ? ok() : cuda_fail(e, "gemv_w2_quant");
}

static int kv_quant_check(const char* fn, const uint16_t* kv, int64_t T, int64_t H, int64_t D,
                          const int32_t* keep4_pos, int64_t n_keep4, const uint8_t* codes3,
                          const uint8_t* codes4, const float* scale) {
  if (T < 0 || H <= 0) return fail(BITLINEAR_ERR_INVALID_ARG, "%s: bad sizes", fn);
  if (D != 64 && D != 128 && D != 256) return fail(BITLINEAR_ERR_UNSUPPORTED, "%s: D must be 64, 128 or 256", fn);
  if (n_keep4 < 0 || n_keep4 > T || (n_keep4 > 0 && (!keep4_pos || !codes4)))
    return fail(BITLINEAR_ERR_INVALID_ARG, "%s: bad 4-bit token list", fn);
  if (T == 0) return BITLINEAR_OK;
  if (!kv || !codes3 || !scale) return fail(BITLINEAR_ERR_INVALID_ARG, "%s: null pointer", fn);
  if (!aligned16(kv) || !aligned16(codes3) || (codes4 && !aligned16(codes4)))
    return fail(BITLINEAR_ERR_ALIGNMENT, "%s: pointers must be 16-byte aligned", fn);
  if (T * H * (D / 8) >= (1LL << 32) - 256 || n_keep4 > 0x7FFFFFFF)
    return fail(BITLINEAR_ERR_UNSUPPORTED, "%s: T * H * D / 8 must stay below 2^32", fn);
  return BITLINEAR_OK;
}

int kv_quant_3bit(const uint16_t* kv, int64_t T, int64_t H, int64_t D, const int32_t* keep4_pos,
                  int64_t n_keep4, uint8_t* codes3, uint8_t* codes4, float* scale,
                  bitlinear_stream_t stream) {
  const int rc = kv_quant_check("kv_quant_3bit", kv, T, H, D, keep4_pos, n_keep4, codes3, codes4, scale);
  if (rc != BITLINEAR_OK) return rc;
  if (T == 0) return ok();
  cudaError_t e = blt::launch_kv_quant(kv, T, H, D, keep4_pos, n_keep4, codes3, codes4, scale, stream);
  return e == cudaSuccess ? ok() : cuda_fail(e, "kv_quant_3bit launch");
}

int kv_quant_3bit_kv(const uint16_t* k, const uint16_t* v, int64_t T, int64_t H, int64_t D,
                     const int32_t* keep4_pos, int64_t n_keep4, uint8_t* k_codes3, uint8_t* k_codes4,
                     float* k_scale, uint8_t* v_codes3, uint8_t* v_codes4, float* v_scale,
                     bitlinear_stream_t stream) {
  int rc = kv_quant_check("kv_quant_3bit_kv (K)", k, T, H, D, keep4_pos, n_keep4, k_codes3, k_codes4, k_scale);
  if (rc != BITLINEAR_OK) return rc;
  rc = kv_quant_check("kv_quant_3bit_kv (V)", v, T, H, D, keep4_pos, n_keep4, v_codes3, v_codes4, v_scale);
  if (rc != BITLINEAR_OK) return rc;
  if (T == 0) return ok();
  cudaError_t e = blt::launch_kv_quant_pair(k, v, T, H, D, keep4_pos, n_keep4, k_codes3, k_codes4, k_scale,
                                           v_codes3, v_codes4, v_scale, stream);
  return e == cudaSuccess ? ok() : cuda_fail(e, "kv_quant_3bit_kv launch");
}

int kv_keep4_positions(const int32_t* token_ids, int64_t T, const int32_t* special_ids,
                       int n_special, int32_t* pos_out, int32_t* count_out,
                       bitlinear_stream_t stream) {
  if (T < 0 || T > 0x7FFFFFFF) return fail(BITLINEAR_ERR_INVALID_ARG, "kv_keep4_positions: bad T");
  if (n_special < 1 || n_special > 8 || !special_ids)
    return fail(BITLINEAR_ERR_INVALID_ARG, "kv_keep4_positions: 1 to 8 special ids");
  if (!count_out || (T > 0 && (!token_ids || !pos_out)))
    return fail(BITLINEAR_ERR_INVALID_ARG, "kv_keep4_positions: null pointer");
  cudaError_t e = blt::launch_keep4_positions(token_ids, T, special_ids, n_special, pos_out, count_out,
                                              stream);
  return e == cudaSuccess ? ok() : cuda_fail(e, "kv_keep4_positions launch");
}

int kv_attention_3bit(const uint16_t* q, int64_t B, int64_t H, int64_t D, int64_t T,
                      const uint8_t* k_codes3, const uint8_t* k_codes4, const float* k_scale,
                      const uint8_t* v_codes3, const uint8_t* v_codes4, const float* v_scale,
                      const int32_t* keep4_pos, int64_t n_keep4, uint16_t* out, int* dev_status,
                      bitlinear_stream_t stream) {
  if (B < 0 || H <= 0 || T <= 0) return fail(BITLINEAR_ERR_INVALID_ARG, "kv_attention_3bit: bad sizes");
  if (D != 128 && D != 256) return fail(BITLINEAR_ERR_UNSUPPORTED, "kv_attention_3bit: D must be 128 or 256");
  if (H % 4 != 0) return fail(BITLINEAR_ERR_UNSUPPORTED, "kv_attention_3bit: H must be a multiple of 4");
  if (n_keep4 < 0 || n_keep4 > T || (n_keep4 > 0 && (!keep4_pos || !k_codes4 || !v_codes4)))
    return fail(BITLINEAR_ERR_INVALID_ARG, "kv_attention_3bit: bad 4-bit token list");
  if (n_keep4 > 1024) return fail(BITLINEAR_ERR_UNSUPPORTED, "kv_attention_3bit: at most 1024 tokens at 4 bits");
  if (H > 65535 || (B + 7) / 8 > 65535 || T >= (1LL << 31) / H)
    return fail(BITLINEAR_ERR_UNSUPPORTED, "kv_attention_3bit: sizes beyond the supported range");
  if (B == 0) return ok();
  if (!q || !k_codes3 || !k_scale || !v_codes3 || !v_scale || !out)
    return fail(BITLINEAR_ERR_INVALID_ARG, "kv_attention_3bit: null pointer");
  if (!aligned16(q) || !aligned16(k_codes3) || !aligned16(v_codes3) || !aligned16(k_scale) ||
      !aligned16(v_scale) || !aligned16(out) ||
      (n_keep4 > 0 && (!aligned16(k_codes4) || !aligned16(v_codes4))))
    return fail(BITLINEAR_ERR_ALIGNMENT, "kv_attention_3bit: q, codes, scales and out must be 16-byte aligned");
  const char* why = nullptr;
  cudaError_t e = blt::launch_kv_attention(q, B, H, D, T, k_codes3, k_codes4, k_scale, v_codes3,
                                           v_codes4, v_scale, keep4_pos, n_keep4, out, dev_status,
                                           static_cast<uint64_t>(g_timeout_ns.load(std::memory_order_relaxed)), stream, &why);
  return e == cudaSuccess ? ok() : cuda_fail(e, "kv_attention_3bit", why);
}

int bitlinear_tensor_peak(int kind, int iters, uint64_t* ns_out, int* units_out, int* dev_status,
                          bitlinear_stream_t stream) {
  if (kind < 0 || kind > 2) return fail(BITLINEAR_ERR_INVALID_ARG, "tensor_peak: kind must be 0, 1 or 2");
  if (iters < 1 || iters > (1 << 22)) return fail(BITLINEAR_ERR_INVALID_ARG, "tensor_peak: iters in 1..2^22");
  if (!ns_out || !units_out) return fail(BITLINEAR_ERR_INVALID_ARG, "tensor_peak: null pointer");
  int units = 0;
  cudaError_t e = blt::launch_tensor_peak(kind, iters, reinterpret_cast<unsigned long long*>(ns_out), dev_status,
                                          static_cast<uint64_t>(g_timeout_ns.load(std::memory_order_relaxed)),
                                          &units, stream);
  if (e != cudaSuccess) return cuda_fail(e, "tensor_peak launch");
  *units_out = units;
  return ok();
}

int bitlinear_check_status(const int* dev_status, bitlinear_stream_t stream) {
  if (!dev_status) return fail(BITLINEAR_ERR_INVALID_ARG, "check_status: null pointer");
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e, "check_status sync");
  int h = 0;
  e = cudaMemcpy(&h, dev_status, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "check_status read");
  if (h & BITLINEAR_STATUS_TIMEOUT) return fail(BITLINEAR_ERR_TIMEOUT, "a kernel gave up a bounded wait");
  return ok();
}

int bitlinear_debug_wait_timeout(int* dev_status, int64_t timeout_ns, bitlinear_stream_t stream) {
  if (!dev_status || timeout_ns <= 0) return fail(BITLINEAR_ERR_INVALID_ARG, "debug_wait_timeout: bad arguments");
  if (timeout_ns > 10000000000LL) return fail(BITLINEAR_ERR_INVALID_ARG, "debug_wait_timeout: at most 10 s");
  cudaError_t e = blt::launch_wait_probe(dev_status, static_cast<uint64_t>(timeout_ns), stream);
  return e == cudaSuccess ? ok() : cuda_fail(e, "debug_wait_timeout launch");
}

}  // extern "C"
