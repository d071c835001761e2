// Internal launchers behind the C ABI (host side). Arguments are already
// validated by the entry points in api.cu.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>
#include "../../include/bitlinear.h"

namespace blt {

cudaError_t launch_quant_act(const uint16_t* x, const uint16_t* up, int64_t M, int64_t K,
                             int64_t ldx, int mode, void* q, float* xs, cudaStream_t s);
cudaError_t launch_topk_i8(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, int64_t k,
                           int8_t* q, float* xs, uint8_t* mask, cudaStream_t s);
cudaError_t launch_kv_attention(const uint16_t* q, int64_t B, int64_t H, int64_t D, int64_t T,
                                const uint8_t* k3, const uint8_t* k4, const float* ks,
                                const uint8_t* v3, const uint8_t* v4, const float* vs,
                                const int32_t* keep4, int64_t n4, uint16_t* out, int* status,
                                uint64_t timeout_ns, cudaStream_t s, const char** why);
cudaError_t launch_keep4_positions(const int32_t* ids, int64_t T, const int32_t* special, int n_special,
                                   int32_t* pos, int32_t* count, cudaStream_t s);
cudaError_t launch_kv_quant(const uint16_t* kv, int64_t T, int64_t H, int64_t D,
                            const int32_t* keep4, int64_t n4, uint8_t* codes3, uint8_t* codes4,
                            float* scale, cudaStream_t s);
cudaError_t launch_kv_quant_pair(const uint16_t* k, const uint16_t* v, int64_t T, int64_t H, int64_t D,
                                 const int32_t* keep4, int64_t n4, uint8_t* k3, uint8_t* k4, float* ks,
                                 uint8_t* v3, uint8_t* v4, float* vs, cudaStream_t s);

// Epilogue of the GEMM kernels.
enum OutMode : int { kOutBf16 = 0, kOutRaw = 1 };

struct GemmArgs {
  const void* xq;        // int8 codes [M x K] or packed e2m1 [M x K/2]
  const float* xs;       // [M] (bf16 output only)
  const uint8_t* Wp;     // [N x K/4]
  const float* gamma;    // [G] (bf16 output only)
  int G;
  int group_end[8];
  int64_t M, N, K;
  void* out;             // bf16 [M x ldo] or raw int32/f32 [M x ldo]
  int64_t ldo;
  int out_mode;
  int* status;
  uint64_t timeout_ns;
};

// fp4 selects e2m1 activations (f8f6f4 kind, fp32 accumulate); otherwise int8.
// Returns a CUDA error, or cudaErrorNotSupported when the tensor-map
// encoder is unavailable (message in *why).
cudaError_t launch_gemm(const GemmArgs& a, bool fp4, cudaStream_t s, const char** why);
cudaError_t launch_gemv(const GemmArgs& a, cudaStream_t s, const char** why);
// Decode path for up to 8 tokens: warp-level MMAs (mma.sync u8 x s8) on the
// masked 2-bit codes, weights streamed by TMA before the dependency wait.
constexpr int kGemvMmaMaxTokens = 8;
bool gemv_mma_supported(int64_t M, int64_t N, int64_t K);
cudaError_t launch_gemv_mma(const GemmArgs& a, cudaStream_t s, const char** why);
// CUDA-core decode path with the activation quantiser inside (dp4a on the
// packed codes), up to 8 tokens.
constexpr int kGemvDp4aMaxTokens = 8;
bool gemv_dp4a_supported(int64_t M, int64_t K);
cudaError_t launch_gemv_dp4a(const GemmArgs& a, cudaStream_t s);
// The same with the per-token quantiser (INT8 / INT4, optional ReLU^2 gate)
// done inside the GEMV on bf16 activations x [M x ldx].
cudaError_t launch_gemv_dp4a_quant(const GemmArgs& a, const uint16_t* x, const uint16_t* up,
                                   int64_t ldx, int mode, cudaStream_t s);
cudaError_t launch_wait_probe(int* status, uint64_t timeout_ns, cudaStream_t s);
// Dense tensor-pipe rate microbenchmark (see bitlinear_tensor_peak); *units
// receives the number of ns_out entries written.
cudaError_t launch_tensor_peak(int kind, int iters, unsigned long long* ns_out, int* status,
                               uint64_t timeout_ns, int* units, cudaStream_t s);

// Driver entry point for cuTensorMapEncodeTiled, resolved once at run time.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn get_encode_tiled();
int num_sms();

// Raise a kernel's dynamic shared-memory limit on the current device to at
// least `bytes` (and, with max_carveout, ask for all of the unified L1 as
// shared memory). Function attributes belong to a device's context, so this
// is kept per (device, kernel); it is thread-safe, and calls that need no
// larger limit only take a lock and a lookup.
cudaError_t set_smem_limit(const void* kern, int bytes, bool max_carveout = false);
template <typename... A>
inline cudaError_t set_smem_limit(void (*kern)(A...), int bytes, bool max_carveout = false) {
  return set_smem_limit(reinterpret_cast<const void*>(kern), bytes, max_carveout);
}

// Process-wide switch (bitlinear_set_launch_overlap): launch with
// programmatic stream serialisation so a kernel may start while the previous
// one in the stream finishes. Every kernel calls pdl_wait() before it reads
// activations or scales or writes an output.
bool launch_overlap();

// Launch with the overlap attribute (when on) and, for cluster_x > 0, a
// cluster of cluster_x CTAs along x.
template <typename... Exp, typename... Act>
inline cudaError_t launch_kernel(void (*kern)(Exp...), dim3 grid, dim3 block, size_t smem,
                                 cudaStream_t s, unsigned cluster_x, Act&&... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  if (cluster_x > 0) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  if (launch_overlap()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Act&&>(args)...);
}

}  // namespace blt
