// Dense tensor-pipe rate of this GPU, for the roofline denominators of the
// BitLinear GEMMs: back-to-back tcgen05 MMAs on operands already resident
// in shared memory (no unpack, no global memory), in the shapes and kinds
// the GEMMs issue. One CTA (or CTA pair) per SM; each records the device
// time of its MMA stream with %globaltimer.
//   kind 0: kind::i8 on CTA pairs, M = 256, N = 256, K = 32 (int8 / INT4 GEMM)
//   kind 1: kind::mxf4 on CTA pairs, M = 256, N = 256, K = 64, unit block
//           scales (FP4 GEMM)
//   kind 2: kind::i8 on one CTA, M = 128, N = 256, K = 32
#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace blt {
namespace peak {

constexpr int THREADS = 128;
constexpr int TILE = 128 * 128;               // one operand tile: 128 rows x 128 B
constexpr int SMEM_BYTES = 120 * 1024;        // A, B (up to 256 rows); sized for one CTA per SM

template <int KIND>
__global__ void __launch_bounds__(THREADS, 1) tensor_peak_kernel(int iters, unsigned long long* ns_out,
                                                                  int* status, uint64_t timeout_ns) {
  constexpr bool PAIR = KIND != 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t s_tmem;
  const int warp = threadIdx.x >> 5;
  pdl_wait();  // never overlap the kernel before it: this one is timed alone
  // operand bytes 0x11: int8 17, or two e2m1 0.5 per byte; values do not matter
  for (int i = threadIdx.x; i < 3 * TILE / 16; i += THREADS)
    reinterpret_cast<uint4*>(smem)[i] = make_uint4(0x11111111u, 0x11111111u, 0x11111111u, 0x11111111u);
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    if (PAIR) { tmem_alloc_pair(&s_tmem, 512); tmem_relinquish_pair(); }
    else      { tmem_alloc(&s_tmem, 512); tmem_relinquish(); }
  }
  __syncthreads();
  if (PAIR) cluster_sync();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  if constexpr (KIND == 1) {
    // unit ue8m0 scales (0x7F) in columns 256..511: A's at 256, B's at 288
    uint32_t ones[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) ones[i] = 0x7F7F7F7Fu;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
#pragma unroll
    for (int col = 256; col < 512; col += 32) tmem_st32(lane_base + col, ones);
    tmem_st_wait();
    tc_fence_before();
    __syncthreads();
    if (PAIR) cluster_sync();
    tc_fence_after();
  }
  const bool leader = !PAIR || cluster_ctarank() == 0;
  unsigned long long t0 = 0;
  if (leader && threadIdx.x == 0) {
    const uint64_t ad = smem_desc_sw128(smem_u32(smem));
    const uint64_t bd = smem_desc_sw128(smem_u32(smem + TILE));
    t0 = globaltimer_ns();
    for (int i = 0; i < iters; ++i) {
#pragma unroll
      for (int k4 = 0; k4 < 4; ++k4) {
        if constexpr (KIND == 0) mma_i8_pair(tmem, ad + 2 * k4, bd + 2 * k4, make_idesc(2, 1, 1, 256, 256), 1u);
        else if constexpr (KIND == 1)
          mma_mxf4_pair(tmem, ad + 2 * k4, bd + 2 * k4, make_idesc_mxf4(256, 256), tmem + 256, tmem + 288, 1u);
        else mma_i8(tmem, ad + 2 * k4, bd + 2 * k4, make_idesc(2, 1, 1, 128, 256), 1u);
      }
    }
    if (PAIR) tc_commit_pair_mc(&bar, 3);
    else      tc_commit(&bar);
  }
  if (threadIdx.x == 0) {
    if (!mbar_wait(&bar, 0, timeout_ns, nullptr)) report_status(status, BITLINEAR_STATUS_TIMEOUT);
    if (leader) ns_out[PAIR ? blockIdx.x / 2 : blockIdx.x] = globaltimer_ns() - t0;
  }
  __syncthreads();
  if (PAIR) cluster_sync();
  if (warp == 0) {
    tc_fence_after();
    if (PAIR) tmem_dealloc_pair(tmem, 512);
    else      tmem_dealloc(tmem, 512);
  }
}

}  // namespace peak

cudaError_t launch_tensor_peak(int kind, int iters, unsigned long long* ns_out, int* status,
                               uint64_t timeout_ns, int* units, cudaStream_t s) {
  using namespace peak;
  const int sms = num_sms();
  const int pairs = sms / 2;
  cudaError_t e;
  switch (kind) {
    case 0:
      e = set_smem_limit(tensor_peak_kernel<0>, SMEM_BYTES);
      if (e != cudaSuccess) return e;
      *units = pairs;
      return launch_kernel(tensor_peak_kernel<0>, dim3(2 * pairs), dim3(THREADS), SMEM_BYTES, s, 2u, iters,
                           ns_out, status, timeout_ns);
    case 1:
      e = set_smem_limit(tensor_peak_kernel<1>, SMEM_BYTES);
      if (e != cudaSuccess) return e;
      *units = pairs;
      return launch_kernel(tensor_peak_kernel<1>, dim3(2 * pairs), dim3(THREADS), SMEM_BYTES, s, 2u, iters,
                           ns_out, status, timeout_ns);
    default:
      e = set_smem_limit(tensor_peak_kernel<2>, SMEM_BYTES);
      if (e != cudaSuccess) return e;
      *units = sms;
      return launch_kernel(tensor_peak_kernel<2>, dim3(sms), dim3(THREADS), SMEM_BYTES, s, 0u, iters, ns_out,
                           status, timeout_ns);
  }
}

}  // namespace blt
