// Decode-time BitLinear (1..64 tokens) on sm_100a tensor cores.
//
// With few tokens the layer is bound by reading the packed weights from
// HBM, so the kernel is arranged around the weight stream ("swap AB"):
//   A = unpacked ternary weights, 128 output features x K   (M side, 128)
//   B = int8 activation codes, Npad tokens x K              (N side, 16..64)
//   D[n, m] in TMEM: lane = output feature, column = token.
// One CTA owns 128 output features and one K slice; the C CTAs of a thread
// block cluster split K and reduce their int32 partials through distributed
// shared memory, so every weight byte is read exactly once and no global
// scratch is used.
//   warp 0     TMA producer (packed weights 128 x 32 B, activations Npad x 128 B)
//   warp 1     TMEM allocator + single-thread MMA issuer
//   warps 4-7  unpack 2-bit weights into the swizzled A ring during the
//              mainloop; afterwards the epilogue (TMEM -> registers -> DSMEM
//              reduction on cluster rank 0 -> bf16 y)
#include <cooperative_groups.h>

#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace blt {
namespace gemv {

constexpr int BNF = 128;                 // output features per CTA
constexpr int BK = 128;
constexpr int S = 8, SA = 4;
constexpr int WP_BYTES = BNF * (BK / 4);  // 4 KB
constexpr int X_BYTES = 64 * 128;         // up to 64 token rows
constexpr int A_BYTES = BNF * 128;        // 16 KB
constexpr int OFF_A = 0;                  // 1024-aligned
constexpr int OFF_X = OFF_A + SA * A_BYTES;
constexpr int OFF_WP = OFF_X + S * X_BYTES;
constexpr int OFF_BAR = OFF_WP + S * WP_BYTES;
constexpr int N_BARS = 2 * S + 2 * SA + 2;
constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
constexpr int THREADS = 256;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(SA * A_BYTES >= 64 * BNF * 4, "partials alias the A ring");

struct Params {
  int M, N, K, npad, num_kb, csize;
  const float* xs;
  const float* gamma;
  int G;
  int group_end[8];
  uint16_t* y;
  int64_t ldy;
  int* status;
  uint64_t timeout_ns;
};

__device__ __forceinline__ float gamma_of(const Params& p, int n) {
  int g = 0;
#pragma unroll
  for (int i = 0; i < 7; ++i) g += (i < p.G - 1 && n >= p.group_end[i]) ? 1 : 0;
  return __ldg(p.gamma + g);
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
__device__ __forceinline__ uint32_t map_to_rank(uint32_t smem_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
  return r;
}
__device__ __forceinline__ int32_t ld_dsmem_s32(uint32_t addr) {
  int32_t v;
  asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

__global__ void __launch_bounds__(THREADS, 1)
bitlinear_gemv_kernel(const __grid_constant__ CUtensorMap tmX,
                      const __grid_constant__ CUtensorMap tmW, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* empty = full + S;
  uint64_t* afull = empty + S;
  uint64_t* aempty = afull + SA;
  uint64_t* tfull = aempty + SA;
  uint64_t* mma_done = tfull + 1;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const uint32_t rank = cluster_rank();
  const int tile = blockIdx.x / p.csize;
  const int n0 = tile * BNF;
  const int kb0 = static_cast<int>((static_cast<int64_t>(p.num_kb) * rank) / p.csize);
  const int kb1 = static_cast<int>((static_cast<int64_t>(p.num_kb) * (rank + 1)) / p.csize);
  const uint32_t tmem_cols = p.npad <= 32 ? 32u : 64u;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    for (int i = 0; i < SA; ++i) { mbar_init(&afull[i], 128); mbar_init(&aempty[i], 1); }
    mbar_init(tfull, 1);
    mbar_init(mma_done, 1);
    *s_abort = 0;
    fence_mbar_init();
    prefetch_tensormap(&tmX);
    prefetch_tensormap(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, tmem_cols);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const uint64_t tmo = p.timeout_ns;
  const uint32_t sA = smem_u32(smem + OFF_A);
  const uint32_t sX = smem_u32(smem + OFF_X);
  const uint32_t sW = smem_u32(smem + OFF_WP);
  auto fail = [&]() {
    *s_abort = 1;
    report_status(p.status, BITLINEAR_STATUS_TIMEOUT);
  };
  bool have_acc = false;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t it = 0;
      const uint32_t tx = WP_BYTES + p.npad * 128;
      for (int kb = kb0; kb < kb1; ++kb, ++it) {
        const uint32_t s = it % S, ph = (it / S) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, tmo, s_abort)) { fail(); break; }
        mbar_arrive_expect_tx(&full[s], tx);
        tma_load_2d(smem + OFF_WP + s * WP_BYTES, &tmW, &full[s], kb * (BK / 4), n0);
        tma_load_2d(smem + OFF_X + s * X_BYTES, &tmX, &full[s], kb * BK, 0);
      }
      const uint32_t inflight = it < S ? it : S;
      for (uint32_t d = 0; d < inflight; ++d) {
        const uint32_t j = it - 1 - d;
        mbar_wait(&full[j % S], (j / S) & 1, tmo, nullptr);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = make_idesc(2, 1, 1, BNF, p.npad);
      uint32_t it = 0;
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb, ++it) {
        const uint32_t s = it % S, ph = (it / S) & 1;
        const uint32_t a = it % SA, aph = (it / SA) & 1;
        if (!mbar_wait(&full[s], ph, tmo, s_abort) || !mbar_wait(&afull[a], aph, tmo, s_abort)) {
          fail(); ok = false; break;
        }
        tc_fence_after();
        const uint64_t adesc = smem_desc_sw128(sA + a * A_BYTES);
        const uint64_t bdesc = smem_desc_sw128(sX + s * X_BYTES);
#pragma unroll
        for (int k4 = 0; k4 < BK / 32; ++k4)
          mma_i8(tmem_base, adesc + 2 * k4, bdesc + 2 * k4, idesc, (kb != kb0) || (k4 != 0));
        tc_commit(&empty[s]);
        tc_commit(&aempty[a]);
      }
      if (ok) tc_commit(tfull);
      tc_commit(mma_done);
      mbar_wait(mma_done, 0, tmo, nullptr);
    }
  } else if (warp >= 4) {
    // --------------------------------------------- unpack, then epilogue
    const int ut = threadIdx.x - 128;  // 0..127
    uint32_t it = 0;
    bool ok = true;
    for (int kb = kb0; kb < kb1; ++kb, ++it) {
      const uint32_t s = it % S, ph = (it / S) & 1;
      const uint32_t a = it % SA, aph = (it / SA) & 1;
      if (!mbar_wait(&full[s], ph, tmo, s_abort) || !mbar_wait(&aempty[a], aph ^ 1, tmo, s_abort)) {
        fail(); ok = false; break;
      }
      const uint32_t src = sW + s * WP_BYTES;
      const uint32_t dst = sA + a * A_BYTES;
#pragma unroll
      for (int i = 0; i < (BNF * BK / 16) / 128; ++i) {
        const int w = ut + 128 * i;
        const int n = w >> 3, j = w & 7;
        const uint32_t word = ld_shared_u32(src + 4 * w);
        const uint4 o = unpack16_s8(word);
        st_shared_v4(dst + (n >> 3) * 1024 + (n & 7) * 128 + ((j ^ (n & 7)) << 4), o.x, o.y, o.z, o.w);
      }
      fence_proxy_async_smem();
      mbar_arrive(&afull[a]);
    }
    if (ok && kb1 > kb0) {
      if (mbar_wait(tfull, 0, tmo, s_abort)) have_acc = true;
      else fail();
    }
  }
  // partial sums: this CTA's [npad x 128] int32 block, aliased on the A ring
  // (every MMA has retired once tfull completed, and the unpack is finished)
  __syncthreads();
  int32_t* part = reinterpret_cast<int32_t*>(smem + OFF_A);
  if (warp >= 4) {
    tc_fence_after();
    const int q = warp & 3;
    const int nl = q * 32 + lane;
    for (int c0 = 0; c0 < p.npad; c0 += 32) {
      uint32_t r[32];
      tmem_ld32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + c0, r);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (c0 + i < p.npad) part[(c0 + i) * BNF + nl] = have_acc ? static_cast<int32_t>(r[i]) : 0;
    }
  }
  cluster_sync_all();
  if (rank == 0 && warp >= 4) {
    const int nl = (warp & 3) * 32 + lane;
    const int n = n0 + nl;
    const float gm = gamma_of(p, n);
    const uint32_t local = smem_u32(part);
    for (int m = 0; m < p.M; ++m) {
      int32_t acc = 0;
      for (int c = 0; c < p.csize; ++c)
        acc += ld_dsmem_s32(map_to_rank(local + 4u * static_cast<uint32_t>(m * BNF + nl), c));
      const float f = __fmul_rn(__fmul_rn(static_cast<float>(acc), __ldg(p.xs + m)), gm);
      p.y[static_cast<int64_t>(m) * p.ldy + n] = __bfloat16_as_ushort(__float2bfloat16_rn(f));
    }
  }
  cluster_sync_all();  // peers keep their shared memory until rank 0 is done
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, tmem_cols);
  }
}

}  // namespace gemv

cudaError_t launch_gemv(const GemmArgs& a, cudaStream_t s, const char** why) {
  using namespace gemv;
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) { *why = "cuTensorMapEncodeTiled unavailable"; return cudaErrorNotSupported; }
  Params p{};
  p.M = static_cast<int>(a.M);
  p.N = static_cast<int>(a.N);
  p.K = static_cast<int>(a.K);
  p.npad = p.M <= 16 ? 16 : (p.M <= 32 ? 32 : (p.M <= 48 ? 48 : 64));
  p.num_kb = p.K / BK;
  const int tiles = p.N / BNF;
  int c = 1;
  // split K over a cluster while the grid still fits in one wave
  while (c < 8 && tiles * 2 * c <= num_sms() && p.num_kb / (2 * c) >= 2) c *= 2;
  p.csize = c;
  p.xs = a.xs;
  p.gamma = a.gamma;
  p.G = a.G;
  for (int i = 0; i < 8; ++i) p.group_end[i] = a.group_end[i];
  p.y = reinterpret_cast<uint16_t*>(a.out);
  p.ldy = a.ldo;
  p.status = a.status;
  p.timeout_ns = a.timeout_ns;

  CUtensorMap tmX, tmW;
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.K), static_cast<cuuint64_t>(a.M)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.K)};
    const cuuint32_t box[2] = {BK, static_cast<cuuint32_t>(p.npad)};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&tmX, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(a.xq), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
      *why = "cuTensorMapEncodeTiled rejected the activation layout";
      return cudaErrorInvalidValue;
    }
  }
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.K / 4), static_cast<cuuint64_t>(a.N)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.K / 4)};
    const cuuint32_t box[2] = {BK / 4, BNF};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&tmW, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(a.Wp), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
      *why = "cuTensorMapEncodeTiled rejected the weight layout";
      return cudaErrorInvalidValue;
    }
  }
  static bool attr_set = false;  // once per process (not during graph capture)
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(bitlinear_gemv_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles * c));
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(c);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, bitlinear_gemv_kernel, tmX, tmW, p);
}

}  // namespace blt
