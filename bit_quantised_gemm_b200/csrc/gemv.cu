// Decode-time BitLinear (1..64 tokens) on sm_100a tensor cores.
//
// With few tokens the layer is bound by reading the packed weights from
// HBM, so the kernel is arranged around the weight stream ("swap AB"):
//   A = unpacked ternary weights, 128 output features x K   (M side, 128)
//   B = int8 activation codes, Npad tokens x K              (N side, 16..64)
//   D[n, m] in TMEM: lane = output feature, column = token.
// One CTA owns 128 output features and one K slice; the C CTAs of a thread
// block cluster split K and reduce their int32 partials through distributed
// shared memory, so every weight byte is read once and no global scratch is
// used. A TMA instruction costs its issuing thread a few hundred ns whatever
// its size, so loads move 512-deep super-stages (16 KB of packed weights,
// Npad x 512 B of activations) from two issuing warps.
//   warp 0      TMA: packed weights, 128 rows x 128 B, 128-byte swizzle
//   warp 1      TMEM allocator + single-thread MMA issuer
//   warp 2      TMA: activation codes, 4 chunks x Npad rows x 128 B (3-D box)
//   warps 4-11  unpack 2-bit weights into the swizzled A ring (one 16-byte
//               read and four 16-byte writes per thread per chunk); warps 4-7
//               then run the epilogue (TMEM -> registers -> DSMEM reduction
//               on cluster rank 0 -> bf16 y)
#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace blt {
namespace gemv {

constexpr int BNF = 128;                  // output features per CTA
constexpr int CH = 128;                   // K chunk (one MMA group of 4 x K=32)
constexpr int SUPER = 4;                  // chunks per TMA super-stage
constexpr int S = 3, SA = 4;              // super-stage ring, unpacked-chunk ring
constexpr int WP_BYTES = BNF * (SUPER * CH / 4);  // 16 KB
constexpr int X_CHUNK = 64 * CH;          // room for 64 token rows per chunk
constexpr int X_BYTES = SUPER * X_CHUNK;  // 32 KB
constexpr int A_BYTES = BNF * CH;         // 16 KB
constexpr int OFF_A = 0;                  // 1024-aligned regions
constexpr int OFF_X = OFF_A + SA * A_BYTES;
constexpr int OFF_WP = OFF_X + S * X_BYTES;
constexpr int OFF_BAR = OFF_WP + S * WP_BYTES;
constexpr int N_BARS = 3 * S + 2 * SA + 2;
constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
constexpr int THREADS = 384;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(SA * A_BYTES >= 64 * BNF * 4, "partials alias the A ring");

struct Params {
  int M, N, K, npad, nchunks, csize;
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
  uint64_t* wfull = reinterpret_cast<uint64_t*>(smem + OFF_BAR);  // packed weights landed [S]
  uint64_t* xfull = wfull + S;                                     // activations landed [S]
  uint64_t* sempty = xfull + S;                                    // super-stage consumed [S]
  uint64_t* afull = sempty + S;                                    // unpacked chunk ready [SA]
  uint64_t* aempty = afull + SA;                                   // MMA done with chunk [SA]
  uint64_t* tfull = aempty + SA;
  uint64_t* mma_done = tfull + 1;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const uint32_t rank = cluster_ctarank();
  const int tile = blockIdx.x / p.csize;
  const int n0 = tile * BNF;
  const int c0 = static_cast<int>((static_cast<int64_t>(p.nchunks) * rank) / p.csize);
  const int c1 = static_cast<int>((static_cast<int64_t>(p.nchunks) * (rank + 1)) / p.csize);
  const int nch = c1 - c0;                          // chunks of this CTA
  const int nsup = (nch + SUPER - 1) / SUPER;       // super-stages of this CTA
  const uint32_t tmem_cols = p.npad <= 32 ? 32u : 64u;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&wfull[i], 1);
      mbar_init(&xfull[i], 1);
      mbar_init(&sempty[i], 1);
    }
    for (int i = 0; i < SA; ++i) { mbar_init(&afull[i], 8); mbar_init(&aempty[i], 1); }
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
  pdl_trigger();  // TMEM is held: the next kernel in the stream may start
  const uint64_t tmo = p.timeout_ns;
  const uint32_t sA = smem_u32(smem + OFF_A);
  const uint32_t sX = smem_u32(smem + OFF_X);
  const uint32_t sW = smem_u32(smem + OFF_WP);
  auto fail = [&]() {
    *s_abort = 1;
    report_status(p.status, BITLINEAR_STATUS_TIMEOUT);
  };
  bool have_acc = false;

  if (warp == 0 || warp == 2) {
    // -------------------------------------------- TMA (weights: warp 0, activations: warp 2)
    if (lane == 0) {
      const bool wts = warp == 0;
      // activation codes come from the previous kernel (the row scales and y
      // are touched after the block-wide barrier that follows this wait)
      if (!wts) pdl_wait();
      int issued = 0;
      for (int j = 0; j < nsup; ++j, ++issued) {
        const uint32_t s = j % S, ph = (j / S) & 1;
        if (!mbar_wait(&sempty[s], ph ^ 1, tmo, s_abort)) { fail(); break; }
        const int kc = c0 + j * SUPER;  // first chunk of the super-stage
        if (wts) {
          mbar_arrive_expect_tx(&wfull[s], WP_BYTES);
          tma_load_2d(smem + OFF_WP + s * WP_BYTES, &tmW, &wfull[s], kc * (CH / 4), n0);
        } else {
          mbar_arrive_expect_tx(&xfull[s], SUPER * p.npad * CH);
          tma_load_3d(smem + OFF_X + s * X_BYTES, &tmX, &xfull[s], 0, 0, kc);
        }
      }
      const int inflight = issued < S ? issued : S;
      for (int d = 0; d < inflight; ++d) {
        const int j = issued - 1 - d;
        mbar_wait(wts ? &wfull[j % S] : &xfull[j % S], (j / S) & 1, tmo, nullptr);
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = make_idesc(2, 1, 1, BNF, p.npad);
      bool ok = true;
      for (int c = 0; ok && c < nch; ++c) {
        const int j = c / SUPER, q = c % SUPER;
        const uint32_t s = j % S, ph = (j / S) & 1;
        const uint32_t a = c % SA, aph = (c / SA) & 1;
        if ((q == 0 && !mbar_wait(&xfull[s], ph, tmo, s_abort)) ||
            !mbar_wait(&afull[a], aph, tmo, s_abort)) {
          fail(); ok = false; break;
        }
        tc_fence_after();
        const uint64_t adesc = smem_desc_sw128(sA + a * A_BYTES);
        const uint64_t bdesc = smem_desc_sw128(sX + s * X_BYTES + q * (p.npad * CH));
#pragma unroll
        for (int k4 = 0; k4 < CH / 32; ++k4)
          mma_i8(tmem_base, adesc + 2 * k4, bdesc + 2 * k4, idesc, (c != 0) || (k4 != 0));
        tc_commit(&aempty[a]);
        if (q == SUPER - 1 || c == nch - 1) tc_commit(&sempty[s]);  // super-stage consumed
      }
      if (ok && nch > 0) tc_commit(tfull);
      tc_commit(mma_done);
      mbar_wait(mma_done, 0, tmo, nullptr);
    }
  } else if (warp >= 4) {
    // --------------------------------------------- unpack, then epilogue
    const int ut = threadIdx.x - 128;  // 0..255: weight row ut/2, half ut%2 of a 32-byte chunk
    const int n = ut >> 1, h = ut & 1;
    bool ok = true;
    for (int c = 0; c < nch; ++c) {
      const int j = c / SUPER, q = c % SUPER;
      const uint32_t s = j % S, ph = (j / S) & 1;
      const uint32_t a = c % SA, aph = (c / SA) & 1;
      if ((q == 0 && !mbar_wait(&wfull[s], ph, tmo, s_abort)) ||
          !mbar_wait(&aempty[a], aph ^ 1, tmo, s_abort)) {
        fail(); ok = false; break;
      }
      // packed row n: 128 B per super-stage, 16-byte unit u = 2q + h, stored
      // at u ^ (n & 7) by the 128-byte swizzle of the weight tile
      const uint32_t u = static_cast<uint32_t>(2 * q + h) ^ static_cast<uint32_t>(n & 7);
      const uint4 wv = ld_shared_v4(sW + s * WP_BYTES + n * 128 + u * 16);
      const uint32_t dst = sA + a * A_BYTES + (n >> 3) * 1024 + (n & 7) * 128;
      const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int cc = 4 * h + i;  // 16-deep K group within the 128-deep chunk
        const uint4 o = unpack16_s8(words[i]);
        st_shared_v4(dst + ((cc ^ (n & 7)) << 4), o.x, o.y, o.z, o.w);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&afull[a]);  // one arrival per unpack warp
    }
    if (ok && nch > 0 && warp < 8) {
      if (mbar_wait(tfull, 0, tmo, s_abort)) have_acc = true;
      else fail();
    }
  }
  // partial sums: this CTA's [npad x 128] int32 block, aliased on the A ring
  // (every MMA has retired once mma_done completed, and the unpack is done)
  __syncthreads();
  int32_t* part = reinterpret_cast<int32_t*>(smem + OFF_A);
  if (warp >= 4 && warp < 8) {
    tc_fence_after();
    const int q = warp & 3;
    const int nl = q * 32 + lane;
    for (int col = 0; col < p.npad; col += 32) {
      uint32_t r[32];
      tmem_ld32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + col, r);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (col + i < p.npad) part[(col + i) * BNF + nl] = have_acc ? static_cast<int32_t>(r[i]) : 0;
    }
  }
  cluster_sync();
  if (rank == 0 && warp >= 4 && warp < 8) {
    const int nl = (warp & 3) * 32 + lane;
    const int nn = n0 + nl;
    const float gm = gamma_of(p, nn);
    const uint32_t local = smem_u32(part);
    uint32_t base[8];
    for (int r = 0; r < p.csize; ++r) base[r] = map_shared_rank(local, r);
    for (int m = 0; m < p.M; ++m) {
      int32_t acc = 0;
      const uint32_t off = 4u * static_cast<uint32_t>(m * BNF + nl);
      for (int r = 0; r < p.csize; ++r) acc += ld_dsmem_s32(base[r] + off);
      const float f = __fmul_rn(static_cast<float>(acc), __fmul_rn(__ldg(p.xs + m), gm));
      p.y[static_cast<int64_t>(m) * p.ldy + nn] = __bfloat16_as_ushort(__float2bfloat16_rn(f));
    }
  }
  cluster_sync();  // peers keep their shared memory until rank 0 is done
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
  p.nchunks = p.K / CH;
  const int tiles = p.N / BNF;
  int c = 1;
  // split K over a cluster while the grid still fits in one wave and every
  // CTA keeps at least two chunks
  while (c < 8 && tiles * 2 * c <= num_sms() && p.nchunks / (2 * c) >= 2) c *= 2;
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
    // activations as [K/128 chunks][M rows][128 B]; a box = SUPER chunks x npad rows
    const cuuint64_t dims[3] = {CH, static_cast<cuuint64_t>(a.M), static_cast<cuuint64_t>(p.nchunks)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(a.K), CH};
    const cuuint32_t box[3] = {CH, static_cast<cuuint32_t>(p.npad), SUPER};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (enc(&tmX, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(a.xq), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
      *why = "cuTensorMapEncodeTiled rejected the activation layout";
      return cudaErrorInvalidValue;
    }
  }
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.K / 4), static_cast<cuuint64_t>(a.N)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.K / 4)};
    const cuuint32_t box[2] = {SUPER * CH / 4, BNF};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&tmW, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(a.Wp), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
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
  return launch_kernel(bitlinear_gemv_kernel, dim3(static_cast<unsigned>(tiles * c)), dim3(THREADS),
                       SMEM_BYTES, s, static_cast<unsigned>(c), tmX, tmW, p);
}

}  // namespace blt
