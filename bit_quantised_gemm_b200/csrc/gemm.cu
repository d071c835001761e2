// Prefill BitLinear GEMM on sm_100a tensor cores.
//
//   acc[m, n] = sum_k a[m, k] * w[k, n],  a = int8 codes (kind::i8, s32 acc)
//                                          or e2m1 codes (kind::f8f6f4, f32 acc)
//   y[m, n]   = bf16(acc * xs[m] * gamma[group(n)])   (or the raw acc)
//
// Persistent, warp-specialised kernel, one 128 x 256 output tile at a time:
//   warp 0      TMA producer: activation tile (128 x 128 B, 128-byte swizzle)
//               and packed-weight tile (256 rows x 32 B) into a 5-stage ring
//   warp 1      TMEM allocator and single-thread MMA issuer (4 MMAs of
//               K = 32 per 128-deep k-block, accumulator in TMEM)
//   warps 4-7   epilogue: tcgen05.ld of the accumulator (lane = row), scale,
//               bf16 pack, 16-byte global stores; TMEM holds two accumulators
//               so the epilogue of tile i overlaps the mainloop of tile i+1
//   warps 8-15  unpack: 2-bit weights -> int8 / padded e2m1 K-major tiles in
//               the 128-byte swizzled layout the MMA descriptors describe
//               (3-stage ring), then fence.proxy.async and an mbarrier arrive
// All waits are bounded (see ptx.cuh); a timeout sets a status bit and the
// CTA unwinds, releasing TMEM.
#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace blt {
namespace gemm {

constexpr int BM = 128, BN = 256, BK = 128;  // BK counted in elements
constexpr int S_TMA = 5, S_B = 3;
constexpr int A_BYTES = BM * 128;            // one 128-byte row per token
constexpr int WP_BYTES = BN * (BK / 4);      // 32 bytes of packed weights per row
constexpr int B_BYTES = BN * 128;
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + S_TMA * A_BYTES;
constexpr int OFF_WP = OFF_B + S_B * B_BYTES;
constexpr int OFF_BAR = OFF_WP + S_TMA * WP_BYTES;
constexpr int N_BARS = 2 * S_TMA + 2 * S_B + 2 * 2 + 1;
constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + slack for 1024-byte alignment
constexpr int THREADS = 512;
constexpr int TMEM_COLS = 512;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

struct Params {
  int M, N, K, num_kb, tiles_m, num_tiles;
  const float* xs;
  const float* gamma;
  int G;
  int group_end[8];
  void* out;
  int64_t ldo;
  int out_mode;
  int* status;
  uint64_t timeout_ns;
};

__device__ __forceinline__ float gamma_of(const Params& p, int n) {
  int g = 0;
#pragma unroll
  for (int i = 0; i < 7; ++i) g += (i < p.G - 1 && n >= p.group_end[i]) ? 1 : 0;
  return __ldg(p.gamma + g);
}

template <bool FP4>
__global__ void __launch_bounds__(THREADS, 1)
bitlinear_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                      const __grid_constant__ CUtensorMap tmW, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* full = bars;                    // TMA landed     [S_TMA]
  uint64_t* empty = full + S_TMA;           // MMA done with A/Wp slot [S_TMA]
  uint64_t* bfull = empty + S_TMA;          // unpacked B ready [S_B]
  uint64_t* bempty = bfull + S_B;           // MMA done with B slot [S_B]
  uint64_t* tfull = bempty + S_B;           // accumulator ready [2]
  uint64_t* tempty = tfull + 2;             // accumulator drained [2]
  uint64_t* mma_done = tempty + 2;          // all MMAs retired (teardown)
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S_TMA; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    for (int i = 0; i < S_B; ++i) { mbar_init(&bfull[i], 256); mbar_init(&bempty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&tfull[i], 1); mbar_init(&tempty[i], 128); }
    mbar_init(mma_done, 1);
    *s_abort = 0;
    fence_mbar_init();
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, TMEM_COLS);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;

  const uint32_t sA = smem_u32(smem + OFF_A);
  const uint32_t sB = smem_u32(smem + OFF_B);
  const uint32_t sW = smem_u32(smem + OFF_WP);
  const uint64_t tmo = p.timeout_ns;

  auto fail = [&]() {
    *s_abort = 1;
    report_status(p.status, BITLINEAR_STATUS_TIMEOUT);
  };

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
        const int m0 = (tile % p.tiles_m) * BM, n0 = (tile / p.tiles_m) * BN;
        for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
          const uint32_t s = it % S_TMA, ph = (it / S_TMA) & 1;
          if (!mbar_wait(&empty[s], ph ^ 1, tmo, s_abort)) { fail(); ok = false; break; }
          // transaction bytes count global bytes: packed e2m1 is half its smem footprint
          mbar_arrive_expect_tx(&full[s], (FP4 ? A_BYTES / 2 : A_BYTES) + WP_BYTES);
          tma_load_2d(smem + OFF_A + s * A_BYTES, &tmA, &full[s], kb * BK, m0);
          tma_load_2d(smem + OFF_WP + s * WP_BYTES, &tmW, &full[s], kb * (BK / 4), n0);
        }
      }
      // Do not leave while copies into this CTA's shared memory are in flight.
      const uint32_t inflight = it < S_TMA ? it : S_TMA;
      for (uint32_t d = 0; d < inflight; ++d) {
        const uint32_t j = it - 1 - d;
        mbar_wait(&full[j % S_TMA], (j / S_TMA) & 1, tmo, nullptr);
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = FP4 ? make_idesc(1, 5, 5, BM, BN) : make_idesc(2, 1, 1, BM, BN);
      uint32_t it = 0, tl = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x, ++tl) {
        const uint32_t acc = tl & 1, aph = (tl >> 1) & 1;
        if (!mbar_wait(&tempty[acc], aph ^ 1, tmo, s_abort)) { fail(); break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
          const uint32_t s = it % S_TMA, ph = (it / S_TMA) & 1;
          const uint32_t b = it % S_B, bph = (it / S_B) & 1;
          if (!mbar_wait(&full[s], ph, tmo, s_abort) || !mbar_wait(&bfull[b], bph, tmo, s_abort)) {
            fail(); ok = false; break;
          }
          tc_fence_after();
          const uint64_t adesc = smem_desc_sw128(sA + s * A_BYTES);
          const uint64_t bdesc = smem_desc_sw128(sB + b * B_BYTES);
#pragma unroll
          for (int k4 = 0; k4 < BK / 32; ++k4) {
            // advance 32 bytes (2 x 16 B) along K inside the swizzled row
            if (FP4) mma_f8f6f4(d_tmem, adesc + 2 * k4, bdesc + 2 * k4, idesc, (kb | k4) != 0);
            else     mma_i8(d_tmem, adesc + 2 * k4, bdesc + 2 * k4, idesc, (kb | k4) != 0);
          }
          tc_commit(&empty[s]);
          tc_commit(&bempty[b]);
        }
        if (ok) tc_commit(&tfull[acc]);
      }
      tc_commit(mma_done);
      mbar_wait(mma_done, 0, tmo, nullptr);
    }
  } else if (warp >= 4 && warp < 8) {
    // ----------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lane quadrant
    uint32_t tl = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++tl) {
      const int m0 = (tile % p.tiles_m) * BM, n0 = (tile / p.tiles_m) * BN;
      const uint32_t acc = tl & 1, aph = (tl >> 1) & 1;
      if (!mbar_wait(&tfull[acc], aph, tmo, s_abort)) { fail(); break; }
      tc_fence_after();
      const int m = m0 + q * 32 + lane;
      const bool row_ok = m < p.M;
      const float xs_m = (row_ok && p.out_mode == kOutBf16) ? __ldg(p.xs + m) : 0.f;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        const int n = n0 + c * 32;
        if (n >= p.N) break;  // warp-uniform
        uint32_t r[32];
        tmem_ld32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * BN + c * 32, r);
        tmem_ld_wait();
        if (!row_ok) continue;
        if (p.out_mode == kOutBf16) {
          uint16_t* yrow = reinterpret_cast<uint16_t*>(p.out) + static_cast<int64_t>(m) * p.ldo + n;
          float gm[32];
          if (p.G == 1) {
            const float g0 = __ldg(p.gamma);
#pragma unroll
            for (int i = 0; i < 32; ++i) gm[i] = g0;
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) gm[i] = gamma_of(p, n + i);
          }
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            if (n + 8 * v >= p.N) break;
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int e = 8 * v + 2 * i;
              float f0, f1;
              if (FP4) { f0 = __uint_as_float(r[e]); f1 = __uint_as_float(r[e + 1]); }
              else { f0 = static_cast<float>(static_cast<int32_t>(r[e]));
                     f1 = static_cast<float>(static_cast<int32_t>(r[e + 1])); }
              f0 = __fmul_rn(__fmul_rn(f0, xs_m), gm[e]);
              f1 = __fmul_rn(__fmul_rn(f1, xs_m), gm[e + 1]);
              w[i] = pack_bf16x2(f0, f1);
            }
            reinterpret_cast<uint4*>(yrow)[v] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        } else {
          uint32_t* orow = reinterpret_cast<uint32_t*>(p.out) + static_cast<int64_t>(m) * p.ldo + n;
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            if (n + 4 * v >= p.N) break;
            reinterpret_cast<uint4*>(orow)[v] =
                make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------- unpack
    const int ut = threadIdx.x - 256;  // 0..255
    uint32_t it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
      for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
        const uint32_t s = it % S_TMA, ph = (it / S_TMA) & 1;
        const uint32_t b = it % S_B, bph = (it / S_B) & 1;
        if (!mbar_wait(&full[s], ph, tmo, s_abort) || !mbar_wait(&bempty[b], bph ^ 1, tmo, s_abort)) {
          fail(); ok = false; break;
        }
        const uint32_t src = sW + s * WP_BYTES;
        const uint32_t dst = sB + b * B_BYTES;
#pragma unroll
        for (int i = 0; i < (BN * BK / 16) / 256; ++i) {
          const int w = ut + 256 * i;     // packed word index in the tile
          const int n = w >> 3, j = w & 7;  // row, 16-byte chunk along K
          const uint32_t word = ld_shared_u32(src + 4 * w);
          const uint4 o = FP4 ? unpack16_e2m1(word) : unpack16_s8(word);
          const uint32_t addr = dst + (n >> 3) * 1024 + (n & 7) * 128 + ((j ^ (n & 7)) << 4);
          st_shared_v4(addr, o.x, o.y, o.z, o.w);
        }
        fence_proxy_async_smem();
        mbar_arrive(&bfull[b]);
      }
    }
  }

  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace gemm

static cudaError_t make_map_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base,
                               uint64_t inner, uint64_t outer, uint64_t row_bytes,
                               uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw,
                               const char** why) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) { *why = "cuTensorMapEncodeTiled unavailable"; return cudaErrorNotSupported; }
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) { *why = "cuTensorMapEncodeTiled rejected the operand layout"; return cudaErrorInvalidValue; }
  return cudaSuccess;
}

cudaError_t launch_gemm(const GemmArgs& a, bool fp4, cudaStream_t s, const char** why) {
  using namespace gemm;
  CUtensorMap tmA, tmW;
  cudaError_t e;
  if (fp4)
    e = make_map_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, a.xq, a.K, a.M, a.K / 2, BK, BM,
                    CU_TENSOR_MAP_SWIZZLE_128B, why);
  else
    e = make_map_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.xq, a.K, a.M, a.K, BK, BM,
                    CU_TENSOR_MAP_SWIZZLE_128B, why);
  if (e != cudaSuccess) return e;
  e = make_map_2d(&tmW, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.Wp, a.K / 4, a.N, a.K / 4, BK / 4, BN,
                  CU_TENSOR_MAP_SWIZZLE_NONE, why);
  if (e != cudaSuccess) return e;

  Params p{};
  p.M = static_cast<int>(a.M);
  p.N = static_cast<int>(a.N);
  p.K = static_cast<int>(a.K);
  p.num_kb = static_cast<int>((a.K + BK - 1) / BK);
  p.tiles_m = static_cast<int>((a.M + BM - 1) / BM);
  const int tiles_n = static_cast<int>((a.N + BN - 1) / BN);
  p.num_tiles = p.tiles_m * tiles_n;
  p.xs = a.xs;
  p.gamma = a.gamma;
  p.G = a.G;
  for (int i = 0; i < 8; ++i) p.group_end[i] = a.group_end[i];
  p.out = a.out;
  p.ldo = a.ldo;
  p.out_mode = a.out_mode;
  p.status = a.status;
  p.timeout_ns = a.timeout_ns;

  auto kern = fp4 ? bitlinear_gemm_kernel<true> : bitlinear_gemm_kernel<false>;
  static bool attr_set[2] = {false, false};  // once per process (not during graph capture)
  if (!attr_set[fp4 ? 1 : 0]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set[fp4 ? 1 : 0] = true;
  }
  const int grid = p.num_tiles < num_sms() ? p.num_tiles : num_sms();
  kern<<<grid, THREADS, SMEM_BYTES, s>>>(tmA, tmW, p);
  return cudaGetLastError();
}

}  // namespace blt
