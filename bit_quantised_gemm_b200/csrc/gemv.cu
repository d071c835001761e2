// Decode-time BitLinear (up to 64 tokens) on sm_100a tensor cores.
//
// With few tokens the layer is bound by reading the packed weights from
// HBM, so the kernel is arranged around the weight stream ("swap AB"):
//   A = unpacked ternary weights, 128 output features x K   (M side, 128)
//   B = int8 activation codes, Npad tokens x K              (N side, 16..64)
//   D[n, m] in TMEM: lane = output feature, column = token.
// The unpacked weights never touch shared memory: each unpack thread owns
// one weight row (= one TMEM lane), expands 2-bit codes to int8 in
// registers and writes them into tensor memory with tcgen05.st; the MMA
// reads A from tensor memory and B (the activation codes) from shared
// memory. Shared memory then carries only the packed weights (once) and the
// activation tiles, so its bandwidth is no longer the limit.
//
// One CTA owns 128 output features and one K slice; the C CTAs of a thread
// block cluster split K and reduce their int32 partials through distributed
// shared memory, so every weight byte is read once and no global scratch is
// used. K moves in chunks of 512: one 16 KB TMA box of packed weights (128
// rows x 128 B, 128-byte swizzle) and one 3-D box of activation codes (4 x
// Npad rows x 128 B), issued by their own warps (two for the weights, which
// take alternate chunks, since a TMA instruction costs its issuing thread a
// few hundred ns).
//   warp 0, 3   TMA: packed weights (even / odd chunks)
//   warp 1      TMEM allocator + single-thread MMA issuer
//   warp 2      TMA: activation codes
//   warps 4-7   unpack even chunks into TMEM, then the epilogue
//   warps 8-11  unpack odd chunks into TMEM
// Tensor memory (512 columns): the accumulator in columns [0, 64), then RA
// slots of 128 columns, one per chunk in flight (512 int8 per lane).
#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace blt {
namespace gemv {

constexpr int BNF = 128;                   // output features per CTA (MMA M, TMEM lanes)
constexpr int CK = 512;                    // K per chunk
constexpr int SUBS = CK / 128;             // 128-deep sub-chunks per chunk (32 TMEM columns each)
constexpr int S_W = 6;                     // packed-weight stages
constexpr int S_X = 3;                     // activation stages
constexpr int RA = 3;                      // unpacked chunks in TMEM
constexpr int D_COLS = 64;                 // accumulator columns (Npad <= 64)
constexpr int TMEM_COLS = 512;
constexpr int W_BYTES = BNF * (CK / 4);    // 16 KB
constexpr int X_BYTES = 64 * CK;           // room for 64 token rows x 512 codes
constexpr int OFF_W = 0;                   // 1024-aligned regions
constexpr int OFF_X = OFF_W + S_W * W_BYTES;
constexpr int OFF_BAR = OFF_X + S_X * X_BYTES;
constexpr int N_BARS = 2 * S_W + 2 * S_X + 2 * RA + 2;
constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
constexpr int OFF_SCALES = OFF_MISC + 16;    // row scales [64], then gamma [8]
constexpr int SMEM_BYTES = OFF_SCALES + (64 + 8) * 4 + 1024;
constexpr int THREADS = 384;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(D_COLS + RA * 128 <= TMEM_COLS, "tensor memory budget");
static_assert(S_W * W_BYTES >= 64 * BNF * 4, "partials alias the weight ring");
static_assert(S_W % 2 == 0, "two weight producers take alternate chunks");

struct Params {
  int M, N, K, npad, nsubs, nchunks, csize;
  const float* xs;
  const float* gamma;
  int G;
  int group_end[8];
  uint16_t* y;
  int64_t ldy;
  int* status;
  uint64_t timeout_ns;
};

// Scale of output feature n's column group, from the copy in shared memory.
__device__ __forceinline__ float gamma_of(const Params& p, const float* gam_s, int n) {
  int g = 0;
#pragma unroll
  for (int i = 0; i < 7; ++i) g += (i < p.G - 1 && n >= p.group_end[i]) ? 1 : 0;
  return gam_s[g];
}

__device__ __forceinline__ int32_t ld_dsmem_s32(uint32_t addr) {
  int32_t v;
  asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

// Expand 128 packed codes (32 bytes of one weight row, as two swizzled
// 16-byte units) into 32 words of four int8 weights, lowest k first.
__device__ __forceinline__ void unpack_row128(uint32_t row_addr, int sub, int n, uint32_t (&r)[32]) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t u = static_cast<uint32_t>(2 * sub + h) ^ static_cast<uint32_t>(n & 7);
    const uint4 wv = ld_shared_v4(row_addr + u * 16);
    const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 o = unpack16_s8(words[i]);
      r[16 * h + 4 * i + 0] = o.x;
      r[16 * h + 4 * i + 1] = o.y;
      r[16 * h + 4 * i + 2] = o.z;
      r[16 * h + 4 * i + 3] = o.w;
    }
  }
}

__global__ void __launch_bounds__(THREADS, 1)
bitlinear_gemv_kernel(const __grid_constant__ CUtensorMap tmX,
                      const __grid_constant__ CUtensorMap tmW, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* wfull = reinterpret_cast<uint64_t*>(smem + OFF_BAR);  // packed weights landed [S_W]
  uint64_t* wempty = wfull + S_W;                                  // packed weights unpacked [S_W]
  uint64_t* xfull = wempty + S_W;                                  // activations landed [S_X]
  uint64_t* xempty = xfull + S_X;                                  // activations consumed [S_X]
  uint64_t* afull = xempty + S_X;                                  // chunk in TMEM [RA]
  uint64_t* aempty = afull + RA;                                   // MMA done with slot [RA]
  uint64_t* tfull = aempty + RA;
  uint64_t* mma_done = tfull + 1;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);
  float* xs_s = reinterpret_cast<float*>(smem + OFF_SCALES);  // row scales [M]
  float* gam_s = xs_s + 64;                                    // group scales [G]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const uint32_t rank = cluster_ctarank();
  const int tile = blockIdx.x / p.csize;
  const int n0 = tile * BNF;
  const int c0 = static_cast<int>((static_cast<int64_t>(p.nchunks) * rank) / p.csize);
  const int c1 = static_cast<int>((static_cast<int64_t>(p.nchunks) * (rank + 1)) / p.csize);
  const int nch = c1 - c0;  // chunks of this CTA

  if (threadIdx.x == 0) {
    for (int i = 0; i < S_W; ++i) { mbar_init(&wfull[i], 1); mbar_init(&wempty[i], 4); }
    for (int i = 0; i < S_X; ++i) { mbar_init(&xfull[i], 1); mbar_init(&xempty[i], 1); }
    for (int i = 0; i < RA; ++i) { mbar_init(&afull[i], 4); mbar_init(&aempty[i], 1); }
    mbar_init(tfull, 1);
    mbar_init(mma_done, 1);
    *s_abort = 0;
    fence_mbar_init();
    prefetch_tensormap(&tmX);
    prefetch_tensormap(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, TMEM_COLS);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  pdl_trigger();  // TMEM is held: the next kernel in the stream may start
  const uint64_t tmo = p.timeout_ns;
  const uint32_t sX = smem_u32(smem + OFF_X);
  const uint32_t sW = smem_u32(smem + OFF_W);
  auto fail = [&]() {
    *s_abort = 1;
    report_status(p.status, BITLINEAR_STATUS_TIMEOUT);
  };
  // 128-deep sub-chunks in this CTA's chunk c (the last chunk of K may be short)
  auto nsub_of = [&](int c) { return min(SUBS, p.nsubs - (c0 + c) * SUBS); };
  bool have_acc = false;

  if (warp == 0 || warp == 3) {
    // ------------------------------------ TMA: packed weights (alternate chunks)
    if (lane == 0) {
      const int par = warp == 0 ? 0 : 1;
      int last = -1;
      for (int c = par; c < nch; c += 2) {
        const uint32_t s = c % S_W, ph = (c / S_W) & 1;
        if (!mbar_wait(&wempty[s], ph ^ 1, tmo, s_abort)) { fail(); break; }
        mbar_arrive_expect_tx(&wfull[s], W_BYTES);
        tma_load_2d(smem + OFF_W + s * W_BYTES, &tmW, &wfull[s], (c0 + c) * (CK / 4), n0);
        last = c;
      }
      // Do not leave while copies into this CTA's shared memory are in
      // flight: the last issue of each slot this producer uses.
      for (int d = 0, c = last; d < S_W / 2 && c >= par; ++d, c -= 2)
        mbar_wait(&wfull[c % S_W], (c / S_W) & 1, tmo, nullptr);
    }
  } else if (warp == 2) {
    // ---------------------------------------------- TMA: activation codes
    // activation codes and row scales come from the previous kernel (y is
    // written after the block-wide barrier that follows this wait). The
    // warp stages the row and group scales in shared memory here, so that
    // the epilogue reads no global memory before its stores.
    pdl_wait();
    for (int m = lane; m < p.M; m += 32) xs_s[m] = __ldg(p.xs + m);
    if (lane < p.G) gam_s[lane] = __ldg(p.gamma + lane);
    if (lane == 0) {
      int last = -1;
      for (int c = 0; c < nch; ++c) {
        const uint32_t s = c % S_X, ph = (c / S_X) & 1;
        if (!mbar_wait(&xempty[s], ph ^ 1, tmo, s_abort)) { fail(); break; }
        mbar_arrive_expect_tx(&xfull[s], SUBS * p.npad * 128);
        tma_load_3d(smem + OFF_X + s * X_BYTES, &tmX, &xfull[s], 0, 0, (c0 + c) * SUBS);
        last = c;
      }
      for (int d = 0, c = last; d < S_X && c >= 0; ++d, --c)
        mbar_wait(&xfull[c % S_X], (c / S_X) & 1, tmo, nullptr);
    }
  } else if (warp == 1) {
    // -------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = make_idesc(2, 1, 1, BNF, p.npad);
      bool ok = true;
      for (int c = 0; ok && c < nch; ++c) {
        const uint32_t sx = c % S_X, xph = (c / S_X) & 1;
        const uint32_t a = c % RA, aph = (c / RA) & 1;
        if (!mbar_wait(&xfull[sx], xph, tmo, s_abort) || !mbar_wait(&afull[a], aph, tmo, s_abort)) {
          fail(); ok = false; break;
        }
        tc_fence_after();
        const int ns = nsub_of(c);
        for (int sub = 0; sub < ns; ++sub) {
          const uint64_t bdesc = smem_desc_sw128(sX + sx * X_BYTES + sub * (p.npad * 128));
          const uint32_t acol = tmem_base + D_COLS + a * 128 + sub * 32;
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4)
            mma_i8_ts(tmem_base, acol + 8 * k4, bdesc + 2 * k4, idesc, (c | sub | k4) != 0);
        }
        tc_commit(&aempty[a]);   // TMEM slot free once these MMAs retire
        tc_commit(&xempty[sx]);  // activation stage too
      }
      if (ok && nch > 0) tc_commit(tfull);
      tc_commit(mma_done);
      mbar_wait(mma_done, 0, tmo, nullptr);
    }
  } else if (warp >= 4) {
    // -------------------------------- unpack into TMEM (then the epilogue)
    const int g = (warp - 4) >> 2;          // group 0: even chunks, 1: odd chunks
    const int q = warp & 3;                 // TMEM lane quarter of this warp
    const int n = q * 32 + lane;            // weight row = TMEM lane
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    bool ok = true;
    for (int c = g; c < nch; c += 2) {
      const uint32_t s = c % S_W, ph = (c / S_W) & 1;
      const uint32_t a = c % RA, aph = (c / RA) & 1;
      if (!mbar_wait(&wfull[s], ph, tmo, s_abort) || !mbar_wait(&aempty[a], aph ^ 1, tmo, s_abort)) {
        fail(); ok = false; break;
      }
      tc_fence_after();  // the MMAs that read this slot before have retired
      const int ns = nsub_of(c);
      const uint32_t row = sW + s * W_BYTES + n * 128;
      for (int sub = 0; sub < ns; ++sub) {
        uint32_t r[32];
        unpack_row128(row, sub, n, r);
        tmem_st32(lane_base + D_COLS + a * 128 + sub * 32, r);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&wempty[s]);  // packed weights read
        mbar_arrive(&afull[a]);   // unpacked chunk in TMEM
      }
    }
    if (ok && nch > 0 && g == 0) {
      if (mbar_wait(tfull, 0, tmo, s_abort)) have_acc = true;
      else fail();
    }
  }
  // partial sums: this CTA's [npad x 128] int32 block, aliased on the weight
  // ring (every load has landed and been unpacked, every MMA has retired)
  __syncthreads();
  int32_t* part = reinterpret_cast<int32_t*>(smem + OFF_W);
  if (warp >= 4 && warp < 8) {
    tc_fence_after();
    const int q = warp & 3;
    const int nl = q * 32 + lane;
    if (p.csize == 1) {
      // K is not split: each thread's accumulator row is final, so it goes
      // from tensor memory to y directly (no partials, no DSMEM round trip)
      const int nn = n0 + nl;
      const float gm = gamma_of(p, gam_s, nn);
      uint16_t* yc = p.y + nn;
      for (int col = 0; col < p.npad && col < p.M; col += 32) {
        uint32_t r[32];
        tmem_ld32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + col, r);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int m = col + i;
          if (m < p.M) {
            const int32_t acc = have_acc ? static_cast<int32_t>(r[i]) : 0;
            const float f = __fmul_rn(static_cast<float>(acc), __fmul_rn(xs_s[m], gm));
            yc[static_cast<int64_t>(m) * p.ldy] = __bfloat16_as_ushort(__float2bfloat16_rn(f));
          }
        }
      }
    } else {
      for (int col = 0; col < p.npad; col += 32) {
        uint32_t r[32];
        tmem_ld32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + col, r);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (col + i < p.npad) part[(col + i) * BNF + nl] = have_acc ? static_cast<int32_t>(r[i]) : 0;
      }
    }
  }
  cluster_sync();
  // the cluster's CTAs share the rows of the final reduction: CTA r sums the
  // partials of rows r, r + csize, ... over every CTA's shared memory. Rows
  // go in groups of 8 so that a thread has 8 DSMEM loads in flight per CTA
  // rather than one dependent load at a time.
  if (p.csize > 1 && warp >= 4 && warp < 8) {
    const int nl = (warp & 3) * 32 + lane;
    const int nn = n0 + nl;
    const float gm = gamma_of(p, gam_s, nn);
    const uint32_t local = smem_u32(part);
    uint32_t base[8];
    for (int r = 0; r < p.csize; ++r) base[r] = map_shared_rank(local, r);
    const int step = p.csize;
    for (int m0 = static_cast<int>(rank); m0 < p.M; m0 += 8 * step) {
      int32_t acc[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[j] = 0;
      for (int r = 0; r < p.csize; ++r) {
        int32_t v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int m = min(m0 + j * step, p.npad - 1);  // rows past M read padding, never stored
          v[j] = ld_dsmem_s32(base[r] + 4u * static_cast<uint32_t>(m * BNF + nl));
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] += v[j];
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int m = m0 + j * step;
        if (m < p.M) {
          const float f = __fmul_rn(static_cast<float>(acc[j]), __fmul_rn(xs_s[m], gm));
          p.y[static_cast<int64_t>(m) * p.ldy + nn] = __bfloat16_as_ushort(__float2bfloat16_rn(f));
        }
      }
    }
  }
  cluster_sync();  // every CTA keeps its shared memory until the others are done
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
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
  p.nsubs = p.K / 128;
  p.nchunks = (p.nsubs + SUBS - 1) / SUBS;
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
    // activations as [K/128 sub-chunks][M rows][128 B]; a box = SUBS sub-chunks x npad rows
    // (rows past M and sub-chunks past K read as zero)
    const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(a.M), static_cast<cuuint64_t>(p.nsubs)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(a.K), 128};
    const cuuint32_t box[3] = {128, static_cast<cuuint32_t>(p.npad), SUBS};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (enc(&tmX, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(a.xq), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
      *why = "cuTensorMapEncodeTiled rejected the activation layout";
      return cudaErrorInvalidValue;
    }
  }
  {
    // packed weights [N rows][K/4 B]; a box = 128 rows x 128 B (512 codes)
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(a.K / 4), static_cast<cuuint64_t>(a.N)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(a.K / 4)};
    const cuuint32_t box[2] = {CK / 4, BNF};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&tmW, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(a.Wp), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
      *why = "cuTensorMapEncodeTiled rejected the weight layout";
      return cudaErrorInvalidValue;
    }
  }
  cudaError_t e = set_smem_limit(bitlinear_gemv_kernel, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  return launch_kernel(bitlinear_gemv_kernel, dim3(static_cast<unsigned>(tiles * c)), dim3(THREADS),
                       SMEM_BYTES, s, static_cast<unsigned>(c), tmX, tmW, p);
}

}  // namespace blt
