// Prefill BitLinear GEMM on sm_100a tensor cores.
//
//   acc[m, n] = sum_k a[m, k] * w[k, n],  a = int8 codes (kind::i8, s32 acc)
//                                          or e2m1 codes (f32 acc: kind::mxf4
//                                          for CTA pairs, kind::f8f6f4 else)
//   y[m, n]   = bf16(acc * (xs[m] * gamma[group(n)]))   (or the raw acc)
//
// FP4 on CTA pairs (K a multiple of 256) runs at the full 4-bit tensor rate
// through the block-scaled kind::mxf4: A and B are packed e2m1 (two per
// byte, 128 bytes = 256 k per swizzled row, half the shared-memory bytes of
// the padded f8f6f4 form that other K take), and every ue8m0 block scale
// is 1.0 (0x7F), written once into tensor memory at start-up, so the
// products and their fp32 sums are those of the unscaled codes. The scale columns take part of tensor memory, so
// these tiles are 192 outputs wide (two accumulators of 192 columns + the
// scales in 512).
//
// Persistent, warp-specialised kernel. In the CTA-pair form (two CTAs of a
// cluster on one TPC, tcgen05 cta_group::2) a pair owns a 256-token x
// 256-output tile (192 for mxf4): each CTA loads its own 128 token rows of
// activations and unpacks its own half of the weight rows, and one MMA of
// M = 256 reads both CTAs' shared memory, so each SM stages half of the
// unpacked weights (the single-CTA form stages all 256 rows and is used for
// M <= 128). A k-block is 256 deep on pairs (512 for mxf4: one 32 KB
// activation box either way), 128 on single CTAs.
//   warp 0      TMA producer of the activation tiles (one box per k-block,
//               128-byte swizzle; on pairs the completion goes to the even
//               CTA's barrier)
//   warp 2      TMA producer of the packed-weight tiles (K/4 bytes per row)
//   warp 1      TMEM allocator; in the even CTA the single-thread MMA issuer
//               (K = 32 per MMA for kind::i8 / f8f6f4, 64 for mxf4; the
//               accumulator in TMEM)
//   warps 4-7   epilogue: tcgen05.ld (lane = token row, 64 columns at a
//               time), scale, bf16 pack, 128-byte-swizzled staging and one
//               TMA store per 32 x 64 block; two TMEM accumulators so the
//               epilogue of one tile overlaps the mainloop of the next
//   warps 8-15  unpack: 2-bit weights -> int8 / e2m1 K-major tiles in the
//               swizzled layout the MMA descriptors describe, then
//               fence.proxy.async and an mbarrier arrive (on the even CTA);
//               for mxf4 two groups of 4 warps take alternate k-blocks
// All waits are bounded (see ptx.cuh); a timeout sets a status bit and the
// CTA unwinds, releasing TMEM.
#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace blt {
namespace gemm {

constexpr int BM = 128;            // token rows per CTA
constexpr int BN = 256;            // output columns per tile
constexpr int SUB = BM * 128;      // one 128-deep K chunk of activations: 128 rows x 128 B
constexpr int THREADS = 512;
constexpr int TMEM_COLS = 512;

// A TMA instruction costs the issuing thread a few hundred ns whatever its
// size, so the CTA-pair form moves 256-deep k-blocks (32 KB of activations in
// one 3-D box) and splits the activation and weight loads over two warps.
// MX: block-scaled FP4 on CTA pairs (packed e2m1 operands, 192-wide tiles);
// a 512-deep k-block keeps its activation box at 32 KB (two 128-byte
// swizzled chunks of 256 k), so one instruction per ring slot still suffices
// at the 4-bit MMA rate.
template <bool PAIR, bool MX = false>
struct Layout {
  static constexpr int BN_T = MX ? 192 : BN;        // output columns per tile
  static constexpr int BK = MX ? 512 : PAIR ? 256 : 128;  // k-block depth in elements
  static constexpr int KSUB = 2;                    // pair: 128-byte swizzled chunks per k-block
  // int8 pairs: a third unpacked-weight slot for one activation slot (q|k|v
  // 24.2 -> 23.5 us, gate|up 36.1 -> 35.0, down_proj 120.9 -> 117.8); the
  // same trade left mxf4 1-2 % slower, so it keeps 4 and 2
  static constexpr int S_TMA = MX ? 4 : PAIR ? 3 : 5;  // activation ring
  static constexpr int S_W = MX ? 2 : PAIR ? 2 : 4;    // packed-weight ring
  static constexpr int S_B = MX ? 2 : PAIR ? 3 : 3;    // unpacked-weight ring
  static constexpr int BROWS = PAIR ? BN_T / 2 : BN_T;  // weight rows staged per CTA
  static constexpr int ROW_BYTES = MX ? BK / 2 : BK;    // bytes of one k-block row in smem
  static constexpr int A_BYTES = BM * ROW_BYTES;
  static constexpr int WP_BYTES = BROWS * (BK / 4);
  static constexpr int B_BYTES = BROWS * ROW_BYTES;
  static constexpr int SF_COL = 2 * BN_T;           // MX: first tensor-memory column of the scales
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + S_TMA * A_BYTES;
  static constexpr int OFF_WP = OFF_B + S_B * B_BYTES;
  static constexpr int OFF_STG = OFF_WP + S_W * WP_BYTES;  // epilogue staging, 4 KB per warp
  static constexpr int OFF_BAR = OFF_STG + 4 * 4096;
  static constexpr int N_BARS = 2 * S_TMA + 2 * S_W + 2 * S_B + 2 * 2 + 2;
  static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + slack for 1024-byte alignment
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(!PAIR || A_BYTES == KSUB * SUB, "pair k-block = two 128-byte chunks");
  static_assert(B_BYTES % 1024 == 0 && (BROWS * 128) % 1024 == 0, "swizzle atoms aligned");
};

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

// The k-block a tile handles at step kb. With long K (16 k-blocks or more)
// tile t starts at k-block t mod num_kb, so the CTAs working on different
// tiles at the same moment read different activation and weight columns:
// down_proj (K = 11008, 43 k-blocks) 131 -> 121 us; at K = 2048 the order
// made no difference. The sums are exact in any order (int32, or fp32 sums
// of multiples of 0.5 below 2^24).
__device__ __forceinline__ int kb_rotation(int tile, int num_kb) { return num_kb >= 16 ? tile % num_kb : 0; }
__device__ __forceinline__ int kb_at(int kb, int rot, int num_kb) {
  const int k = kb + rot;
  return k >= num_kb ? k - num_kb : k;
}

// Every group's weight scale and the group ends, in registers.
struct EpiScales {
  float gam[8];
  int ge[7];  // past the last group: none
  __device__ __forceinline__ void load(const Params& p) {
#pragma unroll
    for (int g = 0; g < 8; ++g) gam[g] = (p.out_mode == kOutBf16 && g < p.G) ? __ldg(p.gamma + g) : 0.f;
#pragma unroll
    for (int g = 0; g < 7; ++g) ge[g] = g < p.G - 1 ? p.group_end[g] : 0x7FFFFFFF;
  }
};

// One 64-column chunk of a tile's accumulator (TMEM columns col .. col + 63,
// lane quadrant q) -> bf16 y[m0 + q * 32 .. + 31][n .. n + 63], staged in the
// 4 KB shared-memory block stg (or the raw accumulators straight to global).
template <bool FP4>
__device__ __forceinline__ void epi_chunk(const Params& p, const CUtensorMap* tmY, uint32_t tmem_base, int lane,
                                          const EpiScales& es, int m0, int n, uint32_t col, int q, uint32_t stg,
                                          float xs_m, bool row_ok, int m) {
  auto grp = [&](int cc) {
    int g = 0;
#pragma unroll
    for (int i = 0; i < 7; ++i) g += cc >= es.ge[i] ? 1 : 0;
    return g;
  };
  uint32_t r[64];
  tmem_ld64(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + col, r);
  tmem_ld_wait();
  if (p.out_mode == kOutBf16) {
    // y = acc * (xs[m] * gamma[group(n)]); one scale per 64-column chunk
    // unless the chunk straddles a group boundary
    const int g0 = grp(n);
    const int g1 = grp(min(n + 63, p.N - 1));
    float s0 = 0.f;
#pragma unroll
    for (int g = 0; g < 8; ++g) s0 = (g == g0) ? es.gam[g] : s0;
    s0 = __fmul_rn(xs_m, s0);  // y = acc * (xs[m] * gamma[group(n)])
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      // FP4: the fp32 accumulator. int8: exact int32 -> fp32 for
      // |acc| < 2^22 (|acc| <= 128 K) on the integer/FMA pipes:
      // (1.5 * 2^23 + acc) - 1.5 * 2^23
      const float f = FP4 ? __uint_as_float(r[i])
                          : __fsub_rn(__int_as_float(static_cast<int32_t>(r[i]) + 0x4B400000), 12582912.f);
      r[i] = __float_as_uint(f);
    }
    if (g0 == g1) {  // warp-uniform: the whole chunk in one scale group
#pragma unroll
      for (int i = 0; i < 64; ++i) r[i] = __float_as_uint(__fmul_rn(__uint_as_float(r[i]), s0));
    } else {
      // the chunk crosses group boundaries: one pass per group touched
      // (a dynamic loop, so the common path above is not predicated)
#pragma unroll 1
      for (int g = g0; g <= g1; ++g) {
        int lo = 0, hi = 0x7FFFFFFF;
#pragma unroll
        for (int j = 0; j < 7; ++j) {
          lo = (j == g - 1) ? es.ge[j] : lo;
          hi = (j == g) ? es.ge[j] : hi;
        }
        float t = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) t = (j == g) ? es.gam[j] : t;
        const float sg = __fmul_rn(xs_m, t);
#pragma unroll
        for (int i = 0; i < 64; ++i)
          r[i] = (n + i >= lo && n + i < hi) ? __float_as_uint(__fmul_rn(__uint_as_float(r[i]), sg))
                                             : r[i];
      }
    }
    // stage the warp's 32 x 64 bf16 block (128 B per row, 16-byte unit v
    // of row r at v ^ (r & 7): the 128-byte swizzle of the output tensor
    // map) and write it with one TMA store; rows past M and columns
    // past N are clipped by the map
    if (lane == 0) bulk_wait_read_all();  // the previous block has left the buffer
    __syncwarp();
#pragma unroll
    for (int v = 0; v < 8; ++v)
      st_shared_v4(stg + lane * 128 + ((v ^ (lane & 7)) << 4),
                   pack_bf16x2(__uint_as_float(r[8 * v + 0]), __uint_as_float(r[8 * v + 1])),
                   pack_bf16x2(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3])),
                   pack_bf16x2(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5])),
                   pack_bf16x2(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7])));
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(tmY, stg, n, m0 + q * 32);
      bulk_commit();
    }
  } else if (row_ok) {
    uint32_t* orow = reinterpret_cast<uint32_t*>(p.out) + static_cast<int64_t>(m) * p.ldo + n;
#pragma unroll
    for (int v = 0; v < 16; ++v) {
      if (n + 4 * v >= p.N) break;
      reinterpret_cast<uint4*>(orow)[v] =
          make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
    }
  }
}

template <bool FP4, bool PAIR, bool MX>
__global__ void __launch_bounds__(THREADS, 1)
bitlinear_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                      const __grid_constant__ CUtensorMap tmW,
                      const __grid_constant__ CUtensorMap tmY, const Params p) {
  static_assert(!MX || (FP4 && PAIR), "mxf4 is the FP4 CTA-pair form");
  using L = Layout<PAIR, MX>;
  constexpr int S_TMA = L::S_TMA, S_W = L::S_W, S_B = L::S_B, BK = L::BK, A_BYTES = L::A_BYTES;
  constexpr int BN = L::BN_T;
  // FP4 on pairs (a light unpack, so its per-k-block waits and arrivals
  // weigh): the 8 unpack warps form two groups of UW = 4 that take alternate
  // k-blocks, one group's waits overlapping the other's work. int8 (an
  // unpack 3x heavier, the shared-memory port already saturated) keeps all
  // 8 warps on every k-block, which measured faster.
  constexpr int UW = MX ? 4 : 8;
  constexpr uint32_t NUG = 8 / UW;  // unpack groups
  constexpr int UT = UW * 32;       // unpack threads per k-block
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* afull = bars;                   // activations landed (even CTA: both CTAs' bytes)
  uint64_t* empty = afull + S_TMA;          // MMA done with activation slot (both CTAs)
  uint64_t* wfull = empty + S_TMA;          // this CTA's packed weights landed
  uint64_t* wempty = wfull + S_W;           // unpack done reading packed-weight slot
  uint64_t* bfull = wempty + S_W;           // unpacked B ready (even CTA: both CTAs' warps)
  uint64_t* bempty = bfull + S_B;           // MMA done with B slot (both CTAs)
  uint64_t* tfull = bempty + S_B;           // accumulator ready (both CTAs)
  uint64_t* tempty = tfull + 2;             // accumulator drained (even CTA: both epilogues)
  uint64_t* mma_done = tempty + 2;          // all MMAs retired (teardown)
  uint64_t* last_acc = mma_done + 1;        // the epilogue warps have this CTA's last accumulator (used once)
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int cta_slot = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int cta_stride = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
  constexpr int TILE_M = PAIR ? 2 * BM : BM;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S_TMA; ++i) { mbar_init(&afull[i], 1); mbar_init(&empty[i], 1); }
    for (int i = 0; i < S_W; ++i) { mbar_init(&wfull[i], 1); mbar_init(&wempty[i], UW); }
    for (int i = 0; i < S_B; ++i) { mbar_init(&bfull[i], PAIR ? 2 * UW : UW); mbar_init(&bempty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&tfull[i], 1); mbar_init(&tempty[i], PAIR ? 8 : 4); }
    mbar_init(mma_done, 1);
    mbar_init(last_acc, 4);
    *s_abort = 0;
    fence_mbar_init();
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmW);
  }
  if (warp == 1) {
    if (PAIR) { tmem_alloc_pair(s_tmem, TMEM_COLS); tmem_relinquish_pair(); }
    else      { tmem_alloc(s_tmem, TMEM_COLS); tmem_relinquish(); }
  }
  __syncthreads();
  if (PAIR) cluster_sync();  // peer barriers initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  if constexpr (MX) {
    // every block scale 1.0: columns SF_COL..511 of all 128 lanes hold 0x7F
    // bytes (the scales of A at SF_COL, of B at SF_COL + 32), written by the
    // four epilogue warps (one lane quarter each) before the first MMA
    if (warp >= 4 && warp < 8) {
      uint32_t ones[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) ones[i] = 0x7F7F7F7Fu;
      const uint32_t lane_base = tmem_base + (static_cast<uint32_t>((warp & 3) * 32) << 16);
#pragma unroll
      for (int c = L::SF_COL; c < TMEM_COLS; c += 32) tmem_st32(lane_base + c, ones);
      tmem_st_wait();
      tc_fence_before();
    }
    __syncthreads();
    if (PAIR) cluster_sync();
    tc_fence_after();
  }
  // Only now (TMEM held) may the next kernel in the stream start its CTAs.
  pdl_trigger();

  const uint32_t sA = smem_u32(smem + L::OFF_A);
  const uint32_t sB = smem_u32(smem + L::OFF_B);
  const uint32_t sW = smem_u32(smem + L::OFF_WP);
  const uint64_t tmo = p.timeout_ns;
  // barrier addresses in the even CTA of the pair (or this CTA)
  auto lead = [&](uint64_t* bar) -> uint32_t {
    return PAIR ? map_shared_rank(smem_u32(bar), 0) : smem_u32(bar);
  };
  auto fail = [&]() {
    *s_abort = 1;
    report_status(p.status, BITLINEAR_STATUS_TIMEOUT);
  };
  // the last tile's epilogue chunks are spread over the warp sets: chunk c
  // by the epilogue warps (c = 0), the unpack warps 8-11 (1) and 12-15 (2),
  // the producer / issuer warps 0-3 (3), each set on all four lane quadrants
  constexpr int NCH = BN / 64;
  // global bytes per activation box (the padded f8f6f4 form reads half of what it stages)
  constexpr uint32_t A_TX = (FP4 && !MX) ? L::A_BYTES / 2 : L::A_BYTES;

  if (warp == 0 || warp == 2) {
    // ----------------------------------------- TMA producers (A: warp 0, W: warp 2)
    if (lane == 0) {
      const bool act = warp == 0;
      // activation codes come from the previous kernel; packed weights do not
      if (act) pdl_wait();
      uint32_t it = 0;
      bool ok = true;
      for (int tile = cta_slot; ok && tile < p.num_tiles; tile += cta_stride) {
        const int m0 = (tile % p.tiles_m) * TILE_M + static_cast<int>(rank) * BM;
        const int n0 = (tile / p.tiles_m) * BN + static_cast<int>(rank) * L::BROWS;
        const int rot = kb_rotation(tile, p.num_kb);
        for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
          const int kg = kb_at(kb, rot, p.num_kb);
          const int S = act ? S_TMA : S_W;
          const uint32_t s = it % S, ph = (it / S) & 1;
          if (!mbar_wait(act ? &empty[s] : &wempty[s], ph ^ 1, tmo, s_abort)) { fail(); ok = false; break; }
          if (act) {
            uint8_t* dst = smem + L::OFF_A + s * A_BYTES;
            if (PAIR) {  // two 128-byte swizzled chunks (int8: 128 k each, e2m1: 256 k)
              if (leader) mbar_arrive_expect_tx(&afull[s], 2 * A_TX);
              tma_load_3d_pair(dst, &tmA, lead(&afull[s]), 0, m0, kg * L::KSUB);
            } else {
              mbar_arrive_expect_tx(&afull[s], A_TX);
              tma_load_2d(dst, &tmA, &afull[s], kg * BK, m0);
            }
          } else {
            mbar_arrive_expect_tx(&wfull[s], L::WP_BYTES);
            tma_load_2d(smem + L::OFF_WP + s * L::WP_BYTES, &tmW, &wfull[s], kg * (BK / 4), n0);
          }
        }
      }
      // Do not leave while copies into this CTA's shared memory are in
      // flight: the weight tiles signal wfull here; the even CTA also waits
      // for the activation tiles of both CTAs (afull). The cluster barrier
      // at exit keeps the odd CTA alive until then.
      const uint32_t S = act ? S_TMA : S_W;
      const uint32_t inflight = it < S ? it : S;
      for (uint32_t d = 0; d < inflight; ++d) {
        const uint32_t j = it - 1 - d;
        if (!act) mbar_wait(&wfull[j % S], (j / S) & 1, tmo, nullptr);
        else if (leader) mbar_wait(&afull[j % S], (j / S) & 1, tmo, nullptr);
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------- MMA issuer
    if (lane == 0 && leader) {
      constexpr uint32_t idesc = MX    ? make_idesc_mxf4(TILE_M, BN)
                                 : FP4 ? make_idesc(1, 5, 5, TILE_M, BN)
                                       : make_idesc(2, 1, 1, TILE_M, BN);
      const uint32_t sfa = tmem_base + L::SF_COL, sfb = tmem_base + L::SF_COL + 32;
      uint32_t it = 0, tl = 0;
      bool ok = true;
      for (int tile = cta_slot; ok && tile < p.num_tiles; tile += cta_stride, ++tl) {
        const uint32_t acc = tl & 1, aph = (tl >> 1) & 1;
        if (!(PAIR ? mbar_wait_cluster(&tempty[acc], aph ^ 1, tmo, s_abort)
                   : mbar_wait(&tempty[acc], aph ^ 1, tmo, s_abort))) { fail(); break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        const int rot = kb_rotation(tile, p.num_kb);
        for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
          const int kg = kb_at(kb, rot, p.num_kb);
          const uint32_t s = it % S_TMA, ph = (it / S_TMA) & 1;
          const uint32_t b = it % S_B, bph = (it / S_B) & 1;
          const bool got = mbar_wait(&afull[s], ph, tmo, s_abort) &&
                           (PAIR ? mbar_wait_cluster(&bfull[b], bph, tmo, s_abort)
                                 : mbar_wait(&bfull[b], bph, tmo, s_abort));
          if (!got) { fail(); ok = false; break; }
          tc_fence_after();
          if constexpr (MX) {
            // 8 MMAs of K = 64 (32 bytes of packed e2m1), 4 along each 128-byte
            // chunk; a chunk wholly past K (the second one of the last
            // k-block when K % 512 = 256) is skipped
#pragma unroll
            for (int kk = 0; kk < BK / 64; ++kk) {
              const int sub = kk >> 2, k4 = kk & 3;
              if (sub > 0 && kg * BK + sub * 256 >= p.K) break;
              const uint64_t adesc = smem_desc_sw128(sA + s * A_BYTES + sub * SUB);
              const uint64_t bdesc = smem_desc_sw128(sB + b * L::B_BYTES + sub * L::BROWS * 128);
              mma_mxf4_pair(d_tmem, adesc + 2 * k4, bdesc + 2 * k4, idesc, sfa, sfb, (kb | kk) != 0);
            }
          } else
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk) {
            // chunk kk / 4 of the k-block; advance 32 bytes (2 x 16 B) along K
            // inside its swizzled 128-byte rows
            const int sub = kk >> 2, k4 = kk & 3;
            const uint64_t adesc = smem_desc_sw128(sA + s * A_BYTES + sub * SUB);
            const uint64_t bdesc = smem_desc_sw128(sB + b * L::B_BYTES + sub * L::BROWS * 128);
            const uint32_t accum = (kb | kk) != 0;
            if (PAIR) {
              if (FP4) mma_f8f6f4_pair(d_tmem, adesc + 2 * k4, bdesc + 2 * k4, idesc, accum);
              else     mma_i8_pair(d_tmem, adesc + 2 * k4, bdesc + 2 * k4, idesc, accum);
            } else {
              if (FP4) mma_f8f6f4(d_tmem, adesc + 2 * k4, bdesc + 2 * k4, idesc, accum);
              else     mma_i8(d_tmem, adesc + 2 * k4, bdesc + 2 * k4, idesc, accum);
            }
          }
          if (PAIR) { tc_commit_pair_mc(&empty[s], 3); tc_commit_pair_mc(&bempty[b], 3); }
          else      { tc_commit(&empty[s]); tc_commit(&bempty[b]); }
        }
        if (ok) {
          if (PAIR) tc_commit_pair_mc(&tfull[acc], 3);
          else      tc_commit(&tfull[acc]);
        }
      }
      if (PAIR) tc_commit_pair_mc(mma_done, 1);
      else      tc_commit(mma_done);
      mbar_wait(mma_done, 0, tmo, nullptr);
    }
  } else if (warp >= 4 && warp < 8) {
    // ----------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lane quadrant
    const uint32_t tempty_addr0 = lead(&tempty[0]);
    const uint32_t stg = smem_u32(smem + L::OFF_STG) + q * 4096;  // this warp's staging block
    EpiScales es;
    es.load(p);
    pdl_wait();  // row scales come from the previous kernel; y may still be read by it
    uint32_t tl = 0;
    for (int tile = cta_slot; tile < p.num_tiles; tile += cta_stride, ++tl) {
      const int m0 = (tile % p.tiles_m) * TILE_M + static_cast<int>(rank) * BM;
      const int n0 = (tile / p.tiles_m) * BN;
      const uint32_t acc = tl & 1, aph = (tl >> 1) & 1;
      const int m = m0 + q * 32 + lane;
      const bool row_ok = m < p.M;
      // the row scale is fetched before waiting, so its latency hides behind the mainloop
      const float xs_m = (row_ok && p.out_mode == kOutBf16) ? __ldg(p.xs + m) : 0.f;
      if (!mbar_wait(&tfull[acc], aph, tmo, s_abort)) { fail(); break; }
      tc_fence_after();
      // the last tile's chunks are shared with the other warps (below): this
      // warp set writes chunk 0 of it, and tells them the accumulator is ready
      // (a barrier of its own: a wait on tfull by parity alone cannot tell the
      // last tile's phase from an earlier one)
      const bool last = tile + cta_stride >= p.num_tiles;
      if (last && lane == 0) mbar_arrive(last_acc);
#pragma unroll 1
      for (int c = 0; c < (last ? 1 : NCH); ++c) {
        const int n = n0 + c * 64;
        if (n >= p.N) break;  // warp-uniform
        epi_chunk<FP4>(p, &tmY, tmem_base, lane, es, m0, n, acc * BN + c * 64, q, stg, xs_m, row_ok, m);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {  // one arrival per epilogue warp, on the even CTA
        if (PAIR) mbar_arrive_cluster(tempty_addr0 + 8u * acc);
        else      mbar_arrive(&tempty[acc]);
      }
    }
    if (lane == 0) bulk_wait_all();  // output stores complete before the CTA exits
  } else if (warp >= 8) {
    // ------------------------------------------------------------- unpack
    const uint32_t ugrp = static_cast<uint32_t>(warp - 8) / UW;  // takes k-blocks it % NUG == ugrp
    const int ut = threadIdx.x - 256 - static_cast<int>(ugrp) * UT;  // 0..UT-1
    const uint32_t bfull_addr0 = lead(&bfull[0]);
    uint32_t it = 0;
    bool ok = true;
    for (int tile = cta_slot; ok && tile < p.num_tiles; tile += cta_stride) {
      for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
        if (it % NUG != ugrp) continue;
        const uint32_t s = it % S_W, ph = (it / S_W) & 1;
        const uint32_t b = it % S_B, bph = (it / S_B) & 1;
        if (!mbar_wait(&wfull[s], ph, tmo, s_abort) || !mbar_wait(&bempty[b], bph ^ 1, tmo, s_abort)) {
          fail(); ok = false; break;
        }
        const uint32_t src = sW + s * L::WP_BYTES;
        const uint32_t dst = sB + b * L::B_BYTES;
        constexpr int WPR = BK / 16;  // packed words per weight row
        if constexpr (MX) {
          // all of a thread's packed words are loaded before its first store
          // (the ordered shared-memory accesses would otherwise serialise
          // the iterations)
          // two packed words (32 k) -> one 16-byte group of 32 e2m1 nibbles
          // (even k low): group j of a row goes to 16-byte column j % 8 of
          // its 128-byte swizzled line in chunk j / 8
          constexpr int GPR = BK / 32;  // groups per weight row
          constexpr int NI = (L::BROWS * GPR) / UT;
          static_assert((L::BROWS * GPR) % UT == 0, "whole groups per thread");
          uint2 wv[NI];
#pragma unroll
          for (int i = 0; i < NI; ++i) {
            const int g = ut + UT * i;
            wv[i] = ld_shared_v2(src + (g / GPR) * (BK / 4) + 8 * (g % GPR));
          }
#pragma unroll
          for (int i = 0; i < NI; ++i) {
            const int g = ut + UT * i;
            const int n = g / GPR, j = g % GPR;
            const int sub = j >> 3, c = j & 7;
            uint4 o;
            e2m1_words(wv[i].x, o.x, o.y);
            e2m1_words(wv[i].y, o.z, o.w);
            st_shared_v4(dst + sub * (L::BROWS * 128) + (n >> 3) * 1024 + (n & 7) * 128 + ((c ^ (n & 7)) << 4),
                         o.x, o.y, o.z, o.w);
          }
        } else {
          // one word at a time: with the shared-memory port saturated by the
          // MMA and TMA traffic, batching the loads was not faster here
          static_assert((L::BROWS * WPR) % UT == 0, "whole words per thread");
#pragma unroll
          for (int i = 0; i < (L::BROWS * WPR) / UT; ++i) {
            const int w = ut + UT * i;           // packed word index in the tile
            const int n = w / WPR, j = w % WPR;  // row, 16-deep K group
            const int sub = j >> 3, c = j & 7;   // 128-deep chunk, 16-byte column in it
            const uint32_t word = ld_shared_u32(src + 4 * w);
            const uint4 o = FP4 ? unpack16_e2m1(word) : unpack16_s8(word);
            const uint32_t addr = dst + sub * (L::BROWS * 128) + (n >> 3) * 1024 + (n & 7) * 128 +
                                  ((c ^ (n & 7)) << 4);
            st_shared_v4(addr, o.x, o.y, o.z, o.w);
          }
        }
        fence_proxy_async_smem();  // each thread's smem writes -> async proxy
        __syncwarp();
        if (lane == 0) {  // one arrival per unpack warp, on the even CTA
          mbar_arrive(&wempty[s]);  // packed slot read: the weight producer may refill it
          if (PAIR) mbar_arrive_cluster(bfull_addr0 + 8u * b);
          else      mbar_arrive(&bfull[b]);
        }
      }
    }
  }

  // ---- the last tile's other chunks: warp set k (1: warps 8-11, 2: 12-15,
  // 3: 0-3) writes chunk k of this CTA's last tile once its accumulator is
  // ready, staging in the unpacked-weight ring (no MMA reads it any more)
  {
    __syncwarp();
    const int set = warp >= 8 ? 1 + ((warp - 8) >> 2) : (warp < 4 ? 3 : 0);
    const int count = cta_slot < p.num_tiles ? (p.num_tiles - 1 - cta_slot) / cta_stride + 1 : 0;
    if (set > 0 && set < NCH && count > 0 && !*s_abort) {
      const int q = warp & 3;
      const uint32_t tl = static_cast<uint32_t>(count - 1);
      const int tile = cta_slot + static_cast<int>(tl) * cta_stride;
      const int m0 = (tile % p.tiles_m) * TILE_M + static_cast<int>(rank) * BM;
      const int n = (tile / p.tiles_m) * BN + set * 64;
      const uint32_t acc = tl & 1;
      const int m = m0 + q * 32 + lane;
      const bool row_ok = m < p.M;
      EpiScales es;
      es.load(p);
      pdl_wait();  // as for the epilogue warps
      const float xs_m = (row_ok && p.out_mode == kOutBf16) ? __ldg(p.xs + m) : 0.f;
      if (!mbar_wait(last_acc, 0, tmo, s_abort)) {
        fail();
      } else if (n < p.N) {
        tc_fence_after();
        epi_chunk<FP4>(p, &tmY, tmem_base, lane, es, m0, n, acc * BN + set * 64, q, sB + ((set - 1) * 4 + q) * 4096,
                       xs_m, row_ok, m);
        if (lane == 0) bulk_wait_all();  // its output stores complete before the CTA exits
      }
    }
  }

  __syncthreads();
  if (PAIR) cluster_sync();  // the pair's MMAs and remote arrivals are finished
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if (PAIR) tmem_dealloc_pair(tmem_base, TMEM_COLS);
    else      tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace gemm

static cudaError_t make_map_3d(CUtensorMap* map, CUtensorMapDataType dt, const void* base,
                               const cuuint64_t (&dims)[3], const cuuint64_t (&strides)[2],
                               const cuuint32_t (&box)[3], const char** why) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) { *why = "cuTensorMapEncodeTiled unavailable"; return cudaErrorNotSupported; }
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) { *why = "cuTensorMapEncodeTiled rejected the activation layout"; return cudaErrorInvalidValue; }
  return cudaSuccess;
}

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

template <bool FP4, bool PAIR, bool MX = false>
static cudaError_t launch_t(const CUtensorMap& tmA, const CUtensorMap& tmW, const CUtensorMap& tmY,
                            const gemm::Params& p, cudaStream_t s) {
  using namespace gemm;
  using L = Layout<PAIR, MX>;
  auto kern = bitlinear_gemm_kernel<FP4, PAIR, MX>;
  cudaError_t e = set_smem_limit(kern, L::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int sms = num_sms();
  if (PAIR) {
    const int pairs = p.num_tiles < sms / 2 ? p.num_tiles : sms / 2;
    return launch_kernel(kern, dim3(static_cast<unsigned>(2 * pairs)), dim3(THREADS),
                         L::SMEM_BYTES, s, 2u, tmA, tmW, tmY, p);
  }
  return launch_kernel(kern, dim3(static_cast<unsigned>(p.num_tiles < sms ? p.num_tiles : sms)),
                       dim3(THREADS), L::SMEM_BYTES, s, 0u, tmA, tmW, tmY, p);
}

cudaError_t launch_gemm(const GemmArgs& a, bool fp4, cudaStream_t s, const char** why) {
  using namespace gemm;
  // CTA pairs once there are two 128-row halves to fill; their 3-D activation
  // view needs whole 128-deep K chunks
  const bool pair = a.M > BM && a.K % 128 == 0;
  // block-scaled FP4 on packed operands; its activation view needs whole
  // 256-deep chunks (other FP4 pairs take kind::f8f6f4 on padded codes)
  const bool mx = pair && fp4 && a.K % 256 == 0;
  const int bn = mx ? Layout<true, true>::BN_T : BN;
  const int brows = pair ? bn / 2 : bn;
  const int BK = mx ? Layout<true, true>::BK : pair ? Layout<true>::BK : Layout<false>::BK;
  CUtensorMap tmA, tmW, tmY;
  cudaError_t e;
  const CUtensorMapDataType adt = fp4 ? CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const uint64_t row_bytes = fp4 ? a.K / 2 : a.K;
  if (mx) {
    // packed e2m1 codes as bytes [K/256 chunks][M rows][128 bytes]: one box
    // = 2 chunks x 128 rows (512 k), two 128-byte-swizzled tiles back to
    // back; a chunk past K reads zeros
    const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(a.M), static_cast<cuuint64_t>(a.K / 256)};
    const cuuint64_t strides[2] = {row_bytes, 128u};
    const cuuint32_t box[3] = {128, BM, static_cast<cuuint32_t>(Layout<true, true>::KSUB)};
    e = make_map_3d(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.xq, dims, strides, box, why);
  } else if (pair) {
    // [K/128 chunks][M rows][128 elements]: one box = 2 chunks x 128 rows,
    // i.e. two standard 128-byte-swizzled 128 x 128 tiles back to back
    const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(a.M), static_cast<cuuint64_t>(a.K / 128)};
    const cuuint64_t strides[2] = {row_bytes, fp4 ? 64u : 128u};
    const cuuint32_t box[3] = {128, BM, static_cast<cuuint32_t>(Layout<true>::KSUB)};
    e = make_map_3d(&tmA, adt, a.xq, dims, strides, box, why);
  } else {
    e = make_map_2d(&tmA, adt, a.xq, a.K, a.M, row_bytes, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B, why);
  }
  if (e != cudaSuccess) return e;
  e = make_map_2d(&tmW, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.Wp, a.K / 4, a.N, a.K / 4, BK / 4, brows,
                  CU_TENSOR_MAP_SWIZZLE_NONE, why);
  if (e != cudaSuccess) return e;
  if (a.out_mode == kOutBf16) {
    // bf16 Y [M x ldo], written by 32 x 64 TMA stores from 128-byte-swizzled staging
    e = make_map_2d(&tmY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.out, a.N, a.M, a.ldo * 2, 64, 32,
                    CU_TENSOR_MAP_SWIZZLE_128B, why);
    if (e != cudaSuccess) return e;
  } else {
    tmY = tmA;  // not used by the raw-accumulator epilogue
  }

  Params p{};
  p.M = static_cast<int>(a.M);
  p.N = static_cast<int>(a.N);
  p.K = static_cast<int>(a.K);
  p.num_kb = static_cast<int>((a.K + BK - 1) / BK);
  const int tile_m = pair ? 2 * BM : BM;
  p.tiles_m = static_cast<int>((a.M + tile_m - 1) / tile_m);
  const int tiles_n = static_cast<int>((a.N + bn - 1) / bn);
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

  if (mx) return launch_t<true, true, true>(tmA, tmW, tmY, p, s);
  if (fp4) return pair ? launch_t<true, true>(tmA, tmW, tmY, p, s) : launch_t<true, false>(tmA, tmW, tmY, p, s);
  return pair ? launch_t<false, true>(tmA, tmW, tmY, p, s) : launch_t<false, false>(tmA, tmW, tmY, p, s);
}

}  // namespace blt
