// Decode-time BitLinear for 1..8 tokens on the warp-level tensor-core path
// (mma.sync m16n8k32, unsigned 8-bit weight codes x signed 8-bit activations,
// int32 accumulate).
//
// Why this path. With a handful of tokens the layer is a matrix-vector
// product whose cost is reading the 2-bit weights from HBM. A tcgen05 MMA of
// M = 128 weight rows takes ~45 SM clocks whatever its N <= 64 (measured), so
// it consumes at most ~92 weights per clock and SM, barely the HBM stream
// (~89 per clock and SM at the measured copy bandwidth), and needs the
// weights unpacked into tensor or shared memory first. The warp-level MMA
// has no such floor: one m16n8k32 covers 16 rows x 32 k for 8 tokens, and at
// the measured ~0.48 per clock and SM it consumes ~245 weights per clock at
// 8 tokens. Its operands come straight from registers, so the 2-bit codes
// need no unpack round trip: four AND masks and one shift per packed word.
//
// Arithmetic. A packed word j of a weight row holds codes c = W_t + 1 in
// {0, 1, 2}; element 16j + 8h + i sits in bits [4i + 2h, 4i + 2h + 2). With
// t = w >> 2 the masks
//     w & 0x03030303 -> c of elements {0, 2, 4, 6}          (scale 1)
//     t & 0x03030303 -> c of elements {8, 10, 12, 14}       (scale 1)
//     w & 0x30303030 -> c of elements {1, 3, 5, 7}          (scale 16)
//     t & 0x30303030 -> c of elements {9, 11, 13, 15}       (scale 16)
// leave one code per byte; the activation bytes are regrouped into the same
// element order once per 16-byte group, so each masked register is directly
// an MMA operand. The scale-1 and scale-16 products go to separate
// accumulators, sum_k c x = acc1 + acc16 / 16 (exact: acc16 is a multiple of
// 16), and
//     acc = sum_k W_t x = sum_k c x - sum_k x
// is exact in int32. The usual epilogue follows:
//     y = bf16_rne((float)acc * (xs[m] * gamma[g(n)])).
//
// Inside one MMA the k order is free as long as A and B agree: for lane
// (g = lane / 4, c = lane % 4) the fragment registers a0 / a2 (rows g) and
// b0 / b1 (token g) hold the same four physical elements each: elements
// {0,2,4,6} and {8,10,12,14} (or {1,3,5,7} and {9,11,13,15}) of the lane's
// word. Lane c of a warp takes words 2c and 2c+1 of a 128-deep k span.
//
// Data flow. Each CTA owns a contiguous range of R output rows (a multiple of
// 8, equal up to 8 rows over the grid, so the weight bytes per SM are
// balanced), processed in blocks of 16 rows. A block arrives as one bulk
// copy per row (the row's K/4 contiguous bytes, every lane of a warp issuing
// one), into a shared-memory slot with a row pitch of K/4 + 16 bytes: the
// padding spreads the rows of an MMA fragment over all 32 banks. The slots
// form a ring; the first ones are requested before the kernel waits for the
// previous one in the stream (the weights do not depend on it), and the CTA
// needs under half an SM, so the next kernel's CTAs sit beside it and stream
// their weights while this one computes. The activation rows are staged the
// same way after the wait. All eight consumer warps work on every block,
// each on its own 128-deep spans of K (four independent accumulators per
// span keep the MMAs overlapped), and add their partial sums into a small
// shared-memory array with atomics; the epilogue reads it once.
//   warps 0-7  consumers (masks, MMAs)
//   warp  8    copies: activation rows, row and group scales, ring refills
// Rows of a 16-row block past R are never copied; their results are
// discarded.
#include <algorithm>

#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace blt {
namespace gemv_mma {

constexpr int WARPS = 8;                   // consumer warps
constexpr int THREADS = (WARPS + 1) * 32;  // + the copy warp
constexpr int SMEM_CTA = 110 * 1024;       // two CTAs fit on one SM
constexpr int MAX_ROWS = 160;              // rows per CTA (10 blocks)

struct Params {
  int M, N, K;
  int nspan;       // 128-deep spans of K
  int NB;          // 16-row blocks of the largest CTA
  int S;           // ring slots (blocks)
  int n8;          // N / 8
  int pitch;       // weight row pitch in shared memory: K / 4 + 16
  int x_pitch;     // activation row pitch: K + 16
  int x_off;       // offsets of the shared-memory regions
  int part_off;
  int bar_off;
  const int8_t* xq;
  const uint8_t* Wp;
  const float* xs;
  const float* gamma;
  int G;
  int group_end[8];
  uint16_t* y;
  int64_t ldy;
  int* status;
  uint64_t timeout_ns;
};

// D (16 x 8, s32) += A (16 x 32, u8) * B (32 x 8, s8)
__device__ __forceinline__ void mma_u8s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 16 activation bytes x0..x15 -> {x0,x2,x4,x6}, {x8,..,x14}, {x1,..,x7}, {x9,..,x15}
__device__ __forceinline__ uint4 regroup16(uint4 v) {
  uint4 r;
  r.x = __byte_perm(v.x, v.y, 0x6420);
  r.y = __byte_perm(v.z, v.w, 0x6420);
  r.z = __byte_perm(v.x, v.y, 0x7531);
  r.w = __byte_perm(v.z, v.w, 0x7531);
  return r;
}

__device__ __forceinline__ void bulk_load_1d(uint32_t dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(dst), "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ int byte_sum(uint4 v) {
  int s = __dp4a(static_cast<int>(v.x), 0x01010101, 0);
  s = __dp4a(static_cast<int>(v.y), 0x01010101, s);
  s = __dp4a(static_cast<int>(v.z), 0x01010101, s);
  return __dp4a(static_cast<int>(v.w), 0x01010101, s);
}

// MMA row g of a 16-row block <-> block row sigma(g) (and 8 + sigma(g)): a
// 16-lane phase of 8-byte shared loads then touches rows {0,2,4,6} (or
// {1,3,5,7}), which the padded pitch places on disjoint banks.
__device__ __forceinline__ int sigma(int g) { return ((g & 3) << 1) | (g >> 2); }

__global__ void __launch_bounds__(THREADS, 2) bitlinear_gemv_mma_kernel(const Params p) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int SLOT = 16 * p.pitch;
  uint8_t* xsm = smem + p.x_off;                                    // [M][x_pitch] activation codes
  int32_t* part = reinterpret_cast<int32_t*>(smem + p.part_off);    // [NB][16][8] sums over warps
  float* xs_s = reinterpret_cast<float*>(part + p.NB * 128);        // [8] row scales
  float* gam_s = xs_s + 8;                                          // [8] group scales
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.bar_off);
  uint64_t* empty = full + p.S;
  uint64_t* xbar = empty + p.S;
  volatile int* s_abort = reinterpret_cast<volatile int*>(xbar + 1);

  const int oct_lo = static_cast<int>((static_cast<int64_t>(blockIdx.x) * p.n8) / gridDim.x);
  const int oct_hi = static_cast<int>((static_cast<int64_t>(blockIdx.x + 1) * p.n8) / gridDim.x);
  const int r0 = 8 * oct_lo;
  const int R = 8 * (oct_hi - oct_lo);
  const int nblocks = (R + 15) >> 4;
  const uint32_t row_bytes = static_cast<uint32_t>(p.K >> 2);

  if (threadIdx.x == 0) {
    for (int i = 0; i < p.S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], WARPS);
    }
    mbar_init(xbar, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < p.NB * 128; i += THREADS) part[i] = 0;
  __syncthreads();
  pdl_trigger();  // the next kernel in the stream may place its CTAs beside this one
  const uint64_t tmo = p.timeout_ns;
  auto fail = [&]() {
    *s_abort = 1;
    report_status(p.status, BITLINEAR_STATUS_TIMEOUT);
  };
  // block b into slot b % S: lane i < rows of the block copies row i (the
  // whole warp calls this; lane 0 announces the bytes first)
  auto issue_block = [&](int b) {
    const int rows = min(16, R - 16 * b);
    uint64_t* bar = &full[b % p.S];
    if (lane == 0) mbar_arrive_expect_tx(bar, static_cast<uint32_t>(rows) * row_bytes);
    __syncwarp();
    if (lane < rows)
      bulk_load_1d(smem_u32(smem + (b % p.S) * SLOT + lane * p.pitch),
                   p.Wp + static_cast<int64_t>(r0 + 16 * b + lane) * row_bytes, row_bytes, bar);
  };

  // the first blocks of the ring, one warp each, before the dependency wait
  for (int b = warp; b < nblocks && b < p.S; b += WARPS + 1) issue_block(b);

  if (warp == WARPS) {
    // ------------------------------------------------------------ copies
    pdl_wait();  // activation codes and row scales come from the previous kernel
    if (lane == 0) mbar_arrive_expect_tx(xbar, static_cast<uint32_t>(p.M * p.K));
    __syncwarp();
    if (lane < p.M) {
      bulk_load_1d(smem_u32(xsm + lane * p.x_pitch), p.xq + static_cast<int64_t>(lane) * p.K,
                   static_cast<uint32_t>(p.K), xbar);
      xs_s[lane] = __ldg(p.xs + lane);
    }
    if (lane < p.G) gam_s[lane] = __ldg(p.gamma + lane);
    int b = p.S;
    for (; b < nblocks; ++b) {
      // the slot's previous block has been consumed by all eight warps
      const bool got = mbar_wait(&empty[b % p.S], ((b / p.S) - 1) & 1, tmo, s_abort);
      if (!__all_sync(0xFFFFFFFFu, got)) {
        if (lane == 0) fail();
        break;
      }
      issue_block(b);
    }
    // do not leave while copies into this CTA's shared memory are in flight
    if (lane == 0) {
      for (int d = 0, j = min(b, nblocks) - 1; d < p.S && j >= 0; ++d, --j)
        mbar_wait(&full[j % p.S], (j / p.S) & 1, tmo, nullptr);
      mbar_wait(xbar, 0, tmo, nullptr);
    }
  } else {
    // ---------------------------------------------------------- consumers
    const int g = lane >> 2, c = lane & 3;
    const int ra = sigma(g), rb = ra + 8;  // block rows of MMA rows g, g + 8
    const bool tok = g < p.M;
    const uint32_t xrow = smem_u32(xsm) + g * p.x_pitch + 32 * c;    // + 128 sp: token g's span bytes
    const int qa = ra * p.pitch + 8 * c, qb = rb * p.pitch + 8 * c;  // + 32 sp: the lane's words
    bool ok = mbar_wait(xbar, 0, tmo, s_abort);
    if (!ok) fail();
    int xsum = 0;  // sum of token g's codes over this warp's spans
    for (int b = 0; ok && b < nblocks; ++b) {
      const int slot = b % p.S;
      if (!mbar_wait(&full[slot], (b / p.S) & 1, tmo, s_abort)) {
        fail();
        break;
      }
      const uint32_t tile = smem_u32(smem + slot * SLOT);
      int a1[4] = {0, 0, 0, 0}, a16[4] = {0, 0, 0, 0}, b1[4] = {0, 0, 0, 0}, b16[4] = {0, 0, 0, 0};
#pragma unroll 2
      for (int sp = warp; sp < p.nspan; sp += WARPS) {
        uint4 xv0 = make_uint4(0u, 0u, 0u, 0u), xv1 = xv0;
        if (tok) {
          xv0 = ld_shared_v4(xrow + 128 * sp);
          xv1 = ld_shared_v4(xrow + 128 * sp + 16);
        }
        if (b == 0) xsum += byte_sum(xv0) + byte_sum(xv1);
        const uint4 x0 = regroup16(xv0), x1 = regroup16(xv1);
        const uint2 wa = ld_shared_v2(tile + qa + 32 * sp);
        const uint2 wb = ld_shared_v2(tile + qb + 32 * sp);
        const uint32_t ta0 = wa.x >> 2, tb0 = wb.x >> 2, ta1 = wa.y >> 2, tb1 = wb.y >> 2;
        // word 2c of the span (wa.x / wb.x) and word 2c + 1, scales 1 and 16
        mma_u8s8(a1, wa.x & 0x03030303u, wb.x & 0x03030303u, ta0 & 0x03030303u, tb0 & 0x03030303u, x0.x, x0.y);
        mma_u8s8(a16, wa.x & 0x30303030u, wb.x & 0x30303030u, ta0 & 0x30303030u, tb0 & 0x30303030u, x0.z, x0.w);
        mma_u8s8(b1, wa.y & 0x03030303u, wb.y & 0x03030303u, ta1 & 0x03030303u, tb1 & 0x03030303u, x1.x, x1.y);
        mma_u8s8(b16, wa.y & 0x30303030u, wb.y & 0x30303030u, ta1 & 0x30303030u, tb1 & 0x30303030u, x1.z, x1.w);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);  // this warp is done with the slot
      if (b == 0) {
        // token sums over this warp's spans: lanes of group g hold token g's
        xsum += __shfl_xor_sync(0xFFFFFFFFu, xsum, 1);
        xsum += __shfl_xor_sync(0xFFFFFFFFu, xsum, 2);
      }
      // D columns 2c, 2c + 1 are tokens 2c, 2c + 1: their sums sit in lanes 8c and 8c + 4
      const int s0 = __shfl_sync(0xFFFFFFFFu, xsum, 8 * c);
      const int s1 = __shfl_sync(0xFFFFFFFFu, xsum, 8 * c + 4);
      int32_t* pb = part + b * 128;
      atomicAdd(&pb[ra * 8 + 2 * c], a1[0] + b1[0] + ((a16[0] + b16[0]) >> 4) - s0);
      atomicAdd(&pb[ra * 8 + 2 * c + 1], a1[1] + b1[1] + ((a16[1] + b16[1]) >> 4) - s1);
      atomicAdd(&pb[rb * 8 + 2 * c], a1[2] + b1[2] + ((a16[2] + b16[2]) >> 4) - s0);
      atomicAdd(&pb[rb * 8 + 2 * c + 1], a1[3] + b1[3] + ((a16[3] + b16[3]) >> 4) - s1);
    }
  }
  pdl_wait();       // the previous kernel may still read y
  __syncthreads();  // every block consumed and summed, the copies landed
  if (*s_abort) return;
  // ----------------------------------------------------------- epilogue
  // output (token m, row r0 + n), n = 16 b + row of the block
  const int total = R * p.M;
  for (int idx = threadIdx.x; idx < total; idx += THREADS) {
    const int m = idx / R, n = idx - m * R;
    const int nn = r0 + n;
    int gi = 0;
#pragma unroll
    for (int i = 0; i < 7; ++i) gi += (i < p.G - 1 && nn >= p.group_end[i]) ? 1 : 0;
    const float sc = __fmul_rn(xs_s[m], gam_s[gi]);
    p.y[static_cast<int64_t>(m) * p.ldy + nn] =
        __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(static_cast<float>(part[n * 8 + m]), sc)));
  }
}

}  // namespace gemv_mma

// Shared memory of one CTA: S weight slots of 16 rows, the M activation rows,
// the block sums, the scales and the barriers.
struct GemvMmaLayout {
  int x_off, part_off, bar_off, total;
};
static GemvMmaLayout gemv_mma_layout(int S, int NB, int M, int K) {
  GemvMmaLayout L;
  const int pitch = K / 4 + 16;
  L.x_off = S * 16 * pitch;
  L.part_off = L.x_off + M * (K + 16);
  L.bar_off = L.part_off + NB * 128 * 4 + 16 * 4;
  L.total = L.bar_off + 8 * (2 * S + 1) + 16;
  return L;
}

bool gemv_mma_supported(int64_t M, int64_t N, int64_t K) {
  if (M < 1 || M > kGemvMmaMaxTokens || N % 128 != 0 || K % 128 != 0) return false;
  // two weight slots beside the staged activation rows
  return gemv_mma_layout(2, gemv_mma::MAX_ROWS / 16, static_cast<int>(M), static_cast<int>(K)).total <=
         227 * 1024;
}

cudaError_t launch_gemv_mma(const GemmArgs& a, cudaStream_t s, const char** why) {
  using namespace gemv_mma;
  Params p{};
  p.M = static_cast<int>(a.M);
  p.N = static_cast<int>(a.N);
  p.K = static_cast<int>(a.K);
  p.nspan = p.K / 128;
  p.n8 = p.N / 8;
  // one CTA per SM (two fit on one), at most MAX_ROWS rows each
  int grid = std::min(num_sms(), p.n8);
  grid = std::max(grid, (p.n8 + MAX_ROWS / 8 - 1) / (MAX_ROWS / 8));
  const int r_hi = 8 * ((p.n8 + grid - 1) / grid);
  p.NB = (r_hi + 15) / 16;
  p.pitch = p.K / 4 + 16;
  p.x_pitch = p.K + 16;
  // as many slots as leave room for a second CTA on the SM (the next
  // kernel's), at least two
  p.S = std::min(p.NB, 2);
  while (p.S < p.NB && gemv_mma_layout(p.S + 1, p.NB, p.M, p.K).total <= SMEM_CTA) ++p.S;
  const GemvMmaLayout L = gemv_mma_layout(p.S, p.NB, p.M, p.K);
  if (L.total > 227 * 1024) {
    *why = "activation rows too long for shared memory";
    return cudaErrorInvalidValue;
  }
  p.x_off = L.x_off;
  p.part_off = L.part_off;
  p.bar_off = L.bar_off;
  p.xq = static_cast<const int8_t*>(a.xq);
  p.Wp = a.Wp;
  p.xs = a.xs;
  p.gamma = a.gamma;
  p.G = a.G;
  for (int i = 0; i < 8; ++i) p.group_end[i] = a.group_end[i];
  p.y = static_cast<uint16_t*>(a.out);
  p.ldy = a.ldo;
  p.status = a.status;
  p.timeout_ns = a.timeout_ns;
  cudaError_t e = set_smem_limit(bitlinear_gemv_mma_kernel, L.total, true);
  if (e != cudaSuccess) return e;
  return launch_kernel(bitlinear_gemv_mma_kernel, dim3(static_cast<unsigned>(grid)), dim3(THREADS),
                       static_cast<size_t>(L.total), s, 0u, p);
}

}  // namespace blt
