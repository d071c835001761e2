// Decode-time BitLinear for 2..8 tokens on the warp-level tensor-core path
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
// {0,2,4,6} and {8,10,12,14} (or {1,3,5,7} and {9,11,13,15}) of one word.
// In a 256-deep k chunk (64 bytes of a row) lane c takes the four words
// 4c .. 4c+3 (one 16-byte load per row), and two MMAs per word cover it.
//
// Data flow. Each CTA owns a contiguous range of R output rows (a multiple of
// 8, equal up to 8 rows over the grid, so the weight bytes per SM are
// balanced), processed in blocks of 16 rows. A block is 16 consecutive rows
// of the packed weights, one contiguous range, so it arrives by a single
// bulk copy into a shared-memory slot (the copy engine's cost is per request,
// and a request per row would throttle it). The slots form a ring; the first
// ones are requested before the kernel waits for the previous one in the
// stream (the weights do not depend on it), and the CTA needs under half an
// SM, so the next kernel's CTAs sit beside it and stream their weights while
// this one computes. The activation rows are staged after the wait and, when
// every warp's share of K is at most two chunks, regrouped once into
// registers for all blocks. All eight consumer warps work on every block,
// each on its own chunks of K (four independent accumulators), and add their
// partial sums into a small shared-memory array with atomics; the epilogue
// reads it once.
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
constexpr int XREG_CHUNKS = 2;             // chunks per warp whose activations stay in registers

struct Params {
  int M, N, K;
  int nchunk;      // 256-deep chunks of K (the last may be 128 deep)
  int NB;          // 16-row blocks of the largest CTA
  int S;           // ring slots (blocks)
  int n8;          // N / 8
  int x_pitch;     // activation row pitch in shared memory: K + 16
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
  asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
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

// The two MMAs of one packed word per row: scale-1 and scale-16 fields of
// word wa (MMA row g) and wb (row g + 8) against the regrouped activations.
__device__ __forceinline__ void word_mma(int (&acc1)[4], int (&acc16)[4], uint32_t wa, uint32_t wb,
                                         const uint4& x) {
  const uint32_t ta = wa >> 2, tb = wb >> 2;
  mma_u8s8(acc1, wa & 0x03030303u, wb & 0x03030303u, ta & 0x03030303u, tb & 0x03030303u, x.x, x.y);
  mma_u8s8(acc16, wa & 0x30303030u, wb & 0x30303030u, ta & 0x30303030u, tb & 0x30303030u, x.z, x.w);
}

// XREG: every warp has at most XREG_CHUNKS chunks, whose regrouped
// activations are loaded once and kept in registers for all blocks.
template <bool XREG>
__global__ void __launch_bounds__(THREADS, 2) bitlinear_gemv_mma_kernel(const Params p) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row_bytes = p.K >> 2;
  const int SLOT = 16 * row_bytes;
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
  // block b (rows r0 + 16 b .. , one contiguous range) into slot b % S
  auto issue_block = [&](int b) {
    const uint32_t bytes = static_cast<uint32_t>(min(16, R - 16 * b) * row_bytes);
    uint64_t* bar = &full[b % p.S];
    mbar_arrive_expect_tx(bar, bytes);
    bulk_load_1d(smem_u32(smem + (b % p.S) * SLOT), p.Wp + static_cast<int64_t>(r0 + 16 * b) * row_bytes,
                 bytes, bar);
  };

  // the first blocks of the ring, one warp each, before the dependency wait
  if (lane == 0)
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
    if (lane == 0) {
      int b = p.S;
      for (; b < nblocks; ++b) {
        // the slot's previous block has been consumed by all eight warps
        if (!mbar_wait(&empty[b % p.S], ((b / p.S) - 1) & 1, tmo, s_abort)) {
          fail();
          break;
        }
        issue_block(b);
      }
      // do not leave while copies into this CTA's shared memory are in flight
      for (int d = 0, j = min(b, nblocks) - 1; d < p.S && j >= 0; ++d, --j)
        mbar_wait(&full[j % p.S], (j / p.S) & 1, tmo, nullptr);
      mbar_wait(xbar, 0, tmo, nullptr);
    }
  } else {
    // ---------------------------------------------------------- consumers
    const int g = lane >> 2, c = lane & 3;
    const int rows_a = (((g & 3) << 1) | (g >> 2));  // block row of MMA row g (rows {0,2,4,6} share a
    const int rows_b = rows_a + 8;                    // half-warp phase of the 16-byte loads)
    const int gx = g < p.M ? g : 0;                   // lanes of absent tokens read row 0 and zero it
    const uint8_t* xrow = xsm + gx * p.x_pitch + 64 * c;  // + 256 chunk: this lane's 64 bytes
    bool ok = mbar_wait(xbar, 0, tmo, s_abort);
    if (!ok) fail();
    // this warp's chunks: warp, warp + 8, ...; a chunk's activations as four
    // regrouped 16-byte groups (token g, k = 256 chunk + 64 c .. + 63)
    auto load_x = [&](int ch, uint4 (&xv)[4], int& xsum) {
      const int kbytes = min(256, p.K - 256 * ch);  // 256, or 128 for a short last chunk
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (64 * c + 16 * i < kbytes) v = *reinterpret_cast<const uint4*>(xrow + 256 * ch + 16 * i);
        if (g >= p.M) v = make_uint4(0u, 0u, 0u, 0u);
        xsum += byte_sum(v);
        xv[i] = regroup16(v);
      }
    };
    uint4 xr[XREG ? XREG_CHUNKS : 1][4];
    int xsum = 0;
    if constexpr (XREG) {
#pragma unroll
      for (int j = 0; j < XREG_CHUNKS; ++j) {
        const int ch = warp + WARPS * j;
        if (ch < p.nchunk) load_x(ch, xr[j], xsum);
        else {
#pragma unroll
          for (int i = 0; i < 4; ++i) xr[j][i] = make_uint4(0u, 0u, 0u, 0u);
        }
      }
    }
    for (int b = 0; ok && b < nblocks; ++b) {
      const int slot = b % p.S;
      if (!mbar_wait(&full[slot], (b / p.S) & 1, tmo, s_abort)) {
        fail();
        break;
      }
      const uint8_t* tile = smem + slot * SLOT;
      const uint8_t* pa = tile + rows_a * row_bytes + 16 * c;
      const uint8_t* pb = tile + rows_b * row_bytes + 16 * c;
      int e1[4] = {0, 0, 0, 0}, e16[4] = {0, 0, 0, 0}, o1[4] = {0, 0, 0, 0}, o16[4] = {0, 0, 0, 0};
      auto chunk = [&](int ch, const uint4 (&xv)[4]) {
        // words 4c .. 4c+3 of the chunk's 64 bytes of rows a and b (zero past K)
        uint4 wa = make_uint4(0u, 0u, 0u, 0u), wb = wa;
        if (256 * ch + 64 * c < p.K) {
          wa = *reinterpret_cast<const uint4*>(pa + 64 * ch);
          wb = *reinterpret_cast<const uint4*>(pb + 64 * ch);
        }
        word_mma(e1, e16, wa.x, wb.x, xv[0]);
        word_mma(o1, o16, wa.y, wb.y, xv[1]);
        word_mma(e1, e16, wa.z, wb.z, xv[2]);
        word_mma(o1, o16, wa.w, wb.w, xv[3]);
      };
      if constexpr (XREG) {
#pragma unroll
        for (int j = 0; j < XREG_CHUNKS; ++j)
          if (warp + WARPS * j < p.nchunk) chunk(warp + WARPS * j, xr[j]);
      } else {
        for (int ch = warp; ch < p.nchunk; ch += WARPS) {
          uint4 xv[4];
          int xs_unused = 0;
          load_x(ch, xv, b == 0 ? xsum : xs_unused);
          chunk(ch, xv);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);  // this warp is done with the slot
      if (b == 0) {
        // token sums over this warp's chunks: lanes of group g hold token g's
        xsum += __shfl_xor_sync(0xFFFFFFFFu, xsum, 1);
        xsum += __shfl_xor_sync(0xFFFFFFFFu, xsum, 2);
      }
      // D columns 2c, 2c + 1 are tokens 2c, 2c + 1: their sums sit in lanes 8c and 8c + 4
      const int s0 = __shfl_sync(0xFFFFFFFFu, xsum, 8 * c);
      const int s1 = __shfl_sync(0xFFFFFFFFu, xsum, 8 * c + 4);
      int32_t* pp = part + b * 128;
      atomicAdd(&pp[rows_a * 8 + 2 * c], e1[0] + o1[0] + ((e16[0] + o16[0]) >> 4) - s0);
      atomicAdd(&pp[rows_a * 8 + 2 * c + 1], e1[1] + o1[1] + ((e16[1] + o16[1]) >> 4) - s1);
      atomicAdd(&pp[rows_b * 8 + 2 * c], e1[2] + o1[2] + ((e16[2] + o16[2]) >> 4) - s0);
      atomicAdd(&pp[rows_b * 8 + 2 * c + 1], e1[3] + o1[3] + ((e16[3] + o16[3]) >> 4) - s1);
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
  L.x_off = S * 16 * (K / 4);
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
  p.nchunk = (p.K + 255) / 256;
  p.n8 = p.N / 8;
  // one CTA per SM (two fit on one), at most MAX_ROWS rows each
  int grid = std::min(num_sms(), p.n8);
  grid = std::max(grid, (p.n8 + MAX_ROWS / 8 - 1) / (MAX_ROWS / 8));
  const int r_hi = 8 * ((p.n8 + grid - 1) / grid);
  p.NB = (r_hi + 15) / 16;
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
  const bool xreg = p.nchunk <= WARPS * XREG_CHUNKS;
  void (*kern)(Params) = xreg ? bitlinear_gemv_mma_kernel<true> : bitlinear_gemv_mma_kernel<false>;
  cudaError_t e = set_smem_limit(kern, L.total, true);
  if (e != cudaSuccess) return e;
  return launch_kernel(kern, dim3(static_cast<unsigned>(grid)), dim3(THREADS), static_cast<size_t>(L.total), s,
                       0u, p);
}

}  // namespace blt
