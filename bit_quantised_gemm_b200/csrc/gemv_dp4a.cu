// Decode-time BitLinear for a few tokens (up to 8) on the CUDA cores.
//
// With up to eight tokens the layer is a matrix-vector product whose cost is
// streaming the 2-bit weights out of HBM (N x K/4 bytes): every weight meets
// at most eight activation codes, and the tensor cores would only add an
// unpack round trip through shared memory. This kernel keeps the weight
// stream in flight with bulk copies and does the arithmetic with 4-way byte
// dot products (dp4a) on the packed codes themselves, without expanding them
// to int8 first.
//
// Arithmetic. The packed word j of a weight row holds codes c = W_t + 1 in
// {0, 1, 2}; element 16j + 8h + i sits at bits [4i+2h, 4i+2h+2). With
// t = w >> 2, the four masks
//     w & 0x03030303 -> c of elements 16j + {0, 2, 4, 6}        (x1)
//     t & 0x03030303 -> c of elements 16j + {8, 10, 12, 14}     (x1)
//     w & 0x30303030 -> c of elements 16j + {1, 3, 5, 7}        (x16)
//     t & 0x30303030 -> c of elements 16j + {9, 11, 13, 15}     (x16)
// leave one code per byte, so dp4a against the activation bytes regrouped in
// that order gives sum_k c[k] x[k] in two integer accumulators (scales 1 and
// 16); with eight tokens each field is shifted down to scale 1 first and one
// accumulator per token and row takes all four. The layer output is acc = sum_k x[k] W_t[k] = sum_k c[k] x[k] - sum_k
// x[k], exact in int32, followed by the usual epilogue
//     y = bf16_rne((float)acc * (xs[m] * gamma[g(n)])).
//
// Work split. Rows of Wp are contiguous (K/4 bytes each), so an item of RW
// consecutive output features is one contiguous range, fetched with a single
// cp.async.bulk into a per-warp ring of `sw` slots. Every CTA owns one
// contiguous, equal share of the items (the weight bytes per SM are balanced)
// and deals it round-robin over its warps, so neighbouring warps read
// neighbouring rows. A lane takes the packed words j = lane, lane + 32, ... of every row of the
// item, so the 4-byte weight reads of a warp and its 16-byte reads of the
// activation codes (all MT tokens, held in shared memory for the whole
// kernel) are contiguous. With one token and K <= 4096 the activation words
// a lane needs (the same for every row) are instead loaded straight into its
// registers after the wait, regrouped there, and their sum is subtracted
// from the lane's partial sums: no shared-memory copy of the activations, no
// block-wide barrier, and only 4-byte weight reads in the inner loop. That
// variant runs as 8-warp CTAs with at most 112 KB of shared memory, two to an
// SM: the CTA of the next kernel in the stream (launched early through
// programmatic dependent launch) becomes resident beside this one and has
// its weights in flight before this kernel ends. The RW x MT partial sums of
// a lane are reduced
// across the warp with a transposing butterfly: log2(RW MT) exchange steps
// that halve the values held per lane, then plain xor steps.
#include <algorithm>

#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace blt {
namespace gemv_cc {

constexpr int MAX_SW = 4;             // ring slots per warp, at most
constexpr int MAX_WARPS = 16;
constexpr int SMEM_LIMIT = 232448;   // one CTA per SM
constexpr int SMEM_PAIR = 114688;    // two CTAs per SM (register-activation variant)
constexpr int PAIR_WARPS = 8;

struct Params {
  int M, N, K;
  int n_items;
  int sw;               // ring slots per warp
  const int8_t* xq;     // activation codes [M x K] (codes given)
  const float* xs;
  const uint16_t* x;    // bf16 activations [M x ldx] (quantised here)
  const uint16_t* up;   // nullable: ReLU^2-gated product with x as the gate
  int64_t ldx;
  float Q;              // 127 (INT8) or 7 (INT4)
  const uint8_t* Wp;
  const float* gamma;
  int G;
  int group_end[8];
  uint16_t* y;
  int64_t ldy;
  int* status;
  uint64_t timeout_ns;
};

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(dst), "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Regroup 16 activation bytes x0..x15 (little-endian words a, b, c, d) into
// {x0,x2,x4,x6}, {x8,x10,x12,x14}, {x1,x3,x5,x7}, {x9,x11,x13,x15}: the
// element order of the four code masks above.
__device__ __forceinline__ uint4 regroup16(uint4 v) {
  uint4 r;
  r.x = __byte_perm(v.x, v.y, 0x6420);
  r.y = __byte_perm(v.z, v.w, 0x6420);
  r.z = __byte_perm(v.x, v.y, 0x7531);
  r.w = __byte_perm(v.z, v.w, 0x7531);
  return r;
}

// Sum of the four signed bytes of each word.
__device__ __forceinline__ int byte_sum16(uint4 v) {
  int s = __dp4a(static_cast<int>(v.x), 0x01010101, 0);
  s = __dp4a(static_cast<int>(v.y), 0x01010101, s);
  s = __dp4a(static_cast<int>(v.z), 0x01010101, s);
  return __dp4a(static_cast<int>(v.w), 0x01010101, s);
}

// Butterfly over the 32 lanes: on return v[0] holds the warp-wide sum of
// value number `idx`, and every lane of a group of 32 / NV consecutive lanes
// holds the same one (idx runs over 0..NV-1 with the group).
template <int NV>
__device__ __forceinline__ int transpose_reduce(int (&v)[NV], int lane, int& idx) {
  static_assert(NV >= 1 && NV <= 32 && (NV & (NV - 1)) == 0, "power of two up to 32");
  idx = 0;
#pragma unroll
  for (int step = 0; (NV >> (step + 1)) >= 1; ++step) {
    const int h = NV >> (step + 1);
    const int o = 16 >> step;
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int j = 0; j < h; ++j) {
      const int send = up ? v[j] : v[j + h];
      const int keep = up ? v[j + h] : v[j];
      v[j] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, o);
    }
    if (up) idx += h;
  }
  int s = v[0];
#pragma unroll
  for (int o = 16 / NV; o >= 1; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
  return s;
}

// dp4a with unsigned bytes in a (the masked codes reach 128) and signed
// bytes in b (the activation codes).
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// One packed word against the MT tokens' regrouped activation words.
// NACC = 4: four masks without a shift, accumulators at scales 1, 4, 16, 64
// (fewest instructions; used for one or two tokens). NACC = 2: one shift,
// accumulators at scales 1 and 16 (half the registers; four tokens).
// NACC = 1: three shifts, every field at scale 1 in one accumulator (a
// quarter of the registers; eight tokens, four rows per item).
template <int MT, int NACC>
__device__ __forceinline__ void word_dot(uint32_t w, const uint4 (&xv)[MT], int (&acc)[MT][NACC]) {
  if constexpr (NACC == 4) {
    const uint32_t m0 = w & 0x03030303u, m1 = w & 0x0C0C0C0Cu;
    const uint32_t m2 = w & 0x30303030u, m3 = w & 0xC0C0C0C0u;
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      acc[t][0] = dp4a_us(m0, xv[t].x, acc[t][0]);
      acc[t][1] = dp4a_us(m1, xv[t].y, acc[t][1]);
      acc[t][2] = dp4a_us(m2, xv[t].z, acc[t][2]);
      acc[t][3] = dp4a_us(m3, xv[t].w, acc[t][3]);
    }
  } else if constexpr (NACC == 1) {
    const uint32_t m0 = w & 0x03030303u, m1 = (w >> 2) & 0x03030303u;
    const uint32_t m2 = (w >> 4) & 0x03030303u, m3 = (w >> 6) & 0x03030303u;
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      acc[t][0] = dp4a_us(m0, xv[t].x, acc[t][0]);
      acc[t][0] = dp4a_us(m1, xv[t].y, acc[t][0]);
      acc[t][0] = dp4a_us(m2, xv[t].z, acc[t][0]);
      acc[t][0] = dp4a_us(m3, xv[t].w, acc[t][0]);
    }
  } else {
    const uint32_t sh = w >> 2;
    const uint32_t m0 = w & 0x03030303u, m1 = sh & 0x03030303u;
    const uint32_t m2 = w & 0x30303030u, m3 = sh & 0x30303030u;
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      acc[t][0] = dp4a_us(m0, xv[t].x, acc[t][0]);
      acc[t][0] = dp4a_us(m1, xv[t].y, acc[t][0]);
      acc[t][1] = dp4a_us(m2, xv[t].z, acc[t][1]);
      acc[t][1] = dp4a_us(m3, xv[t].w, acc[t][1]);
    }
  }
}

// sum_k c[k] x[k] from the scaled accumulators (each is a multiple of its
// scale, so the shifts are exact).
template <int NACC>
__device__ __forceinline__ int combine(const int (&a)[NACC]) {
  if constexpr (NACC == 4) return a[0] + (a[1] >> 2) + (a[2] >> 4) + (a[3] >> 6);
  else if constexpr (NACC == 2) return a[0] + (a[1] >> 4);
  else return a[0];
}

__device__ __forceinline__ float warp_max_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

// FUSED: the kernel quantises the bf16 activations itself (per-token absmax,
// INT8 / INT4, optionally of the ReLU^2-gated product), redundantly in every
// CTA, instead of reading codes written by a separate quantiser launch.
// LW > 0: the activation codes are held in registers, LW packed-word
// columns per lane (K <= 512 LW); codes given (not FUSED) only.
template <int MT, int RW, bool FUSED, int LW>
__global__ void __launch_bounds__(LW > 0 ? PAIR_WARPS * 32 : MAX_WARPS * 32, LW > 0 ? 2 : 1)
bitlinear_gemv_dp4a_kernel(const Params p) {
  static_assert(LW == 0 || (!FUSED && LW % 4 == 0), "register activations: codes given");
  constexpr int NACC = MT <= 2 ? 4 : (MT == 4 ? 2 : 1);
  constexpr int U = MT <= 2 ? 4 : (MT == 4 ? 2 : 1);  // words per lane per batch of loads
  constexpr int NV = RW * MT;
  extern __shared__ __align__(16) uint8_t smem[];
  const int K = p.K;
  const int row_bytes = K >> 2;
  const int slot_bytes = RW * row_bytes;
  const int nwarps = blockDim.x >> 5;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  uint8_t* xsm = smem;                                  // [MT][K] regrouped codes (LW == 0)
  const int SW = p.sw;
  uint8_t* ring = smem + (LW > 0 ? 0 : MT * K);         // [nwarps][SW][slot_bytes]
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring + nwarps * SW * slot_bytes);
  uint64_t* xbar = bars + nwarps * SW;
  int* xsum = reinterpret_cast<int*>(xbar + 1);         // [MT]

  uint8_t* my_ring = ring + warp * SW * slot_bytes;
  uint64_t* my_bar = bars + warp * SW;
  // this CTA's share of the items: [lo, hi)
  const int lo = static_cast<int>(static_cast<int64_t>(blockIdx.x) * p.n_items / gridDim.x);
  const int hi = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * p.n_items / gridDim.x);
  const int n_mine = warp < hi - lo ? (hi - lo - 1 - warp) / nwarps + 1 : 0;
  auto item_of = [&](int s) { return lo + warp + s * nwarps; };

  auto issue = [&](int s) {  // lane 0: fetch the s-th item of this warp
    const int n0 = item_of(s) * RW;
    const int rows = min(RW, p.N - n0);
    const uint32_t bytes = static_cast<uint32_t>(rows * row_bytes);
    uint64_t* bar = my_bar + (s % SW);
    mbar_arrive_expect_tx(bar, bytes);
    bulk_load(smem_u32(my_ring + (s % SW) * slot_bytes),
              p.Wp + static_cast<int64_t>(n0) * row_bytes, bytes, bar);
  };

  // The weight stream does not depend on the previous kernel in the stream:
  // the first items of every warp go out before waiting for it.
  if (lane == 0) {
    for (int i = 0; i < SW; ++i) mbar_init(my_bar + i, 1);
    if (threadIdx.x == 0) mbar_init(xbar, 1);
    fence_mbar_init();
    for (int s = 0; s < min(SW, n_mine); ++s) issue(s);
  }
  __syncwarp();  // the warp's barriers are initialised before any lane waits on them
  float gam[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) gam[i] = i < p.G ? __ldg(p.gamma + i) : 0.f;
  float xsc[MT];
  bool x_ok = true;
  pdl_trigger();
  if constexpr (FUSED) {
    pdl_wait();  // the bf16 activations come from the previous kernel
    float* red = reinterpret_cast<float*>(xsum + MT);  // [nwarps][MT] partial maxima
    if (threadIdx.x < MT) xsum[threadIdx.x] = 0;
    for (int i = p.M * K / 16 + threadIdx.x; i < MT * K / 16; i += blockDim.x)
      reinterpret_cast<uint4*>(xsm)[i] = make_uint4(0u, 0u, 0u, 0u);  // tokens M.. are zero
    const int G16 = K >> 4;  // 16-element groups per row
    const bool relu2 = p.up != nullptr;
    auto load16 = [&](int t, int g, float (&h)[16]) {
      const uint4* xr = reinterpret_cast<const uint4*>(p.x + static_cast<int64_t>(t) * p.ldx) + 2 * g;
      const uint4* ur = relu2 ? reinterpret_cast<const uint4*>(p.up + static_cast<int64_t>(t) * p.ldx) + 2 * g : xr;
      float a[8], b[8];
      act_vals8(__ldg(xr), relu2 ? __ldg(ur) : make_uint4(0u, 0u, 0u, 0u), relu2, a);
      act_vals8(__ldg(xr + 1), relu2 ? __ldg(ur + 1) : make_uint4(0u, 0u, 0u, 0u), relu2, b);
#pragma unroll
      for (int i = 0; i < 8; ++i) { h[i] = a[i]; h[8 + i] = b[i]; }
    };
    // When every thread has at most two 16-element groups, the raw bf16 words
    // stay in registers from the first pass to the second (one round of
    // global loads); otherwise the second pass reads them again.
    const int ngroups = p.M * G16;
    const bool held = ngroups <= 2 * static_cast<int>(blockDim.x);
    uint4 xv[2][2], uv[2][2];
    if (held) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int i = threadIdx.x + r * blockDim.x;
        xv[r][0] = xv[r][1] = uv[r][0] = uv[r][1] = make_uint4(0u, 0u, 0u, 0u);
        if (i < ngroups) {
          const int t = i / G16, g = i - t * G16;
          const uint4* xr = reinterpret_cast<const uint4*>(p.x + static_cast<int64_t>(t) * p.ldx) + 2 * g;
          xv[r][0] = __ldg(xr);
          xv[r][1] = __ldg(xr + 1);
          if (relu2) {
            const uint4* ur = reinterpret_cast<const uint4*>(p.up + static_cast<int64_t>(t) * p.ldx) + 2 * g;
            uv[r][0] = __ldg(ur);
            uv[r][1] = __ldg(ur + 1);
          }
        }
      }
    }
    auto held16 = [&](int r, float (&h)[16]) {
      float a[8], b[8];
      act_vals8(xv[r][0], uv[r][0], relu2, a);
      act_vals8(xv[r][1], uv[r][1], relu2, b);
#pragma unroll
      for (int i = 0; i < 8; ++i) { h[i] = a[i]; h[8 + i] = b[i]; }
    };
    // pass 1: absmax of every token row
    float am[MT];
#pragma unroll
    for (int t = 0; t < MT; ++t) am[t] = 0.f;
    auto absmax16 = [&](int t, const float (&h)[16]) {
      float mx = 0.f;
#pragma unroll
      for (int j = 0; j < 16; ++j) mx = fmaxf(mx, fabsf(h[j]));
#pragma unroll
      for (int u = 0; u < MT; ++u) am[u] = (u == t) ? fmaxf(am[u], mx) : am[u];
    };
    if (held) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int i = threadIdx.x + r * blockDim.x;
        if (i < ngroups) {
          float h[16];
          held16(r, h);
          absmax16(i / G16, h);
        }
      }
    } else {
      for (int i = threadIdx.x; i < ngroups; i += blockDim.x) {
        float h[16];
        load16(i / G16, i % G16, h);
        absmax16(i / G16, h);
      }
    }
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      am[t] = warp_max_f(am[t]);
      if (lane == 0) red[warp * MT + t] = am[t];
    }
    __syncthreads();
    float inv[MT];
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      float a = 0.f;
      for (int w = 0; w < nwarps; ++w) a = fmaxf(a, red[w * MT + t]);
      a = fmaxf(a, kEps);
      inv[t] = __fdiv_rn(p.Q, a);
      xsc[t] = t < p.M ? __fdiv_rn(a, p.Q) : 0.f;
    }
    // pass 2: the codes, regrouped into shared memory, and their row sums
    int part[MT];
#pragma unroll
    for (int t = 0; t < MT; ++t) part[t] = 0;
    auto codes16 = [&](int t, int g, const float (&h)[16]) {
      float iv = 0.f;
#pragma unroll
      for (int u = 0; u < MT; ++u) iv = (u == t) ? inv[u] : iv;
      int q[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) q[j] = quant_code(h[j], iv, -p.Q - 1.f, p.Q);
      const uint4 v = make_uint4(pack_s8x4(q[0], q[1], q[2], q[3]), pack_s8x4(q[4], q[5], q[6], q[7]),
                                 pack_s8x4(q[8], q[9], q[10], q[11]), pack_s8x4(q[12], q[13], q[14], q[15]));
      const int bs = byte_sum16(v);
#pragma unroll
      for (int u = 0; u < MT; ++u) part[u] += (u == t) ? bs : 0;
      *reinterpret_cast<uint4*>(xsm + t * K + 16 * g) = regroup16(v);
    };
    if (held) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int i = threadIdx.x + r * blockDim.x;
        if (i < ngroups) {
          float h[16];
          held16(r, h);
          codes16(i / G16, i % G16, h);
        }
      }
    } else {
      for (int i = threadIdx.x; i < ngroups; i += blockDim.x) {
        float h[16];
        load16(i / G16, i % G16, h);
        codes16(i / G16, i % G16, h);
      }
    }
#pragma unroll
    for (int t = 0; t < MT; ++t) {
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) part[t] += __shfl_xor_sync(0xFFFFFFFFu, part[t], o);
      if (lane == 0 && part[t] != 0) atomicAdd(&xsum[t], part[t]);
    }
    __syncthreads();
  } else if constexpr (LW > 0) {
    pdl_wait();  // activation codes and scales come from the previous kernel
#pragma unroll
    for (int t = 0; t < MT; ++t) xsc[t] = t < p.M ? __ldg(p.xs + t) : 0.f;
  } else {
    pdl_wait();  // activation codes and scales come from the previous kernel
    if (threadIdx.x == 0) {  // the codes are one contiguous M x K block
      const uint32_t xbytes = static_cast<uint32_t>(p.M * K);
      mbar_arrive_expect_tx(xbar, xbytes);
      bulk_load(smem_u32(xsm), p.xq, xbytes, xbar);
    }
#pragma unroll
    for (int t = 0; t < MT; ++t) xsc[t] = t < p.M ? __ldg(p.xs + t) : 0.f;
    if (threadIdx.x < MT) xsum[threadIdx.x] = 0;
    // tokens p.M .. MT-1 are zero codes
    for (int i = p.M * K / 16 + threadIdx.x; i < MT * K / 16; i += blockDim.x)
      reinterpret_cast<uint4*>(xsm)[i] = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();

    // Regroup the codes in place and take their row sums.
    x_ok = mbar_wait(xbar, 0, p.timeout_ns, nullptr);
    if (x_ok) {
      const int groups = p.M * K / 16;
      int part[MT];
#pragma unroll
      for (int t = 0; t < MT; ++t) part[t] = 0;
      for (int i = threadIdx.x; i < groups; i += blockDim.x) {
        uint4* q = reinterpret_cast<uint4*>(xsm) + i;
        const uint4 v = *q;
        const int t = i / (K / 16);
        const int bs = byte_sum16(v);
#pragma unroll
        for (int u = 0; u < MT; ++u) part[u] += (u == t) ? bs : 0;
        *q = regroup16(v);
      }
#pragma unroll
      for (int t = 0; t < MT; ++t) {
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) part[t] += __shfl_xor_sync(0xFFFFFFFFu, part[t], o);
        if (lane == 0 && part[t] != 0) atomicAdd(&xsum[t], part[t]);
      }
    }
    __syncthreads();
  }
  const int words = K >> 4;
  int xsm_sum[MT];
  uint4 xr[LW > 0 ? LW : 1][MT];  // LW > 0: this lane's regrouped activation words
  if constexpr (LW > 0) {
#pragma unroll
    for (int t = 0; t < MT; ++t) xsm_sum[t] = 0;
#pragma unroll
    for (int i = 0; i < LW; ++i) {
      const int j = lane + 32 * i;
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        const uint4 v = (j < words && t < p.M)
                            ? *reinterpret_cast<const uint4*>(p.xq + static_cast<int64_t>(t) * K + 16 * j)
                            : make_uint4(0u, 0u, 0u, 0u);
        xsm_sum[t] += byte_sum16(v);  // this lane's share of sum_k x[k]
        xr[i][t] = regroup16(v);
      }
    }
  } else {
#pragma unroll
    for (int t = 0; t < MT; ++t) xsm_sum[t] = xsum[t];
  }

  const uint32_t x_base = smem_u32(xsm);
  bool timed_out = !x_ok;
  int s = 0;
  for (; s < n_mine && !timed_out; ++s) {
    if (!mbar_wait(my_bar + (s % SW), (s / SW) & 1, p.timeout_ns, nullptr)) {
      timed_out = true;
      break;
    }
    const uint32_t w_base = smem_u32(my_ring + (s % SW) * slot_bytes);
    int acc[RW][MT][NACC];
#pragma unroll
    for (int r = 0; r < RW; ++r)
#pragma unroll
      for (int t = 0; t < MT; ++t)
#pragma unroll
        for (int a = 0; a < NACC; ++a) acc[r][t][a] = 0;

    // U words per lane are loaded before any arithmetic; words past the row
    // end read as code 0, which adds nothing.
    if constexpr (LW > 0) {
#pragma unroll
      for (int i = 0; i < LW; i += 4) {
        uint32_t w[4][RW];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int j = lane + 32 * (i + u);
#pragma unroll
          for (int r = 0; r < RW; ++r) w[u][r] = j < words ? ld_shared_u32(w_base + r * row_bytes + 4 * j) : 0u;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int r = 0; r < RW; ++r) word_dot<MT, NACC>(w[u][r], xr[i + u], acc[r]);
      }
    } else
    for (int j0 = lane; j0 < words; j0 += 32 * U) {
      uint4 xv[U][MT];
      uint32_t w[U][RW];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = j0 + 32 * u;
        const bool in = j < words;
#pragma unroll
        for (int t = 0; t < MT; ++t)
          xv[u][t] = in ? ld_shared_v4(x_base + t * K + 16 * j) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int r = 0; r < RW; ++r) w[u][r] = in ? ld_shared_u32(w_base + r * row_bytes + 4 * j) : 0u;
      }
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int r = 0; r < RW; ++r) word_dot<MT, NACC>(w[u][r], xv[u], acc[r]);
    }
    __syncwarp();  // every lane has read the slot
    if (lane == 0 && s + SW < n_mine) issue(s + SW);

    int v[NV];
#pragma unroll
    for (int r = 0; r < RW; ++r)
#pragma unroll
      for (int t = 0; t < MT; ++t)
        v[r * MT + t] = combine<NACC>(acc[r][t]) - (LW > 0 ? xsm_sum[t] : 0);
    int idx;
    const int sum = transpose_reduce<NV>(v, lane, idx);
    if ((lane & (32 / NV - 1)) == 0) {
      const int r = idx / MT, t = idx % MT;
      const int n = item_of(s) * RW + r;
      if (t < p.M && n < p.N) {
        int ts = 0;
        float xst = 0.f;
#pragma unroll
        for (int u = 0; u < MT; ++u) {
          ts = (u == t) ? xsm_sum[u] : ts;
          xst = (u == t) ? xsc[u] : xst;
        }
        int g = 0;
#pragma unroll
        for (int i = 0; i < 7; ++i) g += (i < p.G - 1 && n >= p.group_end[i]) ? 1 : 0;
        float gm = gam[0];
#pragma unroll
        for (int i = 1; i < 8; ++i) gm = (g == i) ? gam[i] : gm;
        const int acc = LW > 0 ? sum : sum - ts;
        p.y[static_cast<int64_t>(t) * p.ldy + n] = __bfloat16_as_ushort(
            __float2bfloat16_rn(static_cast<float>(acc) * (xst * gm)));
      }
    }
  }
  if (timed_out) {
    report_status(p.status, BITLINEAR_STATUS_TIMEOUT);
    // Let copies still in flight land before the block's shared memory is
    // released (bounded as well).
    if (lane == 0)
      for (int q = s; q < min(s + SW, n_mine); ++q)
        mbar_wait(my_bar + (q % SW), (q / SW) & 1, p.timeout_ns, nullptr);
    if (!FUSED && threadIdx.x == 0 && !x_ok) mbar_wait(xbar, 0, p.timeout_ns, nullptr);
    __syncwarp();
  }
}

}  // namespace gemv_cc

// xk: bytes of activation codes staged in shared memory (mt K, or 0 when
// they are held in registers)
static size_t dp4a_smem_bytes(int mt, int rw, int64_t K, int warps, int sw, int64_t xk) {
  return size_t(xk) + size_t(warps) * sw * rw * (K / 4) + size_t(warps) * sw * 8 + 8 + 8 * 4 +
         size_t(gemv_cc::MAX_WARPS) * mt * 4;
}

static int dp4a_tokens(int64_t M) { return M == 1 ? 1 : M == 2 ? 2 : M <= 4 ? 4 : 8; }

struct Dp4aShape {
  int warps = 0, sw = 0;
  size_t smem = 0;
};

// Warps and ring slots for a CTA that owns `per_cta` items: as many warps as
// there are items (up to the block size), then as many slots as a warp has
// items (up to 4), inside `limit` bytes of shared memory; fewer slots (not
// below 2 while a warp has two items or more), then fewer warps, if it does
// not fit. warps = 0 when even one warp with one slot does not fit.
static Dp4aShape dp4a_shape(int mt, int rw, int64_t K, int per_cta, int max_warps, size_t limit,
                            bool x_in_regs = false) {
  Dp4aShape r;
  for (int w = std::min(max_warps, std::max(per_cta, 1)); w >= 1; --w) {
    const int ipw = (per_cta + w - 1) / w;
    const int top = std::max(1, std::min(gemv_cc::MAX_SW, ipw));
    const int bottom = std::min(2, top);
    for (int sw = top; sw >= bottom; --sw) {
      const size_t b = dp4a_smem_bytes(mt, rw, K, w, sw, x_in_regs ? 0 : mt * K);
      if (b <= limit) {
        r.warps = w;
        r.sw = sw;
        r.smem = b;
        return r;
      }
    }
  }
  return r;
}

bool gemv_dp4a_supported(int64_t M, int64_t K) {
  if (M < 1 || M > kGemvDp4aMaxTokens || K % 64 != 0) return false;
  return dp4a_shape(dp4a_tokens(M), 2, K, 1, 1, gemv_cc::SMEM_LIMIT).warps > 0;  // staged codes
}

// One CTA per SM, each with an equal share of the items. One token with
// K <= 4096 and codes given: activations in registers (8 columns per lane),
// CTAs sized to share the SM with the next kernel's.
template <int MT, int RW, bool FUSED>
static cudaError_t launch_mt(gemv_cc::Params p, cudaStream_t s) {
  p.n_items = (p.N + RW - 1) / RW;
  const int grid = std::min(num_sms(), p.n_items);
  const int per_cta = (p.n_items + grid - 1) / grid;
  constexpr bool kRegs = MT == 1 && !FUSED;
  const bool regs = kRegs && p.K <= 4096;
  const Dp4aShape sh =
      regs ? dp4a_shape(MT, RW, p.K, per_cta, gemv_cc::PAIR_WARPS, gemv_cc::SMEM_PAIR, true)
           : dp4a_shape(MT, RW, p.K, per_cta, gemv_cc::MAX_WARPS, gemv_cc::SMEM_LIMIT, false);
  if (sh.warps == 0) return cudaErrorInvalidValue;
  p.sw = sh.sw;
  auto kern = regs ? gemv_cc::bitlinear_gemv_dp4a_kernel<MT, RW, FUSED, kRegs ? 8 : 0>
                   : gemv_cc::bitlinear_gemv_dp4a_kernel<MT, RW, FUSED, 0>;
  // with register activations, all of the unified L1 as shared memory, so
  // that a second CTA finds room without the SM changing its split
  cudaError_t e = set_smem_limit(kern, static_cast<int>(sh.smem), regs);
  if (e != cudaSuccess) return e;
  return launch_kernel(kern, dim3(grid), dim3(sh.warps * 32), sh.smem, s, 0u, p);
}

// Items of 4 output features when every warp of every CTA gets at least one
// (and two slots per warp fit), else of 2 (more items to spread over the
// warps).
template <int MT, bool FUSED>
static cudaError_t launch_pick_rows(const gemv_cc::Params& p, cudaStream_t s) {
  if constexpr (MT == 1 && !FUSED) {  // register activations: an item or two per warp
    if (p.K <= 4096) {
      if (int64_t(p.N) > int64_t(2) * gemv_cc::PAIR_WARPS * num_sms())
        return launch_mt<MT, 4, FUSED>(p, s);
      return launch_mt<MT, 2, FUSED>(p, s);
    }
  }
  {  // items of 4 rows share each load of the activation words over twice the weights
    constexpr int W = gemv_cc::MAX_WARPS;
    if (int64_t(p.N) >= int64_t(4) * W * num_sms() &&
        dp4a_shape(MT, 4, p.K, 2 * W, W, gemv_cc::SMEM_LIMIT).warps == W)
      return launch_mt<MT, 4, FUSED>(p, s);
  }
  return launch_mt<MT, 2, FUSED>(p, s);
}

template <bool FUSED>
static cudaError_t launch_by_tokens(const gemv_cc::Params& p, cudaStream_t s) {
  switch (dp4a_tokens(p.M)) {
    case 1: return launch_pick_rows<1, FUSED>(p, s);
    case 2: return launch_pick_rows<2, FUSED>(p, s);
    case 4: return launch_pick_rows<4, FUSED>(p, s);
    default: return launch_pick_rows<8, FUSED>(p, s);
  }
}

static gemv_cc::Params dp4a_params(const GemmArgs& a) {
  gemv_cc::Params p{};
  p.M = static_cast<int>(a.M);
  p.N = static_cast<int>(a.N);
  p.K = static_cast<int>(a.K);
  p.xq = static_cast<const int8_t*>(a.xq);
  p.xs = a.xs;
  p.Wp = a.Wp;
  p.gamma = a.gamma;
  p.G = a.G;
  for (int i = 0; i < 8; ++i) p.group_end[i] = a.group_end[i];
  p.y = static_cast<uint16_t*>(a.out);
  p.ldy = a.ldo;
  p.status = a.status;
  p.timeout_ns = a.timeout_ns;
  return p;
}

cudaError_t launch_gemv_dp4a(const GemmArgs& a, cudaStream_t s) {
  return launch_by_tokens<false>(dp4a_params(a), s);
}

cudaError_t launch_gemv_dp4a_quant(const GemmArgs& a, const uint16_t* x, const uint16_t* up,
                                   int64_t ldx, int mode, cudaStream_t s) {
  gemv_cc::Params p = dp4a_params(a);
  p.x = x;
  p.up = up;
  p.ldx = ldx;
  p.Q = mode == BITLINEAR_MODE_INT8 ? 127.f : 7.f;
  return launch_by_tokens<true>(p, s);
}

}  // namespace blt
