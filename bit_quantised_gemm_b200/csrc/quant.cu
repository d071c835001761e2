// Per-token activation quantisers, top-k sparsifier and KV-cache quantiser.
//
// All three are HBM-bound: one pass reads the bf16 rows once (16-byte
// vector loads), reductions run in registers / shared memory, codes are
// written once with vector stores. No fast-math: every scale and rounding is
// an IEEE fp32 operation (explicit __fdiv_rn / __fmul_rn, rintf = RNE).
#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace blt {

constexpr int kQuantThreads = 256;

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float block_max_256(float v, float* red /*[8]*/) {
  v = warp_max(v);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  if (lane == 0) red[wid] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int i = 1; i < kQuantThreads / 32; ++i) r = fmaxf(r, red[i]);
  __syncthreads();
  return r;
}

// Inclusive prefix sum over the 256 threads of the block.
__device__ __forceinline__ uint32_t block_scan_256(uint32_t v, uint32_t* sums /*[8]*/) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) sums[wid] = v;
  __syncthreads();
  if (wid == 0) {
    uint32_t s = lane < 8 ? sums[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) {
      const uint32_t n = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += n;
    }
    if (lane < 8) sums[lane] = s;
  }
  __syncthreads();
  if (wid > 0) v += sums[wid - 1];
  __syncthreads();
  return v;
}

// 8 fp32 -> 8 e2m1 nibbles (even index low), round to nearest even, satfinite.
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float (&v)[8]) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return out;
}

// ------------------------------------------------------------ quant_act
// One block per token row. Pass 1 loads the row (and the up row for the
// ReLU^2 gate), keeps h in shared memory and reduces the absmax; pass 2
// writes the codes.
template <int MODE, bool RELU2>
__global__ void __launch_bounds__(kQuantThreads) quant_act_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ up, int K, int64_t ldx,
    void* __restrict__ q_out, float* __restrict__ xs_out) {
  pdl_wait();  // inputs come from the previous kernel in the stream
  pdl_trigger();
  extern __shared__ float4 s_row4[];
  float* s_row = reinterpret_cast<float*>(s_row4);
  __shared__ float red[kQuantThreads / 32];
  const int64_t m = blockIdx.x;
  const uint4* xr = reinterpret_cast<const uint4*>(x + m * ldx);
  const uint4* ur = reinterpret_cast<const uint4*>(RELU2 ? up + m * ldx : x);
  const int nchunk = K >> 3;

  float amax = 0.f;
  // unrolled so that several rows' worth of 16-byte loads are in flight per thread
#pragma unroll 4
  for (int c = threadIdx.x; c < nchunk; c += kQuantThreads) {
    float h[8];
    bf16x8_to_f32(__ldg(xr + c), h);
    if (RELU2) {
      float u[8];
      bf16x8_to_f32(__ldg(ur + c), u);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float r = h[i] > 0.f ? h[i] : 0.f;
        h[i] = __fmul_rn(__fmul_rn(r, r), u[i]);
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(h[i]));
    s_row4[2 * c] = make_float4(h[0], h[1], h[2], h[3]);
    s_row4[2 * c + 1] = make_float4(h[4], h[5], h[6], h[7]);
  }
  amax = block_max_256(amax, red);  // also orders the shared-memory row

  constexpr float Q = MODE == BITLINEAR_MODE_INT8 ? 127.f : (MODE == BITLINEAR_MODE_INT4 ? 7.f : 6.f);
  const float a = fmaxf(amax, kEps);
  const float inv = __fdiv_rn(Q, a);
  if (threadIdx.x == 0) xs_out[m] = __fdiv_rn(a, Q);

  for (int c = threadIdx.x; c < nchunk; c += kQuantThreads) {
    const float4 p0 = s_row4[2 * c], p1 = s_row4[2 * c + 1];
    const float h[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
    if (MODE == BITLINEAR_MODE_FP4) {
      float v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(h[i], inv);
      reinterpret_cast<uint32_t*>(q_out)[m * (K >> 3) + c] = cvt_e2m1x8(v);
    } else {
      int q[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) q[i] = quant_code(h[i], inv, -Q - 1.f, Q);
      reinterpret_cast<uint2*>(q_out)[m * (K >> 3) + c] =
          make_uint2(pack_s8x4(q[0], q[1], q[2], q[3]), pack_s8x4(q[4], q[5], q[6], q[7]));
    }
  }
  (void)s_row;
}

// Rows of up to 4096 elements: one warp per row, the whole row held in
// registers as bf16 (CPL 16-byte chunks per lane, all loads in flight at
// once), warp-shuffle absmax, no shared memory and no block barrier.
template <int MODE, bool RELU2, int CPL>
__global__ void __launch_bounds__(kQuantThreads) quant_act_warp_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ up, int64_t M, int K,
    int64_t ldx, void* __restrict__ q_out, float* __restrict__ xs_out) {
  pdl_wait();  // inputs come from the previous kernel in the stream
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t m = static_cast<int64_t>(blockIdx.x) * (kQuantThreads / 32) + (threadIdx.x >> 5);
  if (m >= M) return;  // whole warp
  const int nchunk = K >> 3;
  const uint4* xr = reinterpret_cast<const uint4*>(x + m * ldx);
  const uint4* ur = reinterpret_cast<const uint4*>(RELU2 ? up + m * ldx : x);
  uint4 xv[CPL], uv[RELU2 ? CPL : 1];
#pragma unroll
  for (int j = 0; j < CPL; ++j) {
    const int c = lane + 32 * j;
    xv[j] = c < nchunk ? __ldg(xr + c) : make_uint4(0, 0, 0, 0);
    if (RELU2) uv[j] = c < nchunk ? __ldg(ur + c) : make_uint4(0, 0, 0, 0);
  }
  auto row_vals = [&](int j, float (&h)[8]) {
    bf16x8_to_f32(xv[j], h);
    if (RELU2) {
      float u[8];
      bf16x8_to_f32(uv[RELU2 ? j : 0], u);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float r = h[i] > 0.f ? h[i] : 0.f;
        h[i] = __fmul_rn(__fmul_rn(r, r), u[i]);
      }
    }
  };
  float amax = 0.f;
#pragma unroll
  for (int j = 0; j < CPL; ++j) {
    float h[8];
    row_vals(j, h);
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(h[i]));
  }
  amax = warp_max(amax);
  constexpr float Q = MODE == BITLINEAR_MODE_INT8 ? 127.f : (MODE == BITLINEAR_MODE_INT4 ? 7.f : 6.f);
  const float a = fmaxf(amax, kEps);
  const float inv = __fdiv_rn(Q, a);
  if (lane == 0) xs_out[m] = __fdiv_rn(a, Q);
#pragma unroll
  for (int j = 0; j < CPL; ++j) {
    const int c = lane + 32 * j;
    if (c >= nchunk) break;
    float h[8];
    row_vals(j, h);
    if (MODE == BITLINEAR_MODE_FP4) {
      float v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(h[i], inv);
      reinterpret_cast<uint32_t*>(q_out)[m * nchunk + c] = cvt_e2m1x8(v);
    } else {
      int q[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) q[i] = quant_code(h[i], inv, -Q - 1.f, Q);
      reinterpret_cast<uint2*>(q_out)[m * nchunk + c] =
          make_uint2(pack_s8x4(q[0], q[1], q[2], q[3]), pack_s8x4(q[4], q[5], q[6], q[7]));
    }
  }
}

template <int MODE, bool RELU2, int CPL>
static cudaError_t launch_quant_warp(const uint16_t* x, const uint16_t* up, int64_t M, int K,
                                     int64_t ldx, void* q, float* xs, cudaStream_t s) {
  constexpr int RPB = kQuantThreads / 32;
  return launch_kernel(quant_act_warp_kernel<MODE, RELU2, CPL>,
                       dim3(static_cast<unsigned>((M + RPB - 1) / RPB)), dim3(kQuantThreads), 0, s, 0u,
                       x, up, M, K, ldx, q, xs);
}

template <int MODE, bool RELU2>
static cudaError_t launch_quant_t(const uint16_t* x, const uint16_t* up, int64_t M, int K,
                                  int64_t ldx, void* q, float* xs, cudaStream_t s) {
  const int chunks_per_lane = (K / 8 + 31) / 32;
  if (chunks_per_lane <= 1) return launch_quant_warp<MODE, RELU2, 1>(x, up, M, K, ldx, q, xs, s);
  if (chunks_per_lane <= 2) return launch_quant_warp<MODE, RELU2, 2>(x, up, M, K, ldx, q, xs, s);
  if (chunks_per_lane <= 4) return launch_quant_warp<MODE, RELU2, 4>(x, up, M, K, ldx, q, xs, s);
  if (chunks_per_lane <= 8) return launch_quant_warp<MODE, RELU2, 8>(x, up, M, K, ldx, q, xs, s);
  if (!RELU2 && chunks_per_lane <= 16)
    return launch_quant_warp<MODE, RELU2, 16>(x, up, M, K, ldx, q, xs, s);
  const size_t smem = static_cast<size_t>(K) * sizeof(float);
  auto kern = quant_act_kernel<MODE, RELU2>;
  if (smem > 48 * 1024) {
    cudaError_t e = set_smem_limit(kern, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  return launch_kernel(kern, dim3(static_cast<unsigned>(M)), dim3(kQuantThreads), smem, s, 0u,
                       x, up, K, ldx, q, xs);
}

cudaError_t launch_quant_act(const uint16_t* x, const uint16_t* up, int64_t M, int64_t K,
                             int64_t ldx, int mode, void* q, float* xs, cudaStream_t s) {
  const int k = static_cast<int>(K);
  if (up) {
    if (mode == BITLINEAR_MODE_INT8) return launch_quant_t<BITLINEAR_MODE_INT8, true>(x, up, M, k, ldx, q, xs, s);
    if (mode == BITLINEAR_MODE_INT4) return launch_quant_t<BITLINEAR_MODE_INT4, true>(x, up, M, k, ldx, q, xs, s);
    return launch_quant_t<BITLINEAR_MODE_FP4, true>(x, up, M, k, ldx, q, xs, s);
  }
  if (mode == BITLINEAR_MODE_INT8) return launch_quant_t<BITLINEAR_MODE_INT8, false>(x, up, M, k, ldx, q, xs, s);
  if (mode == BITLINEAR_MODE_INT4) return launch_quant_t<BITLINEAR_MODE_INT4, false>(x, up, M, k, ldx, q, xs, s);
  return launch_quant_t<BITLINEAR_MODE_FP4, false>(x, up, M, k, ldx, q, xs, s);
}

// ----------------------------------------------------------------- top-k
// Inclusive prefix sum over the NT threads of the block (NT / 32 <= 8 warps).
template <int NT>
__device__ __forceinline__ uint32_t block_scan(uint32_t v, uint32_t* sums /*[8]*/) {
  constexpr int NWARP = NT / 32;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) sums[wid] = v;
  __syncthreads();
  if (wid == 0) {
    uint32_t s = lane < NWARP ? sums[lane] : 0u;
#pragma unroll
    for (int o = 1; o < NWARP; o <<= 1) {
      const uint32_t n = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += n;
    }
    if (lane < NWARP) sums[lane] = s;
  }
  __syncthreads();
  if (wid > 0) v += sums[wid - 1];
  __syncthreads();
  return v;
}

template <int NT>
__device__ __forceinline__ float block_max(float v, float* red /*[8]*/) {
  v = warp_max(v);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  if (lane == 0) red[wid] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int i = 1; i < NT / 32; ++i) r = fmaxf(r, red[i]);
  return r;
}

// One block of NT threads per row; thread t owns the contiguous elements
// [t*E, t*E+E), held as packed bf16 pairs. Radix select on the 15-bit |bf16|
// key: a 256-bin histogram of key >> 7, then a 128-bin histogram of the low
// bits inside the selected bin, gives the threshold key T and the count of
// keys above it. Keys equal to T are kept in column order until k are kept
// (a block prefix sum of their counts ranks each thread's). Columns past K
// are read as key 0: they come after every real column in the (key
// descending, column ascending) order, so they are never among the k kept
// and the loops need no bounds tests. The per-row work outside the element
// loops (scans, barriers) is the same for any E, so rows of 4096 use 128
// threads of 32 elements.
template <int NT, int E>
__global__ void __launch_bounds__(NT, (E >= 32 ? 1024 : 2048) / NT) topk_i8_kernel(
    const uint16_t* __restrict__ x, int K, int64_t ldx, int k, int8_t* __restrict__ q_out,
    float* __restrict__ xs_out, uint8_t* __restrict__ mask_out) {
  pdl_wait();  // inputs come from the previous kernel in the stream
  pdl_trigger();
  static_assert(E % 8 == 0 && E <= 64, "whole 16-byte groups, 64-bit masks");
  static_assert(NT == 128 || NT == 256, "two or one histogram bins per thread");
  constexpr int NW = E / 2;       // packed pairs per thread
  constexpr int B1 = 256 / NT;    // pass-1 bins per thread
  __shared__ uint32_t hist[256];
  __shared__ uint32_t sums[8];
  __shared__ float red[8];
  __shared__ uint32_t sel[2];  // selected bin, count of keys above the bin
  const int t = threadIdx.x;
  const int64_t m = blockIdx.x;
  const int base = t * E;
  const int nvalid = max(0, min(E, K - base));  // multiple of 8

  uint32_t w[NW];
#pragma unroll
  for (int c = 0; c < E / 8; ++c) {
    uint4 u = make_uint4(0u, 0u, 0u, 0u);
    if (c * 8 < nvalid) u = __ldg(reinterpret_cast<const uint4*>(x + m * ldx + base) + c);
    w[4 * c] = u.x; w[4 * c + 1] = u.y; w[4 * c + 2] = u.z; w[4 * c + 3] = u.w;
  }
  auto key_lo = [](uint32_t v) { return v & 0x7FFFu; };
  auto key_hi = [](uint32_t v) { return (v >> 16) & 0x7FFFu; };

  // pass 1: high 8 bits of the key
#pragma unroll
  for (int b = 0; b < B1; ++b) hist[t + NT * b] = 0u;
  __syncthreads();
#pragma unroll
  for (int j = 0; j < NW; ++j) {
    atomicAdd(&hist[(w[j] >> 7) & 0xFFu], 1u);
    atomicAdd(&hist[(w[j] >> 23) & 0xFFu], 1u);
  }
  __syncthreads();
  {
    // thread t holds bins 255 - B1 t - i, i < B1 (descending)
    uint32_t cb[B1], c = 0u;
#pragma unroll
    for (int i = 0; i < B1; ++i) { cb[i] = hist[255 - B1 * t - i]; c += cb[i]; }
    uint32_t above = block_scan<NT>(c, sums) - c;  // keys in higher bins
#pragma unroll
    for (int i = 0; i < B1; ++i) {
      if (above < static_cast<uint32_t>(k) && above + cb[i] >= static_cast<uint32_t>(k)) {
        sel[0] = 255 - B1 * t - i;
        sel[1] = above;
      }
      above += cb[i];
    }
  }
  __syncthreads();
  const uint32_t b1 = sel[0], above1 = sel[1];
  __syncthreads();

  // pass 2: low 7 bits inside bin b1
  if (t < 128) hist[t] = 0u;
  __syncthreads();
#pragma unroll
  for (int j = 0; j < NW; ++j) {
    const uint32_t lo = key_lo(w[j]), hi = key_hi(w[j]);
    if ((lo >> 7) == b1) atomicAdd(&hist[lo & 127u], 1u);
    if ((hi >> 7) == b1) atomicAdd(&hist[hi & 127u], 1u);
  }
  __syncthreads();
  {
    const uint32_t c = t < 128 ? hist[127 - t] : 0u;
    const uint32_t s = block_scan<NT>(c, sums);
    const uint32_t need = static_cast<uint32_t>(k) - above1;
    if (t < 128 && s >= need && s - c < need) {
      sel[0] = 127 - t;
      sel[1] = s - c;
    }
  }
  __syncthreads();
  const uint32_t T = (b1 << 7) | sel[0];
  const uint32_t need_eq = static_cast<uint32_t>(k) - above1 - sel[1];  // >= 1

  // keys above T are kept; keys equal to T are kept in column order until
  // k are kept (the block prefix of their counts ranks this thread's)
  uint64_t gt = 0u, eq = 0u;
  uint32_t kmax = 0u;  // the row's largest key: the largest kept one (k >= 1 here)
#pragma unroll
  for (int i = 0; i < E; ++i) {
    const uint32_t key = (i & 1) ? key_hi(w[i >> 1]) : key_lo(w[i >> 1]);
    gt |= static_cast<uint64_t>(key > T ? 1u : 0u) << i;
    eq |= static_cast<uint64_t>(key == T ? 1u : 0u) << i;
    kmax = max(kmax, key);
  }
  const uint32_t n_eq = static_cast<uint32_t>(__popcll(eq));
  const uint32_t rank = block_scan<NT>(n_eq, sums) - n_eq;  // equal keys in earlier threads
  uint64_t keep = gt;
  if (eq) {  // rare: this thread holds keys equal to T; keep its first ones
    const uint32_t take = rank < need_eq ? min(need_eq - rank, n_eq) : 0u;
    uint64_t e = eq;
    for (uint32_t j = 0; j < take; ++j) {
      keep |= e & (~e + 1u);  // lowest set bit
      e &= e - 1u;
    }
  }
  const float amax = block_max<NT>(__uint_as_float(kmax << 16), red);
  const float a = fmaxf(amax, kEps);
  const float inv = __fdiv_rn(127.f, a);
  if (t == 0) xs_out[m] = __fdiv_rn(a, 127.f);

#pragma unroll
  for (int c = 0; c < E / 8; ++c) {
    if (c * 8 < nvalid) {
      const uint32_t kb = static_cast<uint32_t>(keep >> (8 * c)) & 0xFFu;  // this group's 8 bits
      int q[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t v = w[4 * c + (i >> 1)];
        const float xv = __uint_as_float((i & 1) ? (v & 0xFFFF0000u) : (v << 16));
        q[i] = ((kb >> i) & 1u) ? quant_code(xv, inv, -128.f, 127.f) : 0;
      }
      reinterpret_cast<uint2*>(q_out + m * K + base)[c] =
          make_uint2(pack_s8x4(q[0], q[1], q[2], q[3]), pack_s8x4(q[4], q[5], q[6], q[7]));
      if (mask_out) mask_out[m * (K >> 3) + (base >> 3) + c] = static_cast<uint8_t>(kb);
    }
  }
}

cudaError_t launch_topk_i8(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, int64_t k,
                           int8_t* q, float* xs, uint8_t* mask, cudaStream_t s) {
  const int kk = static_cast<int>(k), KK = static_cast<int>(K);
  const unsigned grid = static_cast<unsigned>(M);
  auto go = [&](auto kern, int threads) {
    return launch_kernel(kern, dim3(grid), dim3(threads), 0, s, 0u, x, KK, ldx, kk, q, xs, mask);
  };
  if (K <= 8 * 128) return go(topk_i8_kernel<128, 8>, 128);
  if (K <= 16 * 128) return go(topk_i8_kernel<128, 16>, 128);
  if (K <= 32 * 128) return go(topk_i8_kernel<128, 32>, 128);
  if (K <= 32 * 256) return go(topk_i8_kernel<256, 32>, 256);
  return go(topk_i8_kernel<256, 64>, 256);
}

// ------------------------------------------------------------ KV 3-bit
// Each thread quantises 16 consecutive head dims (two 16-byte loads); the
// G = D/16 threads of one (token, head) row reduce their absmax with a
// segmented warp shuffle, so the per-row work (the shuffles, the divisions,
// the 4-bit list search) is shared by 16 elements a thread. A warp covers
// 32/G whole rows whose 3-bit streams (6 bytes per thread) form 192
// contiguous bytes, staged in shared memory and written as 48 aligned words.
// The list of 4-bit tokens is copied to shared memory once per block (up to
// kKeepSmem entries) and searched there by row ranges (token p holds rows
// [p H, p H + H)), so no division by H is needed on the 3-bit path.

// The rounding bias's share of the packed 3-bit words (fields 0..10 of the
// low word, 11..15 of the high one), modulo 2^32.
constexpr uint32_t kv3_bias(int first, int last, int base) {
  uint32_t b = 0u;
  for (int i = first; i <= last; ++i) b += 0x4B400000u << (3 * i - base);
  return b;
}
constexpr uint32_t kKv3BiasLo = kv3_bias(0, 10, 0);
constexpr uint32_t kKv3BiasHi = kv3_bias(11, 15, 32);
constexpr int kKeepSmem = 1024;
constexpr int KV_TILES = 2;  // warp tiles per warp (2 x 16-byte loads in flight per thread each)

template <int G>
__global__ void __launch_bounds__(kQuantThreads) kv_quant_kernel(
    const uint16_t* __restrict__ kv, uint32_t rows, uint32_t H, const int32_t* __restrict__ keep4,
    int n4, uint8_t* __restrict__ codes3, uint8_t* __restrict__ codes4, float* __restrict__ scale) {
  pdl_wait();  // inputs come from the previous kernel in the stream
  pdl_trigger();
  constexpr int D = 16 * G;
  constexpr int RPW = 32 / G;  // rows per warp tile
  __shared__ __align__(16) uint8_t stage[kQuantThreads / 32][192];
  __shared__ int32_t s_keep[kKeepSmem];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int n4s = n4 < kKeepSmem ? n4 : kKeepSmem;
  for (int i = threadIdx.x; i < n4s; i += kQuantThreads) s_keep[i] = __ldg(keep4 + i);
  const int g = lane % G;
  // this warp's KV_TILES consecutive warp tiles: all loads issued up front
  const uint32_t tile0 = (blockIdx.x * (kQuantThreads / 32) + wid) * KV_TILES;
  float f[KV_TILES][16];
#pragma unroll
  for (int j = 0; j < KV_TILES; ++j) {
    const uint32_t row = (tile0 + j) * RPW + lane / G;
#pragma unroll
    for (int i = 0; i < 16; ++i) f[j][i] = 0.f;
    if (row < rows) {
      const uint4* src = reinterpret_cast<const uint4*>(kv + static_cast<size_t>(row) * D) + 2 * g;
      float lo[8], hi[8];
      bf16x8_to_f32(__ldg(src), lo);
      bf16x8_to_f32(__ldg(src + 1), hi);
#pragma unroll
      for (int i = 0; i < 8; ++i) { f[j][i] = lo[i]; f[j][8 + i] = hi[i]; }
    }
  }
  __syncthreads();  // s_keep ready
#pragma unroll
  for (int j = 0; j < KV_TILES; ++j) {
    const uint32_t warp_row0 = (tile0 + j) * RPW;
    const uint32_t row = warp_row0 + lane / G;
    const bool valid = row < rows;
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(f[j][i]));
#pragma unroll
    for (int o = G / 2; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    int jk = -1;  // index of this row's token among the 4-bit tokens
    if (valid && n4 > 0) {
      // token p holds rows [p H, p H + H): compare rows, no division
      int lo = 0, hi = n4 - 1;
      while (lo <= hi) {
        const int mid = (lo + hi) >> 1;
        const uint32_t r0 = static_cast<uint32_t>(mid < kKeepSmem ? s_keep[mid] : __ldg(keep4 + mid)) * H;
        if (row >= r0 && row - r0 < H) { jk = mid; break; }
        if (r0 < row) lo = mid + 1; else hi = mid - 1;
      }
    }
    const bool four = jk >= 0;
    const float Q = four ? 7.f : 3.f;
    const float a = fmaxf(amax, kEps);
    const float inv = __fdiv_rn(Q, a);
    uint64_t pk = 0u;  // 48 bits of 3-bit codes
    if (four) {
      uint32_t q0 = 0u, q1 = 0u;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        q0 |= static_cast<uint32_t>(quant_code(f[j][i], inv, -8.f, 7.f) + 8) << (4 * i);
        q1 |= static_cast<uint32_t>(quant_code(f[j][8 + i], inv, -8.f, 7.f) + 8) << (4 * i);
      }
      const uint32_t h = row % H;
      if (valid)
        reinterpret_cast<uint2*>(codes4 + (static_cast<size_t>(jk) * H + h) * (D / 2))[g] = make_uint2(q0, q1);
    } else {
      // code + 4 comes out of the rounding itself: x * inv + (1.5 * 2^23 + 4)
      // has the bits 0x4B400000 + code + 4. Every |x * inv| <= 3 (1 + 2^-24),
      // so each code lies in [-3, 3] and needs no clamp. The biased bits,
      // shifted to their 3-bit fields, are summed modulo 2^32 (the fields do
      // not overlap) and the bias's share is removed once per word; field 10
      // straddles the two words.
      uint32_t lo = 0u, hi = 0u, r10 = 0u;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const uint32_t r = __float_as_uint(__fadd_rn(__fmul_rn(f[j][i], inv), 12582916.f));
        if (i <= 10) lo += r << (3 * i);
        else hi += r << (3 * i - 32);
        if (i == 10) r10 = r;
      }
      pk = (static_cast<uint64_t>(hi - kKv3BiasHi + ((r10 >> 2) & 1u)) << 32) | (lo - kKv3BiasLo);
    }
    const uint32_t p0 = static_cast<uint32_t>(pk), p1 = static_cast<uint32_t>(pk >> 32);
    if (valid && g == 0) scale[row] = __fdiv_rn(a, Q);
    // 6 bytes at offset 6 lane: a 4-byte and a 2-byte store in either order
    uint8_t* sp = &stage[wid][6 * lane];
    if ((lane & 1) == 0) {
      *reinterpret_cast<uint32_t*>(sp) = p0;
      *reinterpret_cast<uint16_t*>(sp + 4) = static_cast<uint16_t>(p1);
    } else {
      *reinterpret_cast<uint16_t*>(sp) = static_cast<uint16_t>(p0);
      *reinterpret_cast<uint32_t*>(sp + 2) = (p0 >> 16) | (p1 << 16);
    }
    __syncwarp();
    const int64_t rows_here = static_cast<int64_t>(rows) - warp_row0;
    const int nbytes = rows_here >= RPW ? 192 : static_cast<int>(rows_here > 0 ? rows_here : 0) * 6 * G;
    uint32_t* dst = reinterpret_cast<uint32_t*>(codes3 + static_cast<size_t>(warp_row0) * (6 * G));
    const uint32_t* src = reinterpret_cast<const uint32_t*>(stage[wid]);
    if (lane * 4 < nbytes) dst[lane] = src[lane];
    if ((lane + 32) * 4 < nbytes) dst[lane + 32] = src[lane + 32];
    __syncwarp();
  }
}

cudaError_t launch_kv_quant(const uint16_t* kv, int64_t T, int64_t H, int64_t D,
                            const int32_t* keep4, int64_t n4, uint8_t* codes3, uint8_t* codes4,
                            float* scale, cudaStream_t s) {
  const uint32_t rows = static_cast<uint32_t>(T * H);  // the entry point bounds rows * G < 2^32
  const int G = static_cast<int>(D / 16);
  const uint64_t threads = static_cast<uint64_t>(rows) * G;
  const uint64_t per_block = static_cast<uint64_t>(kQuantThreads) * KV_TILES;
  const unsigned grid = static_cast<unsigned>((threads + per_block - 1) / per_block);
  const int n = static_cast<int>(n4);
  const uint32_t h = static_cast<uint32_t>(H);
  auto go = [&](auto kern) {
    return launch_kernel(kern, dim3(grid), dim3(kQuantThreads), 0, s, 0u, kv, rows, h, keep4, n,
                         codes3, codes4, scale);
  };
  if (G == 4) return go(kv_quant_kernel<4>);
  if (G == 8) return go(kv_quant_kernel<8>);
  return go(kv_quant_kernel<16>);
}

// ------------------------------------------------ 4-bit token positions
// One block walks the token ids in chunks of 256 x 4: each thread tests its
// 4 consecutive ids against the special ids, a block prefix sum of the
// matches gives every thread its output offset, and the running total moves
// on to the next chunk, so the positions come out in increasing order.
struct SpecialIds {
  int32_t id[8];
  int n;
};

__global__ void __launch_bounds__(kQuantThreads) keep4_positions_kernel(
    const int32_t* __restrict__ ids, int64_t T, SpecialIds sp, int32_t* __restrict__ pos,
    int32_t* __restrict__ count) {
  pdl_wait();
  pdl_trigger();
  __shared__ uint32_t sums[8];
  uint32_t total = 0;
  for (int64_t base = 0; base < T; base += 4 * kQuantThreads) {
    const int64_t t0 = base + 4 * static_cast<int64_t>(threadIdx.x);
    uint32_t hit = 0u, n = 0u;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      bool m = false;
      if (t0 + i < T) {
        const int32_t v = __ldg(ids + t0 + i);
#pragma unroll
        for (int j = 0; j < 8; ++j) m |= (j < sp.n && v == sp.id[j]);
      }
      hit |= (m ? 1u : 0u) << i;
      n += m ? 1u : 0u;
    }
    const uint32_t incl = block_scan_256(n, sums);
    uint32_t o = total + incl - n;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if ((hit >> i) & 1u) pos[o++] = static_cast<int32_t>(t0 + i);
    total += sums[kQuantThreads / 32 - 1];  // the chunk's matches
    __syncthreads();                         // sums is rewritten by the next chunk
  }
  if (threadIdx.x == 0) *count = static_cast<int32_t>(total);
}

cudaError_t launch_keep4_positions(const int32_t* ids, int64_t T, const int32_t* special, int n_special,
                                   int32_t* pos, int32_t* count, cudaStream_t s) {
  SpecialIds sp{};
  for (int j = 0; j < n_special; ++j) sp.id[j] = special[j];
  sp.n = n_special;
  return launch_kernel(keep4_positions_kernel, dim3(1), dim3(kQuantThreads), 0, s, 0u, ids, T, sp,
                       pos, count);
}


}  // namespace blt
