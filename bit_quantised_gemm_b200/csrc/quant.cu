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

// Rows of up to 4096 columns: one block of NWR warps per row. Thread t
// holds the 16-byte chunks t, t + 32 NWR, t + 64 NWR, ... of the row (so each
// warp load and store is one contiguous run, and chunk order is column
// order), as packed bf16 pairs; chunks past K read as key 0 (they come last
// in column order, so they are never kept).
// The 15-bit key |x| is selected in one counting pass, not two: a shared-
// memory histogram at full key resolution over a window of W keys whose top
// is the row's largest key. With the guard bit 0x8000 set over each half's
// sign, one 32-bit subtraction gives both halves' bin numbers; a packed
// 16-bit max sends keys below the window to a per-lane slot (bins 0..31, no
// shared hot bin), a packed min sends keys above it (later windows only) to
// slots above the window. A descending scan (thread sums, block suffix scan,
// then the 4-bin groups of the crossing thread) gives the threshold key T
// and the count of keys above it. If T lies below the window the pass
// repeats over the next window down (top = the largest key below the last
// window); the window base drops by at least W a pass, so 32768 / W + 1
// passes end it.
// The keep pass compares every key with T + 1 (kept) and T (tied) by the same
// guard-bit subtraction, quantises each value (the code is the low byte of
// fl(fl(x * (127 / a)) + 1.5 * 2^23)) and zeroes the dropped codes with a
// byte mask built from the guard bits. Tied keys are kept in column order
// until k are kept: column order is (round, warp, lane) order, so a prefix
// over the warps' per-round tie counts finds the (round, warp) where the
// quota runs out, a lane prefix sum there the lane, and the threads that keep
// ties rewrite those few codes after the vector stores. When every tied key
// is kept the pass keeps keys >= T directly.
template <int W, int NWR>
struct TopkBins {
  static constexpr int kThreads = 32 * NWR;
  static constexpr int kBins = ((W + 64 + 4 * kThreads - 1) / (4 * kThreads)) * (4 * kThreads);
  static constexpr int kPerThread = kBins / kThreads;  // multiple of 4
  static constexpr int kGroups = kPerThread / 4;       // <= 32
};

template <int NWR>
__device__ __forceinline__ uint32_t block_max_u32(uint32_t v, uint32_t* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  if (NWR == 1) return v;
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  uint32_t r = red[0];
#pragma unroll
  for (int i = 1; i < NWR; ++i) r = max(r, red[i]);
  __syncthreads();  // red is reused
  return r;
}

template <int E, int W, int NWR, bool MASK>
__global__ void __launch_bounds__(32 * NWR, 32 / NWR) topk_row_kernel(
    const uint16_t* __restrict__ x, int K, int64_t ldx, int k, int8_t* __restrict__ q_out,
    float* __restrict__ xs_out, uint8_t* __restrict__ mask_out) {
  pdl_wait();  // inputs come from the previous kernel in the stream
  pdl_trigger();
  static_assert(E % 8 == 0 && E <= 64, "whole 16-byte chunks");
  constexpr int NT = 32 * NWR;
  constexpr int NC = E / 8;   // chunks (rounds) per thread
  constexpr int NW = E / 2;   // packed pairs per thread
  constexpr int NB = TopkBins<W, NWR>::kBins, PT = TopkBins<W, NWR>::kPerThread;
  constexpr int NG = TopkBins<W, NWR>::kGroups;
  static_assert(NG <= 32 && NC * NWR <= 32, "one group / one (round, warp) per lane");
  __shared__ __align__(16) uint32_t hist[NB];
  __shared__ uint32_t s_red[NWR];
  __shared__ uint32_t s_sel[4];
  __shared__ float s_inv;
  __shared__ uint32_t s_cnt[NC * NWR];  // ties per (round, warp), column order
  const int t = threadIdx.x, lane = t & 31, v = t >> 5;
  const int64_t m = blockIdx.x;
  const uint32_t hist_s = smem_u32(hist);
  uint4* my_bins = reinterpret_cast<uint4*>(hist + t * PT);
#pragma unroll
  for (int g = 0; g < PT / 4; ++g) my_bins[g] = make_uint4(0u, 0u, 0u, 0u);

  const int nchunk = K >> 3;  // valid chunks of the row
  const uint4* xr = reinterpret_cast<const uint4*>(x + m * ldx);
  uint32_t w[NW];
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    const int ch = NT * c + t;
    uint4 u = make_uint4(0u, 0u, 0u, 0u);
    if (ch < nchunk) u = __ldg(xr + ch);
    w[4 * c] = u.x; w[4 * c + 1] = u.y; w[4 * c + 2] = u.z; w[4 * c + 3] = u.w;
  }
  // the row's largest key (a NaN counts as the largest); four running maxima
  uint32_t am[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int j = 0; j < NW; ++j) am[j & 3] = absmax_bf16x2(am[j & 3], w[j]);
  const uint32_t am2 = absmax_bf16x2(absmax_bf16x2(am[0], am[1]), absmax_bf16x2(am[2], am[3]));
  // (the block maximum's barrier also orders the cleared bins before the adds)
  const uint32_t kmax = block_max_u32<NWR>(max(am2 & 0x7FFFu, (am2 >> 16) & 0x7FFFu), s_red);
  if (NWR == 1) __syncwarp();

  const uint32_t uk = static_cast<uint32_t>(k);
  uint32_t top = kmax, T = 0u, above = 0u, cnt_T = 0u;
  for (int pass = 0; pass <= 0x8000 / W; ++pass) {
    const int base = max(static_cast<int>(top) - (W - 1), 0);
    // half = 0x8000 + 32 + key - base: no borrow or carry between the halves
    // for any key <= top, and for every finite key above it
    const uint32_t sub = static_cast<uint32_t>(base - 32) * 0x10001u;
    const uint32_t slot_lo = (0x8000u + static_cast<uint32_t>(lane)) * 0x10001u;
    const uint32_t slot_hi = (0x8000u + 32u + W + static_cast<uint32_t>(lane)) * 0x10001u;
#pragma unroll
    for (int j = 0; j < NW; ++j) {
      uint32_t d = vmax_u16x2((w[j] | 0x80008000u) - sub, slot_lo);
      if (pass > 0) d = vmin_u16x2(d, slot_hi);
      red_add_shared(hist_s + ((d << 2) & 0x1FFFCu), 1u);
      red_add_shared(hist_s + ((d >> 14) & 0x1FFFCu), 1u);
    }
    __syncthreads();
    // descending scan: this thread's bins, suffix over the block, crossing thread L
    uint32_t s = 0u;
#pragma unroll
    for (int g = 0; g < PT / 4; ++g) {
      const uint4 b = my_bins[g];
      s += b.x + b.y + b.z + b.w;
    }
    uint32_t suf = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t u = __shfl_down_sync(0xffffffffu, suf, o);
      if (lane + o < 32) suf += u;
    }
    if (NWR > 1) {
      if (lane == 0) s_red[v] = suf;  // the warp's total
      __syncthreads();
#pragma unroll
      for (int i = 1; i < NWR; ++i)
        if (i > v) suf += s_red[i];
    }
    if (suf >= uk && suf - s < uk) { s_sel[0] = static_cast<uint32_t>(t); s_sel[1] = suf - s; }
    __syncthreads();
    if (v == 0) {
      // the groups of 4 bins of thread L, one per lane
      const int L = static_cast<int>(s_sel[0]);
      const uint32_t above_L = s_sel[1];
      uint4 gv = make_uint4(0u, 0u, 0u, 0u);
      if (lane < NG) gv = reinterpret_cast<const uint4*>(hist + L * PT)[lane];
      const uint32_t gsum = gv.x + gv.y + gv.z + gv.w;
      uint32_t gsuf = gsum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t u = __shfl_down_sync(0xffffffffu, gsuf, o);
        if (lane + o < 32) gsuf += u;
      }
      if (lane < NG && above_L + gsuf >= uk && above_L + gsuf - gsum < uk) {
        uint32_t c = above_L + gsuf - gsum, cnt, b;
        if (c + gv.w >= uk) { b = 3; cnt = gv.w; }
        else if (c + gv.w + gv.z >= uk) { c += gv.w; b = 2; cnt = gv.z; }
        else if (c + gv.w + gv.z + gv.y >= uk) { c += gv.w + gv.z; b = 1; cnt = gv.y; }
        else { c += gv.w + gv.z + gv.y; b = 0; cnt = gv.x; }
        s_sel[1] = c;
        s_sel[2] = static_cast<uint32_t>(L * PT + 4 * lane) + b;
        s_sel[3] = cnt;
      }
      if (pass == 0 && lane == 0) {
        // the row scale, once: the largest key is kept
        const float a = fmaxf(__uint_as_float(kmax << 16), kEps);
        s_inv = __fdiv_rn(127.f, a);
        xs_out[m] = __fdiv_rn(a, 127.f);
      }
    }
    __syncthreads();
    const int bin = static_cast<int>(s_sel[2]);
    above = s_sel[1];
    cnt_T = s_sel[3];
    if (bin >= 32 || base == 0) {  // block-uniform; base == 0: nothing lies below the window
      T = bin >= 32 ? static_cast<uint32_t>(base + bin - 32) : 0u;
      break;
    }
    // T is below the window: the next window ends at the largest key below it
    uint32_t nb = 0u;
#pragma unroll
    for (int j = 0; j < NW; ++j) {
      const uint32_t lo = w[j] & 0x7FFFu, hi = (w[j] >> 16) & 0x7FFFu;
      if (lo < static_cast<uint32_t>(base)) nb = max(nb, lo);
      if (hi < static_cast<uint32_t>(base)) nb = max(nb, hi);
    }
#pragma unroll
    for (int g = 0; g < PT / 4; ++g) my_bins[g] = make_uint4(0u, 0u, 0u, 0u);
    top = block_max_u32<NWR>(nb, s_red);  // its barrier orders the cleared bins
    if (NWR == 1) __syncwarp();
  }
  const uint32_t need_eq = uk - above;  // >= 1 of the cnt_T keys equal to T
  const bool all_ties = need_eq == cnt_T;  // block-uniform

  const float inv = s_inv;
  const uint32_t s_eq = T * 0x10001u;
  const uint32_t s_keep = all_ties ? s_eq : s_eq + 0x10001u;  // guard bit: kept without a rank
  uint32_t tie[(NC + 3) / 4], kbits[(NC + 3) / 4];  // a byte per chunk
#pragma unroll
  for (int i = 0; i < (NC + 3) / 4; ++i) { tie[i] = 0u; kbits[i] = 0u; }
  int8_t* qrow = q_out + m * K;
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    const int ch = NT * c + t;
    uint32_t code[2], tacc = 0u, kacc = 0u;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t r[4], dd[2];
#pragma unroll
      for (int p = 0; p < 2; ++p) {
        const int q = 2 * h + p;  // word within the chunk
        const uint32_t wv = w[4 * c + q];
        const uint32_t wg = wv | 0x80008000u;
        const uint32_t d = wg - s_keep;
        if (!all_ties) tacc += ((wg - s_eq) & ~d & 0x80008000u) >> (15 - 2 * q);
        if (MASK) kacc += (d & 0x80008000u) >> (15 - 2 * q);
        dd[p] = d;
        float lo = __uint_as_float(wv << 16), hi = __uint_as_float(wv & 0xFFFF0000u);
        mul_then_add_rn(lo, hi, inv, 12582912.f);
        r[2 * p] = __float_as_uint(lo);
        r[2 * p + 1] = __float_as_uint(hi);
      }
      const uint32_t packed = prmt(prmt(r[0], r[1], 0x0040u), prmt(r[2], r[3], 0x0040u), 0x5410u);
      code[h] = packed & prmt(dd[0], dd[1], 0xFDB9u);  // 0xFF where the guard bit is set
    }
    if (ch < nchunk) reinterpret_cast<uint2*>(qrow)[ch] = make_uint2(code[0], code[1]);
    // flags of word q sit at bits 2q (lo) and 16 + 2q (hi): one byte, column order
    if (!all_ties) {
      const uint32_t t8 = (tacc & 0x55u) | ((tacc >> 15) & 0xAAu);
      tie[c >> 2] |= t8 << (8 * (c & 3));
      const uint32_t n = __reduce_add_sync(0xffffffffu, __popc(t8));
      if (lane == 0) s_cnt[c * NWR + v] = n;
    }
    if (MASK) kbits[c >> 2] |= ((kacc & 0x55u) | ((kacc >> 15) & 0xAAu)) << (8 * (c & 3));
  }
  if (!all_ties) {
    __syncthreads();
    // the (round, warp) where the quota of tied keys runs out: a prefix over
    // lanes j = round * NWR + warp (column order)
    const uint32_t nj = lane < NC * NWR ? s_cnt[lane] : 0u;
    uint32_t cum = nj;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t u = __shfl_up_sync(0xffffffffu, cum, o);
      if (lane >= o) cum += u;
    }
    const int jstar = __ffs(__ballot_sync(0xffffffffu, cum >= need_eq)) - 1;  // exists: all ties counted
    const uint32_t quota = need_eq - __shfl_sync(0xffffffffu, cum - nj, jstar);
    const int cstar = jstar / NWR, vstar = jstar % NWR;
    // in that round and warp, lanes before the boundary keep all their ties, the boundary lane its first ones
    uint32_t nst = 0u;
#pragma unroll
    for (int c = 0; c < NC; ++c)
      if (c == cstar) nst = __popc((tie[c >> 2] >> (8 * (c & 3))) & 0xFFu);
    uint32_t incl = nst;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    const uint32_t before = incl - nst;
    const uint32_t take_star =
        v < vstar ? nst : (v > vstar ? 0u : (before < quota ? min(quota - before, nst) : 0u));
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      if (c > cstar) break;  // block-uniform
      uint32_t bits = (tie[c >> 2] >> (8 * (c & 3))) & 0xFFu;
      if (c == cstar) {
        uint32_t keepb = 0u, b = bits;  // the first take_star of them
        for (uint32_t i = 0; i < take_star; ++i) { keepb |= b & (~b + 1u); b &= b - 1u; }
        bits = keepb;
      }
      if (MASK) kbits[c >> 2] |= bits << (8 * (c & 3));
      const int ch = NT * c + t;
      while (bits) {
        const int i = __ffs(bits) - 1;
        bits &= bits - 1u;
        const int col = 8 * ch + i;
        const uint32_t xb = __ldg(x + m * ldx + col);
        qrow[col] = static_cast<int8_t>(quant_code(__uint_as_float(xb << 16), inv, -128.f, 127.f));
      }
    }
  }
  if (MASK) {
    uint8_t* mrow = mask_out + m * (K >> 3);
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      const int ch = NT * c + t;
      if (ch < nchunk) mrow[ch] = static_cast<uint8_t>(kbits[c >> 2] >> (8 * (c & 3)));
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
  if (K <= 4096) {
    const bool m_ = mask != nullptr;
#define BLT_TOPK_ROW(E_, W_, NWR_)                                                        \
  return m_ ? go(topk_row_kernel<E_, W_, NWR_, true>, 32 * NWR_)                         \
            : go(topk_row_kernel<E_, W_, NWR_, false>, 32 * NWR_)
    if (K <= 256) BLT_TOPK_ROW(8, 1024, 1);
    if (K <= 512) BLT_TOPK_ROW(16, 1024, 1);
    if (K <= 1024) BLT_TOPK_ROW(16, 1024, 2);
    if (K <= 2048) BLT_TOPK_ROW(32, 1024, 2);
    BLT_TOPK_ROW(64, 1024, 2);  // 2 warps of 64 columns a thread: 19.2 us against 21.1 for 4 of 32
#undef BLT_TOPK_ROW
  }
  if (K <= 32 * 256) return go(topk_i8_kernel<256, 32>, 256);
  return go(topk_i8_kernel<256, 64>, 256);
}

// ------------------------------------------------------------ KV 3-bit
// A persistent grid: each warp walks warp tiles of 32 / GP rows (2 KB: GP =
// D / 32 lanes per (token, head) row, 32 consecutive head dims a lane, four
// 16-byte loads), loading the next tile into registers before it quantises
// the current one. A row's absmax is a packed |bf16| max over the lane's
// words and a segmented warp shuffle; the codes come from an IEEE fp32
// multiply, then add (x * inv + (1.5 * 2^23 + 4) has the bits 0x4B400000 +
// code + 4), and the 32 3-bit fields of a lane (96 bits) are summed into
// three words by shifted adds, the bias's share removed once per word. A
// lane's 12 bytes start 4-byte aligned, so they are stored directly. The list
// of 4-bit tokens is copied to shared memory once per block (up to kKeepSmem
// entries) and searched there by row ranges (token p holds rows
// [p H, p H + H)), so no division by H is needed. (A ring of 16-byte
// asynchronous copies into shared memory, three tiles deep per warp, measured
// slower: 31.0 us for K and V against 19.4.)

// The rounding bias's share of fields first..last of a packed word whose bit
// 0 is field bit `base`, modulo 2^32 (every shift lies in [0, 31]).
constexpr uint32_t kv3_bias(int first, int last, int base) {
  uint32_t b = 0u;
  for (int i = first; i <= last; ++i) b += 0x4B400000u << (3 * i - base);
  return b;
}
constexpr uint32_t kKv3Bias0 = kv3_bias(0, 10, 0);    // fields 0..10 (field 10: bits 0, 1)
constexpr uint32_t kKv3Bias1 = kv3_bias(11, 21, 32);  // fields 11..21 (field 21: bit 0)
constexpr uint32_t kKv3Bias2 = kv3_bias(22, 31, 64);  // fields 22..31
constexpr int kKeepSmem = 1024;
constexpr int kKvThreads = 256;

// One launch quantises one or two tensors of the same shape (K and V of a
// layer): tile t of the 2 ntiles belongs to tensor t / ntiles.
struct KvSet {
  const uint16_t* kv;
  uint8_t* codes3;
  uint8_t* codes4;
  float* scale;
};
struct KvSets {
  KvSet s[2];
  int n;
};

template <int GP>
__global__ void __launch_bounds__(kKvThreads, 4) kv_quant_kernel(
    const KvSets sets, uint32_t rows, uint32_t H, const int32_t* __restrict__ keep4, int n4) {
  pdl_wait();  // inputs come from the previous kernel in the stream
  pdl_trigger();
  constexpr int D = 32 * GP;
  constexpr int RPT = 32 / GP;  // rows per warp tile (2 KB)
  __shared__ int32_t s_keep[kKeepSmem];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int n4s = n4 < kKeepSmem ? n4 : kKeepSmem;
  for (int i = threadIdx.x; i < n4s; i += kKvThreads) s_keep[i] = __ldg(keep4 + i);
  __syncthreads();
  const int g = lane % GP;
  const uint32_t ntiles = (rows + RPT - 1) / RPT;  // per tensor
  const uint32_t total = ntiles * static_cast<uint32_t>(sets.n);
  const uint32_t nwarps = gridDim.x * (kKvThreads / 32);

  auto load = [&](uint32_t gt, uint4 (&b)[4]) {
    const int set = gt >= ntiles ? 1 : 0;
    const uint32_t row = (gt - (set ? ntiles : 0u)) * RPT + lane / GP;
#pragma unroll
    for (int i = 0; i < 4; ++i) b[i] = make_uint4(0u, 0u, 0u, 0u);
    if (row < rows) {
      const uint16_t* kvp = set ? sets.s[1].kv : sets.s[0].kv;
      const uint4* src = reinterpret_cast<const uint4*>(kvp + static_cast<size_t>(row) * D) + 4 * g;
#pragma unroll
      for (int i = 0; i < 4; ++i) b[i] = __ldg(src + i);
    }
  };
  auto quantise = [&](uint32_t gt, const uint4 (&b)[4]) {
    const int set = gt >= ntiles ? 1 : 0;
    uint8_t* __restrict__ codes3 = set ? sets.s[1].codes3 : sets.s[0].codes3;
    uint8_t* __restrict__ codes4 = set ? sets.s[1].codes4 : sets.s[0].codes4;
    float* __restrict__ scale = set ? sets.s[1].scale : sets.s[0].scale;
    const uint32_t row = (gt - (set ? ntiles : 0u)) * RPT + lane / GP;
    const bool valid = row < rows;
    const uint32_t w[16] = {b[0].x, b[0].y, b[0].z, b[0].w, b[1].x, b[1].y, b[1].z, b[1].w,
                            b[2].x, b[2].y, b[2].z, b[2].w, b[3].x, b[3].y, b[3].z, b[3].w};
    uint32_t am[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int j = 0; j < 16; ++j) am[j & 3] = absmax_bf16x2(am[j & 3], w[j]);
    const uint32_t am2 = absmax_bf16x2(absmax_bf16x2(am[0], am[1]), absmax_bf16x2(am[2], am[3]));
    uint32_t key = max(am2 & 0x7FFFu, (am2 >> 16) & 0x7FFFu);
#pragma unroll
    for (int o = GP / 2; o > 0; o >>= 1) key = max(key, __shfl_xor_sync(0xffffffffu, key, o));
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
    const float a = fmaxf(__uint_as_float(key << 16), kEps);
    const float inv = __fdiv_rn(Q, a);
    if (valid && g == 0) scale[row] = __fdiv_rn(a, Q);
    uint32_t p0 = 0u, p1 = 0u, p2 = 0u;  // a 4-bit row keeps zeros in the 3-bit store
    if (!four) {
      // |x * inv| <= 3 (1 + 2^-24): every code lies in [-3, 3], no clamp
      uint32_t r10 = 0u, r21 = 0u;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        float lo = __uint_as_float(w[j] << 16), hi = __uint_as_float(w[j] & 0xFFFF0000u);
        mul_then_add_rn(lo, hi, inv, 12582916.f);
        const uint32_t r[2] = {__float_as_uint(lo), __float_as_uint(hi)};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int i = 2 * j + h;
          if (i <= 10) p0 += r[h] << (3 * i);
          else if (i <= 21) p1 += r[h] << (3 * i - 32);
          else p2 += r[h] << (3 * i - 64);
          if (i == 10) r10 = r[h];
          if (i == 21) r21 = r[h];
        }
      }
      p0 -= kKv3Bias0;
      p1 = p1 - kKv3Bias1 + ((r10 >> 2) & 1u);
      p2 = p2 - kKv3Bias2 + ((r21 >> 1) & 3u);
    } else {
      uint32_t q[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        q[t] = 0u;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t v = w[4 * t + (i >> 1)];
          const float xv = __uint_as_float((i & 1) ? (v & 0xFFFF0000u) : (v << 16));
          q[t] |= static_cast<uint32_t>(quant_code(xv, inv, -8.f, 7.f) + 8) << (4 * i);
        }
      }
      const uint32_t h = row % H;
      reinterpret_cast<uint4*>(codes4 + (static_cast<size_t>(jk) * H + h) * (D / 2))[g] =
          make_uint4(q[0], q[1], q[2], q[3]);
    }
    if (valid) {
      uint32_t* dst = reinterpret_cast<uint32_t*>(codes3 + static_cast<size_t>(row) * (3 * D / 8) + 12 * g);
      dst[0] = p0; dst[1] = p1; dst[2] = p2;
    }
  };

  uint32_t tile = blockIdx.x * (kKvThreads / 32) + wid;
  uint4 A[4], B[4];
  if (tile < total) load(tile, A);
  while (tile < total) {
    uint32_t nt = tile + nwarps;
    if (nt < total) load(nt, B);
    quantise(tile, A);
    tile = nt;
    if (tile >= total) break;
    nt = tile + nwarps;
    if (nt < total) load(nt, A);
    quantise(tile, B);
    tile = nt;
  }
}

static cudaError_t launch_kv_sets(const KvSets& sets, int64_t T, int64_t H, int64_t D, const int32_t* keep4,
                                  int64_t n4, cudaStream_t s) {
  const uint32_t rows = static_cast<uint32_t>(T * H);  // the entry point bounds rows * D / 8 < 2^32
  const int GP = static_cast<int>(D / 32);
  const uint64_t tiles = static_cast<uint64_t>(sets.n) * ((static_cast<uint64_t>(rows) * GP + 31) / 32);
  const int n = static_cast<int>(n4);
  const uint32_t h = static_cast<uint32_t>(H);
  auto go = [&](auto kern) {
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kKvThreads, 0);
    if (e != cudaSuccess) return e;
    const uint64_t want = (tiles + kKvThreads / 32 - 1) / (kKvThreads / 32);
    const uint64_t cap = static_cast<uint64_t>(num_sms()) * static_cast<uint64_t>(per_sm > 0 ? per_sm : 1);
    const unsigned grid = static_cast<unsigned>(want < cap ? want : cap);
    return launch_kernel(kern, dim3(grid), dim3(kKvThreads), 0, s, 0u, sets, rows, h, keep4, n);
  };
  if (GP == 2) return go(kv_quant_kernel<2>);
  if (GP == 4) return go(kv_quant_kernel<4>);
  return go(kv_quant_kernel<8>);
}

cudaError_t launch_kv_quant(const uint16_t* kv, int64_t T, int64_t H, int64_t D,
                            const int32_t* keep4, int64_t n4, uint8_t* codes3, uint8_t* codes4,
                            float* scale, cudaStream_t s) {
  KvSets sets{};
  sets.s[0] = KvSet{kv, codes3, codes4, scale};
  sets.s[1] = sets.s[0];
  sets.n = 1;
  return launch_kv_sets(sets, T, H, D, keep4, n4, s);
}

cudaError_t launch_kv_quant_pair(const uint16_t* k, const uint16_t* v, int64_t T, int64_t H, int64_t D,
                                 const int32_t* keep4, int64_t n4, uint8_t* k3, uint8_t* k4, float* ks,
                                 uint8_t* v3, uint8_t* v4, float* vs, cudaStream_t s) {
  KvSets sets{};
  sets.s[0] = KvSet{k, k3, k4, ks};
  sets.s[1] = KvSet{v, v3, v4, vs};
  sets.n = 2;
  return launch_kv_sets(sets, T, H, D, keep4, n4, s);
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
