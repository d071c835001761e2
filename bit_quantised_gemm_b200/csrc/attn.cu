// Decode attention over the 3-bit KV cache written by kv_quant_3bit.
//
// For every query (b, h) and every cached token t of head h:
//   s_t = (q . k_t) / sqrt(D),  p = softmax_t(s),  o = sum_t p_t v_t
// with k_t, v_t the dequantised cache rows ((code - 4) * scale, or
// (code - 8) * scale for the tokens kept at 4 bits). The cache is read once,
// straight from its packed form: nothing is expanded in HBM.
//
// Work split ("split-T"): a cluster of S CTAs owns one head and one group of
// up to BG queries; CTA r of the cluster walks tokens [T r / S, T (r+1) / S)
// in tiles of 128 with an online softmax (running max m, running sum l and
// the running weighted value sum o per query), and the S partial results are
// merged through distributed shared memory by cluster rank 0, so no global
// scratch is needed. Within a tile:
//   * thread i owns token i: it loads the token's packed K row (3D/8 bytes,
//     8-byte loads) and its scale, and forms s_b for every query b against
//     the queries held in shared memory (broadcast reads); the codes become
//     floats with one OR and one subtract (2^23 + code trick);
//   * the block reduces the tile maximum and the sum of exp per query;
//   * the V rows of the tile are staged in shared memory; thread d then
//     accumulates dimension d over the tile's tokens.
#include <cmath>

#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace blt {
namespace attn {

constexpr int TT = 128;             // tokens per tile = threads per CTA
constexpr int MAX_BG = 8;           // queries per CTA
constexpr int MAX_KEEP = 1024;      // 4-bit token list held in shared memory

struct Params {
  const uint16_t* q;                // bf16 [B x H x D]
  const uint8_t* k3; const uint8_t* k4; const float* ks;
  const uint8_t* v3; const uint8_t* v4; const float* vs;
  const int32_t* keep4;
  int n4;
  int B, H, T;
  float qk_scale;                   // 1 / sqrt(D)
  uint16_t* out;                    // bf16 [B x H x D]
};

__device__ __forceinline__ float ld_dsmem_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

// code d of a little-endian 3-bit stream held in 32-bit words, minus 4, as
// a float: (2^23 | code) - (2^23 + 4).
template <int NW>
__device__ __forceinline__ float code3f(const uint32_t (&w)[NW], int d) {
  const int bit = 3 * d, i = bit >> 5, sh = bit & 31;
  uint32_t v = w[i] >> sh;
  if (sh > 29) v |= w[i + 1] << (32 - sh);
  return __int_as_float(static_cast<int>((v & 7u) | 0x4B000000u)) - 8388612.f;
}

// code d of a 4-bit row (low nibble first), minus 8, as a float.
__device__ __forceinline__ float code4f(const uint8_t* row, int d) {
  const uint32_t b = row[d >> 1];
  const uint32_t c = (d & 1) ? (b >> 4) : (b & 15u);
  return __int_as_float(static_cast<int>(c | 0x4B000000u)) - 8388616.f;
}

// index of token t in the sorted 4-bit list, or -1
__device__ __forceinline__ int keep_index(const int32_t* list, int n, int t) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (list[mid] < t) lo = mid + 1; else hi = mid;
  }
  return (lo < n && list[lo] == t) ? lo : -1;
}

template <int D, int BG>
__global__ void __launch_bounds__(TT)
kv_attention_kernel(const Params p) {
  constexpr int RB = 3 * D / 8;     // packed 3-bit row bytes
  constexpr int NW = RB / 4;        // ... in 32-bit words
  constexpr int DPT = D / TT > 0 ? D / TT : 1;  // value dims per thread (D = 256: 2)
  __shared__ float qs[BG][D];       // queries, pre-scaled by 1/sqrt(D)
  __shared__ float pv[BG][TT];      // softmax weight x value scale of the tile's tokens
  __shared__ __align__(16) uint32_t vrow[TT][NW + 1];  // the tile's packed V rows (padded)
  __shared__ int vkeep[TT];         // 4-bit list index of the tile's tokens, or -1
  __shared__ float red[TT / 32][BG];
  __shared__ float stat[2][BG];     // tile max / sum broadcast
  __shared__ int32_t s_keep[MAX_KEEP];
  __shared__ float part_m[BG], part_l[BG];
  __shared__ float part_o[BG][D];

  pdl_wait();  // the queries and the cache come from earlier kernels
  pdl_trigger();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t rank = cluster_ctarank();
  const int S = static_cast<int>(gridDim.x);
  const int h = blockIdx.y;
  const int b0 = blockIdx.z * BG;
  const int nb = min(BG, p.B - b0);
  const int t_begin = static_cast<int>((static_cast<int64_t>(p.T) * rank) / S);
  const int t_end = static_cast<int>((static_cast<int64_t>(p.T) * (rank + 1)) / S);
  const int n4 = min(p.n4, MAX_KEEP);

  for (int i = tid; i < n4; i += TT) s_keep[i] = __ldg(p.keep4 + i);
  for (int i = tid; i < BG * D; i += TT) {
    const int b = i / D, d = i - b * D;
    float v = 0.f;
    if (b < nb) {
      const uint16_t bits = __ldg(p.q + (static_cast<int64_t>(b0 + b) * p.H + h) * D + d);
      v = __fmul_rn(__uint_as_float(static_cast<uint32_t>(bits) << 16), p.qk_scale);
    }
    qs[b][d] = v;
  }
  __syncthreads();

  float m_run[BG], l_run[BG], o_run[BG][DPT];
#pragma unroll
  for (int b = 0; b < BG; ++b) {
    m_run[b] = -INFINITY;
    l_run[b] = 0.f;
#pragma unroll
    for (int j = 0; j < DPT; ++j) o_run[b][j] = 0.f;
  }

  for (int t0 = t_begin; t0 < t_end; t0 += TT) {
    // ---- scores: thread tid owns token t
    const int t = t0 + tid;
    const bool valid = t < t_end;
    float s[BG];
    int kj = -1;
    float vsc = 0.f;
    if (valid) {
      const int64_t row = static_cast<int64_t>(t) * p.H + h;
      kj = n4 > 0 ? keep_index(s_keep, n4, t) : -1;
      const float ksc = __ldg(p.ks + row);
      vsc = __ldg(p.vs + row);
      float acc[BG];
#pragma unroll
      for (int b = 0; b < BG; ++b) acc[b] = 0.f;
      if (kj < 0) {
        uint32_t w[NW + 1];
        const uint2* src = reinterpret_cast<const uint2*>(p.k3 + row * RB);
#pragma unroll
        for (int i = 0; i < NW / 2; ++i) {
          const uint2 u = __ldg(src + i);
          w[2 * i] = u.x;
          w[2 * i + 1] = u.y;
        }
        w[NW] = 0u;
#pragma unroll
        for (int d = 0; d < D; ++d) {
          const float c = code3f(w, d);
#pragma unroll
          for (int b = 0; b < BG; ++b) acc[b] = fmaf(qs[b][d], c, acc[b]);
        }
        // the V row of this token, for the value pass
        const uint2* vsrc = reinterpret_cast<const uint2*>(p.v3 + row * RB);
#pragma unroll
        for (int i = 0; i < NW / 2; ++i) {
          const uint2 u = __ldg(vsrc + i);
          vrow[tid][2 * i] = u.x;
          vrow[tid][2 * i + 1] = u.y;
        }
        vrow[tid][NW] = 0u;
      } else {
        const uint8_t* k4row = p.k4 + (static_cast<int64_t>(kj) * p.H + h) * (D / 2);
        for (int d = 0; d < D; ++d) {
          const float c = code4f(k4row, d);
#pragma unroll
          for (int b = 0; b < BG; ++b) acc[b] = fmaf(qs[b][d], c, acc[b]);
        }
      }
#pragma unroll
      for (int b = 0; b < BG; ++b) s[b] = __fmul_rn(acc[b], ksc);
    } else {
#pragma unroll
      for (int b = 0; b < BG; ++b) s[b] = -INFINITY;
    }
    vkeep[tid] = valid ? kj : -2;  // -2: no token

    // ---- tile maximum per query
#pragma unroll
    for (int b = 0; b < BG; ++b) {
      float v = s[b];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
      if (lane == 0) red[warp][b] = v;
    }
    __syncthreads();
    if (tid < BG) {
      float v = red[0][tid];
#pragma unroll
      for (int w = 1; w < TT / 32; ++w) v = fmaxf(v, red[w][tid]);
      stat[0][tid] = v;
    }
    __syncthreads();
    float m_new[BG], corr[BG];
#pragma unroll
    for (int b = 0; b < BG; ++b) {
      m_new[b] = fmaxf(m_run[b], stat[0][b]);
      corr[b] = expf(m_run[b] - m_new[b]);  // 0 on the first tile (m_run = -inf)
      const float e = valid ? expf(s[b] - m_new[b]) : 0.f;
      pv[b][tid] = __fmul_rn(e, vsc);
      float v = e;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
      if (lane == 0) red[warp][b] = v;
    }
    __syncthreads();
    if (tid < BG) {
      float v = red[0][tid];
#pragma unroll
      for (int w = 1; w < TT / 32; ++w) v += red[w][tid];
      stat[1][tid] = v;
    }
    __syncthreads();
#pragma unroll
    for (int b = 0; b < BG; ++b) {
      l_run[b] = fmaf(l_run[b], corr[b], stat[1][b]);
      m_run[b] = m_new[b];
    }

    // ---- values: thread tid owns dimensions d = tid + TT j
    const int ntok = min(TT, t_end - t0);
#pragma unroll
    for (int j = 0; j < DPT; ++j) {
      const int d = tid + TT * j;
      if (d >= D) break;
      float acc[BG];
#pragma unroll
      for (int b = 0; b < BG; ++b) acc[b] = 0.f;
      const int bit = 3 * d, wi = bit >> 5, sh = bit & 31;
      for (int i = 0; i < ntok; ++i) {
        float c;
        const int kk = vkeep[i];
        if (kk < 0) {
          uint32_t v = vrow[i][wi] >> sh;
          if (sh > 29) v |= vrow[i][wi + 1] << (32 - sh);
          c = __int_as_float(static_cast<int>((v & 7u) | 0x4B000000u)) - 8388612.f;
        } else {
          c = code4f(p.v4 + (static_cast<int64_t>(kk) * p.H + h) * (D / 2), d);
        }
#pragma unroll
        for (int b = 0; b < BG; ++b) acc[b] = fmaf(pv[b][i], c, acc[b]);
      }
#pragma unroll
      for (int b = 0; b < BG; ++b) o_run[b][j] = fmaf(o_run[b][j], corr[b], acc[b]);
    }
    __syncthreads();  // the tile's shared rows are reused by the next tile
  }

  // ---- merge the S partial results on cluster rank 0
  // every thread holds the same m_run / l_run; thread b publishes query b
#pragma unroll
  for (int b = 0; b < BG; ++b)
    if (tid == b) { part_m[b] = m_run[b]; part_l[b] = l_run[b]; }
#pragma unroll
  for (int b = 0; b < BG; ++b)
#pragma unroll
    for (int j = 0; j < DPT; ++j)
      if (tid + TT * j < D) part_o[b][tid + TT * j] = o_run[b][j];
  cluster_sync();
  if (rank == 0) {
    for (int i = tid; i < nb * D; i += TT) {
      const int b = i / D, d = i - b * D;
      float M = -INFINITY;
      for (int r = 0; r < S; ++r)
        M = fmaxf(M, ld_dsmem_f32(map_shared_rank(smem_u32(&part_m[b]), r)));
      float num = 0.f, den = 0.f;
      for (int r = 0; r < S; ++r) {
        const float mr = ld_dsmem_f32(map_shared_rank(smem_u32(&part_m[b]), r));
        const float w = mr == -INFINITY ? 0.f : expf(mr - M);
        den = fmaf(w, ld_dsmem_f32(map_shared_rank(smem_u32(&part_l[b]), r)), den);
        num = fmaf(w, ld_dsmem_f32(map_shared_rank(smem_u32(&part_o[b][d]), r)), num);
      }
      p.out[(static_cast<int64_t>(b0 + b) * p.H + h) * D + d] =
          __bfloat16_as_ushort(__float2bfloat16_rn(num / den));
    }
  }
  cluster_sync();  // peers keep their shared memory until rank 0 is done
}

}  // namespace attn

template <int D, int BG>
static cudaError_t launch_attn_t(const attn::Params& p, int S, cudaStream_t s) {
  const dim3 grid(static_cast<unsigned>(S), static_cast<unsigned>(p.H),
                  static_cast<unsigned>((p.B + BG - 1) / BG));
  return launch_kernel(attn::kv_attention_kernel<D, BG>, grid, dim3(attn::TT), 0, s,
                       static_cast<unsigned>(S), p);
}

cudaError_t launch_kv_attention(const uint16_t* q, int64_t B, int64_t H, int64_t D, int64_t T,
                                const uint8_t* k3, const uint8_t* k4, const float* ks,
                                const uint8_t* v3, const uint8_t* v4, const float* vs,
                                const int32_t* keep4, int64_t n4, uint16_t* out, cudaStream_t s) {
  attn::Params p{};
  p.q = q;
  p.k3 = k3; p.k4 = k4; p.ks = ks;
  p.v3 = v3; p.v4 = v4; p.vs = vs;
  p.keep4 = keep4;
  p.n4 = static_cast<int>(n4);
  p.B = static_cast<int>(B);
  p.H = static_cast<int>(H);
  p.T = static_cast<int>(T);
  p.qk_scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
  p.out = out;
  const int BG = B == 1 ? 1 : attn::MAX_BG;
  const int64_t ctas = H * ((B + BG - 1) / BG);
  // split T over a cluster until the grid fills the SMs (and each CTA keeps a full tile)
  int S = 1;
  while (S < 8 && ctas * S * 2 <= 2 * num_sms() && T / (2 * S) >= attn::TT) S *= 2;
  if (D == 64) return BG == 1 ? launch_attn_t<64, 1>(p, S, s) : launch_attn_t<64, 8>(p, S, s);
  if (D == 128) return BG == 1 ? launch_attn_t<128, 1>(p, S, s) : launch_attn_t<128, 8>(p, S, s);
  return BG == 1 ? launch_attn_t<256, 1>(p, S, s) : launch_attn_t<256, 8>(p, S, s);
}

}  // namespace blt
