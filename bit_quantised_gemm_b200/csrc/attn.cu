// Decode attention over the 3-bit KV cache written by kv_quant_3bit.
//
// For every query (b, h) and every cached token t of head h:
//   s_t = (q . k_t) / sqrt(D),  p = softmax_t(s),  o = sum_t p_t v_t
// with k_t, v_t the dequantised cache rows ((code - 4) * scale, or
// (code - 8) * scale for the tokens kept at 4 bits). The cache is read once,
// straight from its packed form: nothing is expanded in HBM.
//
// Work split ("split-T"): a cluster of S CTAs owns one head and one group of
// queries; CTA r of the cluster walks tokens [T r / S, T (r+1) / S) in tiles
// with an online softmax (running max m, running sum l and the running
// weighted value sum o per query), and the S partial results are merged
// through distributed shared memory by cluster rank 0, so no global scratch
// is needed. The rows of one head are 3D/8 bytes every H * 3D/8 bytes in the
// cache, so each tile's K rows, V rows and their scales arrive by TMA (2-D
// boxes, one row per token) into a ring of stages: the next tiles are in
// flight while the current one is computed.
//
// D = 128 (`kv_attention_mma_kernel`, below): both products on the warp-level
// bf16 tensor-core MMA, 4 or 8 queries per cluster.
//
// Other head dimensions (`kv_attention_kernel`): 256-token tiles, one CTA of
// 256 threads, up to 8 queries per cluster. Within a tile:
//   * thread i owns token i: it reads the token's packed K row from shared
//     memory and forms s_b for every query b against the queries held in
//     shared memory (broadcast reads); codes become floats with one OR and
//     one subtract (2^23 + code trick);
//   * the block reduces the tile maximum and the sum of exp per query;
//   * thread (half, d) accumulates dimension d over half of the tile's
//     tokens straight from the staged V rows; the halves meet in shared memory.
#include <cmath>

#include <cuda_bf16.h>

#include "common.cuh"
#include "launch.h"
#include "ptx.cuh"

namespace blt {
namespace attn {

constexpr int TT = 256;             // tokens per tile = threads per CTA
constexpr int VT = 128;             // threads per half in the value pass
constexpr int NS = 2;               // tile stages
constexpr int MAX_BG = 8;           // queries per CTA
constexpr int MAX_KEEP = 1024;      // 4-bit token list held in shared memory

struct Params {
  const uint16_t* q;                // bf16 [B x H x D]
  const uint8_t* k4; const uint8_t* v4;  // 4-bit rows [n4 x H x D/2]
  const int32_t* keep4;
  int n4;
  int B, H, T;
  float qk_scale;                   // 1 / sqrt(D)
  const float* ks; const float* vs; // scales [T x H]
  uint16_t* out;                    // bf16 [B x H x D]
  int* status;
  uint64_t timeout_ns;
};

template <int D, int BG>
struct Smem {
  static constexpr int RB = 3 * D / 8;   // packed 3-bit row bytes
  uint8_t krow[NS][TT][RB];         // staged K rows of the tile (TMA)
  uint8_t vrow[NS][TT][RB];         // staged V rows
  float ksc[NS][TT][4];             // scales of the 4-head group holding h
  float vsc[NS][TT][4];
  float qs[BG][D];                  // queries, pre-scaled by 1/sqrt(D)
  float pv[BG][TT];                 // softmax weight x value scale of the tile's tokens
  int k4_tok[TT];                   // the tile's 4-bit tokens: list index ...
  float k4_w[BG][TT];               // ... and softmax weight x value scale
  float red[TT / 32][BG];
  float stat[2][BG];                // tile max / sum broadcast
  int32_t s_keep[MAX_KEEP];
  float part_m[BG], part_l[BG];
  float part_o[BG][D];
  float vpart[BG][D];               // second half of the value pass
  uint64_t full[NS];
  int k4_n;
};

__device__ __forceinline__ void st_dsmem_f32(uint32_t addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

__device__ __forceinline__ void st_dsmem_v4f32(uint32_t addr, float4 v) {
  asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
               : "memory");
}

__device__ __forceinline__ float ld_dsmem_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

// The merged output of one (query, dim) from the S partial results of a
// cluster (S <= 16): every rank's m, l and o come through distributed shared
// memory, all loads issued before any is used (one round trip, not 3 S).
__device__ __forceinline__ float merge_partials(int S, uint32_t m_addr, uint32_t l_addr, uint32_t o_addr) {
  float mr[16], lr[16], orr[16];
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    mr[r] = -INFINITY; lr[r] = 0.f; orr[r] = 0.f;
    if (r < S) {
      mr[r] = ld_dsmem_f32(map_shared_rank(m_addr, static_cast<uint32_t>(r)));
      lr[r] = ld_dsmem_f32(map_shared_rank(l_addr, static_cast<uint32_t>(r)));
      orr[r] = ld_dsmem_f32(map_shared_rank(o_addr, static_cast<uint32_t>(r)));
    }
  }
  float M = -INFINITY;
#pragma unroll
  for (int r = 0; r < 16; ++r) M = fmaxf(M, mr[r]);
  float num = 0.f, den = 0.f;
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    const float w = mr[r] == -INFINITY ? 0.f : expf(mr[r] - M);
    den = fmaf(w, lr[r], den);
    num = fmaf(w, orr[r], num);
  }
  return num / den;
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
kv_attention_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmKs, const __grid_constant__ CUtensorMap tmVs,
                    const Params p) {
  using SM = Smem<D, BG>;
  constexpr int RB = SM::RB;
  constexpr int NW = RB / 4;        // packed row in 32-bit words
  constexpr int DPT = D / VT;       // value dims per thread
  constexpr uint32_t STAGE_TX = 2 * TT * RB + 2 * TT * 16;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  SM& sm = *reinterpret_cast<SM*>(smem_raw);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t rank = cluster_ctarank();
  const int S = static_cast<int>(gridDim.x);
  const int h = blockIdx.y;
  const int h4 = h & ~3, hl = h & 3;
  const int b0 = blockIdx.z * BG;
  const int nb = min(BG, p.B - b0);
  const int t_begin = static_cast<int>((static_cast<int64_t>(p.T) * rank) / S);
  const int t_end = static_cast<int>((static_cast<int64_t>(p.T) * (rank + 1)) / S);
  const int n_tiles = (t_end - t_begin + TT - 1) / TT;
  const int n4 = min(p.n4, MAX_KEEP);

  if (tid == 0) {
    for (int i = 0; i < NS; ++i) mbar_init(&sm.full[i], 1);
    fence_mbar_init();
  }
  __syncthreads();
  pdl_wait();  // the queries and the cache come from earlier kernels
  pdl_trigger();
  auto issue = [&](int k) {  // thread 0: tile k into stage k % NS
    const int st = k % NS, t0 = t_begin + k * TT;
    mbar_arrive_expect_tx(&sm.full[st], STAGE_TX);
    tma_load_2d(&sm.krow[st][0][0], &tmK, &sm.full[st], h * RB, t0);
    tma_load_2d(&sm.vrow[st][0][0], &tmV, &sm.full[st], h * RB, t0);
    tma_load_2d(&sm.ksc[st][0][0], &tmKs, &sm.full[st], h4, t0);
    tma_load_2d(&sm.vsc[st][0][0], &tmVs, &sm.full[st], h4, t0);
  };
  if (tid == 0)
    for (int k = 0; k < min(NS, n_tiles); ++k) issue(k);

  for (int i = tid; i < n4; i += TT) sm.s_keep[i] = __ldg(p.keep4 + i);
  for (int i = tid; i < BG * D; i += TT) {
    const int b = i / D, d = i - b * D;
    float v = 0.f;
    if (b < nb) {
      const uint16_t bits = __ldg(p.q + (static_cast<int64_t>(b0 + b) * p.H + h) * D + d);
      v = __fmul_rn(__uint_as_float(static_cast<uint32_t>(bits) << 16), p.qk_scale);
    }
    sm.qs[b][d] = v;
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

  bool ok = true;
  int k = 0;
  for (; k < n_tiles; ++k) {
    const int st = k % NS, t0 = t_begin + k * TT;
    if (!mbar_wait(&sm.full[st], (k / NS) & 1, p.timeout_ns, nullptr)) ok = false;
    if (__syncthreads_or(!ok)) { ok = false; break; }  // the whole block leaves together
    // ---- scores: thread tid owns token t
    const int t = t0 + tid;
    const bool valid = t < t_end;
    const int kj = (valid && n4 > 0) ? keep_index(sm.s_keep, n4, t) : -1;
    const float vsc = sm.vsc[st][tid][hl];
    float s[BG];
    if (valid) {
      float acc[BG][4];  // four independent chains per query
#pragma unroll
      for (int b = 0; b < BG; ++b)
#pragma unroll
        for (int u = 0; u < 4; ++u) acc[b][u] = 0.f;
      if (kj < 0) {
        uint32_t w[NW + 1];
        const uint2* src = reinterpret_cast<const uint2*>(&sm.krow[st][tid][0]);
#pragma unroll
        for (int i = 0; i < NW / 2; ++i) {
          const uint2 u = src[i];
          w[2 * i] = u.x;
          w[2 * i + 1] = u.y;
        }
        w[NW] = 0u;
#pragma unroll
        for (int d = 0; d < D; ++d) {
          const float c = code3f(w, d);
#pragma unroll
          for (int b = 0; b < BG; ++b) acc[b][d & 3] = fmaf(sm.qs[b][d], c, acc[b][d & 3]);
        }
      } else {
        const uint8_t* k4row = p.k4 + (static_cast<int64_t>(kj) * p.H + h) * (D / 2);
        for (int d = 0; d < D; ++d) {
          const float c = code4f(k4row, d);
#pragma unroll
          for (int b = 0; b < BG; ++b) acc[b][d & 3] = fmaf(sm.qs[b][d], c, acc[b][d & 3]);
        }
      }
      const float ksc = sm.ksc[st][tid][hl];
#pragma unroll
      for (int b = 0; b < BG; ++b)
        s[b] = __fmul_rn((acc[b][0] + acc[b][1]) + (acc[b][2] + acc[b][3]), ksc);
    } else {
#pragma unroll
      for (int b = 0; b < BG; ++b) s[b] = -INFINITY;
    }
    if (tid == 0) sm.k4_n = 0;

    // ---- tile maximum per query
#pragma unroll
    for (int b = 0; b < BG; ++b) {
      float v = s[b];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
      if (lane == 0) sm.red[warp][b] = v;
    }
    __syncthreads();
    if (tid < BG) {
      float v = sm.red[0][tid];
#pragma unroll
      for (int w = 1; w < TT / 32; ++w) v = fmaxf(v, sm.red[w][tid]);
      sm.stat[0][tid] = v;
    }
    __syncthreads();
    float m_new[BG], corr[BG];
#pragma unroll
    for (int b = 0; b < BG; ++b) {
      m_new[b] = fmaxf(m_run[b], sm.stat[0][b]);
      corr[b] = expf(m_run[b] - m_new[b]);  // 0 on the first tile (m_run = -inf)
      const float e = valid ? expf(s[b] - m_new[b]) : 0.f;
      // absent and 4-bit tokens weigh nothing in the 3-bit value pass
      sm.pv[b][tid] = kj < 0 ? __fmul_rn(e, vsc) : 0.f;
      s[b] = __fmul_rn(e, vsc);  // kept for a 4-bit token below
      float v = e;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
      if (lane == 0) sm.red[warp][b] = v;
    }
    __syncthreads();
    if (tid < BG) {
      float v = sm.red[0][tid];
#pragma unroll
      for (int w = 1; w < TT / 32; ++w) v += sm.red[w][tid];
      sm.stat[1][tid] = v;
    }
    if (kj >= 0) {  // a 4-bit token of this tile (rare): its own list for the value pass
      const int slot = atomicAdd(&sm.k4_n, 1);
      sm.k4_tok[slot] = kj;
#pragma unroll
      for (int b = 0; b < BG; ++b) sm.k4_w[b][slot] = s[b];
    }
    __syncthreads();
#pragma unroll
    for (int b = 0; b < BG; ++b) {
      l_run[b] = fmaf(l_run[b], corr[b], sm.stat[1][b]);
      m_run[b] = m_new[b];
    }

    // ---- values: thread tid owns dimensions d = dl + VT j of one half of the
    // tile's tokens (half = tid / VT), read straight from the staged rows
    // (rows with weight 0 add nothing), with four independent chains.
    const int nk4 = sm.k4_n;
    const int half = tid / VT, dl = tid % VT;
    float vsum[BG][DPT];
#pragma unroll
    for (int j = 0; j < DPT; ++j) {
      const int d = dl + VT * j;
      float acc[BG][4];
#pragma unroll
      for (int b = 0; b < BG; ++b)
#pragma unroll
        for (int u = 0; u < 4; ++u) acc[b][u] = 0.f;
      const int bit = 3 * d, wi = bit >> 5, sh = bit & 31;
      const int i0 = half * VT;
      const uint8_t* vbase = &sm.vrow[st][0][0];
#pragma unroll 4
      for (int i = i0; i < i0 + VT; i += 4) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t* row = reinterpret_cast<const uint32_t*>(vbase + (i + u) * RB);
          uint32_t v = row[wi] >> sh;
          if (sh > 29) v |= row[wi + 1] << (32 - sh);
          const float c = __int_as_float(static_cast<int>((v & 7u) | 0x4B000000u)) - 8388612.f;
#pragma unroll
          for (int b = 0; b < BG; ++b) acc[b][u] = fmaf(sm.pv[b][i + u], c, acc[b][u]);
        }
      }
      for (int kk = half; kk < nk4; kk += 2) {
        const float c = code4f(p.v4 + (static_cast<int64_t>(sm.k4_tok[kk]) * p.H + h) * (D / 2), d);
#pragma unroll
        for (int b = 0; b < BG; ++b) acc[b][0] = fmaf(sm.k4_w[b][kk], c, acc[b][0]);
      }
#pragma unroll
      for (int b = 0; b < BG; ++b) vsum[b][j] = (acc[b][0] + acc[b][1]) + (acc[b][2] + acc[b][3]);
    }
    if (half == 1) {
#pragma unroll
      for (int j = 0; j < DPT; ++j)
#pragma unroll
        for (int b = 0; b < BG; ++b) sm.vpart[b][dl + VT * j] = vsum[b][j];
    }
    __syncthreads();  // every thread is done with stage st; the halves meet
    if (half == 0) {
#pragma unroll
      for (int j = 0; j < DPT; ++j)
#pragma unroll
        for (int b = 0; b < BG; ++b)
          o_run[b][j] = fmaf(o_run[b][j], corr[b], vsum[b][j] + sm.vpart[b][dl + VT * j]);
    }
    if (tid == 0 && k + NS < n_tiles) issue(k + NS);  // refill the stage just read
  }
  if (!ok) {
    report_status(p.status, BITLINEAR_STATUS_TIMEOUT);
    // copies still in flight land before the block's shared memory is released
    if (tid == 0)
      for (int j = k; j < min(k + NS, n_tiles); ++j)
        mbar_wait(&sm.full[j % NS], (j / NS) & 1, p.timeout_ns, nullptr);
  }

  // ---- merge the S partial results on cluster rank 0
  // every thread holds the same m_run / l_run; thread b publishes query b
#pragma unroll
  for (int b = 0; b < BG; ++b)
    if (tid == b) { sm.part_m[b] = m_run[b]; sm.part_l[b] = l_run[b]; }
  if (tid < VT) {  // the value sums live in the first half
#pragma unroll
    for (int b = 0; b < BG; ++b)
#pragma unroll
      for (int j = 0; j < DPT; ++j) sm.part_o[b][tid + VT * j] = o_run[b][j];
  }
  cluster_sync();
  if (rank == 0 && ok) {
    for (int i = tid; i < nb * D; i += TT) {
      const int b = i / D, d = i - b * D;
      const float o = merge_partials(S, smem_u32(&sm.part_m[b]), smem_u32(&sm.part_l[b]),
                                     smem_u32(&sm.part_o[b][d]));
      p.out[(static_cast<int64_t>(b0 + b) * p.H + h) * D + d] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
    }
  }
  cluster_sync();  // peers keep their shared memory until rank 0 is done
}


// ---------------------------------------------------------------------------
// D = 128, up to QG queries per (head, query group): both products on the
// warp-level bf16 tensor-core MMA (m16n8k16, fp32 accumulation). A CTA of 8
// warps walks its token range in 256-token tiles staged by TMA (a
// three-stage ring, one CTA an SM); warp w owns tokens [32 w, 32 w + 32) of
// every tile, in two steps of 16.
//
// Scores, S[t][n] = sum_k K[t][k] Q[k][n]: A = 16 tokens x 16 dims of
// 3-bit codes, B = 16 dims x 8 query columns. The order of the dimensions
// inside an MMA is free (the same on both sides), so lane (g, t4) takes the
// 32 codes of word-aligned chunk t4 of its two token rows (bits 96 t4 ..) and
// pairs code a with code a + 4: shifted so that code a lands at bits 4..6
// and code a + 4 at bits 16..18, one mask-and-or with 0x43004300 gives the
// two bf16 values 128 + 16 c_a and 128 + c_(a+4), and one packed bf16
// subtraction (exact) leaves 16 (c_a - 4) and c_(a+4) - 4. The query takes
// q_a / 16 (exact) at that position, so every product is q_d (c_d - 4)
// exactly and the MMA sums them in fp32.
//
// Values, O[d][n] = sum_t V[t][d] W[t][n]: A = 16 dims x 16 tokens of
// codes, B = 16 tokens x 8 columns of softmax weight x value scale. Lane
// (g, t4) owns the 16 dimensions 16 g .. 16 g + 15 (6 bytes of every row)
// and tokens 2 t4, 2 t4 + 1, 2 t4 + 8, 2 t4 + 9 of the step; a byte permute
// puts the byte holding dimension d of two tokens' rows into the two bf16
// halves (from the row, or from the row shifted by 4 bits where the code
// would reach past bit 4 of its byte), the same mask-and-or and subtraction
// give 2^j (c - 4), and the output of dimension d is unscaled by 2^-j at
// the end. The weights enter as bf16 hi + lo pairs (hi = bf16(w), lo =
// bf16(w - hi), w to ~2^-17): with QG = 4 columns 2 q and 2 q + 1 hold hi
// and lo of query q, with QG = 8 a second MMA takes the lo parts.
//
// Column n of the score MMA holds query n / 2 (QG = 4) or n (QG = 8), so a
// lane's scores and its value accumulators belong to the same queries and
// the online softmax stays in registers; 4 (QG = 4) or 8 shuffles per step
// hand the weights to the lanes that hold them in the value MMA. Scores
// are kept in base 2 (log2 e folded into the scale), so the softmax and the
// merges use exp2.
//
// Tokens kept at 4 bits are left out of the token loop (a per-warp bit mask
// from the sorted list) and added after it, each as one more online-softmax
// step: every lane forms the partial score over its 16 dimensions, the
// lanes sum them, and each lane adds its 16 dimensions of the value row.
// Their rows are prefetched into L2 when the kernel starts. The 8 warps then
// merge through shared memory; every CTA stores its partial result (m, l, o)
// into rank 0's shared memory (distributed shared-memory stores ordered by
// the cluster barrier), and rank 0 merges them. Both merges take their
// factors 2^(m - M) once per query.
constexpr int MQ_WARPS = 8;
constexpr int MQ_TT = 32 * MQ_WARPS;  // tokens per tile = threads per CTA
constexpr int MQ_NS = 3;

template <int QG>
struct SmemMQ {
  union {
    struct {
      uint8_t krow[MQ_NS][MQ_TT][48];
      uint8_t vrow[MQ_NS][MQ_TT][48];
    } st;                              // the tile stages (TMA)
    float wo[MQ_WARPS][QG][128];      // after the token loop: each warp's partial output
  } u;
  float ksc[MQ_NS][MQ_TT][4];
  float vsc[MQ_NS][MQ_TT][4];
  int32_t s_keep[MAX_KEEP];
  float wm[MQ_WARPS][QG], wl[MQ_WARPS][QG];
  float wf[MQ_WARPS][QG];             // the warps' merge factors
  float rf[QG][16];                   // the cluster's merge factors (rank 0)
  // rank 0 only: the partial results (m, l, o) of every CTA of the cluster,
  // written by each CTA into rank 0's copy before the cluster barrier
  float cm[16][QG], cl[16][QG];
  alignas(16) float co[16][QG][128];
  uint64_t full[MQ_NS], empty[MQ_NS];
};

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
               "{%0,%1,%2,%3};"
               : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
               : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// x + y for packed bf16 pairs, exact where the sums are representable
__device__ __forceinline__ uint32_t bf16x2_add_exact(uint32_t x, uint32_t y) {
  uint32_t r;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(x), "r"(0x3F803F80u), "r"(y));
  return r;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Score operand for pair PI (0..15) of a 96-bit chunk X[0..2] (X[3] = 0):
// codes a = 8 (PI / 4) + PI % 4 and a + 4 as bf16 16 (c_a - 4) | (c_(a+4) - 4).
template <int PI>
__device__ __forceinline__ uint32_t k_operand(const uint32_t (&X)[4]) {
  constexpr int a = 8 * (PI >> 2) + (PI & 3);
  constexpr int n = 3 * a - 4;  // stream bit that lands at bit 0
  uint32_t x;
  if constexpr (n < 0) x = X[0] << (-n);
  else if constexpr ((n & 31) == 0) x = X[n >> 5];
  else x = __funnelshift_r(X[n >> 5], X[(n >> 5) + 1], n & 31);
  // bf16 (-192, -132): subtracts 128 + 4 * 16 from the low half and 128 + 4 from the high half
  return bf16x2_add_exact((x & 0x00070070u) | 0x43004300u, 0xC304C340u);
}

// Where local dimension DL (0..15) of a 6-byte group sits among the group
// words {A0, A1, A0 >> 4, A1 >> 4} (funnel-shifted), and its scale 2^j.
template <int DL>
struct VPos {
  static constexpr int b = 3 * DL;
  static constexpr bool shifted = (b & 7) > 4;
  static constexpr int bb = shifted ? b - 4 : b;
  static constexpr int word = (shifted ? 2 : 0) + (bb >> 5);
  static constexpr int byte = (bb & 31) >> 3;
  static constexpr int j = bb & 7;
};

__host__ __device__ constexpr int vpos_j(int dl) { return ((3 * dl) & 7) > 4 ? ((3 * dl) & 7) - 4 : (3 * dl) & 7; }

// Value operand of local dimension DL for two tokens: 2^j (c - 4) of
// token a in the low half, of token b in the high half.
template <int DL>
__device__ __forceinline__ uint32_t v_operand(const uint32_t (&wa)[4], const uint32_t (&wb)[4]) {
  using P = VPos<DL>;
  constexpr uint32_t sel = P::byte | (P::byte << 4) | ((4 + P::byte) << 8) | ((4 + P::byte) << 12);
  constexpr uint32_t mask = (7u << P::j) | (7u << (16 + P::j));
  // -(128 + 4 * 2^j) in both halves
  constexpr uint32_t nb = P::j == 0 ? 0xC304u : P::j == 1 ? 0xC308u : P::j == 2 ? 0xC310u : P::j == 3 ? 0xC320u : 0xC340u;
  const uint32_t r = prmt(wa[P::word], wb[P::word], sel);
  return bf16x2_add_exact((r & mask) | 0x43004300u, nb | (nb << 16));
}

template <int QG>
constexpr int mq_ctas_per_sm() { return 1; }  // shared memory: one CTA an SM

__device__ __forceinline__ int lower_bound_i32(const int32_t* a, int lo, int hi, int key) {
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] < key) lo = mid + 1; else hi = mid;
  }
  return lo;
}

__device__ __forceinline__ void prefetch_l2(const void* ptr) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(ptr));
}

template <int QG>
__global__ void __launch_bounds__(MQ_TT, mq_ctas_per_sm<QG>())
kv_attention_mma_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        const __grid_constant__ CUtensorMap tmKs, const __grid_constant__ CUtensorMap tmVs,
                        const Params p) {
  static_assert(QG == 4 || QG == 8, "4 queries (hi and lo columns in one MMA) or 8 (two MMAs)");
  constexpr int D = 128, RB = 48;
  constexpr int NQL = QG == 4 ? 1 : 2;  // queries of a lane
  constexpr uint32_t STAGE_TX = 2 * MQ_TT * RB + 2 * MQ_TT * 16;
  using SM = SmemMQ<QG>;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  SM& sm = *reinterpret_cast<SM*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t4 = lane & 3;
  const uint32_t rank = cluster_ctarank();
  const int S = static_cast<int>(gridDim.x);
  const int h = blockIdx.y, b0 = blockIdx.z * QG;
  const int nb = min(QG, p.B - b0);
  const int h4 = h & ~3, hl = h & 3;
  const int t_begin = static_cast<int>((static_cast<int64_t>(p.T) * rank) / S);
  const int t_end = static_cast<int>((static_cast<int64_t>(p.T) * (rank + 1)) / S);
  const int n_tiles = (t_end - t_begin + MQ_TT - 1) / MQ_TT;
  const int n4 = min(p.n4, MAX_KEEP);
  const float kql = p.qk_scale * 1.4426950408889634f;  // scores in base 2: exp(x) = 2^(x log2 e)

  if (tid == 0) {
    for (int i = 0; i < MQ_NS; ++i) {
      mbar_init(&sm.full[i], 1);
      mbar_init(&sm.empty[i], MQ_WARPS);
    }
    fence_mbar_init();
  }
  __syncthreads();
  pdl_wait();  // the queries and the cache come from earlier kernels
  pdl_trigger();
  // the query words and the 4-bit list first: issued after the tile copies
  // they would queue behind them
  const int qcol = QG == 4 ? (g >> 1) : g;  // query of this lane's column of the score MMA
  uint32_t qw[16];  // dims 32 t4 .. 32 t4 + 31 as bf16 pairs
#pragma unroll
  for (int i = 0; i < 16; ++i) qw[i] = 0u;
  if (qcol < nb) {
    const uint4* src = reinterpret_cast<const uint4*>(p.q + (static_cast<int64_t>(b0 + qcol) * p.H + h) * D + 32 * t4);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 u = __ldg(src + c);
      qw[4 * c] = u.x; qw[4 * c + 1] = u.y; qw[4 * c + 2] = u.z; qw[4 * c + 3] = u.w;
    }
  }
  auto issue = [&](int k) {  // thread 0: tile k into stage k % MQ_NS
    const int st = k % MQ_NS, t0 = t_begin + k * MQ_TT;
    mbar_arrive_expect_tx(&sm.full[st], STAGE_TX);
    tma_load_2d(&sm.u.st.krow[st][0][0], &tmK, &sm.full[st], h * RB, t0);
    tma_load_2d(&sm.u.st.vrow[st][0][0], &tmV, &sm.full[st], h * RB, t0);
    tma_load_2d(&sm.ksc[st][0][0], &tmKs, &sm.full[st], h4, t0);
    tma_load_2d(&sm.vsc[st][0][0], &tmVs, &sm.full[st], h4, t0);
  };
  for (int i = tid; i < n4; i += MQ_TT) sm.s_keep[i] = __ldg(p.keep4 + i);
  // tile 0 alone first: with every CTA's later tiles in flight too, the
  // first ones would land only with the whole cache; the next MQ_NS - 1 are
  // issued once tile 0 is in, and stream while it is computed
  int n_issued = 0;
  if (tid == 0 && n_tiles > 0) issue(n_issued++);

  // the query operand of the score MMA: pair pi of chunk t4, bf16 q_a / 16 | q_(a+4)
  uint32_t qb[16];
  {
    auto qf = [&](int d) { return __uint_as_float((d & 1) ? (qw[d >> 1] & 0xFFFF0000u) : (qw[d >> 1] << 16)); };
#pragma unroll
    for (int pi = 0; pi < 16; ++pi) {
      const int a = 8 * (pi >> 2) + (pi & 3);
      qb[pi] = pack_bf16x2(qf(a) * 0.0625f, qf(a + 4));  // exact: a power-of-two scale of bf16 values
    }
  }
  // this lane's queries in both MMAs (QG = 4: t4; QG = 8: 2 t4, 2 t4 + 1)
  float m_run[NQL], l_run[NQL];
#pragma unroll
  for (int i = 0; i < NQL; ++i) { m_run[i] = -INFINITY; l_run[i] = 0.f; }
  float acc[8][4], acl[QG == 8 ? 8 : 1][4];  // value accumulators (hi, and lo for QG = 8)
#pragma unroll
  for (int m = 0; m < 8; ++m)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[m][c] = 0.f;
#pragma unroll
  for (int m = 0; m < (QG == 8 ? 8 : 1); ++m)
#pragma unroll
    for (int c = 0; c < 4; ++c) acl[m][c] = 0.f;
  const int vbase = 4 * ((3 * g - (g & 1)) >> 1);  // byte offset of the word holding byte 6 g (or 6 g - 2)
  const int vsh = 16 * (g & 1);
  __syncthreads();  // the 4-bit token list
  // the 4-bit tokens of this CTA's range are list entries [k4lo, k4hi): the
  // token loop leaves them out, and they are added once it is done; their
  // rows go to L2 now
  int k4lo = 0, k4hi = 0;
  if (n4 > 0) {
    k4lo = lower_bound_i32(sm.s_keep, 0, n4, t_begin);
    k4hi = lower_bound_i32(sm.s_keep, k4lo, n4, t_end);
    if (lane == 0 && k4lo + warp < k4hi) {
      const int64_t row = static_cast<int64_t>(k4lo + warp) * p.H + h;
      prefetch_l2(p.k4 + row * (D / 2));
      prefetch_l2(p.v4 + row * (D / 2));
    }
  }

  bool ok = true;
  int k = 0;
  for (; k < n_tiles; ++k) {
    const int st = k % MQ_NS, t0 = t_begin + k * MQ_TT;
    if (!mbar_wait(&sm.full[st], (k / MQ_NS) & 1, p.timeout_ns, nullptr)) { ok = false; break; }
    if (tid == 0 && k == 0)  // into the stages not used yet
      while (n_issued < min(MQ_NS, n_tiles)) issue(n_issued++);
    const int tw0 = t0 + 32 * warp;
    uint32_t m4 = 0u;  // bit i: token tw0 + i is kept at 4 bits
    if (k4lo < k4hi) {
      const int e = lower_bound_i32(sm.s_keep, k4lo, k4hi, tw0) + lane;
      const int te = e < k4hi ? sm.s_keep[e] : 0x7FFFFFFF;
      m4 = __reduce_or_sync(0xFFFFFFFFu, te < tw0 + 32 ? 1u << (te - tw0) : 0u);
    }
    // ---- scores of the warp's 32 tokens: step u, C rows g (r = 0) and g + 8 (r = 1)
    float sv[2][2][NQL];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int rA = 32 * warp + 16 * u + g;
      const uint32_t* ka = reinterpret_cast<const uint32_t*>(&sm.u.st.krow[st][rA][12 * t4]);
      const uint32_t* kb = reinterpret_cast<const uint32_t*>(&sm.u.st.krow[st][rA + 8][12 * t4]);
      const uint32_t XA[4] = {ka[0], ka[1], ka[2], 0u}, XB[4] = {kb[0], kb[1], kb[2], 0u};
      float c[4] = {0.f, 0.f, 0.f, 0.f};
#define BLT_KSTEP(S_)                                                                          \
      {                                                                                        \
        const uint32_t a[4] = {k_operand<2 * S_>(XA), k_operand<2 * S_>(XB),                   \
                               k_operand<2 * S_ + 1>(XA), k_operand<2 * S_ + 1>(XB)};          \
        mma_bf16_16816(c, a, qb[2 * S_], qb[2 * S_ + 1]);                                      \
      }
      BLT_KSTEP(0) BLT_KSTEP(1) BLT_KSTEP(2) BLT_KSTEP(3) BLT_KSTEP(4) BLT_KSTEP(5) BLT_KSTEP(6) BLT_KSTEP(7)
#undef BLT_KSTEP
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int row = rA + 8 * r, t = t0 + row;
        const bool live = t < t_end && !((m4 >> (16 * u + g + 8 * r)) & 1u);
        const float kq = __fmul_rn(sm.ksc[st][row][hl], kql);
#pragma unroll
        for (int i = 0; i < NQL; ++i) sv[u][r][i] = live ? __fmul_rn(c[2 * r + (QG == 8 ? i : 0)], kq) : -INFINITY;
      }
    }
    // ---- online softmax over the warp's 32 tokens, per query of the lane (base 2)
    float corr[NQL], w[2][2][NQL];
#pragma unroll
    for (int i = 0; i < NQL; ++i) {
      float mt = fmaxf(fmaxf(sv[0][0][i], sv[0][1][i]), fmaxf(sv[1][0][i], sv[1][1][i]));
#pragma unroll
      for (int o_ = 4; o_ < 32; o_ <<= 1) mt = fmaxf(mt, __shfl_xor_sync(0xFFFFFFFFu, mt, o_));
      const float m_new = fmaxf(m_run[i], mt);
      corr[i] = m_new == -INFINITY ? 1.f : exp2f(m_run[i] - m_new);
      float ls = 0.f;
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const float e = sv[u][r][i] == -INFINITY ? 0.f : exp2f(sv[u][r][i] - m_new);
          ls += e;
          w[u][r][i] = __fmul_rn(e, sm.vsc[st][32 * warp + 16 * u + g + 8 * r][hl]);
        }
#pragma unroll
      for (int o_ = 4; o_ < 32; o_ <<= 1) ls += __shfl_xor_sync(0xFFFFFFFFu, ls, o_);
      l_run[i] = fmaf(l_run[i], corr[i], ls);
      m_run[i] = m_new;
    }
#pragma unroll
    for (int m = 0; m < 8; ++m)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        acc[m][c] = __fmul_rn(acc[m][c], corr[QG == 8 ? (c & 1) : 0]);
        if constexpr (QG == 8) acl[m][c] = __fmul_rn(acl[m][c], corr[c & 1]);
      }
    // ---- values, step u: tokens 2 t4, 2 t4 + 1, 2 t4 + 8, 2 t4 + 9
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      // B: the weights of column g's query at those tokens, from the lanes
      // that hold them (token i of the step: lane 4 (i % 8) + its query slot)
      const int src0 = 4 * (2 * t4), src1 = 4 * (2 * t4 + 1);
      const int sq = g >> 1;
      uint32_t bh0, bh1, bl0 = 0u, bl1 = 0u;
      if constexpr (QG == 4) {  // column g: query g / 2, hi (g even) or lo (g odd)
        float v[4] = {__shfl_sync(0xFFFFFFFFu, w[u][0][0], src0 + sq), __shfl_sync(0xFFFFFFFFu, w[u][0][0], src1 + sq),
                      __shfl_sync(0xFFFFFFFFu, w[u][1][0], src0 + sq), __shfl_sync(0xFFFFFFFFu, w[u][1][0], src1 + sq)};
        if (g & 1) {
#pragma unroll
          for (int e = 0; e < 4; ++e) v[e] = v[e] - __bfloat162float(__float2bfloat16_rn(v[e]));
        }
        bh0 = pack_bf16x2(v[0], v[1]);
        bh1 = pack_bf16x2(v[2], v[3]);
      } else {  // column g: query g; lane 4 i + g / 2 holds queries g & ~1 and g | 1
        float v0[4], v1[4], v[4], lo[4];
        v0[0] = __shfl_sync(0xFFFFFFFFu, w[u][0][0], src0 + sq); v1[0] = __shfl_sync(0xFFFFFFFFu, w[u][0][1], src0 + sq);
        v0[1] = __shfl_sync(0xFFFFFFFFu, w[u][0][0], src1 + sq); v1[1] = __shfl_sync(0xFFFFFFFFu, w[u][0][1], src1 + sq);
        v0[2] = __shfl_sync(0xFFFFFFFFu, w[u][1][0], src0 + sq); v1[2] = __shfl_sync(0xFFFFFFFFu, w[u][1][1], src0 + sq);
        v0[3] = __shfl_sync(0xFFFFFFFFu, w[u][1][0], src1 + sq); v1[3] = __shfl_sync(0xFFFFFFFFu, w[u][1][1], src1 + sq);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          v[e] = (g & 1) ? v1[e] : v0[e];
          lo[e] = v[e] - __bfloat162float(__float2bfloat16_rn(v[e]));
        }
        bh0 = pack_bf16x2(v[0], v[1]);
        bh1 = pack_bf16x2(v[2], v[3]);
        bl0 = pack_bf16x2(lo[0], lo[1]);
        bl1 = pack_bf16x2(lo[2], lo[3]);
      }
      // A: group g's 6 bytes of the four token rows, aligned, and shifted by 4 bits
      uint32_t wr[4][4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int row = 32 * warp + 16 * u + 2 * t4 + (e & 1) + 8 * (e >> 1);
        const uint8_t* vr = &sm.u.st.vrow[st][row][vbase];
        const uint32_t x0 = *reinterpret_cast<const uint32_t*>(vr);
        const uint32_t x1 = *reinterpret_cast<const uint32_t*>(vr + 4);
        wr[e][0] = __funnelshift_r(x0, x1, vsh);
        wr[e][1] = x1 >> vsh;
        wr[e][2] = __funnelshift_r(wr[e][0], wr[e][1], 4);
        wr[e][3] = wr[e][1] >> 4;
      }
#define BLT_VSTEP(M_)                                                                        \
      {                                                                                      \
        const uint32_t a[4] = {v_operand<2 * M_>(wr[0], wr[1]), v_operand<2 * M_ + 1>(wr[0], wr[1]), \
                               v_operand<2 * M_>(wr[2], wr[3]), v_operand<2 * M_ + 1>(wr[2], wr[3])}; \
        mma_bf16_16816(acc[M_], a, bh0, bh1);                                                \
        if constexpr (QG == 8) mma_bf16_16816(acl[M_ & (QG == 8 ? 7 : 0)], a, bl0, bl1);     \
      }
      BLT_VSTEP(0) BLT_VSTEP(1) BLT_VSTEP(2) BLT_VSTEP(3) BLT_VSTEP(4) BLT_VSTEP(5) BLT_VSTEP(6) BLT_VSTEP(7)
#undef BLT_VSTEP
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.empty[st]);  // this warp is done with the stage
    if (tid == 0 && n_issued < n_tiles) {
      if (!mbar_wait(&sm.empty[st], (k / MQ_NS) & 1, p.timeout_ns, nullptr)) { ok = false; break; }
      issue(n_issued++);
    }
  }
  if (tid == 0)  // copies still in flight land before the stages are reused or released
    for (int j = k; j < n_issued; ++j) mbar_wait(&sm.full[j % MQ_NS], (j / MQ_NS) & 1, p.timeout_ns, nullptr);
  const bool bad = __syncthreads_or(!ok);
  if (bad && tid == 0) report_status(p.status, BITLINEAR_STATUS_TIMEOUT);

  // ---- the 4-bit tokens of the range, one online-softmax step each: warp w
  // takes entries k4lo + w, k4lo + w + 8, ...; lane (g, t4) forms the partial
  // score over dimensions 16 g .. 16 g + 15 for its queries (summed over g)
  // and adds its 16 dimensions of the value row
  for (int e = k4lo + warp; e < k4hi; e += MQ_WARPS) {
    const int t = sm.s_keep[e];
    const int64_t row = static_cast<int64_t>(e) * p.H + h;
    const uint2 kc = __ldg(reinterpret_cast<const uint2*>(p.k4 + row * (D / 2)) + g);
    const uint2 vc = __ldg(reinterpret_cast<const uint2*>(p.v4 + row * (D / 2)) + g);
    const float kq = __fmul_rn(__ldg(p.ks + static_cast<int64_t>(t) * p.H + h), kql);
    const float vscl = __ldg(p.vs + static_cast<int64_t>(t) * p.H + h);
#pragma unroll
    for (int q = 0; q < NQL; ++q) {
      const int qi = QG == 4 ? t4 : 2 * t4 + q;
      float dot = 0.f;
      if (qi < nb) {
        const uint4* qs = reinterpret_cast<const uint4*>(p.q + (static_cast<int64_t>(b0 + qi) * p.H + h) * D + 16 * g);
        const uint4 qa = __ldg(qs), qz = __ldg(qs + 1);
        const uint32_t qq[8] = {qa.x, qa.y, qa.z, qa.w, qz.x, qz.y, qz.z, qz.w};
#pragma unroll
        for (int dl = 0; dl < 16; ++dl) {
          const float qd = __uint_as_float((dl & 1) ? (qq[dl >> 1] & 0xFFFF0000u) : (qq[dl >> 1] << 16));
          const uint32_t cw = dl < 8 ? kc.x : kc.y;
          dot = fmaf(qd, static_cast<float>(static_cast<int>((cw >> (4 * (dl & 7))) & 15u) - 8), dot);
        }
      }
#pragma unroll
      for (int o_ = 4; o_ < 32; o_ <<= 1) dot += __shfl_xor_sync(0xFFFFFFFFu, dot, o_);
      const float s = __fmul_rn(dot, kq);
      const float m_new = fmaxf(m_run[q], s);
      const float cr = exp2f(m_run[q] - m_new);  // 0 while m_run = -inf
      const float ee = exp2f(s - m_new);
      l_run[q] = fmaf(l_run[q], cr, ee);
      m_run[q] = m_new;
      const float wv = __fmul_rn(ee, vscl);
#pragma unroll
      for (int m = 0; m < 8; ++m)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (QG == 4 || (c & 1) == q) {
            acc[m][c] = __fmul_rn(acc[m][c], cr);
            if constexpr (QG == 8) acl[m][c] = __fmul_rn(acl[m][c], cr);
          }
        }
#pragma unroll
      for (int dl = 0; dl < 16; ++dl) {
        const uint32_t cw = dl < 8 ? vc.x : vc.y;
        const float cd = static_cast<float>(static_cast<int>((cw >> (4 * (dl & 7))) & 15u) - 8);
        float& a = acc[dl >> 1][2 * (dl & 1) + (QG == 8 ? q : 0)];
        a = fmaf(__fmul_rn(wv, static_cast<float>(1 << vpos_j(dl))), cd, a);
      }
    }
  }

  // ---- each warp's partial outputs (unscaled by 2^-j), then the 8 warps, then the cluster
#pragma unroll
  for (int m = 0; m < 8; ++m)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int dl = 2 * m + hh;
      const float us = 1.f / static_cast<float>(1 << vpos_j(dl));
#pragma unroll
      for (int q = 0; q < NQL; ++q) {
        const int qi = QG == 4 ? t4 : 2 * t4 + q;
        const float o = QG == 4 ? acc[m][2 * hh] + acc[m][2 * hh + 1]
                                : acc[m][2 * hh + q] + acl[m & (QG == 8 ? 7 : 0)][2 * hh + q];
        sm.u.wo[warp][qi][16 * g + dl] = o * us;
      }
    }
  if (g == 0)
#pragma unroll
    for (int q = 0; q < NQL; ++q) {
      const int qi = QG == 4 ? t4 : 2 * t4 + q;
      sm.wm[warp][qi] = m_run[q];
      sm.wl[warp][qi] = l_run[q];
    }
  __syncthreads();
  // the warps' factors 2^(m_w - M), and this CTA's (M, L, O) written into
  // rank 0's slots (distributed shared memory stores, ordered by the
  // release / acquire of the cluster barrier)
  if (tid < QG) {
    float M = -INFINITY;
#pragma unroll
    for (int ww = 0; ww < MQ_WARPS; ++ww) M = fmaxf(M, sm.wm[ww][tid]);
    float L = 0.f;
#pragma unroll
    for (int ww = 0; ww < MQ_WARPS; ++ww) {
      const float f = sm.wm[ww][tid] == -INFINITY ? 0.f : exp2f(sm.wm[ww][tid] - M);
      sm.wf[ww][tid] = f;
      L = fmaf(f, sm.wl[ww][tid], L);
    }
    st_dsmem_f32(map_shared_rank(smem_u32(&sm.cm[rank][tid]), 0u), M);
    st_dsmem_f32(map_shared_rank(smem_u32(&sm.cl[rank][tid]), 0u), L);
  }
  __syncthreads();
  for (int i = tid; i < QG * D / 4; i += MQ_TT) {  // 4 dimensions an item
    const int q = i / (D / 4), d = 4 * (i - q * (D / 4));
    float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int ww = 0; ww < MQ_WARPS; ++ww) {
      const float f = sm.wf[ww][q];
      const float4 x = *reinterpret_cast<const float4*>(&sm.u.wo[ww][q][d]);
      O.x = fmaf(f, x.x, O.x); O.y = fmaf(f, x.y, O.y); O.z = fmaf(f, x.z, O.z); O.w = fmaf(f, x.w, O.w);
    }
    st_dsmem_v4f32(map_shared_rank(smem_u32(&sm.co[rank][q][d]), 0u), O);
  }
  cluster_sync();
  // rank 0 merges the S partial results from its own shared memory; the
  // other CTAs are done (nothing reads their shared memory any more)
  if (rank == 0 && !bad) {  // block-uniform
    if (tid < nb) {  // the ranks' factors 2^(m_r - M) / L
      float M = -INFINITY;
      for (int r = 0; r < S; ++r) M = fmaxf(M, sm.cm[r][tid]);
      float L = 0.f;
      for (int r = 0; r < S; ++r) {
        const float f = sm.cm[r][tid] == -INFINITY ? 0.f : exp2f(sm.cm[r][tid] - M);
        sm.rf[tid][r] = f;
        L = fmaf(f, sm.cl[r][tid], L);
      }
      const float inv = 1.f / L;
      for (int r = 0; r < S; ++r) sm.rf[tid][r] *= inv;
    }
    __syncthreads();
    for (int i = tid; i < nb * D; i += MQ_TT) {
      const int q = i / D, d = i - q * D;
      float o = 0.f;
      for (int r = 0; r < S; ++r) o = fmaf(sm.rf[q][r], sm.co[r][q][d], o);
      p.out[(static_cast<int64_t>(b0 + q) * p.H + h) * D + d] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
    }
  }
}
}  // namespace attn

template <int D, int BG>
static cudaError_t launch_attn_t(const CUtensorMap (&maps)[4], const attn::Params& p, int S,
                                 cudaStream_t s) {
  cudaError_t e = set_smem_limit(attn::kv_attention_kernel<D, BG>,
                                  static_cast<int>(sizeof(attn::Smem<D, BG>)));
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>(S), static_cast<unsigned>(p.H),
                  static_cast<unsigned>((p.B + BG - 1) / BG));
  return launch_kernel(attn::kv_attention_kernel<D, BG>, grid, dim3(attn::TT),
                       sizeof(attn::Smem<D, BG>), s, static_cast<unsigned>(S), maps[0], maps[1],
                       maps[2], maps[3], p);
}

cudaError_t launch_kv_attention(const uint16_t* q, int64_t B, int64_t H, int64_t D, int64_t T,
                                const uint8_t* k3, const uint8_t* k4, const float* ks,
                                const uint8_t* v3, const uint8_t* v4, const float* vs,
                                const int32_t* keep4, int64_t n4, uint16_t* out, int* status,
                                uint64_t timeout_ns, cudaStream_t s, const char** why) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) { *why = "cuTensorMapEncodeTiled unavailable"; return cudaErrorNotSupported; }
  const uint64_t RB = static_cast<uint64_t>(3 * D / 8);
  CUtensorMap maps[4];
  // packed rows: [T rows][H * RB bytes]; a box = 256 rows x RB bytes (one head)
  for (int i = 0; i < 2; ++i) {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(H) * RB, static_cast<cuuint64_t>(T)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(H) * RB};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(RB), static_cast<cuuint32_t>(attn::TT)};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&maps[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(i == 0 ? k3 : v3), dims,
            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
      *why = "cuTensorMapEncodeTiled rejected the packed cache layout";
      return cudaErrorInvalidValue;
    }
  }
  // scales: [T rows][H floats]; a box = 256 rows x the 4 heads holding h
  for (int i = 0; i < 2; ++i) {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(T)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(H) * 4};
    const cuuint32_t box[2] = {4, static_cast<cuuint32_t>(attn::TT)};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&maps[2 + i], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(i == 0 ? ks : vs),
            dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
      *why = "cuTensorMapEncodeTiled rejected the scale layout";
      return cudaErrorInvalidValue;
    }
  }
  attn::Params p{};
  p.q = q;
  p.k4 = k4;
  p.v4 = v4;
  p.keep4 = keep4;
  p.n4 = static_cast<int>(n4);
  p.B = static_cast<int>(B);
  p.H = static_cast<int>(H);
  p.T = static_cast<int>(T);
  p.qk_scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
  p.ks = ks;
  p.vs = vs;
  p.out = out;
  p.status = status;
  p.timeout_ns = timeout_ns;
  if (D == 128) {
    // D = 128, any number of queries: both products on the bf16 tensor-core
    // MMA, 4 or 8 queries per CTA, clusters of up to 16 CTAs per (head, query
    // group) with two tiles or more each, one wave of CTAs
    CUtensorMap qm[4];
    for (int i = 0; i < 4; ++i) {
      const bool codes = i < 2;
      const cuuint64_t dims[2] = {codes ? static_cast<cuuint64_t>(H) * RB : static_cast<cuuint64_t>(H),
                                  static_cast<cuuint64_t>(T)};
      const cuuint64_t strides[1] = {codes ? static_cast<cuuint64_t>(H) * RB : static_cast<cuuint64_t>(H) * 4};
      const cuuint32_t box[2] = {codes ? static_cast<cuuint32_t>(RB) : 4u, static_cast<cuuint32_t>(attn::MQ_TT)};
      const cuuint32_t estr[2] = {1, 1};
      void* base = i == 0 ? const_cast<uint8_t*>(k3) : i == 1 ? const_cast<uint8_t*>(v3)
                 : i == 2 ? static_cast<void*>(const_cast<float*>(ks)) : static_cast<void*>(const_cast<float*>(vs));
      if (enc(&qm[i], codes ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims,
              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
        *why = "cuTensorMapEncodeTiled rejected the cache layout";
        return cudaErrorInvalidValue;
      }
    }
    const int QG = B <= 4 ? 4 : 8;
    const int64_t groups = (B + QG - 1) / QG;
    int S = 1;
    const int per_sm = QG == 4 ? attn::mq_ctas_per_sm<4>() : attn::mq_ctas_per_sm<8>();
    while (S < 16 && T / (4 * S) >= attn::MQ_TT && H * groups * S * 2 <= per_sm * num_sms()) S *= 2;
    auto go = [&](auto kern, int smem) -> cudaError_t {
      cudaError_t e = set_smem_limit(kern, smem);
      if (e != cudaSuccess) return e;
      if (S > 8) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
      }
      return launch_kernel(kern, dim3(static_cast<unsigned>(S), static_cast<unsigned>(H), static_cast<unsigned>(groups)),
                           dim3(attn::MQ_TT), static_cast<size_t>(smem), s, static_cast<unsigned>(S),
                           qm[0], qm[1], qm[2], qm[3], p);
    };
    return QG == 4 ? go(attn::kv_attention_mma_kernel<4>, static_cast<int>(sizeof(attn::SmemMQ<4>)))
                   : go(attn::kv_attention_mma_kernel<8>, static_cast<int>(sizeof(attn::SmemMQ<8>)));
  }
  const int BG = B == 1 ? 1 : attn::MAX_BG;
  const int64_t ctas = H * ((B + BG - 1) / BG);
  // split T over a cluster while the grid stays within two waves and every
  // CTA keeps at least one full tile
  int S = 1;
  while (S < 8 && ctas * S * 2 <= 2 * num_sms() && T / (2 * S) >= attn::TT) S *= 2;
  if (D == 128) return BG == 1 ? launch_attn_t<128, 1>(maps, p, S, s) : launch_attn_t<128, 8>(maps, p, S, s);
  return BG == 1 ? launch_attn_t<256, 1>(maps, p, S, s) : launch_attn_t<256, 8>(maps, p, S, s);
}

}  // namespace blt
