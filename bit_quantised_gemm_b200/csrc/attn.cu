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
// in tiles of 256 with an online softmax (running max m, running sum l and
// the running weighted value sum o per query), and the S partial results are
// merged through distributed shared memory by cluster rank 0, so no global
// scratch is needed.
//
// The rows of one head are 3D/8 bytes every H * 3D/8 bytes in the cache, so
// each tile's K rows, V rows and their scales arrive by TMA (2-D boxes of 256
// rows) into a two-stage ring: the next tile is in flight while the current
// one is computed. Within a tile:
//   * thread i owns token i: it reads the token's packed K row from shared
//     memory and forms s_b for every query b against the queries held in
//     shared memory (broadcast reads); codes become floats with one OR and
//     one subtract (2^23 + code trick);
//   * the block reduces the tile maximum and the sum of exp per query;
//   * thread (half, d) accumulates dimension d over half of the tile's
//     tokens straight from the staged V rows; the halves meet in shared memory.
#include <cmath>

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
// One query per (batch, head), D = 128: warp-independent tiles.
// A CTA of 4 warps walks its token range in 128-token tiles staged by TMA;
// warp w owns tokens [32 w, 32 w + 32) of every
// tile and keeps its own online softmax (running max, running sum, running
// weighted value sum), so a tile needs no block barrier: each warp releases
// the stage through an mbarrier the loading thread waits on before it reuses
// it. Scores: 4 lanes per token, 32 dimensions a lane, the query slice in
// registers, the codes taken from the staged row three 32-bit words at a
// time (conflict-free: lane (token g, part j) reads words 12 g + 3 j ...).
// Values: the two half-warps take alternate tokens, a lane 8 consecutive
// dimensions (24 bits of the row: two 32-bit words and a funnel shift).
// Every code becomes the float (2^23 + c) by one OR, then c - 4 by a paired
// fp32 add, and the products run on the paired fp32 multiply-add. The 4
// warps merge once at the end, then the CTAs of a cluster through
// distributed shared memory as above.
constexpr int Q1_NS = 2;
constexpr int Q1_WARPS = 4;
constexpr int Q1_TT = 32 * Q1_WARPS;  // tokens per tile = threads per CTA

template <int D>
struct SmemQ1 {
  static constexpr int RB = 3 * D / 8;
  uint8_t krow[Q1_NS][Q1_TT][RB];
  uint8_t vrow[Q1_NS][Q1_TT][RB];
  float ksc[Q1_NS][Q1_TT][4];
  float vsc[Q1_NS][Q1_TT][4];
  int32_t s_keep[MAX_KEEP];
  float wm[Q1_WARPS], wl[Q1_WARPS];
  float wo[Q1_WARPS][D];
  float part_m, part_l;
  float part_o[D];
  uint64_t full[Q1_NS], empty[Q1_NS];
};

// the float 2^23 + (3-bit code at bit `bit` of the words w)
template <int NW>
__device__ __forceinline__ float code_f(const uint32_t (&w)[NW], int bit) {
  const int i = bit >> 5, sh = bit & 31;
  const uint32_t v = sh <= 29 ? (w[i] >> sh) : __funnelshift_r(w[i], w[i + 1], sh);
  return __int_as_float(static_cast<int>((v & 7u) | 0x4B000000u));
}

template <int D>
__global__ void __launch_bounds__(Q1_TT, 6)
kv_attention_q1_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmKs, const __grid_constant__ CUtensorMap tmVs,
                       const Params p) {
  static_assert(D == 128, "4 lanes of 32 dimensions per token; 8 dimensions per lane in the value pass");
  using SM = SmemQ1<D>;
  constexpr int RB = SM::RB;        // 48 bytes a packed row
  constexpr uint32_t STAGE_TX = 2 * Q1_TT * RB + 2 * Q1_TT * 16;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  SM& sm = *reinterpret_cast<SM*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t rank = cluster_ctarank();
  const int S = static_cast<int>(gridDim.x);
  const int h = blockIdx.y, bq = blockIdx.z;
  const int h4 = h & ~3, hl = h & 3;
  const int t_begin = static_cast<int>((static_cast<int64_t>(p.T) * rank) / S);
  const int t_end = static_cast<int>((static_cast<int64_t>(p.T) * (rank + 1)) / S);
  const int n_tiles = (t_end - t_begin + Q1_TT - 1) / Q1_TT;
  const int n4 = min(p.n4, MAX_KEEP);

  if (tid == 0) {
    for (int i = 0; i < Q1_NS; ++i) {
      mbar_init(&sm.full[i], 1);
      mbar_init(&sm.empty[i], Q1_WARPS);
    }
    fence_mbar_init();
  }
  __syncthreads();
  pdl_wait();  // the queries and the cache come from earlier kernels
  pdl_trigger();
  auto issue = [&](int k) {  // thread 0: tile k into stage k % Q1_NS
    const int st = k % Q1_NS, t0 = t_begin + k * Q1_TT;
    mbar_arrive_expect_tx(&sm.full[st], STAGE_TX);
    tma_load_2d(&sm.krow[st][0][0], &tmK, &sm.full[st], h * RB, t0);
    tma_load_2d(&sm.vrow[st][0][0], &tmV, &sm.full[st], h * RB, t0);
    tma_load_2d(&sm.ksc[st][0][0], &tmKs, &sm.full[st], h4, t0);
    tma_load_2d(&sm.vsc[st][0][0], &tmVs, &sm.full[st], h4, t0);
  };
  int n_issued = 0;
  if (tid == 0)
    for (; n_issued < min(Q1_NS, n_tiles); ++n_issued) issue(n_issued);
  for (int i = tid; i < n4; i += Q1_TT) sm.s_keep[i] = __ldg(p.keep4 + i);

  // this lane's query slice, pre-scaled by 1/sqrt(D)
  const int sub = lane & 3;
  float2 qv[16];  // dims 32 sub + 2 i, 32 sub + 2 i + 1
  {
    const uint4* qsrc = reinterpret_cast<const uint4*>(p.q + (static_cast<int64_t>(bq) * p.H + h) * D + 32 * sub);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 u = __ldg(qsrc + c);
      const uint32_t ww[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
        qv[4 * c + i] = make_float2(__fmul_rn(__uint_as_float(ww[i] << 16), p.qk_scale),
                                    __fmul_rn(__uint_as_float(ww[i] & 0xFFFF0000u), p.qk_scale));
    }
  }
  const float2 kMinus4 = make_float2(-8388612.f, -8388612.f), kMinus8 = make_float2(-8388616.f, -8388616.f);
  __syncthreads();  // the 4-bit token list

  const int half = lane >> 4, dl = lane & 15;       // value pass: dims 8 dl .. 8 dl + 7
  const int vi0 = (24 * dl) >> 5, vsh = (24 * dl) & 31;
  const int vi1 = min(vi0 + 1, RB / 4 - 1);
  float m_w = -INFINITY, l_w = 0.f;
  float2 o[4];  // dims 8 dl + 2 i, 8 dl + 2 i + 1
#pragma unroll
  for (int i = 0; i < 4; ++i) o[i] = make_float2(0.f, 0.f);

  bool ok = true;
  int k = 0;
  for (; k < n_tiles; ++k) {
    const int st = k % Q1_NS, t0 = t_begin + k * Q1_TT;
    if (!mbar_wait(&sm.full[st], (k / Q1_NS) & 1, p.timeout_ns, nullptr)) { ok = false; break; }
    // 4-bit tokens in this warp's 32 (rare): the list is sorted
    const int tw0 = t0 + 32 * warp;
    bool rare = false;
    if (n4 > 0) {
      int lo = 0, hi = n4;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (sm.s_keep[mid] < tw0) lo = mid + 1; else hi = mid;
      }
      rare = lo < n4 && sm.s_keep[lo] < min(tw0 + 32, t_end);
    }
    // ---- scores: token 8 pp + lane / 4 of the warp, dims 32 sub .. 32 sub + 31
    float sc[4], w3[4], w4[4];
    int kj[4];
#pragma unroll
    for (int pp = 0; pp < 4; ++pp) {
      const int row = 32 * warp + 8 * pp + (lane >> 2);
      const int t = t0 + row;
      const uint32_t* kr = reinterpret_cast<const uint32_t*>(&sm.krow[st][row][12 * sub]);
      const uint32_t kw[4] = {kr[0], kr[1], kr[2], 0u};
      float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
#pragma unroll
      for (int d = 0; d < 32; d += 2) {
        const float2 c = __fadd2_rn(make_float2(code_f(kw, 3 * d), code_f(kw, 3 * d + 3)), kMinus4);  // code - 4
        if ((d >> 1) & 1) a1 = __ffma2_rn(qv[d >> 1], c, a1);
        else a0 = __ffma2_rn(qv[d >> 1], c, a0);
      }
      float sp = (a0.x + a0.y) + (a1.x + a1.y);
      kj[pp] = -1;
      if (rare) {  // a 4-bit token: its own row, dims 32 sub .. from the 4-bit store
        int lo = 0, hi = n4;
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (sm.s_keep[mid] < t) lo = mid + 1; else hi = mid;
        }
        if (lo < n4 && sm.s_keep[lo] == t && t < t_end) {
          kj[pp] = lo;
          const uint4* r4 = reinterpret_cast<const uint4*>(p.k4 + (static_cast<int64_t>(lo) * p.H + h) * (D / 2)) + sub;
          const uint4 u = __ldg(r4);
          const uint32_t ww[4] = {u.x, u.y, u.z, u.w};
          float2 b = make_float2(0.f, 0.f);
#pragma unroll
          for (int d = 0; d < 32; d += 2) {
            const uint32_t x = ww[d >> 3] >> (4 * (d & 7));
            const float2 c = __fadd2_rn(make_float2(__int_as_float(static_cast<int>((x & 15u) | 0x4B000000u)),
                                                    __int_as_float(static_cast<int>(((x >> 4) & 15u) | 0x4B000000u))),
                                        kMinus8);  // code - 8
            b = __ffma2_rn(qv[d >> 1], c, b);
          }
          sp = b.x + b.y;
        }
      }
      sp += __shfl_xor_sync(0xFFFFFFFFu, sp, 1);
      sp += __shfl_xor_sync(0xFFFFFFFFu, sp, 2);
      sc[pp] = t < t_end ? __fmul_rn(sp, sm.ksc[st][row][hl]) : -INFINITY;
    }
    // ---- this warp's online softmax over its 32 tokens
    float mt = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
#pragma unroll
    for (int o_ = 4; o_ < 32; o_ <<= 1) mt = fmaxf(mt, __shfl_xor_sync(0xFFFFFFFFu, mt, o_));
    const float m_new = fmaxf(m_w, mt);
    const float corr = m_new == -INFINITY ? 1.f : expf(m_w - m_new);  // 0 while m_w = -inf
    float ls = 0.f;
#pragma unroll
    for (int pp = 0; pp < 4; ++pp) {
      const int row = 32 * warp + 8 * pp + (lane >> 2);
      const float e = sc[pp] == -INFINITY ? 0.f : expf(sc[pp] - m_new);
      ls += e;
      const float we = __fmul_rn(e, sm.vsc[st][row][hl]);
      w3[pp] = kj[pp] < 0 ? we : 0.f;  // absent and 4-bit tokens weigh nothing in the 3-bit pass
      w4[pp] = we;
    }
#pragma unroll
    for (int o_ = 4; o_ < 32; o_ <<= 1) ls += __shfl_xor_sync(0xFFFFFFFFu, ls, o_);
    l_w = fmaf(l_w, corr, ls);
    m_w = m_new;
    // ---- values: tokens 2 uu + half of the warp, dims 8 dl .. 8 dl + 7
    const float2 corr2 = make_float2(corr, corr);
#pragma unroll
    for (int i = 0; i < 4; ++i) o[i] = __fmul2_rn(o[i], corr2);
#pragma unroll
    for (int uu = 0; uu < 16; ++uu) {
      const int u = 2 * uu + half;
      const float wt = __shfl_sync(0xFFFFFFFFu, w3[uu >> 2], 4 * (u & 7));
      const float2 wt2 = make_float2(wt, wt);
      const uint32_t* vr = reinterpret_cast<const uint32_t*>(&sm.vrow[st][32 * warp + u][0]);
      const uint32_t v = __funnelshift_r(vr[vi0], vr[vi1], vsh);
#pragma unroll
      for (int j = 0; j < 8; j += 2) {
        const float2 c = __fadd2_rn(make_float2(__int_as_float(static_cast<int>(((v >> (3 * j)) & 7u) | 0x4B000000u)),
                                                __int_as_float(static_cast<int>(((v >> (3 * j + 3)) & 7u) | 0x4B000000u))),
                                    kMinus4);
        o[j >> 1] = __ffma2_rn(wt2, c, o[j >> 1]);
      }
    }
    if (rare) {  // 4-bit tokens of this warp: half 0 adds them
#pragma unroll
      for (int pp = 0; pp < 4; ++pp) {
        for (int g = 0; g < 8; ++g) {
          const int kjg = __shfl_sync(0xFFFFFFFFu, kj[pp], 4 * g);
          const float wg = __shfl_sync(0xFFFFFFFFu, w4[pp], 4 * g);
          if (kjg >= 0 && half == 0) {
            const uint32_t x = __ldg(reinterpret_cast<const uint32_t*>(
                p.v4 + (static_cast<int64_t>(kjg) * p.H + h) * (D / 2)) + dl);
#pragma unroll
            for (int j = 0; j < 8; j += 2) {
              const float2 c = __fadd2_rn(make_float2(__int_as_float(static_cast<int>(((x >> (4 * j)) & 15u) | 0x4B000000u)),
                                                      __int_as_float(static_cast<int>(((x >> (4 * j + 4)) & 15u) | 0x4B000000u))),
                                          kMinus8);
              o[j >> 1] = __ffma2_rn(make_float2(wg, wg), c, o[j >> 1]);
            }
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.empty[st]);  // this warp is done with the stage
    if (tid == 0 && n_issued < n_tiles) {
      // refill stage st once every warp has released it
      if (!mbar_wait(&sm.empty[st], (k / Q1_NS) & 1, p.timeout_ns, nullptr)) { ok = false; break; }
      issue(n_issued++);
    }
  }
  if (tid == 0)  // copies still in flight land before the block's shared memory is released
    for (int j = k; j < n_issued; ++j) mbar_wait(&sm.full[j % Q1_NS], (j / Q1_NS) & 1, p.timeout_ns, nullptr);
  const bool bad = __syncthreads_or(!ok);
  if (bad && tid == 0) report_status(p.status, BITLINEAR_STATUS_TIMEOUT);

  // ---- merge the 8 warps, then the S CTAs of the cluster on rank 0
#pragma unroll
  for (int i = 0; i < 4; ++i) {  // the two halves
    o[i].x += __shfl_xor_sync(0xFFFFFFFFu, o[i].x, 16);
    o[i].y += __shfl_xor_sync(0xFFFFFFFFu, o[i].y, 16);
  }
  if (lane < 16) {
#pragma unroll
    for (int i = 0; i < 4; ++i) { sm.wo[warp][8 * dl + 2 * i] = o[i].x; sm.wo[warp][8 * dl + 2 * i + 1] = o[i].y; }
  }
  if (lane == 0) { sm.wm[warp] = m_w; sm.wl[warp] = l_w; }
  __syncthreads();
  if (tid < D) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < Q1_WARPS; ++w) M = fmaxf(M, sm.wm[w]);
    float L = 0.f, O = 0.f;
#pragma unroll
    for (int w = 0; w < Q1_WARPS; ++w) {
      const float f = sm.wm[w] == -INFINITY ? 0.f : expf(sm.wm[w] - M);
      L = fmaf(f, sm.wl[w], L);
      O = fmaf(f, sm.wo[w][tid], O);
    }
    sm.part_o[tid] = O;
    if (tid == 0) { sm.part_m = M; sm.part_l = L; }
  }
  cluster_sync();
  if (rank == 0 && !bad && tid < D) {
    const float o = merge_partials(S, smem_u32(&sm.part_m), smem_u32(&sm.part_l), smem_u32(&sm.part_o[tid]));
    p.out[(static_cast<int64_t>(bq) * p.H + h) * D + tid] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
  }
  cluster_sync();  // peers keep their shared memory until rank 0 is done
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
  p.out = out;
  p.status = status;
  p.timeout_ns = timeout_ns;
  if (B == 1 && D == 128) {
    // one query per head: warp-independent 128-token tiles, clusters of up
    // to 16 CTAs per head with two tiles or more each, one wave of CTAs
    CUtensorMap qm[4];
    for (int i = 0; i < 4; ++i) {
      const bool codes = i < 2;
      const cuuint64_t dims[2] = {codes ? static_cast<cuuint64_t>(H) * RB : static_cast<cuuint64_t>(H),
                                  static_cast<cuuint64_t>(T)};
      const cuuint64_t strides[1] = {codes ? static_cast<cuuint64_t>(H) * RB : static_cast<cuuint64_t>(H) * 4};
      const cuuint32_t box[2] = {codes ? static_cast<cuuint32_t>(RB) : 4u, static_cast<cuuint32_t>(attn::Q1_TT)};
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
    int S = 1;
    while (S < 16 && T / (4 * S) >= attn::Q1_TT && H * S * 2 <= 6 * num_sms()) S *= 2;
    auto kern = attn::kv_attention_q1_kernel<128>;
    const int smem = static_cast<int>(sizeof(attn::SmemQ1<128>));
    cudaError_t e = set_smem_limit(kern, smem);
    if (e != cudaSuccess) return e;
    if (S > 8) {
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) return e;
    }
    return launch_kernel(kern, dim3(static_cast<unsigned>(S), static_cast<unsigned>(H), 1u), dim3(attn::Q1_TT),
                         static_cast<size_t>(smem), s, static_cast<unsigned>(S), qm[0], qm[1], qm[2], qm[3], p);
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
