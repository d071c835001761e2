"""CPU oracle for the BitNet a4.8 BitLinear forward: TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this module. The product path (the CUDA library and its
Python binding) never calls it and shares no code with it.

What it computes, and where the pages say so
--------------------------------------------
Sources (five web pages on one subject):
  [R]  "BitNet a4.8: 4-bit Activations for 1-bit LLMs", Telegram review
       (t.center/ru/toshoseti/992), sections "Метод" and "Эксперименты".
  [A]  "BitNet a4.8: 4-bit Activations for 1-bit LLMs", arXiv 2411.04965
       summary page, section "摘要（原文）" (the English abstract) and
       section "方法详解" (method details, "技术框架" / "关键设计").
  [N]  "This AI Paper Introduces BitNet a4.8 ..." (9pt.com news article),
       paragraph on activation sparsity.

  * weights are ternary {-1, 0, +1}            -- [R] "Метод" (BitNet b1.58 lineage)
  * 4-bit activations (INT4 or FP4) on the inputs of the attention and
    FFN projections (q, k, v, gate, up)         -- [A] abstract; [R] "Метод"
  * FP4 as the alternative to INT4              -- [R] "Метод"
  * the o_proj input is sparsified by top-k at 50% and then quantised to
    8 bits                                      -- [R] "Метод"; [A] abstract; [N]
  * the FFN gate uses ReLU^2, and the down_proj input (the gated product)
    is quantised to 8 bits                      -- [R] "Метод"; [A] abstract
  * activations were absmax-quantised to INT8 in the predecessor  -- [R] "Метод"
  * KV cache at 3 bits except the <bos>/<eos> tokens at 4 bits   -- [R] "Эксперименты"

The pages give no formula for any quantiser, no rounding rule, no epsilon,
no packing format and no tie rule. The readings used here (the same ones the
CUDA library implements from its own code) are:

  C1 ternarisation: per column group g, gamma_g = (float32)(sum |W| in fp64,
     summed sequentially in row-major (k, then n) order / count);
     gamma' = max(gamma_g, 1e-5); W_t = clamp(rne(W / gamma'), -1, 1) with
     fp32 division.
  C2 packing: code c = W_t + 1 in {0,1,2}; row n of Wp holds K/4 bytes; the
     32-bit little-endian word j of a row covers k = 16j .. 16j+15 and holds
     element 16j + 8h + i (h in {0,1}, i in 0..7) in bits [4i + 2h, 4i + 2h + 2).
  C3 per-token absmax INT8 / INT4 (Q = 127 / 7), fp32: a = max|x|,
     a' = max(a, 1e-5), inv = Q / a', q = clamp(rne(x * inv), -Q-1, Q),
     xs = a' / Q.
  C4 per-token FP4 (e2m1): inv = 6 / a', v = x * inv; round v to the e2m1
     grid {0, .5, 1, 1.5, 2, 3, 4, 6} to nearest, ties to the even code,
     saturating at 6; the sign bit is the sign of v; xs = a' / 6.
  C5 top-k: k = ceil(K/2); key = |x| as the bf16 magnitude bits; keep the k
     largest keys, ties at the threshold kept lowest column index first;
     the rest become 0; then C3 with Q = 127.
  C6 ReLU^2 gate: r = (g > 0 ? g : 0), h = (r * r) * u in fp32, then C3.
  C7 accumulators: integer sum of codes x ternary weights (exact); FP4:
     sum of e2m1 values x ternary weights (exact in fp32 and fp64).
  C8 output: y = bf16_rne(acc * xs[m] * gamma[g(n)]), evaluated here in fp64.
  C9 KV: per (token, head), a' = max(max_d |x|, 1e-5); Q = 3, codes
     clamp(rne(x * (Q / a')), -4, 3), stored as code + 4 in a little-endian
     3-bit stream (code d in bits [3d, 3d+3)); tokens listed in keep4_pos use
     Q = 7, clamp [-8, 7], stored as code + 8, two per byte, low nibble first;
     their 3-bit row is all zero bytes. scale = a' / Q. The listed tokens are
     those whose id is one of the special ids (bos, eos), in position order.
  C10 decode attention over that cache (the pages name only its storage
     precision): softmax((q . k_t) / sqrt(D)) over every cached token t of
     the query's head, weights applied to the dequantised v_t; fp64 here.

Quantisation decisions are taken in fp32 (the precision of the kernels),
because a float decides an integer there; everything else is fp64 or exact.
"""
from __future__ import annotations

import math

import numpy as np

EPS = np.float32(1e-5)
Q_INT8 = 127
Q_INT4 = 7
Q_FP4 = 6  # the largest e2m1 magnitude
E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)

MODE_INT8, MODE_INT4, MODE_FP4 = 0, 1, 2


# ---------------------------------------------------------------- bf16 helpers
def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> fp32 (exact: bf16 is the top half of fp32)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(x) -> np.ndarray:
    """fp32 values -> bf16 bits, round to nearest even (finite inputs)."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return b.astype(np.uint16)


def bf16_ulp_diff(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    """Distance in bf16 ulps between two arrays of bf16 bit patterns."""
    def ordered(bits):
        b = np.asarray(bits, dtype=np.uint16).astype(np.int32)
        return np.where(b & 0x8000, -(b & 0x7FFF), b)
    return np.abs(ordered(a_bits) - ordered(b_bits))


# ------------------------------------------------------- C1/C2 weights (offline)
def ternarize(W: np.ndarray, group_ends) -> tuple[np.ndarray, np.ndarray]:
    """Absmean ternarisation per column group (C1).

    W: fp32 [K x N] (in x out). group_ends: increasing column ends, last == N.
    Returns W_t int8 [K x N] in {-1,0,1} and gamma fp32 [G] (already max'ed with eps).
    """
    W = np.asarray(W, dtype=np.float32)
    K, N = W.shape
    assert group_ends[-1] == N
    Wt = np.empty((K, N), dtype=np.int8)
    gammas = []
    start = 0
    for end in group_ends:
        blk = W[:, start:end]
        # sequential fp64 sum in row-major order (cumsum is strictly sequential)
        total = np.cumsum(np.abs(blk.astype(np.float64)).ravel(order="C"))[-1]
        g = np.float32(total / float(blk.size))
        g = max(g, EPS)
        r = np.rint(blk / np.float32(g))  # fp32 IEEE division, then RNE
        Wt[:, start:end] = np.clip(r, -1, 1).astype(np.int8)
        gammas.append(g)
        start = end
    return Wt, np.array(gammas, dtype=np.float32)


def gamma_per_column(gamma: np.ndarray, group_ends) -> np.ndarray:
    out = np.empty(group_ends[-1], dtype=np.float32)
    start = 0
    for g, end in zip(gamma, group_ends):
        out[start:end] = g
        start = end
    return out


def pack_ternary(Wt: np.ndarray) -> np.ndarray:
    """C2: W_t [K x N] -> Wp uint8 [N x K/4]."""
    K, N = Wt.shape
    assert K % 16 == 0
    c = (Wt.T.astype(np.int64) + 1)  # [N x K], codes 0..2
    words = np.zeros((N, K // 16), dtype=np.int64)
    for h in range(2):
        for i in range(8):
            # element 16j + 8h + i of every word j
            words |= c[:, 8 * h + i::16] << (4 * i + 2 * h)
    out = np.zeros((N, K // 4), dtype=np.uint8)
    for b in range(4):
        out[:, b::4] = ((words >> (8 * b)) & 0xFF).astype(np.uint8)
    return out


def unpack_ternary(Wp: np.ndarray, K: int) -> np.ndarray:
    """Inverse of C2: Wp uint8 [N x K/4] -> W_t int8 [K x N]."""
    N = Wp.shape[0]
    b = Wp.astype(np.int64)
    words = b[:, 0::4] | (b[:, 1::4] << 8) | (b[:, 2::4] << 16) | (b[:, 3::4] << 24)
    Wt = np.empty((N, K), dtype=np.int8)
    for h in range(2):
        for i in range(8):
            code = (words >> (4 * i + 2 * h)) & 3
            Wt[:, 8 * h + i::16] = (code - 1).astype(np.int8)
    return Wt.T.copy()


# ------------------------------------------------- C3/C4/C6 activation quantisers
def row_absmax(x: np.ndarray) -> np.ndarray:
    return np.max(np.abs(x), axis=1) if x.shape[1] else np.zeros(x.shape[0], np.float32)


def quant_int(x: np.ndarray, Q: int) -> tuple[np.ndarray, np.ndarray]:
    """C3: per-token absmax quantiser on fp32 rows. Returns (codes int8, xs fp32)."""
    x = np.asarray(x, dtype=np.float32)
    a = np.maximum(row_absmax(x).astype(np.float32), EPS)
    inv = (np.float32(Q) / a).astype(np.float32)
    q = np.clip(np.rint(x * inv[:, None]), -Q - 1, Q).astype(np.int8)
    xs = (a / np.float32(Q)).astype(np.float32)
    return q, xs


def e2m1_code(v: np.ndarray) -> np.ndarray:
    """C4 rounding of fp32 values to e2m1 nibbles (sign<<3 | magnitude index).

    Magnitude index by the midpoints of the grid {0,.5,1,1.5,2,3,4,6}:
    a value exactly on a midpoint goes to the even index (even mantissa);
    anything above 5 saturates to 6 (index 7)."""
    v = np.asarray(v, dtype=np.float32)
    m = np.abs(v)
    idx = np.zeros(v.shape, dtype=np.uint8)
    # (lower midpoint, inclusive-at-midpoint?) for each step up the grid
    idx = np.where(m > 0.25, 1, idx)
    idx = np.where(m >= 0.75, 2, idx)   # 0.75 ties up to index 2 (even)
    idx = np.where(m > 1.25, 3, idx)    # 1.25 ties down to index 2
    idx = np.where(m >= 1.75, 4, idx)   # 1.75 ties up to index 4
    idx = np.where(m > 2.5, 5, idx)     # 2.5 ties down to index 4
    idx = np.where(m >= 3.5, 6, idx)    # 3.5 ties up to index 6
    idx = np.where(m > 5.0, 7, idx)     # 5 ties down to index 6; saturate above
    sign = np.signbit(v).astype(np.uint8)
    return (sign << 3) | idx.astype(np.uint8)


def e2m1_value(code: np.ndarray) -> np.ndarray:
    code = np.asarray(code, dtype=np.uint8)
    mag = E2M1_GRID[code & 7]
    return np.where(code & 8, -mag, mag)


def quant_fp4(x: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """C4: per-token absmax to e2m1. Returns (nibble codes uint8 [M x K], xs fp32)."""
    x = np.asarray(x, dtype=np.float32)
    a = np.maximum(row_absmax(x).astype(np.float32), EPS)
    inv = (np.float32(Q_FP4) / a).astype(np.float32)
    codes = e2m1_code(x * inv[:, None])
    xs = (a / np.float32(Q_FP4)).astype(np.float32)
    return codes, xs


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """[M x K] nibbles -> [M x K/2] bytes, even k in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[:, 0::2] & 0xF) | ((c[:, 1::2] & 0xF) << 4)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = p & 0xF
    out[:, 1::2] = p >> 4
    return out


def relu2_gate(gate_bits: np.ndarray, up_bits: np.ndarray) -> np.ndarray:
    """C6: h = (r*r)*u with r = g if g > 0 else 0, all in fp32."""
    g = bf16_to_f32(gate_bits)
    u = bf16_to_f32(up_bits)
    r = np.where(g > 0, g, np.float32(0.0)).astype(np.float32)
    return ((r * r) * u).astype(np.float32)


def quant_act(x_bits: np.ndarray, mode: int, up_bits: np.ndarray | None = None):
    """The per-token activation quantiser on bf16 input rows.

    mode INT8 / INT4 -> (codes int8 [M x K], xs)
    mode FP4         -> (packed e2m1 uint8 [M x K/2], xs)
    With up_bits given, the row quantised is the ReLU^2-gated product (C6)."""
    x = relu2_gate(x_bits, up_bits) if up_bits is not None else bf16_to_f32(x_bits)
    if mode == MODE_INT8:
        return quant_int(x, Q_INT8)
    if mode == MODE_INT4:
        return quant_int(x, Q_INT4)
    if mode == MODE_FP4:
        codes, xs = quant_fp4(x)
        return pack_nibbles(codes), xs
    raise ValueError(mode)


# ------------------------------------------------------------------ C5 top-k
def topk_keep_mask(x_bits: np.ndarray, k: int) -> np.ndarray:
    """C5: boolean [M x K]; per row the k largest |x| (bf16 magnitude bits),
    equal magnitudes ordered by lower column index first."""
    key = (np.asarray(x_bits, dtype=np.uint16) & 0x7FFF).astype(np.int32)
    M, K = key.shape
    order = np.argsort(-key, axis=1, kind="stable")[:, :k]
    mask = np.zeros((M, K), dtype=bool)
    np.put_along_axis(mask, order, True, axis=1)
    return mask


def topk_sparsify_i8(x_bits: np.ndarray, k: int = 0):
    """C5 then C3 (Q=127). Returns (codes int8, xs fp32, keep mask bool)."""
    K = x_bits.shape[1]
    if k <= 0:
        k = (K + 1) // 2
    mask = topk_keep_mask(x_bits, k)
    x = np.where(mask, bf16_to_f32(x_bits), np.float32(0.0)).astype(np.float32)
    q, xs = quant_int(x, Q_INT8)
    return q, xs, mask


def pack_mask_bits(mask: np.ndarray) -> np.ndarray:
    """bool [M x K] -> uint8 [M x ceil(K/8)], bit (k % 8) of byte k // 8."""
    return np.packbits(mask, axis=1, bitorder="little")


# ------------------------------------------------------- C7/C8 GEMM and output
def gemm_acc_int(xq: np.ndarray, Wt: np.ndarray) -> np.ndarray:
    """C7: exact integer accumulators acc[m, n] = sum_k xq[m,k] * Wt[k,n].

    Float64 matmul of small integers is exact (every partial sum is an
    integer below 2^53), so this is the plain definition."""
    acc = np.asarray(xq, dtype=np.float64) @ np.asarray(Wt, dtype=np.float64)
    return acc.astype(np.int64)


def gemm_acc_fp4(codes: np.ndarray, Wt: np.ndarray) -> np.ndarray:
    """C7 for e2m1 codes (unpacked nibbles): exact sums of multiples of 0.5."""
    return e2m1_value(codes) @ np.asarray(Wt, dtype=np.float64)


def epilogue_bf16(acc: np.ndarray, xs: np.ndarray, gamma_col: np.ndarray) -> np.ndarray:
    """C8: y = bf16(acc * xs[m] * gamma[n]) evaluated in fp64, rounded once."""
    y = np.asarray(acc, dtype=np.float64) * xs.astype(np.float64)[:, None] \
        * gamma_col.astype(np.float64)[None, :]
    return f64_to_bf16(y)


def f64_to_bf16(y: np.ndarray) -> np.ndarray:
    """Correct bf16 rounding of fp64 values, vectorised.

    Split y = t + r where t is y truncated to bf16 (toward zero) and compare
    the remainder with half a bf16 ulp, exactly in fp64."""
    y = np.atleast_1d(np.asarray(y, dtype=np.float64))
    f = np.ascontiguousarray(y.astype(np.float32))  # may round; corrected below using exact fp64 compares
    t = (f.view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32).astype(np.float64)
    # make t the truncation (toward zero) of y to bf16
    over = np.abs(t) > np.abs(y)
    tb = (t.astype(np.float32).view(np.uint32)).astype(np.int64)
    tb = np.where(over, tb - 0x10000, tb)
    t = tb.astype(np.uint32).view(np.float32).astype(np.float64)
    nb = tb + 0x10000
    nxt = nb.astype(np.uint32).view(np.float32).astype(np.float64)
    d_lo = np.abs(y - t)
    d_hi = np.abs(nxt - y)
    even = ((tb >> 16) & 1) == 0
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & ~even)
    pick_hi &= (y != 0.0)
    res = np.where(pick_hi, nb, np.where(y == 0.0, 0, tb))
    return (res >> 16).astype(np.uint16)


def bitlinear_int(xq, xs, Wt, gamma, group_ends):
    acc = gemm_acc_int(xq, Wt)
    return acc, epilogue_bf16(acc, xs, gamma_per_column(gamma, group_ends))


def bitlinear_fp4(xf4_packed, xs, Wt, gamma, group_ends):
    acc = gemm_acc_fp4(unpack_nibbles(xf4_packed), Wt)
    return acc, epilogue_bf16(acc, xs, gamma_per_column(gamma, group_ends))


# -------------------------------------------------------------- C9 KV cache
def keep4_positions(token_ids, special_ids):
    """C9: the positions whose token id is one of special_ids (the bos and eos
    ids), in increasing order, as int32."""
    ids = np.asarray(token_ids, dtype=np.int64)
    hit = np.zeros(ids.shape, dtype=bool)
    for v in special_ids:
        hit |= ids == int(v)
    return np.flatnonzero(hit).astype(np.int32)


def kv_quant_3bit(kv_bits: np.ndarray, keep4_pos=(0,)):
    """C9 per (token, head) KV quantiser.

    kv_bits: bf16 bits [T x H x D] (D % 8 == 0). keep4_pos: sorted token
    positions stored at 4 bits. Returns (codes3 uint8 [T x H x 3D/8],
    codes4 uint8 [n4 x H x D/2], scale fp32 [T x H])."""
    kv = bf16_to_f32(kv_bits)
    T, H, D = kv.shape
    keep = np.zeros(T, dtype=bool)
    keep4_pos = np.asarray(keep4_pos, dtype=np.int64)
    keep[keep4_pos] = True
    a = np.maximum(np.max(np.abs(kv), axis=2), EPS).astype(np.float32)  # [T x H]
    Q = np.where(keep, np.float32(7), np.float32(3)).astype(np.float32)[:, None]
    inv = (Q / a).astype(np.float32)
    r = np.rint(kv * inv[:, :, None])
    lo = np.where(keep, -8, -4)[:, None, None]
    hi = np.where(keep, 7, 3)[:, None, None]
    code = np.clip(r, lo, hi).astype(np.int64)
    scale = (a / Q).astype(np.float32)

    codes3 = np.zeros((T, H, 3 * D // 8), dtype=np.uint8)
    u3 = code + 4
    for d in range(D):
        for b in range(3):
            pos = 3 * d + b
            codes3[:, :, pos // 8] |= (((u3[:, :, d] >> b) & 1) << (pos % 8)).astype(np.uint8)
    codes3[keep] = 0
    u4 = (code[keep4_pos] + 8).astype(np.uint8)  # [n4 x H x D]
    codes4 = (u4[:, :, 0::2] & 0xF) | ((u4[:, :, 1::2] & 0xF) << 4)
    return codes3, codes4.astype(np.uint8), scale


def kv_dequant(codes3, codes4, scale, keep4_pos, D):
    """Decode C9 storage back to fp64 values code * scale (for tests)."""
    T, H, _ = codes3.shape
    out = np.zeros((T, H, D), dtype=np.float64)
    bits = np.unpackbits(codes3, axis=2, bitorder="little")  # [T x H x 3D]
    u3 = bits[:, :, 0::3] | (bits[:, :, 1::3] << 1) | (bits[:, :, 2::3] << 2)
    out[:] = (u3.astype(np.int64) - 4) * scale[:, :, None]
    for j, t in enumerate(np.asarray(keep4_pos, dtype=np.int64)):
        u4 = np.empty((H, D), dtype=np.int64)
        u4[:, 0::2] = codes4[j] & 0xF
        u4[:, 1::2] = codes4[j] >> 4
        out[t] = (u4 - 8) * scale[t][:, None]
    return out


def kv_attention_probs_f64(q_bits, k_store, keep4_pos):
    """The softmax weights of the decode attention below (reading C10), fp64:
    p[b, h, t] = softmax_t((q[b,h] . k_t) / sqrt(D)) over every cached token
    t of head h, k_t the dequantised cache row. Returns p [B x H x T]."""
    q = bf16_to_f32(q_bits).astype(np.float64)
    D = q.shape[2]
    k = kv_dequant(*k_store, keep4_pos, D)  # [T x H x D]
    s = np.einsum("bhd,thd->bht", q, k) / math.sqrt(D)
    s = s - s.max(axis=2, keepdims=True)
    p = np.exp(s)
    return p / p.sum(axis=2, keepdims=True)


def kv_attention_f64(q_bits, k_store, v_store, keep4_pos):
    """Decode attention over the C9 cache (the consumer of the 3-bit KV
    quantiser; [R] "Эксперименты": 3-bit KV cache). The pages state only the
    storage precision; the attention is the plain scaled dot-product one
    (reading C10): for each query (b, h) and every cached token t of head h,
      s_t = (q . k_t) / sqrt(D),  p = softmax_t(s),  o = sum_t p_t v_t
    with k_t, v_t the dequantised cache rows (code * scale) and q the bf16
    query. Everything in fp64.

    q_bits: bf16 bits [B x H x D]; k_store, v_store: (codes3, codes4, scale)
    as returned by kv_quant_3bit. Returns o as fp64 [B x H x D]."""
    D = np.asarray(q_bits).shape[2]
    p = kv_attention_probs_f64(q_bits, k_store, keep4_pos)
    v = kv_dequant(*v_store, keep4_pos, D)
    return np.einsum("bht,thd->bhd", p, v)


def kv_attention_3bit(q_bits, k_store, v_store, keep4_pos):
    """kv_attention_f64 rounded to bf16 (nearest even)."""
    return f64_to_bf16(kv_attention_f64(q_bits, k_store, v_store, keep4_pos))


def ceil_half(K: int) -> int:
    return (K + 1) // 2


def zero_fraction_gaussian_ternary() -> float:
    """Closed form: fraction of zeros after absmean ternarisation of i.i.d.
    Gaussian weights, P(|Z| < 0.5 * E|Z|) = erf(0.5 * sqrt(2/pi) / sqrt(2))."""
    return math.erf(0.5 * math.sqrt(2.0 / math.pi) / math.sqrt(2.0))
