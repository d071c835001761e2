"""Pins for the CPU oracle: worked examples, closed forms, invariants,
library special cases and brute force on tiny inputs. CPU only."""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

from conftest import golden
from oracle import bitlinear_oracle as O
import workloads as W


def f32(vals):
    return np.array([float(v) for v in vals], dtype=np.float32)


def bits_of(vals):
    return O.f32_to_bf16(f32(vals))


# ------------------------------------------------------------------ bf16 helpers
def test_f32_to_bf16_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(10000).astype(np.float32) * 100,
                        f32([0.0, -0.0, 1.0, 1.00390625, 1.001953125, -3.0e-39, 65504.0])])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(O.f32_to_bf16(x), ref)
    assert np.array_equal(O.bf16_to_f32(ref), torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).float().numpy())


def _nearest_bf16_bruteforce(v: float) -> int:
    """Exact nearest-even bf16 of a double by rational comparison of neighbours."""
    if v == 0.0:
        return 0
    fv = Fraction(v)
    t = int(np.float32(v).view(np.uint32)) & 0xFFFF0000
    cands = [t - 0x10000, t, t + 0x10000, t + 0x20000]
    best = None
    for c in cands:
        val = Fraction(float(np.uint32(c & 0xFFFFFFFF).view(np.float32)))
        d = abs(val - fv)
        key = (d, (c >> 16) & 1)  # prefer even mantissa on ties
        if best is None or key < best[0]:
            best = (key, c)
    return (best[1] >> 16) & 0xFFFF


def test_bf16_ulp_diff_hand_pairs():
    """The checker behind every bf16 parity verdict, on pairs whose distance
    follows from the bf16 format (1 sign, 8 exponent, 7 mantissa bits)."""
    pairs = [
        (0x3F80, 0x3F81, 1),       # 1.0 and the next value up: one mantissa step
        (0x3F80, 0x3F7F, 1),       # 1.0 and the value below it (exponent changes)
        (0x0001, 0x8001, 2),       # +/- smallest subnormal: -d -> 0 -> +d
        (0x0000, 0x8000, 0),       # +0 and -0 are the same value
        (0x8000, 0x0001, 1),       # -0 (= 0) to the smallest subnormal
        (0x7F7F, 0x7F7E, 1),       # largest finite and the one below it
        (0xFF7F, 0xFF7E, 1),       # the same pair, negative
        (0x3F80, 0x4000, 128),     # 1.0 -> 2.0: the 2^7 mantissa steps of one binade
        (0xBF80, 0x3F80, 2 * 0x3F80),  # -1 -> +1: every step from 0 to 1, twice
        (0xC2F6, 0xC2F6, 0),       # equal patterns
    ]
    a = np.array([p[0] for p in pairs], np.uint16)
    b = np.array([p[1] for p in pairs], np.uint16)
    assert O.bf16_ulp_diff(a, b).tolist() == [p[2] for p in pairs]
    assert O.bf16_ulp_diff(b, a).tolist() == [p[2] for p in pairs]  # symmetric


def test_bf16_ulp_diff_matches_rank_of_finite_values():
    """Brute force: the distance equals the difference of the two values'
    ranks among all distinct finite bf16 values in increasing order (+0 and
    -0 one value), computed from the decoded floats alone."""
    allbits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = O.bf16_to_f32(allbits)
    finite = np.isfinite(vals)
    ranks_of = np.unique(vals[finite])  # sorted distinct values, -0 == +0
    rng = np.random.default_rng(7)
    fb = allbits[finite]
    a = rng.choice(fb, 20000)
    b = np.where(rng.random(20000) < 0.5, rng.choice(fb, 20000),
                 (a.astype(np.int32) + rng.integers(-3, 4, 20000)).astype(np.uint16))
    ok = np.isfinite(O.bf16_to_f32(b))
    a, b = a[ok], b[ok]
    ra = np.searchsorted(ranks_of, O.bf16_to_f32(a))
    rb = np.searchsorted(ranks_of, O.bf16_to_f32(b))
    assert np.array_equal(O.bf16_ulp_diff(a, b), np.abs(ra - rb))


def test_f64_to_bf16_exact_rounding():
    rng = np.random.default_rng(1)
    vals = list(rng.standard_normal(300) * 10.0 ** rng.integers(-5, 5, 300))
    # exact ties between bf16 neighbours (1 + 2^-8 is halfway between 1 and 1+2^-7)
    vals += [1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 1.0 + 2.0 ** -8 + 2.0 ** -40,
             1.0 + 2.0 ** -8 - 2.0 ** -40, 3.0 * (1.0 + 2.0 ** -8)]
    got = O.f64_to_bf16(np.array(vals))
    want = np.array([_nearest_bf16_bruteforce(v) for v in vals], dtype=np.uint16)
    assert np.array_equal(got, want)


# --------------------------------------------------------------- C1 ternarise
@pytest.mark.parametrize("case", ["A", "B", "C"])
def test_ternarize_golden(case):
    g = golden("ternarize_ties.txt")
    Wm = f32(g[f"W_{case}"]).reshape(2, 2)
    Wt, gamma = O.ternarize(Wm, (2,))
    assert Wt.ravel().tolist() == [int(v) for v in g[f"Wt_{case}"]]
    if f"gamma_{case}" in g:
        assert gamma[0] == np.float32(float(g[f"gamma_{case}"][0]))


def test_ternarize_closed_form_and_invariants():
    Wm = W.weights(np.random.default_rng(7), 256, 512)
    Wt, gamma = O.ternarize(Wm, (256, 512))
    assert set(np.unique(Wt)) <= {-1, 0, 1}
    # zero fraction of absmean-ternarised Gaussian weights (closed form 0.3101)
    assert abs((Wt == 0).mean() - O.zero_fraction_gaussian_ternary()) < 0.01
    # gamma per group equals the correctly rounded mean |W| (fsum) within 1 fp32 ulp
    for gi, (s, e) in enumerate([(0, 256), (256, 512)]):
        ref = math.fsum(abs(float(v)) for v in Wm[:, s:e].ravel()) / Wm[:, s:e].size
        assert abs(float(gamma[gi]) - ref) <= float(np.spacing(np.float32(ref)))
    # the dequantised weight is a nearest point of {-g, 0, g} to W
    gcol = O.gamma_per_column(gamma, (256, 512)).astype(np.float64)
    dq = Wt * gcol[None, :]
    cands = np.stack([-gcol, 0 * gcol, gcol])[:, None, :]
    dist = np.abs(Wm.astype(np.float64)[None] - cands)
    assert np.all(np.abs(Wm - dq) <= dist.min(axis=0) * (1 + 1e-6) + 1e-12)


def test_ternarize_group_scale_equivariance():
    Wm = W.weights(np.random.default_rng(8), 64, 96)
    Wt, gamma = O.ternarize(Wm, (32, 96))
    W2 = Wm.copy()
    W2[:, 32:] *= np.float32(8.0)  # power of two: exact in fp32
    Wt2, gamma2 = O.ternarize(W2, (32, 96))
    assert np.array_equal(Wt, Wt2)
    assert gamma2[0] == gamma[0] and gamma2[1] == np.float32(8.0) * gamma[1]


# ------------------------------------------------------------------ C2 packing
def test_pack_golden():
    g = golden("pack_layout.txt")
    col = np.array([int(v) for v in g["Wt_col"]], dtype=np.int8).reshape(16, 1)
    Wp = O.pack_ternary(col)
    assert Wp[0].tolist() == [int(b, 16) for b in g["bytes"]]


def test_pack_roundtrip_and_no_code3():
    rng = np.random.default_rng(3)
    Wt = rng.integers(-1, 2, size=(128, 40)).astype(np.int8)
    Wp = O.pack_ternary(Wt)
    assert Wp.shape == (40, 32)
    assert np.array_equal(O.unpack_ternary(Wp, 128), Wt)
    fields = np.stack([(Wp >> s) & 3 for s in (0, 2, 4, 6)])
    assert not np.any(fields == 3)
    # moving one weight moves exactly one 2-bit field
    Wt2 = Wt.copy()
    Wt2[37, 5] = 1 if Wt[37, 5] != 1 else -1
    diff = np.argwhere(O.pack_ternary(Wt2) != Wp)
    assert diff.shape[0] == 1 and diff[0, 0] == 5 and diff[0, 1] // 4 == 37 // 16


# -------------------------------------------------------------- C3 INT8 / INT4
def test_quant_int_golden():
    g = golden("quant_int_rows.txt")
    x = f32(g["x"]).reshape(1, 4)
    q8, xs8 = O.quant_int(x, 127)
    q4, xs4 = O.quant_int(x, 7)
    assert q8[0].tolist() == [int(v) for v in g["int8_codes"]]
    assert q4[0].tolist() == [int(v) for v in g["int4_codes"]]
    assert xs8[0] == np.float32(4) / np.float32(127)
    assert xs4[0] == np.float32(4) / np.float32(7)
    qz, xsz = O.quant_int(np.zeros((1, 4), np.float32), 127)
    assert qz[0].tolist() == [int(v) for v in g["zero_row_codes"]]
    assert xsz[0] == np.float32(1e-5) / np.float32(127)


@pytest.mark.parametrize("Q", [7, 127])
def test_quant_int_invariants(Q):
    rng = np.random.default_rng(Q)
    x = O.bf16_to_f32(W.student_t_bf16(rng, 64, 300))
    q, xs = O.quant_int(x, Q)
    assert q.min() >= -Q and q.max() <= Q
    am = np.argmax(np.abs(x), axis=1)
    assert np.all(np.abs(q[np.arange(64), am]) == Q)
    a = np.abs(x).max(axis=1).astype(np.float64)
    err = np.abs(x.astype(np.float64) - q.astype(np.float64) * xs.astype(np.float64)[:, None])
    assert np.all(err <= (a / (2 * Q) * (1 + 1e-5))[:, None])
    # sign is preserved wherever the code is non-zero
    assert np.all(np.sign(q[q != 0]) == np.sign(x[q != 0]))


# ------------------------------------------------------------------- C4 e2m1
def test_e2m1_golden_table():
    rows = golden("e2m1_table.txt")["_rows"]
    v = f32([r[0] for r in rows])
    want = [int(r[1], 16) for r in rows]
    assert O.e2m1_code(v).tolist() == want


def test_e2m1_bruteforce_nearest_even():
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    vals = np.concatenate([np.linspace(-7, 7, 20001, dtype=np.float32), f32(mids),
                           np.nextafter(f32(mids), np.float32(10)),
                           np.nextafter(f32(mids), np.float32(-10)), -f32(mids)])
    codes = O.e2m1_code(vals)
    for v, c in zip(vals.astype(np.float64), codes):
        m = min(abs(v), 6.0)
        d = np.abs(grid - m)
        best = np.flatnonzero(d == d.min())
        idx = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]
        assert (c & 7) == idx, (v, c)
        assert (c >> 3) == (1 if np.signbit(np.float32(v)) else 0)


def test_quant_fp4_invariants():
    rng = np.random.default_rng(11)
    x = O.bf16_to_f32(W.normal_bf16(rng, (32, 256)))
    codes, xs = O.quant_fp4(x)
    am = np.argmax(np.abs(x), axis=1)
    assert np.all((codes[np.arange(32), am] & 7) == 7)
    val = O.e2m1_value(codes) * xs.astype(np.float64)[:, None]
    a = np.abs(x).max(axis=1).astype(np.float64)
    # the largest gap of the grid is 2 (between 4 and 6): error <= 1 step of xs
    assert np.all(np.abs(val - x) <= (a / 6.0 * 1.0 + 1e-9)[:, None])
    packed = O.pack_nibbles(codes)
    assert np.array_equal(O.unpack_nibbles(packed), codes)
    assert (packed[0, 0] & 0xF) == codes[0, 0] and (packed[0, 0] >> 4) == codes[0, 1]


# ------------------------------------------------------------------ C5 top-k
def test_topk_golden_ties():
    g = golden("topk_ties.txt")
    xb = bits_of(g["x"]).reshape(1, -1)
    for k in (3, 4, 5):
        assert O.topk_keep_mask(xb, k)[0].astype(int).tolist() == [int(v) for v in g[f"mask_k{k}"]]
    q, xs, mask = O.topk_sparsify_i8(xb, 4)
    assert q[0].tolist() == [int(v) for v in g["codes_k4"]]
    assert O.pack_mask_bits(mask).tolist() == [[int(g["mask_k4_byte"][0], 16)]]


@pytest.mark.parametrize("K", [64, 255, 4096])
def test_topk_invariants(K):
    rng = np.random.default_rng(K)
    # coarse values: many exact ties in |x|
    x = np.round(rng.standard_t(3, size=(16, K)) * 4) / 4
    xb = O.f32_to_bf16(x.astype(np.float32))
    k = (K + 1) // 2
    q, xs, mask = O.topk_sparsify_i8(xb)
    key = (xb & 0x7FFF).astype(np.int64)
    assert np.all(mask.sum(axis=1) == k)
    for r in range(16):
        kept, dropped = key[r][mask[r]], key[r][~mask[r]]
        assert kept.min() >= dropped.max()
        thr = kept.min()
        ki = np.flatnonzero(mask[r] & (key[r] == thr))
        di = np.flatnonzero(~mask[r] & (key[r] == thr))
        if len(di):
            assert ki.max() < di.min()
    assert np.all(q[~mask] == 0)
    assert np.count_nonzero(q, axis=1).max() <= k


# ----------------------------------------------------------------- C6 ReLU^2
def test_relu2_gate():
    rng = np.random.default_rng(5)
    g = W.normal_bf16(rng, (8, 512))
    u = W.normal_bf16(rng, (8, 512))
    h = O.relu2_gate(g, u)
    gf, uf = O.bf16_to_f32(g).astype(np.float64), O.bf16_to_f32(u).astype(np.float64)
    assert np.all(h[gf <= 0] == 0)
    ref = np.maximum(gf, 0) ** 2 * uf
    assert np.all(np.abs(h - ref) <= np.abs(ref) * 2.0 ** -22)
    assert 0.45 < (h == 0).mean() < 0.55  # half the gate values are <= 0


# -------------------------------------------------------------- C7/C8 GEMMs
def test_gemm_int_bruteforce():
    rng = np.random.default_rng(9)
    M, K, N = 5, 48, 7
    xq = rng.integers(-128, 128, size=(M, K)).astype(np.int8)
    Wt = rng.integers(-1, 2, size=(K, N)).astype(np.int8)
    acc = O.gemm_acc_int(xq, Wt)
    for m in range(M):
        for n in range(N):
            assert acc[m, n] == sum(int(xq[m, k]) * int(Wt[k, n]) for k in range(K))
    big_x = rng.integers(-128, 128, size=(64, 2048)).astype(np.int64)
    big_w = rng.integers(-1, 2, size=(2048, 96)).astype(np.int64)
    assert np.array_equal(O.gemm_acc_int(big_x, big_w), big_x @ big_w)  # int64 matmul


def test_gemm_fp4_bruteforce():
    rng = np.random.default_rng(10)
    codes = rng.integers(0, 16, size=(4, 32)).astype(np.uint8)
    Wt = rng.integers(-1, 2, size=(32, 5)).astype(np.int8)
    acc = O.gemm_acc_fp4(codes, Wt)
    mags = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3),
            Fraction(4), Fraction(6)]
    for m in range(4):
        for n in range(5):
            s = sum((-mags[c & 7] if c & 8 else mags[c & 7]) * int(Wt[k, n])
                    for k, c in enumerate(codes[m]))
            assert Fraction(acc[m, n]) == s


def test_epilogue_exact_rounding_and_zero():
    rng = np.random.default_rng(12)
    acc = rng.integers(-5000, 5000, size=(6, 9))
    acc[0, 0] = 0
    xs = rng.uniform(0.001, 1, 6).astype(np.float32)
    gcol = rng.uniform(0.001, 0.1, 9).astype(np.float32)
    y = O.epilogue_bf16(acc, xs, gcol)
    for m in range(6):
        for n in range(9):
            exact = Fraction(int(acc[m, n])) * Fraction(float(xs[m])) * Fraction(float(gcol[n]))
            assert y[m, n] == _nearest_bf16_bruteforce(float(exact))
    assert np.array_equal(y == 0, acc == 0)


def test_bitlinear_tracks_float_matmul():
    """The quantised layer approximates X @ W (catches transposed operands)."""
    d = W.single_w2a4()
    Wm = d["proj"].W
    Wt, gamma = O.ternarize(Wm, (256,))
    xf = O.bf16_to_f32(d["x"]).astype(np.float64)
    ref = xf @ (Wt * gamma[0]).astype(np.float64)
    for mode in (O.MODE_INT8, O.MODE_INT4):
        q, xs = O.quant_act(d["x"], mode)
        acc, y = O.bitlinear_int(q, xs, Wt, gamma, (256,))
        got = O.bf16_to_f32(y).astype(np.float64)
        cos = (got * ref).sum() / np.linalg.norm(got) / np.linalg.norm(ref)
        assert cos > (0.999 if mode == O.MODE_INT8 else 0.97)
    f4, xs4 = O.quant_act(d["x"], O.MODE_FP4)
    acc, y = O.bitlinear_fp4(f4, xs4, Wt, gamma, (256,))
    got = O.bf16_to_f32(y).astype(np.float64)
    assert (got * ref).sum() / np.linalg.norm(got) / np.linalg.norm(ref) > 0.97
    # the ternary layer itself tracks the full-precision one loosely
    full = xf @ Wm.astype(np.float64)
    assert (ref * full).sum() / np.linalg.norm(ref) / np.linalg.norm(full) > 0.8


# ------------------------------------------------------------------- C9 KV
def test_kv_golden():
    g = golden("kv_pack.txt")
    x = f32(g["x"])
    kv = O.f32_to_bf16(np.stack([x, x]).reshape(2, 1, 8))
    c3, c4, s = O.kv_quant_3bit(kv, (0,))
    assert c3[1, 0].tolist() == [int(b, 16) for b in g["codes3_t1"]]
    assert c3[0, 0].tolist() == [int(b, 16) for b in g["codes3_t0"]]
    assert c4[0, 0].tolist() == [int(b, 16) for b in g["codes4_t0"]]
    assert s[1, 0] == np.float32(float(g["scale_t1"][0]))
    assert s[0, 0] == np.float32(3) / np.float32(7)


def test_keep4_positions_golden():
    g = golden("keep4_ids.txt")
    ids = np.array([int(v) for v in g["ids"]], np.int32)
    got = O.keep4_positions(ids, [int(v) for v in g["special"]])
    assert got.dtype == np.int32 and got.tolist() == [int(v) for v in g["positions"]]
    got = O.keep4_positions(ids, [int(v) for v in g["special_bos"]])
    assert got.tolist() == [int(v) for v in g["positions_bos"]]
    assert O.keep4_positions(np.zeros(0, np.int32), [1]).size == 0
    assert O.keep4_positions(ids, [99]).size == 0


def test_kv_invariants_and_roundtrip():
    rng = np.random.default_rng(13)
    T, H, D = 20, 4, 128
    kv = W.normal_bf16(rng, (T, H, D))
    keep = (0, 7)
    c3, c4, s = O.kv_quant_3bit(kv, keep)
    assert c3.shape == (T, H, 48) and c4.shape == (2, H, 64) and s.shape == (T, H)
    deq = O.kv_dequant(c3, c4, s, keep, D)
    x = O.bf16_to_f32(kv).astype(np.float64)
    a = np.maximum(np.abs(x).max(axis=2), 1e-5)
    Q = np.full(T, 3.0)
    Q[list(keep)] = 7.0
    err = np.abs(deq - x)
    assert np.all(err <= (a / (2 * Q[:, None]) * (1 + 1e-5))[:, :, None])
    bits = np.unpackbits(c3, axis=2, bitorder="little")
    u3 = bits[:, :, 0::3] | (bits[:, :, 1::3] << 1) | (bits[:, :, 2::3] << 2)
    rest = [t for t in range(T) if t not in keep]
    assert u3[rest].min() >= 1 and u3[rest].max() <= 7   # codes in [-3, 3]
    assert np.all(c3[list(keep)] == 0)


# ---------------------------------------------------------- C10 attention
def _kv_store(rng, T, H, D, keep):
    kv = W.normal_bf16(rng, (T, H, D))
    return O.kv_quant_3bit(kv, keep), kv


def test_attention_single_token_returns_its_value_row():
    """One cached token: softmax weight 1, the output is that token's
    dequantised value row (exactly, before the bf16 rounding)."""
    rng = np.random.default_rng(40)
    (ks, _), (vs, _) = _kv_store(rng, 1, 2, 64, (0,)), _kv_store(rng, 1, 2, 64, (0,))
    q = W.normal_bf16(rng, (3, 2, 64))
    o = O.kv_attention_f64(q, ks, vs, (0,))
    v = O.kv_dequant(*vs, (0,), 64)
    assert np.array_equal(o, np.broadcast_to(v[0], (3, 2, 64)))


def test_attention_zero_query_is_the_mean_value():
    rng = np.random.default_rng(41)
    T, H, D = 37, 3, 128
    ks, _ = _kv_store(rng, T, H, D, (0, 5))
    vs, _ = _kv_store(rng, T, H, D, (0, 5))
    q = np.zeros((1, H, D), dtype=np.uint16)  # +0.0 in bf16
    o = O.kv_attention_f64(q, ks, vs, (0, 5))
    v = O.kv_dequant(*vs, (0, 5), D)
    assert np.allclose(o[0], v.mean(axis=0), rtol=1e-12, atol=1e-14)


def test_attention_two_tokens_closed_form():
    """Two tokens, one head: o = (e^a v0 + e^b v1) / (e^a + e^b) with a, b
    the two scaled scores, written out with scalar math."""
    rng = np.random.default_rng(42)
    D = 64
    ks, _ = _kv_store(rng, 2, 1, D, ())
    vs, _ = _kv_store(rng, 2, 1, D, ())
    q = W.normal_bf16(rng, (1, 1, D))
    k = O.kv_dequant(*ks, (), D)[:, 0]
    v = O.kv_dequant(*vs, (), D)[:, 0]
    qf = O.bf16_to_f32(q)[0, 0].astype(np.float64)
    a = sum(float(qf[d]) * float(k[0, d]) for d in range(D)) / math.sqrt(D)
    b = sum(float(qf[d]) * float(k[1, d]) for d in range(D)) / math.sqrt(D)
    ea, eb = math.exp(a - max(a, b)), math.exp(b - max(a, b))
    want = [(ea * float(v[0, d]) + eb * float(v[1, d])) / (ea + eb) for d in range(D)]
    o = O.kv_attention_f64(q, ks, vs, ())
    assert np.allclose(o[0, 0], want, rtol=1e-12, atol=1e-14)


def test_attention_token_order_invariance():
    """Permuting the cached tokens (and the 4-bit list with them) leaves the
    output unchanged."""
    rng = np.random.default_rng(43)
    T, H, D = 29, 2, 64
    k_bits = W.normal_bf16(rng, (T, H, D))
    v_bits = W.normal_bf16(rng, (T, H, D))
    keep = (0, 11)
    q = W.normal_bf16(rng, (2, H, D))
    o1 = O.kv_attention_f64(q, O.kv_quant_3bit(k_bits, keep), O.kv_quant_3bit(v_bits, keep), keep)
    perm = rng.permutation(T)
    inv = np.argsort(perm)
    keep2 = tuple(sorted(int(inv[t]) for t in keep))
    o2 = O.kv_attention_f64(q, O.kv_quant_3bit(k_bits[perm], keep2), O.kv_quant_3bit(v_bits[perm], keep2),
                            keep2)
    assert np.allclose(o1, o2, rtol=1e-12, atol=1e-14)
