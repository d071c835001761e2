"""GPU parity: every C-ABI entry point against the CPU oracle on the same
seeded inputs. Integer work (codes, masks, int32 accumulators, packed bytes)
must match bit for bit; bf16 outputs within 2 bf16 ulp; FP4 fp32
accumulators within 1e-5 relative (they are exact in practice)."""
import numpy as np
import pytest
import torch

import bit_quantised_gemm_b200 as B
from conftest import attention_tolerance
from oracle import bitlinear_oracle as O
import workloads as W

pytestmark = pytest.mark.gpu
BF16_ULP_TOL = 2
FP4_REL_TOL = 1e-5
DEV = "cuda:0"


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(DEV).view(torch.bfloat16)


def host(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy()


def bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def assert_bf16_close(got_bits, want_bits, tol=BF16_ULP_TOL):
    d = O.bf16_ulp_diff(got_bits, want_bits)
    assert d.max() <= tol, f"max ulp diff {d.max()} at {np.unravel_index(d.argmax(), d.shape)}"


@pytest.fixture(autouse=True)
def _clean_status():
    B.status_buffer().zero_()
    yield
    B.check_status()


# ----------------------------------------------------------- quantisers
@pytest.mark.parametrize("mode", [O.MODE_INT8, O.MODE_INT4, O.MODE_FP4])
@pytest.mark.parametrize("M,K", [(1, 256), (17, 2048), (130, 4096 + 128), (3, 11008)])
@pytest.mark.parametrize("relu2", [False, True])
def test_quant_act_parity(mode, M, K, relu2):
    rng = np.random.default_rng(M * K + mode)
    x = W.student_t_bf16(rng, M, K)
    up = W.normal_bf16(rng, (M, K)) if relu2 else None
    q, xs = B.quant_act(dev_bf16(x), mode, up=dev_bf16(up) if relu2 else None)
    q_o, xs_o = O.quant_act(x, mode, up)
    assert np.array_equal(host(xs), xs_o)
    assert np.array_equal(host(q).view(np.uint8), q_o.view(np.uint8))


def test_quant_act_strided_rows_and_zero_row():
    rng = np.random.default_rng(5)
    x = W.normal_bf16(rng, (9, 512))
    x[4] = 0
    xt = dev_bf16(x)[:, :384]  # row stride 512, K = 384
    for mode in (O.MODE_INT8, O.MODE_INT4, O.MODE_FP4):
        q, xs = B.quant_act(xt, mode)
        q_o, xs_o = O.quant_act(np.ascontiguousarray(x[:, :384]), mode)
        assert np.array_equal(host(xs), xs_o)
        assert np.array_equal(host(q).view(np.uint8), q_o.view(np.uint8))


def test_fp4_rounding_midpoints():
    """Rows whose absmax is 6 (scale 1): every e2m1 midpoint and its bf16
    neighbours, both signs, and signed zeros."""
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    vals = []
    for m in mids:
        b = O.f32_to_bf16(np.float32(m))
        vals += [m, float(np.ravel(O.bf16_to_f32(b + 1))[0]), float(np.ravel(O.bf16_to_f32(b - 1))[0])]
    vals += [0.0, -0.0, 0.1, -0.1, 6.0, 4.0, 3.0]
    vals += [-v for v in vals]
    row = np.array(vals + [0.0] * (-len(vals) % 16), np.float32)
    row[0] = 6.0
    x = O.f32_to_bf16(np.stack([row, row * np.float32(0.5)]))
    q, xs = B.quant_act(dev_bf16(x), O.MODE_FP4)
    q_o, xs_o = O.quant_act(x, O.MODE_FP4)
    assert np.array_equal(host(q), q_o)
    assert np.array_equal(host(xs), xs_o)


@pytest.mark.parametrize("K", [64, 256, 4096, 11008, 16384])
@pytest.mark.parametrize("k", [0, 1, 7, None])
def test_topk_parity(K, k):
    rng = np.random.default_rng(K + (k or 0))
    M = 19
    xf = rng.standard_t(3, size=(M, K)).astype(np.float32)
    xf[1] = np.round(xf[1] * 2) / 2        # heavy ties
    xf[2] = 1.0                            # all equal
    xf[3] = 0.0                            # all zero
    x = O.f32_to_bf16(xf)
    kk = K if k is None else k
    q, xs, mask = B.topk_sparsify_i8(dev_bf16(x), k=kk, mask=True)
    q_o, xs_o, m_o = O.topk_sparsify_i8(x, kk if kk else 0)
    assert np.array_equal(host(mask), O.pack_mask_bits(m_o))
    assert np.array_equal(host(q), q_o)
    assert np.array_equal(host(xs), xs_o)


@pytest.mark.parametrize("K", [16, 272, 528, 1040, 2064, 4096])
def test_topk_extreme_rows(K):
    """Rows whose selection takes the rarer routes: a threshold far below the
    row maximum (wide dynamic range, a lone outlier, mostly zeros), every
    finite bf16 bit pattern, subnormal-only rows, k = 1 and k = K; one
    column count per lane width, M not a multiple of the rows per block."""
    rng = np.random.default_rng(K)
    M = 7
    xf = rng.standard_normal((M, K)).astype(np.float32)
    xf[0] = np.exp(rng.uniform(-80, 80, K)) * np.sign(rng.standard_normal(K))
    xf[1] *= 1e-3
    xf[1, K // 3] = 1e30
    xf[2, : K - K // 8] = 0.0
    x = O.f32_to_bf16(xf)
    x[3] = rng.integers(0, 0x7F80, K).astype(np.uint16) | (rng.integers(0, 2, K).astype(np.uint16) << 15)
    x[4] = rng.integers(0, 0x80, K).astype(np.uint16) | (rng.integers(0, 2, K).astype(np.uint16) << 15)
    for kk in (1, K // 2, K - 1, K):
        q, xs, mask = B.topk_sparsify_i8(dev_bf16(x), k=kk, mask=True)
        q_o, xs_o, m_o = O.topk_sparsify_i8(x, kk)
        assert np.array_equal(host(mask), O.pack_mask_bits(m_o)), kk
        assert np.array_equal(host(q), q_o), kk
        assert np.array_equal(host(xs), xs_o), kk


def test_topk_full_size_o_proj():
    d = W.o_proj_sparse(make_weights=False, M=1024)  # the o_proj input recipe, 1024 rows
    q, xs, mask = B.topk_sparsify_i8(dev_bf16(d["x"]), mask=True)
    q_o, xs_o, m_o = O.topk_sparsify_i8(d["x"])
    assert np.array_equal(host(q), q_o) and np.array_equal(host(xs), xs_o)
    assert np.array_equal(host(mask), O.pack_mask_bits(m_o))


@pytest.mark.parametrize("T,special,p", [(0, (1,), 0.0), (1, (1, 2), 1.0), (9, (1, 2), 0.3),
                                         (1024, (1, 2), 0.01), (5000, (7,), 0.5), (70000, (1, 2), 0.002),
                                         (3000, (1, 2), 0.0), (2049, (3, 1, 2, 9), 1.0)])
def test_keep4_positions_parity(T, special, p):
    """Token ids -> the sorted positions kept at 4 bits (bit-exact), several
    1024-id chunks, ragged tails, none and all matching."""
    rng = np.random.default_rng(T + len(special))
    ids = rng.integers(10, 32000, size=T).astype(np.int32)
    hit = rng.random(T) < p
    ids[hit] = rng.choice(np.array(special, np.int32), size=int(hit.sum()))
    got = B.kv_keep4_positions(torch.from_numpy(ids).to(DEV), special)
    assert np.array_equal(host(got), O.keep4_positions(ids, special))


def test_kv_quant_with_positions_from_token_ids():
    """bos / eos ids -> positions -> the 3-bit cache, against the oracle's."""
    rng = np.random.default_rng(3)
    T, H, D = 300, 4, 128
    ids = rng.integers(3, 32000, size=T).astype(np.int32)
    ids[[0, 120, 121]] = 1
    ids[[119, 299]] = 2
    kv = W.normal_bf16(rng, (T, H, D))
    pos = B.kv_keep4_positions(torch.from_numpy(ids).to(DEV), (1, 2))
    keep = O.keep4_positions(ids, (1, 2))
    assert np.array_equal(host(pos), keep)
    c3, c4, s = B.kv_quant_3bit(dev_bf16(kv), pos)
    c3_o, c4_o, s_o = O.kv_quant_3bit(kv, tuple(keep))
    assert np.array_equal(host(c3), c3_o) and np.array_equal(host(c4), c4_o)
    assert np.array_equal(host(s), s_o)


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("keep", [(0,), (0, 5, 6, 37), ()])
def test_kv_quant_parity(D, keep):
    rng = np.random.default_rng(D + len(keep))
    T, H = 41, 3
    kv = W.normal_bf16(rng, (T, H, D))
    kv[7, 1] = 0  # an all-zero head row
    kp = torch.tensor(keep, dtype=torch.int32, device=DEV) if keep else None
    c3, c4, s = B.kv_quant_3bit(dev_bf16(kv), kp)
    c3_o, c4_o, s_o = O.kv_quant_3bit(kv, keep)
    assert np.array_equal(host(s), s_o)
    assert np.array_equal(host(c3), c3_o)
    if keep:
        assert np.array_equal(host(c4), c4_o)


@pytest.mark.parametrize("D,T", [(64, 41), (128, 300), (256, 17)])
def test_kv_quant_pair_parity(D, T):
    """K and V in one launch: each cache equals the oracle's for that tensor,
    with the 4-bit tokens shared and ragged tile counts on both halves."""
    rng = np.random.default_rng(100 + D)
    H = 5
    k, v = W.normal_bf16(rng, (T, H, D)), W.normal_bf16(rng, (T, H, D))
    k[3, 2] = 0
    v[T - 1, 0] = 0
    keep = tuple(sorted({0, 1, T // 2, T - 1}))
    kp = torch.tensor(keep, dtype=torch.int32, device=DEV)
    (k3, k4, ks), (v3, v4, vs) = B.kv_quant_3bit_kv(dev_bf16(k), dev_bf16(v), kp)
    for (c3, c4, s), x in (((k3, k4, ks), k), ((v3, v4, vs), v)):
        c3_o, c4_o, s_o = O.kv_quant_3bit(x, keep)
        assert np.array_equal(host(s), s_o)
        assert np.array_equal(host(c3), c3_o)
        assert np.array_equal(host(c4), c4_o)
    (k3n, _, ksn), (v3n, _, vsn) = B.kv_quant_3bit_kv(dev_bf16(k), dev_bf16(v), None)
    for (c3, s), x in (((k3n, ksn), k), ((v3n, vsn), v)):
        c3_o, _, s_o = O.kv_quant_3bit(x, ())
        assert np.array_equal(host(s), s_o) and np.array_equal(host(c3), c3_o)


# ------------------------------------------------------------------ GEMMs
def prep_weights(K, N, groups, seed):
    Wm = W.weights(np.random.default_rng(seed), K, N)
    Wt, gamma = O.ternarize(Wm, groups)
    Wp = O.pack_ternary(Wt)
    return Wt, gamma, torch.from_numpy(Wp).to(DEV), torch.from_numpy(gamma).to(DEV)


GEMM_SHAPES = [  # (M, N, K): single tile, ragged M/N, half k-block, many tiles
    (16, 256, 256), (1, 16, 64), (130, 272, 320), (257, 512, 1024), (2048, 4096, 256),
    (300, 768, 2048 + 64), (384, 400, 384), (300, 400, 768)]


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_gemm_int8_accumulators_bit_exact(M, N, K):
    rng = np.random.default_rng(M + N + K)
    xq = rng.integers(-128, 128, size=(M, K)).astype(np.int8)
    Wt, _, Wp, _ = prep_weights(K, N, (N,), K)
    acc = B.gemm_w2a8_acc(torch.from_numpy(xq).to(DEV), Wp)
    B.check_status()
    assert np.array_equal(host(acc).astype(np.int64), O.gemm_acc_int(xq, Wt))


@pytest.mark.parametrize("M,N,K", [s for s in GEMM_SHAPES if s[2] % 128 == 0])
def test_gemm_fp4_accumulators(M, N, K):
    rng = np.random.default_rng(M * 3 + N + K)
    codes = rng.integers(0, 16, size=(M, K)).astype(np.uint8)
    xf4 = O.pack_nibbles(codes)
    Wt, _, Wp, _ = prep_weights(K, N, (N,), K + 1)
    acc = B.gemm_w2fp4_acc(torch.from_numpy(xf4).to(DEV), Wp)
    B.check_status()
    want = O.gemm_acc_fp4(codes, Wt)
    got = host(acc).astype(np.float64)
    assert np.all(np.abs(got - want) <= FP4_REL_TOL * np.maximum(np.abs(want), 1.0))
    assert np.array_equal(got, want)  # exact in practice (multiples of 0.5 < 2^24)


@pytest.mark.parametrize("mode", [O.MODE_INT8, O.MODE_INT4, O.MODE_FP4])
@pytest.mark.parametrize("M,N,K,groups", [(16, 256, 256, (256,)), (200, 768, 2048, (256, 512, 768)),
                                          (129, 1056, 512, (528, 1056))])
def test_bitlinear_layer_end_to_end(mode, M, N, K, groups):
    """bf16 X -> quantiser -> GEMM -> bf16 Y, both sides from the same X and W."""
    rng = np.random.default_rng(M + mode)
    x = W.outlier_bf16(rng, M, K)[0]
    Wt, gamma, Wp, gamma_d = prep_weights(K, N, groups, 7)
    xq_o, xs_o = O.quant_act(x, mode)
    q, xs = B.quant_act(dev_bf16(x), mode)
    if mode == O.MODE_FP4:
        y = B.gemm_w2fp4(q, xs, Wp, gamma_d, groups)
        _, y_o = O.bitlinear_fp4(xq_o, xs_o, Wt, gamma, groups)
    else:
        fn = B.gemm_w2a8 if mode == O.MODE_INT8 else B.gemm_w2a4
        y = fn(q, xs, Wp, gamma_d, groups)
        _, y_o = O.bitlinear_int(xq_o, xs_o, Wt, gamma, groups)
    B.check_status()
    assert_bf16_close(bits(y), y_o)


# M <= 8 runs the CUDA-core (dp4a) path, larger M the tensor-core path.
@pytest.mark.parametrize("M", [1, 2, 3, 4, 6, 8, 9, 17, 64])
@pytest.mark.parametrize("N,K", [(128, 128), (4096, 4096), (4096, 11008), (1024, 512)])
def test_gemv_parity(M, N, K):
    rng = np.random.default_rng(M + N + K)
    xq = rng.integers(-128, 128, size=(M, K)).astype(np.int8)
    xs = rng.uniform(0.01, 1, M).astype(np.float32)
    Wt, gamma, Wp, gamma_d = prep_weights(K, N, (N,), 11)
    y = B.gemv_w2(torch.from_numpy(xq).to(DEV), torch.from_numpy(xs).to(DEV), Wp, gamma_d, (N,))
    B.check_status()
    _, y_o = O.bitlinear_int(xq, xs, Wt, gamma, (N,))
    assert_bf16_close(bits(y), y_o)


@pytest.mark.parametrize("M,N,K", [(1, 12288, 4096), (4, 22016, 4096), (8, 12288, 4096), (6, 22016, 4096)])
def test_gemv_decode_full_size(M, N, K):
    """Fused q/k/v and gate/up projections of the decode layer at full size."""
    rng = np.random.default_rng(N + M)
    xq = rng.integers(-8, 8, size=(M, K)).astype(np.int8)
    xs = rng.uniform(0.01, 1, M).astype(np.float32)
    groups = (N // 3, 2 * N // 3, N) if N % 3 == 0 else (N // 2, N)
    Wt, gamma, Wp, gamma_d = prep_weights(K, N, groups, 13)
    y = B.gemv_w2(torch.from_numpy(xq).to(DEV), torch.from_numpy(xs).to(DEV), Wp, gamma_d, groups)
    B.check_status()
    _, y_o = O.bitlinear_int(xq, xs, Wt, gamma, groups)
    assert_bf16_close(bits(y), y_o)


_DECODE_LAUNCHES = {  # the benchmark's decode-layer launches: (N, K, column groups)
    "qkv": (12288, 4096, (4096, 8192, 12288)),
    "o": (4096, 4096, (4096,)),
    "gate_up": (22016, 4096, (11008, 22016)),
    "down": (4096, 11008, (4096,)),
}


@pytest.mark.parametrize("M,proj", [(64, "qkv"), (64, "o"), (64, "gate_up"), (64, "down"),
                                    (9, "qkv"), (33, "qkv"), (9, "gate_up"), (33, "gate_up"),
                                    (16, "down"), (48, "o")])
def test_gemv_decode_bench_launches(M, proj):
    """The tensor-core decode GEMV in exactly the launch configurations the
    benchmark times (fused q|k|v with 3 scale groups, gate|up with 2, o and
    down), every output element against the oracle."""
    N, K, groups = _DECODE_LAUNCHES[proj]
    rng = np.random.default_rng(M * 31 + N + K)
    xq = rng.integers(-128, 128, size=(M, K)).astype(np.int8)
    xs = rng.uniform(0.01, 1, M).astype(np.float32)
    Wt, gamma, Wp, gamma_d = prep_weights(K, N, groups, 23)
    y = B.gemv_w2(torch.from_numpy(xq).to(DEV), torch.from_numpy(xs).to(DEV), Wp, gamma_d, groups)
    B.check_status()
    _, y_o = O.bitlinear_int(xq, xs, Wt, gamma, groups)
    assert_bf16_close(bits(y), y_o)


def test_gemv_extreme_codes():
    """All codes at -128 against all-+1 / all--1 weight rows: the largest
    accumulators the decode path can see at K = 11008."""
    M, N, K = 2, 256, 11008
    xq = np.full((M, K), -128, dtype=np.int8)
    xs = np.ones(M, dtype=np.float32)
    Wf = np.where((np.arange(N) % 2) == 0, 1.0, -1.0)[None, :].repeat(K, 0).astype(np.float32)
    Wf[:, 5] = 0.0
    Wt, gamma = O.ternarize(Wf, (N,))
    Wp = torch.from_numpy(O.pack_ternary(Wt)).to(DEV)
    y = B.gemv_w2(torch.from_numpy(xq).to(DEV), torch.from_numpy(xs).to(DEV), Wp,
                  torch.from_numpy(gamma).to(DEV), (N,))
    B.check_status()
    _, y_o = O.bitlinear_int(xq, xs, Wt, gamma, (N,))
    assert_bf16_close(bits(y), y_o)


@pytest.mark.parametrize("M", [1, 3, 33])
def test_gemv_matches_gemm(M):
    rng = np.random.default_rng(3)
    N, K = 2048, 2048
    xq = torch.from_numpy(rng.integers(-8, 8, size=(M, K)).astype(np.int8)).to(DEV)
    xs = torch.from_numpy(rng.uniform(0.01, 1, M).astype(np.float32)).to(DEV)
    _, _, Wp, gamma_d = prep_weights(K, N, (1024, 2048), 12)
    y1 = B.gemv_w2(xq, xs, Wp, gamma_d, (1024, 2048))
    y2 = B.gemm_w2a4(xq, xs, Wp, gamma_d, (1024, 2048))
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def _extreme_weights(K, N):
    """Columns of all +1, all -1 and all 0 weights, then random ternary ones."""
    rng = np.random.default_rng(K + N)
    Wf = rng.normal(0.0, 0.02, size=(K, N)).astype(np.float32)
    Wf[:, 0::4] = 1.0
    Wf[:, 1::4] = -1.0
    Wf[:, 2::4] = 0.0
    Wt, gamma = O.ternarize(Wf, (N,))
    return Wt, gamma, torch.from_numpy(O.pack_ternary(Wt)).to(DEV), torch.from_numpy(gamma).to(DEV)


@pytest.mark.parametrize("M", [257, 64])
def test_gemm_max_k_extreme_accumulators(M):
    """K = 32768, the largest the GEMMs take: codes of -128 (and 127) against
    columns of all +1 / -1 weights reach |acc| = 2^22, the edge of the exact
    int32 -> fp32 conversion; raw accumulators bit-exact, bf16 within 2 ulp.
    M = 257 runs the CTA-pair kernel, M = 64 the single-CTA one."""
    N, K = 32, 32768
    xq = np.full((M, K), -128, dtype=np.int8)
    xq[1::3] = 127
    xq[2::3] = np.random.default_rng(5).integers(-128, 128, size=xq[2::3].shape)
    Wt, gamma, Wp, gamma_d = _extreme_weights(K, N)
    xd = torch.from_numpy(xq).to(DEV)
    acc = B.gemm_w2a8_acc(xd, Wp)
    B.check_status()
    want = O.gemm_acc_int(xq, Wt)
    assert np.abs(want).max() == 128 * K
    assert np.array_equal(host(acc).astype(np.int64), want)
    xs = np.full(M, 1.0 / 127.0, dtype=np.float32)
    y = B.gemm_w2a8(xd, torch.from_numpy(xs).to(DEV), Wp, gamma_d, (N,))
    B.check_status()
    _, y_o = O.bitlinear_int(xq, xs, Wt, gamma, (N,))
    assert_bf16_close(bits(y), y_o)


def test_gemm_fp4_max_k_extreme_accumulators():
    """FP4 at K = 32768 with every code +-6 (the e2m1 extremes): the fp32
    accumulators reach 6 K = 196608, still exact."""
    M, N, K = 257, 32, 32768
    codes = np.full((M, K), 0x7, dtype=np.uint8)  # +6
    codes[1::2] = 0xF                              # -6
    Wt, _, Wp, _ = _extreme_weights(K, N)
    acc = B.gemm_w2fp4_acc(torch.from_numpy(O.pack_nibbles(codes)).to(DEV), Wp)
    B.check_status()
    want = O.gemm_acc_fp4(codes, Wt)
    assert np.abs(want).max() == 6 * K
    assert np.array_equal(host(acc).astype(np.float64), want)


@pytest.mark.parametrize("M", [1, 8, 64])
def test_gemv_max_k_extreme_codes(M):
    """The decode paths at K = 32768 (CUDA-core for one token, tensor-core for
    64) with codes of -128 against all-+1 / all--1 rows."""
    N, K = 256, 32768
    xq = np.full((M, K), -128, dtype=np.int8)
    xs = np.full(M, 1.0 / 127.0, dtype=np.float32)
    Wt, gamma, Wp, gamma_d = _extreme_weights(K, N)
    y = B.gemv_w2(torch.from_numpy(xq).to(DEV), torch.from_numpy(xs).to(DEV), Wp, gamma_d, (N,))
    B.check_status()
    _, y_o = O.bitlinear_int(xq, xs, Wt, gamma, (N,))
    assert_bf16_close(bits(y), y_o)


def test_empty_inputs_are_noops():
    e = torch.empty((0, 256), dtype=torch.bfloat16, device=DEV)
    q, xs = B.quant_act(e, O.MODE_INT8)
    assert q.shape == (0, 256)
    _, _, Wp, g = prep_weights(256, 256, (256,), 1)
    y = B.gemm_w2a8(torch.empty((0, 256), dtype=torch.int8, device=DEV), xs, Wp, g, (256,))
    assert y.shape == (0, 256)


def test_bounded_wait_reports_timeout_and_context_survives():
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    B.debug_wait_timeout(st, 2_000_000)  # 2 ms on a barrier nothing arrives on
    with pytest.raises(B.BitlinearError) as ei:
        B.check_status(st)
    assert ei.value.code == -5
    assert int(st.item()) == 1
    # the context is still usable
    rng = np.random.default_rng(0)
    xq = rng.integers(-128, 128, size=(32, 256)).astype(np.int8)
    Wt, _, Wp, _ = prep_weights(256, 256, (256,), 0)
    acc = B.gemm_w2a8_acc(torch.from_numpy(xq).to(DEV), Wp)
    assert np.array_equal(host(acc).astype(np.int64), O.gemm_acc_int(xq, Wt))


def test_library_prep_feeds_gpu_gemm():
    """Weights prepared by the library's host call (not the oracle) give the
    same GEMM result as the oracle's own ternarisation."""
    d = W.single_w2a4()
    Wp_l, gamma_l = B.ternarize_pack(d["proj"].W, (256,))
    Wt, gamma = O.ternarize(d["proj"].W, (256,))
    q, xs = B.quant_act(dev_bf16(d["x"]), O.MODE_INT4)
    y = B.gemm_w2a4(q, xs, torch.from_numpy(Wp_l).to(DEV), torch.from_numpy(gamma_l).to(DEV), (256,))
    xq_o, xs_o = O.quant_act(d["x"], O.MODE_INT4)
    _, y_o = O.bitlinear_int(xq_o, xs_o, Wt, gamma, (256,))
    assert_bf16_close(bits(y), y_o)


def _dependent_chain(x_dec, x_pre, wts):
    """Kernels that each read the output of the one just before them:
    decode (quantiser -> GEMV -> quantiser -> GEMV -> top-k -> GEMV) and
    prefill (quantiser -> GEMM -> top-k -> GEMM -> KV quantiser)."""
    (Wp1, g1), (Wp2, g2), (Wp3, g3) = wts
    outs = []
    q, xs = B.quant_act(x_dec, O.MODE_INT4)
    y = B.gemv_w2(q, xs, Wp1, g1, (1024,))
    q, xs = B.quant_act(y, O.MODE_INT8)
    y = B.gemv_w2(q, xs, Wp2, g2, (1024,))
    q, xs = B.topk_sparsify_i8(y)[:2]
    outs.append(B.gemv_w2(q, xs, Wp3, g3, (1024,)))
    if outs[-1].shape[0] <= 8:  # the fused quantiser + GEMV reads the previous output directly
        outs.append(B.gemv_w2_quant(outs[-1], O.MODE_INT8, Wp1, g1, (1024,), up=outs[-1]))
    q, xs = B.quant_act(x_pre, O.MODE_INT4)
    y = B.gemm_w2a4(q, xs, Wp1, g1, (1024,))
    q, xs = B.topk_sparsify_i8(y)[:2]
    y = B.gemm_w2a8(q, xs, Wp2, g2, (1024,))
    outs.append(y)
    codes3, _, scale = B.kv_quant_3bit(y.view(-1, 8, 128), None)
    outs += [codes3, scale]
    return [o.clone() for o in outs]


@pytest.mark.parametrize("M", [1, 6, 40])
def test_launch_overlap_dependent_chain(M):
    """With launch overlap on, every kernel must still see its producer's
    finished output: the chain gives the same bits as with overlap off."""
    wts = [prep_weights(1024, 1024, (1024,), 30 + i)[2:] for i in range(3)]
    runs = []
    for overlap in (False, True, True):
        B.set_launch_overlap(overlap)
        try:
            res = []
            for it in range(6):
                x_dec = dev_bf16(W.normal_bf16(np.random.default_rng(it), (M, 1024)))
                x_pre = dev_bf16(W.normal_bf16(np.random.default_rng(100 + it), (300, 1024)))
                res.append(_dependent_chain(x_dec, x_pre, wts))
            torch.cuda.synchronize()
            B.check_status()
        finally:
            B.set_launch_overlap(False)
        runs.append(res)
    for other in runs[1:]:
        for a, b in zip(runs[0], other):
            for ta, tb in zip(a, b):
                assert torch.equal(ta.view(torch.uint8), tb.view(torch.uint8))


# ---------------------------------------------- the bench's workloads, full size
# Every kernel runs on the whole workload in the bench's launch configuration;
# the oracle checks a seeded sample of token rows (each output row depends on
# its own input row only) plus the full quantiser output where that is cheap.
def _sample_rows(M, n, seed):
    return np.sort(np.random.default_rng(seed).choice(M, n, replace=False))


def _device_weights(proj):
    Wp, gamma = B.ternarize_pack(proj.W, proj.group_ends)
    return torch.from_numpy(Wp).to(DEV), torch.from_numpy(gamma).to(DEV)


@pytest.mark.parametrize("mode", [O.MODE_INT4, O.MODE_FP4])
def test_prefill_workload_full_size(mode):
    """X [2048 x 2048] (1% outlier channels) through q|k|v [2048 x 6144] and
    gate|up [2048 x 11264], as the bench's step runs them."""
    d = W.input_projection_prefill(seed=1)
    q, xs = B.quant_act(dev_bf16(d["x"]), mode)
    q_o, xs_o = O.quant_act(d["x"], mode)
    assert np.array_equal(host(q), q_o) and np.array_equal(host(xs), xs_o)
    rows = _sample_rows(2048, 48, 11 + mode)
    for proj in d["projs"]:
        Wp, g = _device_weights(proj)
        Wt, gamma = O.ternarize(proj.W, proj.group_ends)
        if mode == O.MODE_FP4:
            y = B.gemm_w2fp4(q, xs, Wp, g, proj.group_ends)
            _, y_o = O.bitlinear_fp4(q_o[rows], xs_o[rows], Wt, gamma, proj.group_ends)
        else:
            y = B.gemm_w2a4(q, xs, Wp, g, proj.group_ends)
            _, y_o = O.bitlinear_int(q_o[rows], xs_o[rows], Wt, gamma, proj.group_ends)
        B.check_status()
        assert_bf16_close(bits(y)[rows], y_o)


def test_o_proj_workload_full_size():
    """Top-k 50% + INT8 of X [4096 x 4096] (Student-t) and the o_proj GEMM."""
    d = W.o_proj_sparse()
    q, xs, _ = B.topk_sparsify_i8(dev_bf16(d["x"]))
    rows = _sample_rows(4096, 48, 21)
    q_o, xs_o, _ = O.topk_sparsify_i8(d["x"][rows])
    assert np.array_equal(host(q)[rows], q_o) and np.array_equal(host(xs)[rows], xs_o)
    Wp, g = _device_weights(d["proj"])
    y = B.gemm_w2a8(q, xs, Wp, g, d["proj"].group_ends)
    B.check_status()
    Wt, gamma = O.ternarize(d["proj"].W, d["proj"].group_ends)
    _, y_o = O.bitlinear_int(q_o, xs_o, Wt, gamma, d["proj"].group_ends)
    assert_bf16_close(bits(y)[rows], y_o)


def test_down_proj_workload_full_size():
    """ReLU^2(gate) * up + INT8 of [4096 x 11008] and the down_proj GEMM."""
    d = W.down_proj_relu2()
    q, xs = B.quant_act(dev_bf16(d["gate"]), O.MODE_INT8, up=dev_bf16(d["up"]))
    rows = _sample_rows(4096, 32, 31)
    q_o, xs_o = O.quant_act(d["gate"][rows], O.MODE_INT8, up_bits=d["up"][rows])
    assert np.array_equal(host(q)[rows], q_o) and np.array_equal(host(xs)[rows], xs_o)
    Wp, g = _device_weights(d["proj"])
    y = B.gemm_w2a8(q, xs, Wp, g, d["proj"].group_ends)
    B.check_status()
    Wt, gamma = O.ternarize(d["proj"].W, d["proj"].group_ends)
    _, y_o = O.bitlinear_int(q_o, xs_o, Wt, gamma, d["proj"].group_ends)
    assert_bf16_close(bits(y)[rows], y_o)


def test_kv_workload_full_size():
    """K and V caches [4096 x 32 x 128] with the bos token at 4 bits."""
    d = W.decode_layer(batch=1, make_weights=False)
    keep = torch.tensor([0], dtype=torch.int32, device=DEV)
    for name in ("k_cache", "v_cache"):
        kv = d[name]
        c3, c4, sc = B.kv_quant_3bit(dev_bf16(kv), keep)
        c3o, c4o, sco = O.kv_quant_3bit(kv, (0,))
        assert np.array_equal(host(c3), c3o)
        assert np.array_equal(host(c4), c4o)
        assert np.array_equal(host(sc), sco)


@pytest.mark.parametrize("M", [1, 3, 8])
@pytest.mark.parametrize("mode,relu2", [(O.MODE_INT4, False), (O.MODE_INT8, False), (O.MODE_INT8, True)])
@pytest.mark.parametrize("N,K", [(4096, 4096), (4096, 11008), (128, 128)])
def test_gemv_quant_fused(M, mode, relu2, N, K):
    """The quantiser inside the GEMV gives the oracle's quantiser + BitLinear,
    and the same bits as the two separate calls."""
    rng = np.random.default_rng(M * 7 + K + mode)
    x = W.outlier_bf16(rng, M, K)[0]
    up = W.normal_bf16(rng, (M, K)) if relu2 else None
    groups = (N // 2, N)
    Wt, gamma, Wp, gamma_d = prep_weights(K, N, groups, 17)
    xd = dev_bf16(x)
    ud = dev_bf16(up) if relu2 else None
    y = B.gemv_w2_quant(xd, mode, Wp, gamma_d, groups, up=ud)
    B.check_status()
    xq_o, xs_o = O.quant_act(x, mode, up_bits=up)
    _, y_o = O.bitlinear_int(xq_o, xs_o, Wt, gamma, groups)
    assert_bf16_close(bits(y), y_o)
    q, xs = B.quant_act(xd, mode, up=ud)
    y2 = B.gemv_w2(q, xs, Wp, gamma_d, groups)
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))


@pytest.mark.parametrize("M,mode,relu2,N", [(8, O.MODE_INT4, False, 12288), (5, O.MODE_INT8, True, 22016)])
def test_gemv_quant_fused_wide(M, mode, relu2, N):
    """Five to eight tokens against the fused q/k/v and gate/up widths: items
    of four weight rows, one accumulator per token and row."""
    K = 4096
    rng = np.random.default_rng(M * 11 + N)
    x = W.outlier_bf16(rng, M, K)[0]
    up = W.normal_bf16(rng, (M, K)) if relu2 else None
    groups = (N // 3, 2 * N // 3, N) if N % 3 == 0 else (N // 2, N)
    Wt, gamma, Wp, gamma_d = prep_weights(K, N, groups, 19)
    xd = dev_bf16(x)
    ud = dev_bf16(up) if relu2 else None
    y = B.gemv_w2_quant(xd, mode, Wp, gamma_d, groups, up=ud)
    B.check_status()
    xq_o, xs_o = O.quant_act(x, mode, up_bits=up)
    _, y_o = O.bitlinear_int(xq_o, xs_o, Wt, gamma, groups)
    assert_bf16_close(bits(y), y_o)


def test_gemv_quant_fused_strided_rows():
    """Rows with a stride above K (a view into a wider buffer)."""
    M, K, N = 5, 4096, 1024
    rng = np.random.default_rng(5)
    wide = W.normal_bf16(rng, (M, K + 64))
    Wt, gamma, Wp, gamma_d = prep_weights(K, N, (N,), 18)
    xd = dev_bf16(wide)[:, :K]
    y = B.gemv_w2_quant(xd, O.MODE_INT4, Wp, gamma_d, (N,))
    B.check_status()
    xq_o, xs_o = O.quant_act(np.ascontiguousarray(wide[:, :K]), O.MODE_INT4)
    _, y_o = O.bitlinear_int(xq_o, xs_o, Wt, gamma, (N,))
    assert_bf16_close(bits(y), y_o)


# ------------------------------------------------------ 3-bit KV attention
def _attn_case(rng, Bq, H, D, T, keep):
    k_bits = W.normal_bf16(rng, (T, H, D))
    v_bits = W.normal_bf16(rng, (T, H, D))
    q = W.normal_bf16(rng, (Bq, H, D))
    ks, vs = O.kv_quant_3bit(k_bits, keep), O.kv_quant_3bit(v_bits, keep)
    return q, ks, vs


def _check_attention(q, ks, vs, keep, out=None):
    """The kernel's bf16 output against the fp64 oracle within the bound of
    conftest.attention_tolerance (one bf16 ulp + 2^-16 of sum_t p_t |v_t| + |o|)."""
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(DEV)
    if out is None:
        kd = (dev(ks[0]), dev(ks[1]) if len(keep) else None, dev(ks[2]))
        vd = (dev(vs[0]), dev(vs[1]) if len(keep) else None, dev(vs[2]))
        kp = torch.tensor(keep, dtype=torch.int32, device=DEV) if len(keep) else None
        out = B.kv_attention_3bit(dev_bf16(q), kd, vd, kp)
    torch.cuda.synchronize()
    want, tol = attention_tolerance(q, ks, vs, keep)
    got = O.bf16_to_f32(bits(out)).astype(np.float64)
    err = np.abs(got - want)
    assert np.all(err <= tol), f"max excess {np.max(err - tol)} at {np.unravel_index(np.argmax(err - tol), err.shape)}"


@pytest.mark.parametrize("Bq,H,D,T,keep", [
    (1, 4, 128, 1, (0,)), (1, 4, 128, 37, ()), (3, 4, 128, 300, (0, 5, 130)), (8, 4, 256, 513, (0,)),
    (11, 8, 128, 1000, (0, 999)), (1, 4, 128, 4096, (0,)), (2, 4, 128, 129, tuple(range(0, 129, 3))),
    (1, 4, 256, 2000, ()),
    # D = 128 (the tensor-core kernel): 4-bit tokens on warp and tile edges, many 4-bit tokens (up
    # to the 1024 the entry point takes, several in every warp), token counts that split unevenly
    # over the cluster, 5 queries (8-query groups with 3 empty) and 12 (a group of 8 and one of 4)
    (1, 8, 128, 1000, (0, 31, 32, 255, 256, 511, 999)), (1, 4, 128, 2049, tuple(range(0, 2049, 7))),
    (1, 4, 128, 8191, (0, 4095, 8190)), (2, 4, 128, 4096, tuple(range(0, 4096, 4))),
    (5, 4, 128, 777, (0, 1, 2, 3, 776)), (12, 4, 128, 300, (0, 150))])
def test_kv_attention_parity(Bq, H, D, T, keep):
    q, ks, vs = _attn_case(np.random.default_rng(Bq * 100 + T), Bq, H, D, T, keep)
    _check_attention(q, ks, vs, keep)


@pytest.mark.parametrize("Bq", [1, 8])
def test_kv_attention_full_size(Bq):
    """The decode layer's cache: 4096 tokens x 32 heads x 128, bos at 4 bits,
    K and V quantised by the library's own kernel."""
    d = W.decode_layer(batch=1, make_weights=False)
    keep = torch.tensor([0], dtype=torch.int32, device=DEV)
    kst = B.kv_quant_3bit(dev_bf16(d["k_cache"]), keep)
    vst = B.kv_quant_3bit(dev_bf16(d["v_cache"]), keep)
    q = W.normal_bf16(np.random.default_rng(9), (Bq, 32, 128))
    out = B.kv_attention_3bit(dev_bf16(q), kst, vst, keep)
    _check_attention(q, tuple(host(t) for t in kst), tuple(host(t) for t in vst), (0,), out=out)


@pytest.mark.parametrize("Bq", [1, 3])
def test_kv_attention_full_size_planted_edges(Bq):
    """Every token at a 32-token boundary (t % 32 in {0, 31}, which includes
    each 256-token tile edge and each split of the tokens over a cluster)
    carries value rows 16x larger, so a boundary token lost or counted twice
    moves its head's output by far more than the bound."""
    d = W.decode_layer(batch=1, make_weights=False)
    T = d["v_cache"].shape[0]
    v = O.bf16_to_f32(d["v_cache"])
    edge = (np.arange(T) % 32 == 0) | (np.arange(T) % 32 == 31)
    v[edge] *= np.float32(16.0)
    v_bits = O.f32_to_bf16(v)
    keep = torch.tensor([0], dtype=torch.int32, device=DEV)
    kst = B.kv_quant_3bit(dev_bf16(d["k_cache"]), keep)
    vst = B.kv_quant_3bit(dev_bf16(v_bits), keep)
    q = W.normal_bf16(np.random.default_rng(10), (Bq, 32, 128))
    out = B.kv_attention_3bit(dev_bf16(q), kst, vst, keep)
    _check_attention(q, tuple(host(t) for t in kst), tuple(host(t) for t in vst), (0,), out=out)


def test_tensor_peak_measures_the_pipe():
    """The measurement helper runs every kind without a timeout and reports
    rates in the range a B200's tensor pipe can give (dense int8 near
    4.5 POPS nominal, block-scaled FP4 near 9)."""
    r = {k: B.tensor_peak(k, 512) for k in (0, 1, 2)}
    B.check_status()
    assert r[0]["units"] * 2 == r[2]["units"] // 2 * 2 and r[0]["units"] >= 1
    assert 1000 < r[0]["tops"] < 6000 and 1000 < r[2]["tops"] < 6000
    assert 2000 < r[1]["tops"] < 12000
