"""C-ABI checks that need no GPU: the library loads, exports every function
the header declares, the host weight-prep call matches the oracle bit for
bit, and bad arguments are rejected on the host before any launch."""
import ctypes

import numpy as np
import pytest

import bit_quantised_gemm_b200 as B
from bit_quantised_gemm_b200 import _lib
from conftest import golden
from oracle import bitlinear_oracle as O
import workloads as W


def test_library_exports_every_declared_function():
    L = B.lib()
    declared = B.header_functions()
    assert len(declared) >= 14
    for name in declared:
        assert hasattr(L, name), name
    assert set(declared) == set(_lib._SIGS)
    assert B.version() == 106


@pytest.mark.parametrize("K,N,groups,seed", [
    (256, 256, (256,), 0), (64, 96, (32, 96), 1), (2048, 384, (128, 256, 384), 2),
    (16, 16, (16,), 3)])
def test_ternarize_pack_matches_oracle(K, N, groups, seed):
    Wm = W.weights(np.random.default_rng(seed), K, N)
    Wp, gamma = B.ternarize_pack(Wm, groups)
    Wt_o, gamma_o = O.ternarize(Wm, groups)
    assert np.array_equal(gamma, gamma_o)
    assert np.array_equal(Wp, O.pack_ternary(Wt_o))


def test_ternarize_pack_golden_ties():
    g = golden("ternarize_ties.txt")
    for case in "ABC":
        Wm = np.array([float(v) for v in g[f"W_{case}"]], np.float32).reshape(2, 2)
        # K must be a multiple of 16: repeat the 2 x 2 block 8 times down K
        # (the mean |W| and so every code are unchanged)
        Wp, gamma = B.ternarize_pack(np.tile(Wm, (8, 1)), (2,))
        Wt = O.unpack_ternary(Wp, 16)
        want = np.array([int(v) for v in g[f"Wt_{case}"]]).reshape(2, 2)
        assert np.array_equal(Wt, np.tile(want, (8, 1)))


def test_ternarize_pack_golden_layout():
    g = golden("pack_layout.txt")
    col = np.array([int(v) for v in g["Wt_col"]], np.float32).reshape(16, 1)
    # values +-1 with mean |W| = 3/16: +-1/gamma rounds to +-5 -> clamps to +-1
    Wp, gamma = B.ternarize_pack(col, (1,))
    assert Wp[0].tolist() == [int(b, 16) for b in g["bytes"]]


FAKE = 1 << 20  # a 16-byte aligned non-null address; never dereferenced on a host-side error
ge1 = np.array([256], np.int64)


def _gemm(fn, **kw):
    a = dict(xq=FAKE, xs=FAKE, Wp=FAKE, gamma=FAKE, ge=ge1.ctypes.data, G=1, M=16, N=256, K=256,
             y=FAKE, ldy=256)
    a.update(kw)
    return getattr(B.lib(), fn)(a["xq"], a["xs"], a["Wp"], a["gamma"], a["ge"], a["G"], a["M"],
                                a["N"], a["K"], a["y"], a["ldy"], None, None)


@pytest.mark.parametrize("fn", ["bitlinear_gemm_w2a8", "bitlinear_gemm_w2a4",
                                "bitlinear_gemm_w2fp4", "bitlinear_gemv_w2"])
def test_gemm_argument_errors(fn):
    assert _gemm(fn, K=200) == _lib.ERR_INVALID_ARG
    assert _gemm(fn, N=250) == _lib.ERR_INVALID_ARG
    assert _gemm(fn, M=-1) == _lib.ERR_INVALID_ARG
    assert _gemm(fn, xq=None) == _lib.ERR_INVALID_ARG
    assert _gemm(fn, xq=FAKE + 4) == _lib.ERR_ALIGNMENT
    assert _gemm(fn, ldy=100) == _lib.ERR_INVALID_ARG
    bad = np.array([100, 200], np.int64)
    assert _gemm(fn, ge=bad.ctypes.data, G=2) == _lib.ERR_INVALID_ARG  # last end != N
    dec = np.array([200, 100, 256], np.int64)
    assert _gemm(fn, ge=dec.ctypes.data, G=3) == _lib.ERR_INVALID_ARG
    assert _gemm(fn, G=9) == _lib.ERR_INVALID_ARG
    assert _gemm(fn, M=0) == _lib.OK  # empty: nothing launched


def test_gemv_and_fp4_specific_limits():
    assert _gemm("bitlinear_gemv_w2", M=65) == _lib.ERR_INVALID_ARG
    assert _gemm("bitlinear_gemm_w2fp4", K=192) == _lib.ERR_INVALID_ARG  # K % 128


def test_fused_gemv_argument_errors():
    def call(**kw):
        a = dict(x=FAKE, up=None, ldx=256, mode=1, Wp=FAKE, gamma=FAKE, ge=ge1.ctypes.data, G=1,
                 M=4, N=256, K=256, y=FAKE, ldy=256)
        a.update(kw)
        return B.lib().bitlinear_gemv_w2_quant(a["x"], a["up"], a["ldx"], a["mode"], a["Wp"], a["gamma"],
                                               a["ge"], a["G"], a["M"], a["N"], a["K"], a["y"], a["ldy"],
                                               None, None)
    assert call(mode=2) == _lib.ERR_INVALID_ARG        # FP4 is not a GEMV code kind
    assert call(M=9) == _lib.ERR_UNSUPPORTED            # more tokens: quantiser + GEMV
    assert call(K=192) == _lib.ERR_INVALID_ARG          # K % 128
    assert call(ldx=128) == _lib.ERR_INVALID_ARG        # ldx < K
    assert call(ldx=260) == _lib.ERR_INVALID_ARG        # ldx % 8
    assert call(x=FAKE + 2) == _lib.ERR_ALIGNMENT
    assert call(up=FAKE + 2) == _lib.ERR_ALIGNMENT
    assert call(x=None) == _lib.ERR_INVALID_ARG
    assert call(M=0) == _lib.OK


def test_kv_attention_argument_errors():
    L = B.lib()
    def call(**kw):
        a = dict(q=FAKE, B=2, H=4, D=128, T=64, k3=FAKE, k4=None, ks=FAKE, v3=FAKE, v4=None, vs=FAKE,
                 keep=None, n4=0, out=FAKE)
        a.update(kw)
        return L.kv_attention_3bit(a["q"], a["B"], a["H"], a["D"], a["T"], a["k3"], a["k4"], a["ks"],
                                   a["v3"], a["v4"], a["vs"], a["keep"], a["n4"], a["out"], None, None)
    assert call(D=96) == _lib.ERR_UNSUPPORTED
    assert call(D=64) == _lib.ERR_UNSUPPORTED               # 24-byte rows: no TMA box
    assert call(H=6) == _lib.ERR_UNSUPPORTED                # scale rows: H % 4
    assert call(T=0) == _lib.ERR_INVALID_ARG
    assert call(n4=1) == _lib.ERR_INVALID_ARG               # no list / 4-bit rows
    assert call(n4=65, keep=FAKE, k4=FAKE, v4=FAKE) == _lib.ERR_INVALID_ARG  # more than T
    assert call(q=None) == _lib.ERR_INVALID_ARG
    assert call(out=FAKE + 2) == _lib.ERR_ALIGNMENT
    assert call(n4=1, keep=FAKE, k4=FAKE + 8, v4=FAKE) == _lib.ERR_ALIGNMENT  # 4-bit rows: 16-byte aligned
    assert call(n4=1, keep=FAKE, k4=FAKE, v4=FAKE + 4) == _lib.ERR_ALIGNMENT
    assert call(B=0) == _lib.OK


def test_keep4_positions_argument_errors():
    L = B.lib()
    sp = (ctypes.c_int32 * 2)(1, 2)
    many = (ctypes.c_int32 * 9)(*range(9))
    addr = ctypes.addressof
    assert L.kv_keep4_positions(FAKE, 16, addr(sp), 0, FAKE, FAKE, None) == _lib.ERR_INVALID_ARG
    assert L.kv_keep4_positions(FAKE, 16, addr(many), 9, FAKE, FAKE, None) == _lib.ERR_INVALID_ARG
    assert L.kv_keep4_positions(FAKE, 16, None, 2, FAKE, FAKE, None) == _lib.ERR_INVALID_ARG
    assert L.kv_keep4_positions(FAKE, -1, addr(sp), 2, FAKE, FAKE, None) == _lib.ERR_INVALID_ARG
    assert L.kv_keep4_positions(None, 16, addr(sp), 2, FAKE, FAKE, None) == _lib.ERR_INVALID_ARG
    assert L.kv_keep4_positions(FAKE, 16, addr(sp), 2, FAKE, None, None) == _lib.ERR_INVALID_ARG


def test_quantiser_argument_errors():
    L = B.lib()
    assert L.bitlinear_quant_act(FAKE, None, 4, 250, 256, 0, FAKE, FAKE, None) == _lib.ERR_INVALID_ARG
    assert L.bitlinear_quant_act(FAKE, None, 4, 256, 256, 7, FAKE, FAKE, None) == _lib.ERR_INVALID_ARG
    assert L.bitlinear_quant_act(FAKE, None, 4, 256, 100, 0, FAKE, FAKE, None) == _lib.ERR_INVALID_ARG
    assert L.bitlinear_quant_act(FAKE + 2, None, 4, 256, 256, 0, FAKE, FAKE, None) == _lib.ERR_ALIGNMENT
    assert L.bitlinear_quant_act(FAKE, None, 0, 256, 256, 0, FAKE, FAKE, None) == _lib.OK
    assert L.bitlinear_topk_sparsify_i8(FAKE, 4, 32768, 32768, 0, FAKE, FAKE, None, None) == _lib.ERR_UNSUPPORTED
    assert L.bitlinear_topk_sparsify_i8(FAKE, 4, 256, 256, -1, FAKE, FAKE, None, None) == _lib.ERR_INVALID_ARG
    assert L.kv_quant_3bit(FAKE, 4, 2, 96, None, 0, FAKE, None, FAKE, None) == _lib.ERR_UNSUPPORTED
    assert L.kv_quant_3bit(FAKE, 4, 2, 128, None, 1, FAKE, FAKE, FAKE, None) == _lib.ERR_INVALID_ARG
    assert L.kv_quant_3bit(FAKE, 0, 2, 128, None, 0, FAKE, None, FAKE, None) == _lib.OK
    # K and V in one launch: each tensor is checked as kv_quant_3bit checks it
    assert L.kv_quant_3bit_kv(FAKE, FAKE, 4, 2, 96, None, 0, FAKE, None, FAKE, FAKE, None, FAKE,
                              None) == _lib.ERR_UNSUPPORTED
    assert L.kv_quant_3bit_kv(FAKE, FAKE, 4, 2, 128, FAKE, 1, FAKE, FAKE, FAKE, FAKE, None, FAKE,
                              None) == _lib.ERR_INVALID_ARG
    assert L.kv_quant_3bit_kv(FAKE, None, 4, 2, 128, None, 0, FAKE, None, FAKE, FAKE, None, FAKE,
                              None) == _lib.ERR_INVALID_ARG
    assert L.kv_quant_3bit_kv(FAKE, FAKE + 8, 4, 2, 128, None, 0, FAKE, None, FAKE, FAKE, None, FAKE,
                              None) == _lib.ERR_ALIGNMENT
    assert L.kv_quant_3bit_kv(FAKE, FAKE, 0, 2, 128, None, 0, FAKE, None, FAKE, FAKE, None, FAKE,
                              None) == _lib.OK
    assert L.bitlinear_set_wait_timeout_ns(0) == _lib.ERR_INVALID_ARG
    msg = L.bitlinear_last_error().decode()
    assert "timeout" in msg


def test_error_raises_python_exception():
    with pytest.raises(B.BitlinearError) as ei:
        B.set_wait_timeout_ns(-5)
    assert ei.value.code == _lib.ERR_INVALID_ARG
    B.set_wait_timeout_ns(2_000_000_000)


def test_binding_rejects_malformed_tensors():
    """The C ABI sees only pointers and sizes, so the binding checks dtypes,
    shapes and layouts first (CPU tensors: a well-formed call gets as far as
    the CUDA-tensor check)."""
    import torch
    M, K, N = 4, 256, 128
    xq = torch.zeros((M, K), dtype=torch.int8)
    xs = torch.ones(M, dtype=torch.float32)
    Wp = torch.zeros((N, K // 4), dtype=torch.uint8)
    g = torch.ones(1, dtype=torch.float32)
    with pytest.raises(ValueError, match="CUDA"):
        B.gemm_w2a8(xq, xs, Wp, g, (N,))
    with pytest.raises(ValueError, match="activation codes: dtype"):
        B.gemm_w2a8(xq.to(torch.int32), xs, Wp, g, (N,))
    with pytest.raises(ValueError, match="activation codes: must be contiguous"):
        B.gemm_w2a8(torch.zeros((M, 2 * K), dtype=torch.int8)[:, ::2], xs, Wp, g, (N,))
    with pytest.raises(ValueError, match="activation codes: dtype"):
        B.gemm_w2fp4(xq, xs, Wp, g, (N,))  # FP4 codes are packed uint8
    with pytest.raises(ValueError, match="xs: dtype"):
        B.gemv_w2(xq, xs.double(), Wp, g, (N,))
    with pytest.raises(ValueError, match="xs: 3 scales"):
        B.gemm_w2a8(xq, xs[:3], Wp, g, (N,))
    with pytest.raises(ValueError, match="Wp: rows of"):
        B.gemm_w2a8(xq, xs, Wp[:, :32].contiguous(), g, (N,))
    with pytest.raises(ValueError, match="gamma: 1 scales for 2"):
        B.gemm_w2a8(xq, xs, Wp, g, (64, N))
    with pytest.raises(ValueError, match="y: shape"):
        B.gemm_w2a8(xq, xs, Wp, g, (N,), y=torch.empty((M, N + 1), dtype=torch.bfloat16))
    x = torch.zeros((M, K), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        B.quant_act(x, _lib.MODE_INT4)
    with pytest.raises(ValueError, match="x: dtype"):
        B.quant_act(x.float(), _lib.MODE_INT4)
    with pytest.raises(ValueError, match="out: shape"):
        B.quant_act(x, _lib.MODE_FP4, out=torch.empty((M, K), dtype=torch.uint8))
    with pytest.raises(ValueError, match="out: dtype"):
        B.topk_sparsify_i8(x, out=torch.empty((M, K), dtype=torch.uint8))
    with pytest.raises(ValueError, match="CUDA"):
        B.gemv_w2_quant(x, _lib.MODE_INT4, Wp, g, (N,))
    with pytest.raises(ValueError, match="Wp: dtype"):
        B.gemv_w2_quant(x, _lib.MODE_INT4, Wp.to(torch.int8), g, (N,))


def test_binding_rejects_malformed_acc_and_kv_tensors():
    """The raw-accumulator GEMMs and the KV calls check every operand against
    the sizes they pass to the C ABI before any launch (a short Wp or v3
    would otherwise send a tensor map past the end of an allocation)."""
    import torch
    M, K, N = 4, 256, 128
    xq = torch.zeros((M, K), dtype=torch.int8)
    Wp = torch.zeros((N, K // 4), dtype=torch.uint8)
    with pytest.raises(ValueError, match="CUDA"):
        B.gemm_w2a8_acc(xq, Wp)
    with pytest.raises(ValueError, match="Wp: rows of"):
        B.gemm_w2a8_acc(xq, Wp[:, :32].contiguous())
    with pytest.raises(ValueError, match="activation codes: dtype"):
        B.gemm_w2a8_acc(xq.to(torch.int16), Wp)
    with pytest.raises(ValueError, match="Wp: dtype"):
        B.gemm_w2a8_acc(xq, Wp.to(torch.int8))
    f4 = torch.zeros((M, K // 2), dtype=torch.uint8)
    with pytest.raises(ValueError, match="CUDA"):
        B.gemm_w2fp4_acc(f4, Wp)
    with pytest.raises(ValueError, match="Wp: rows of"):
        B.gemm_w2fp4_acc(f4[:, :64].contiguous(), Wp)
    with pytest.raises(ValueError, match="must be contiguous"):
        B.gemm_w2fp4_acc(torch.zeros((M, K), dtype=torch.uint8)[:, ::2], Wp)

    T, H, D = 40, 4, 128
    kv = torch.zeros((T, H, D), dtype=torch.bfloat16)
    keep = torch.tensor([0], dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):
        B.kv_quant_3bit(kv, keep)
    with pytest.raises(ValueError, match="codes3: shape"):
        B.kv_quant_3bit(kv, keep, codes3=torch.empty((T, H, D // 4), dtype=torch.uint8))
    with pytest.raises(ValueError, match="codes4: shape"):
        B.kv_quant_3bit(kv, keep, codes4=torch.empty((2, H, D // 2), dtype=torch.uint8))
    with pytest.raises(ValueError, match="scale: dtype"):
        B.kv_quant_3bit(kv, keep, scale=torch.empty((T, H), dtype=torch.float64))
    with pytest.raises(ValueError, match="keep4_pos: dtype"):
        B.kv_quant_3bit(kv, keep.long())
    with pytest.raises(ValueError, match="kv: dtype"):
        B.kv_quant_3bit(kv.float(), keep)
    with pytest.raises(ValueError, match="CUDA"):
        B.kv_quant_3bit_kv(kv, kv.clone(), keep)
    with pytest.raises(ValueError, match="one shape"):
        B.kv_quant_3bit_kv(kv, kv[:8].contiguous(), keep)
    with pytest.raises(ValueError, match="v: dtype"):
        B.kv_quant_3bit_kv(kv, kv.float(), keep)
    with pytest.raises(ValueError, match="v codes3: shape"):
        B.kv_quant_3bit_kv(kv, kv, keep, v_store=(torch.empty((T, H, D // 4), dtype=torch.uint8),
                                                 torch.empty((1, H, D // 2), dtype=torch.uint8),
                                                 torch.empty((T, H), dtype=torch.float32)))

    q = torch.zeros((2, H, D), dtype=torch.bfloat16)
    c3 = torch.zeros((T, H, 3 * D // 8), dtype=torch.uint8)
    c4 = torch.zeros((1, H, D // 2), dtype=torch.uint8)
    sc = torch.ones((T, H), dtype=torch.float32)
    good = (c3, c4, sc)
    with pytest.raises(ValueError, match="CUDA"):
        B.kv_attention_3bit(q, good, good, keep)
    with pytest.raises(ValueError, match="v codes3: shape"):
        B.kv_attention_3bit(q, good, (c3[:T - 1].contiguous(), c4, sc), keep)
    with pytest.raises(ValueError, match="v scale: shape"):
        B.kv_attention_3bit(q, good, (c3, c4, sc[:, :2].contiguous()), keep)
    with pytest.raises(ValueError, match="k codes4: missing"):
        B.kv_attention_3bit(q, (c3, None, sc), good, keep)
    with pytest.raises(ValueError, match="k codes3: shape"):
        B.kv_attention_3bit(torch.zeros((2, H, 256), dtype=torch.bfloat16), good, good, keep)
    with pytest.raises(ValueError, match="out: shape"):
        B.kv_attention_3bit(q, good, good, keep, out=torch.empty((1, H, D), dtype=torch.bfloat16))
