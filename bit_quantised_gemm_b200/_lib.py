"""ctypes binding of libbitlinear.so: argument marshalling only.

Every computation happens in the CUDA library; this module passes device
pointers, sizes and the current CUDA stream, allocates outputs with torch,
and turns error codes into exceptions. There is no CPU fallback: if the
library is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import re

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbitlinear.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "bitlinear.h")

MODE_INT8, MODE_INT4, MODE_FP4 = 0, 1, 2
OK, ERR_INVALID_ARG, ERR_ALIGNMENT, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT = 0, -1, -2, -3, -4, -5
STATUS_TIMEOUT = 1


class BitlinearError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"bitlinear error {code}: {msg}")
        self.code = code


_c = ctypes
_P = _c.c_void_p
_I64 = _c.c_int64
_INT = _c.c_int

_SIGS = {
    "bitlinear_last_error": ([], _c.c_char_p),
    "bitlinear_version": ([], _INT),
    "bitlinear_set_wait_timeout_ns": ([_I64], _INT),
    "bitlinear_set_launch_overlap": ([_INT], _INT),
    "bitlinear_ternarize_pack": ([_P, _I64, _I64, _P, _INT, _P, _P], _INT),
    "bitlinear_quant_act": ([_P, _P, _I64, _I64, _I64, _INT, _P, _P, _P], _INT),
    "bitlinear_topk_sparsify_i8": ([_P, _I64, _I64, _I64, _I64, _P, _P, _P, _P], _INT),
    "bitlinear_gemm_w2a8": ([_P, _P, _P, _P, _P, _INT, _I64, _I64, _I64, _P, _I64, _P, _P], _INT),
    "bitlinear_gemm_w2a4": ([_P, _P, _P, _P, _P, _INT, _I64, _I64, _I64, _P, _I64, _P, _P], _INT),
    "bitlinear_gemm_w2fp4": ([_P, _P, _P, _P, _P, _INT, _I64, _I64, _I64, _P, _I64, _P, _P], _INT),
    "bitlinear_gemm_w2a8_acc": ([_P, _P, _I64, _I64, _I64, _P, _P, _P], _INT),
    "bitlinear_gemm_w2fp4_acc": ([_P, _P, _I64, _I64, _I64, _P, _P, _P], _INT),
    "bitlinear_gemv_w2": ([_P, _P, _P, _P, _P, _INT, _I64, _I64, _I64, _P, _I64, _P, _P], _INT),
    "kv_attention_3bit": ([_P, _I64, _I64, _I64, _I64, _P, _P, _P, _P, _P, _P, _P, _I64, _P, _P, _P],
                          _INT),
    "bitlinear_gemv_w2_quant": ([_P, _P, _I64, _INT, _P, _P, _P, _INT, _I64, _I64, _I64, _P, _I64, _P, _P],
                                _INT),
    "kv_quant_3bit": ([_P, _I64, _I64, _I64, _P, _I64, _P, _P, _P, _P], _INT),
    "kv_quant_3bit_kv": ([_P, _P, _I64, _I64, _I64, _P, _I64, _P, _P, _P, _P, _P, _P, _P], _INT),
    "kv_keep4_positions": ([_P, _I64, _P, _INT, _P, _P, _P], _INT),
    "bitlinear_check_status": ([_P, _P], _INT),
    "bitlinear_tensor_peak": ([_INT, _INT, _P, _P, _P, _P], _INT),
    "bitlinear_debug_wait_timeout": ([_P, _I64, _P], _INT),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load libbitlinear.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m bit_quantised_gemm_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def header_functions() -> list[str]:
    """Names of the functions declared in include/bitlinear.h."""
    text = open(HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", text, flags=re.M)))


def _check(rc: int):
    if rc != OK:
        raise BitlinearError(rc, lib().bitlinear_last_error().decode())


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return t.data_ptr()


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _require_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("expected a CUDA tensor")


# bf16 values, or their 16-bit patterns
_BF16_LIKE = tuple(d for d in (torch.bfloat16, torch.int16, getattr(torch, "uint16", None)) if d is not None)


def _need(t, name: str, dtypes, dim: int | None = None, contiguous: bool = False):
    """Metadata checks the C ABI cannot make (it sees only pointers and sizes)."""
    if t.dtype not in dtypes:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {' or '.join(str(d) for d in dtypes)}")
    if dim is not None and t.dim() != dim:
        raise ValueError(f"{name}: {t.dim()}-D, expected {dim}-D")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")


def _check_gemm_operands(a, code_dtype, xs, Wp, gamma, n_groups: int, K: int, y):
    """Codes [M x *] contiguous, xs fp32 [>= M], Wp uint8 [N x K/4], gamma fp32
    [>= G], y (when given) bf16 [M x N] with unit column stride."""
    _need(a, "activation codes", (code_dtype,), 2, contiguous=True)
    M = a.shape[0]
    _need(xs, "xs", (torch.float32,), 1, contiguous=True)
    if xs.numel() < M:
        raise ValueError(f"xs: {xs.numel()} scales for {M} rows")
    _need(Wp, "Wp", (torch.uint8,), 2, contiguous=True)
    if Wp.shape[1] * 4 != K:
        raise ValueError(f"Wp: rows of {Wp.shape[1]} bytes, expected K/4 = {K // 4}")
    _need(gamma, "gamma", (torch.float32,), 1, contiguous=True)
    if gamma.numel() < n_groups:
        raise ValueError(f"gamma: {gamma.numel()} scales for {n_groups} column groups")
    if y is not None:
        _need(y, "y", _BF16_LIKE, 2)
        if tuple(y.shape) != (M, Wp.shape[0]) or y.stride(1) != 1:
            raise ValueError(f"y: shape {tuple(y.shape)} / strides {y.stride()}, expected "
                             f"({M}, {Wp.shape[0]}) with unit column stride")


def _rows(t: torch.Tensor) -> tuple[int, int, int]:
    """(M, K, ld) of a 2-D tensor whose rows are contiguous."""
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError("expected a 2-D tensor with contiguous rows")
    return t.shape[0], t.shape[1], t.stride(0)


_status = {}


def status_buffer(device=None) -> torch.Tensor:
    """Per-device int32 status word passed to the GEMM kernels (zeroed)."""
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    key = dev.index if dev.index is not None else torch.cuda.current_device()
    if key not in _status:
        _status[key] = torch.zeros(1, dtype=torch.int32, device=f"cuda:{key}")
    return _status[key]


# ------------------------------------------------------------------ API
def version() -> int:
    return lib().bitlinear_version()


def set_launch_overlap(enable: bool):
    """Programmatic dependent launch for later calls (see bitlinear.h)."""
    _check(lib().bitlinear_set_launch_overlap(1 if enable else 0))


def set_wait_timeout_ns(ns: int):
    _check(lib().bitlinear_set_wait_timeout_ns(int(ns)))


def ternarize_pack(W: np.ndarray, group_ends) -> tuple[np.ndarray, np.ndarray]:
    """Host weight prep: fp32 W [K x N] -> (Wp uint8 [N x K/4], gamma fp32 [G])."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    K, N = W.shape
    ge = np.ascontiguousarray(group_ends, dtype=np.int64)
    Wp = np.zeros((N, K // 4), dtype=np.uint8)
    gamma = np.zeros(len(ge), dtype=np.float32)
    _check(lib().bitlinear_ternarize_pack(_ptr(W), K, N, _ptr(ge), len(ge), _ptr(Wp), _ptr(gamma)))
    return Wp, gamma


def quant_act(x: torch.Tensor, mode: int, up: torch.Tensor | None = None, out=None, xs=None,
              stream=None):
    """Per-token quantiser (INT8 / INT4 / FP4), optionally of relu(x)^2 * up."""
    _need(x, "x", _BF16_LIKE)
    if up is not None:
        _need(up, "up", _BF16_LIKE)
    M, K, ld = _rows(x)
    if out is not None:
        fp4 = mode == MODE_FP4
        _need(out, "out", (torch.uint8,) if fp4 else (torch.int8,), 2, contiguous=True)
        if tuple(out.shape) != (M, K // 2 if fp4 else K):
            raise ValueError(f"out: shape {tuple(out.shape)} for {M} rows of {K} values")
    if xs is not None:
        _need(xs, "xs", (torch.float32,), 1, contiguous=True)
        if xs.numel() < M:
            raise ValueError(f"xs: {xs.numel()} scales for {M} rows")
    _require_cuda(x, up)
    if up is not None and (up.shape != x.shape or up.stride() != x.stride()):
        raise ValueError("up must match x in shape and strides")
    if out is None:
        out = (torch.empty((M, K // 2), dtype=torch.uint8, device=x.device) if mode == MODE_FP4
               else torch.empty((M, K), dtype=torch.int8, device=x.device))
    if xs is None:
        xs = torch.empty(M, dtype=torch.float32, device=x.device)
    _check(lib().bitlinear_quant_act(_ptr(x), _ptr(up), M, K, ld, mode, _ptr(out), _ptr(xs),
                                     _stream(stream)))
    return out, xs


def topk_sparsify_i8(x: torch.Tensor, k: int = 0, mask: bool = False, out=None, xs=None,
                     stream=None):
    """Keep the k (default ceil(K/2)) largest |x| per row, zero the rest, INT8."""
    _need(x, "x", _BF16_LIKE)
    M, K, ld = _rows(x)
    if out is not None:
        _need(out, "out", (torch.int8,), 2, contiguous=True)
        if tuple(out.shape) != (M, K):
            raise ValueError(f"out: shape {tuple(out.shape)} for {M} rows of {K} values")
    if xs is not None:
        _need(xs, "xs", (torch.float32,), 1, contiguous=True)
        if xs.numel() < M:
            raise ValueError(f"xs: {xs.numel()} scales for {M} rows")
    _require_cuda(x)
    if out is None:
        out = torch.empty((M, K), dtype=torch.int8, device=x.device)
    if xs is None:
        xs = torch.empty(M, dtype=torch.float32, device=x.device)
    mk = torch.empty((M, K // 8), dtype=torch.uint8, device=x.device) if mask else None
    _check(lib().bitlinear_topk_sparsify_i8(_ptr(x), M, K, ld, int(k), _ptr(out), _ptr(xs),
                                            _ptr(mk), _stream(stream)))
    return out, xs, mk


def _gemm(fn: str, a: torch.Tensor, xs, Wp, gamma, group_ends, K: int, y=None, status=None,
          stream=None):
    ge = np.ascontiguousarray(group_ends, dtype=np.int64)
    _check_gemm_operands(a, torch.uint8 if fn.endswith("fp4") else torch.int8, xs, Wp, gamma,
                         len(ge), K, y)
    _require_cuda(a, xs, Wp, gamma)
    M = a.shape[0]
    N = Wp.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=a.device)
    if status is None:
        status = status_buffer(a.device)
    _check(getattr(lib(), fn)(_ptr(a), _ptr(xs), _ptr(Wp), _ptr(gamma), _ptr(ge), len(ge), M, N, K,
                              _ptr(y), y.stride(0), _ptr(status), _stream(stream)))
    return y


def gemm_w2a8(xq, xs, Wp, gamma, group_ends, y=None, status=None, stream=None):
    """y = bf16((xq @ W_t) * xs[m] * gamma[group(n)]) on tensor cores (int8 codes)."""
    return _gemm("bitlinear_gemm_w2a8", xq, xs, Wp, gamma, group_ends, xq.shape[1], y, status, stream)


def gemm_w2a4(xq, xs, Wp, gamma, group_ends, y=None, status=None, stream=None):
    """As gemm_w2a8 for INT4 codes held in int8."""
    return _gemm("bitlinear_gemm_w2a4", xq, xs, Wp, gamma, group_ends, xq.shape[1], y, status, stream)


def gemm_w2fp4(xf4, xs, Wp, gamma, group_ends, y=None, status=None, stream=None):
    """As gemm_w2a8 for packed e2m1 activations [M x K/2]."""
    return _gemm("bitlinear_gemm_w2fp4", xf4, xs, Wp, gamma, group_ends, 2 * xf4.shape[1], y,
                 status, stream)


def gemv_w2(xq, xs, Wp, gamma, group_ends, y=None, status=None, stream=None):
    """Decode-time variant of gemm_w2a8 for 1..64 tokens."""
    return _gemm("bitlinear_gemv_w2", xq, xs, Wp, gamma, group_ends, xq.shape[1], y, status, stream)


def gemv_w2_quant(x, mode, Wp, gamma, group_ends, up=None, y=None, status=None, stream=None):
    """Decode-time BitLinear on bf16 activations (1..8 tokens): the per-token
    INT8 / INT4 quantiser (ReLU^2-gated by `up` when given) runs inside the GEMV."""
    _need(x, "x", _BF16_LIKE)
    if up is not None:
        _need(up, "up", _BF16_LIKE)
    if x.dim() != 2 or x.stride(1) != 1 or (up is not None and up.stride() != x.stride()):
        raise ValueError("x (and up) must be row-major [M x K] with the same row stride")
    M, K = x.shape
    ge = np.ascontiguousarray(group_ends, dtype=np.int64)
    _need(Wp, "Wp", (torch.uint8,), 2, contiguous=True)
    if Wp.shape[1] * 4 != K:
        raise ValueError(f"Wp: rows of {Wp.shape[1]} bytes, expected K/4 = {K // 4}")
    _need(gamma, "gamma", (torch.float32,), 1, contiguous=True)
    if gamma.numel() < len(ge):
        raise ValueError(f"gamma: {gamma.numel()} scales for {len(ge)} column groups")
    if y is not None:
        _need(y, "y", _BF16_LIKE, 2)
        if tuple(y.shape) != (M, Wp.shape[0]) or y.stride(1) != 1:
            raise ValueError(f"y: shape {tuple(y.shape)}, expected ({M}, {Wp.shape[0]}) with unit column stride")
    _require_cuda(x, up, Wp, gamma)
    N = Wp.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    if status is None:
        status = status_buffer(x.device)
    _check(lib().bitlinear_gemv_w2_quant(_ptr(x), _ptr(up), x.stride(0), int(mode), _ptr(Wp), _ptr(gamma),
                                         _ptr(ge), len(ge), M, N, K, _ptr(y), y.stride(0), _ptr(status),
                                         _stream(stream)))
    return y


def _check_acc_operands(a, code_dtype, Wp, K: int):
    """Codes [M x *] contiguous, Wp uint8 [N x K/4] contiguous."""
    _need(a, "activation codes", (code_dtype,), 2, contiguous=True)
    _need(Wp, "Wp", (torch.uint8,), 2, contiguous=True)
    if Wp.shape[1] * 4 != K:
        raise ValueError(f"Wp: rows of {Wp.shape[1]} bytes, expected K/4 = {K // 4}")


def gemm_w2a8_acc(xq, Wp, status=None, stream=None):
    """Raw int32 accumulators [M x N] of the int8 GEMM."""
    _check_acc_operands(xq, torch.int8, Wp, xq.shape[1])
    _require_cuda(xq, Wp)
    M, K = xq.shape
    N = Wp.shape[0]
    acc = torch.empty((M, N), dtype=torch.int32, device=xq.device)
    status = status if status is not None else status_buffer(xq.device)
    _check(lib().bitlinear_gemm_w2a8_acc(_ptr(xq), _ptr(Wp), M, N, K, _ptr(acc), _ptr(status),
                                         _stream(stream)))
    return acc


def gemm_w2fp4_acc(xf4, Wp, status=None, stream=None):
    """Raw fp32 accumulators [M x N] of the FP4 GEMM."""
    _check_acc_operands(xf4, torch.uint8, Wp, 2 * xf4.shape[1])
    _require_cuda(xf4, Wp)
    M, Kh = xf4.shape
    N = Wp.shape[0]
    acc = torch.empty((M, N), dtype=torch.float32, device=xf4.device)
    status = status if status is not None else status_buffer(xf4.device)
    _check(lib().bitlinear_gemm_w2fp4_acc(_ptr(xf4), _ptr(Wp), M, N, 2 * Kh, _ptr(acc),
                                          _ptr(status), _stream(stream)))
    return acc


def _check_kv_store(prefix: str, codes3, codes4, scale, T: int, H: int, D: int, n4: int):
    """The (codes3, codes4, scale) of a 3-bit cache of T tokens, H heads, head
    dim D with n4 tokens at 4 bits: uint8 [T x H x 3D/8], uint8 [n4 x H x D/2]
    (None when n4 == 0), fp32 [T x H], all contiguous."""
    for t, name, dt, shape in ((codes3, "codes3", torch.uint8, (T, H, 3 * D // 8)),
                               (scale, "scale", torch.float32, (T, H)),
                               (codes4, "codes4", torch.uint8, (n4, H, D // 2))):
        if t is None:
            if name == "codes4" and n4 == 0:
                continue
            raise ValueError(f"{prefix}{name}: missing")
        _need(t, prefix + name, (dt,), len(shape), contiguous=True)
        if tuple(t.shape) != shape:
            raise ValueError(f"{prefix}{name}: shape {tuple(t.shape)}, expected {shape}")


def kv_quant_3bit(kv: torch.Tensor, keep4_pos: torch.Tensor | None, codes3=None, codes4=None,
                  scale=None, stream=None):
    """3-bit per-(token, head) KV quantiser; listed tokens at 4 bits."""
    if kv.dim() != 3 or not kv.is_contiguous():
        raise ValueError("kv must be a contiguous [T x H x D] tensor")
    _need(kv, "kv", _BF16_LIKE)
    T, H, D = kv.shape
    n4 = 0 if keep4_pos is None else keep4_pos.numel()
    if keep4_pos is not None:
        _need(keep4_pos, "keep4_pos", (torch.int32,), 1, contiguous=True)
    if codes3 is None:
        codes3 = torch.empty((T, H, 3 * D // 8), dtype=torch.uint8, device=kv.device)
    if codes4 is None and n4:
        codes4 = torch.empty((n4, H, D // 2), dtype=torch.uint8, device=kv.device)
    if scale is None:
        scale = torch.empty((T, H), dtype=torch.float32, device=kv.device)
    _check_kv_store("", codes3, codes4, scale, T, H, D, n4)
    _require_cuda(kv, keep4_pos, codes3, codes4, scale)
    _check(lib().kv_quant_3bit(_ptr(kv), T, H, D, _ptr(keep4_pos), n4, _ptr(codes3), _ptr(codes4),
                               _ptr(scale), _stream(stream)))
    return codes3, codes4, scale


def kv_quant_3bit_kv(k: torch.Tensor, v: torch.Tensor, keep4_pos: torch.Tensor | None, k_store=None,
                     v_store=None, stream=None):
    """kv_quant_3bit of a layer's K and V in one launch; returns the two
    (codes3, codes4, scale) triples."""
    for name, t in (("k", k), ("v", v)):
        if t.dim() != 3 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous [T x H x D] tensor")
        _need(t, name, _BF16_LIKE)
    if tuple(k.shape) != tuple(v.shape):
        raise ValueError(f"k {tuple(k.shape)} and v {tuple(v.shape)} must have one shape")
    T, H, D = k.shape
    n4 = 0 if keep4_pos is None else keep4_pos.numel()
    if keep4_pos is not None:
        _need(keep4_pos, "keep4_pos", (torch.int32,), 1, contiguous=True)

    def store(given):
        if given is not None:
            return given
        c3 = torch.empty((T, H, 3 * D // 8), dtype=torch.uint8, device=k.device)
        c4 = torch.empty((n4, H, D // 2), dtype=torch.uint8, device=k.device) if n4 else None
        return c3, c4, torch.empty((T, H), dtype=torch.float32, device=k.device)
    ks, vs = store(k_store), store(v_store)
    _check_kv_store("k ", *ks, T, H, D, n4)
    _check_kv_store("v ", *vs, T, H, D, n4)
    _require_cuda(k, v, keep4_pos, *ks, *vs)
    _check(lib().kv_quant_3bit_kv(_ptr(k), _ptr(v), T, H, D, _ptr(keep4_pos), n4, _ptr(ks[0]), _ptr(ks[1]),
                                  _ptr(ks[2]), _ptr(vs[0]), _ptr(vs[1]), _ptr(vs[2]), _stream(stream)))
    return ks, vs


def kv_keep4_positions(token_ids: torch.Tensor, special_ids, stream=None) -> torch.Tensor:
    """Sorted positions t with token_ids[t] in special_ids (e.g. bos and eos),
    the 4-bit list of kv_quant_3bit; the count is read back to size it."""
    _require_cuda(token_ids)
    if token_ids.dtype != torch.int32 or token_ids.dim() != 1 or not token_ids.is_contiguous():
        raise ValueError("token_ids must be a contiguous 1-D int32 tensor")
    sp = (_c.c_int32 * len(special_ids))(*[int(v) for v in special_ids])
    T = token_ids.numel()
    pos = torch.empty(max(T, 1), dtype=torch.int32, device=token_ids.device)
    count = torch.zeros(1, dtype=torch.int32, device=token_ids.device)
    _check(lib().kv_keep4_positions(_ptr(token_ids), T, _c.addressof(sp), len(special_ids), _ptr(pos),
                                    _ptr(count), _stream(stream)))
    (stream or torch.cuda.current_stream(token_ids.device)).synchronize()
    return pos[:int(count.item())]


def kv_attention_3bit(q: torch.Tensor, k_store, v_store, keep4_pos: torch.Tensor | None, out=None,
                      status=None, stream=None):
    """Decode attention of q [B x H x D] (bf16) over a 3-bit KV cache; k_store
    and v_store are the (codes3, codes4, scale) triples of kv_quant_3bit."""
    k3, k4, ks = k_store
    v3, v4, vs = v_store
    if q.dim() != 3 or not q.is_contiguous():
        raise ValueError("q must be a contiguous [B x H x D] tensor")
    _need(q, "q", _BF16_LIKE)
    B, H, D = q.shape
    if k3.dim() != 3:
        raise ValueError("k codes3 must be [T x H x 3D/8]")
    T = k3.shape[0]
    n4 = 0 if keep4_pos is None else keep4_pos.numel()
    if keep4_pos is not None:
        _need(keep4_pos, "keep4_pos", (torch.int32,), 1, contiguous=True)
    _check_kv_store("k ", k3, k4, ks, T, H, D, n4)
    _check_kv_store("v ", v3, v4, vs, T, H, D, n4)
    if out is not None:
        _need(out, "out", _BF16_LIKE, 3, contiguous=True)
        if tuple(out.shape) != (B, H, D):
            raise ValueError(f"out: shape {tuple(out.shape)}, expected {(B, H, D)}")
    _require_cuda(q, k3, k4, ks, v3, v4, vs, keep4_pos, out)
    if out is None:
        out = torch.empty((B, H, D), dtype=torch.bfloat16, device=q.device)
    if status is None:
        status = status_buffer(q.device)
    _check(lib().kv_attention_3bit(_ptr(q), B, H, D, T, _ptr(k3), _ptr(k4), _ptr(ks), _ptr(v3), _ptr(v4),
                                   _ptr(vs), _ptr(keep4_pos), n4, _ptr(out), _ptr(status), _stream(stream)))
    return out


def tensor_peak(kind: int, iters: int = 4096, status=None, stream=None) -> dict:
    """Dense tensor-pipe rate in the GEMMs' MMA shapes (bitlinear_tensor_peak):
    kind 0 = kind::i8 CTA pairs 256x256x32, 1 = kind::mxf4 pairs 256x256x64,
    2 = kind::i8 one CTA 128x256x32. Returns {'tops', 'units', 'max_ns'}."""
    dev = torch.device("cuda", torch.cuda.current_device())
    ns = torch.zeros(torch.cuda.get_device_properties(dev).multi_processor_count, dtype=torch.int64, device=dev)
    units = _c.c_int(0)
    status = status if status is not None else status_buffer(dev)
    _check(lib().bitlinear_tensor_peak(int(kind), int(iters), _ptr(ns), _c.addressof(units), _ptr(status),
                                       _stream(stream)))
    (stream or torch.cuda.current_stream()).synchronize()
    n = units.value
    max_ns = int(ns[:n].max().item())
    M, N, K = {0: (256, 256, 32), 1: (256, 256, 64), 2: (128, 256, 32)}[int(kind)]
    return {"tops": n * 4 * iters * 2 * M * N * K / max_ns * 1e-3, "units": n, "max_ns": max_ns}


def check_status(status: torch.Tensor | None = None, stream=None):
    """Synchronise and raise BitlinearError(ERR_TIMEOUT) if a kernel gave up a wait."""
    status = status if status is not None else status_buffer()
    _check(lib().bitlinear_check_status(_ptr(status), _stream(stream)))


def debug_wait_timeout(status: torch.Tensor, timeout_ns: int, stream=None):
    _check(lib().bitlinear_debug_wait_timeout(_ptr(status), int(timeout_ns), _stream(stream)))
