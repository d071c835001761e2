"""The attention parity bound can see a lost or doubled token (CPU only).

A kernel that skips token t of a head, or counts it twice, returns o moved by
p_t (o - v_t) / (1 - p_t) or p_t (v_t - o) / (1 + p_t). The GPU parity tests
allow |kernel - oracle| <= tol (conftest.attention_tolerance), so such a slip
is caught as soon as the shift exceeds 2 tol in one output element of the
head. Here, on the oracle alone, the full decode cache of the benchmark
(4096 tokens x 32 heads x 128, bos at 4 bits) is checked for how many tokens
that holds: nearly all of them, the tokens at every 256-token tile edge
included."""
import numpy as np
import pytest

from conftest import attention_tolerance
from oracle import bitlinear_oracle as O
import workloads as W


def _shifts(q, ks, vs, keep, tol=None):
    """Per (query, head, token): is a drop / a double count of that token
    seen by the bound (some output element moves by more than 2 tol)?"""
    o, tol_new = attention_tolerance(q, ks, vs, keep)
    tol = tol_new if tol is None else tol
    p = O.kv_attention_probs_f64(q, ks, keep)                       # [b, h, t]
    v = O.kv_dequant(*vs, keep, q.shape[2]).transpose(1, 0, 2)      # [h, t, d]
    seen_drop = np.empty(p.shape, bool)
    seen_double = np.empty(p.shape, bool)
    for b in range(p.shape[0]):  # one query at a time keeps the arrays small
        dv = v - o[b][:, None, :]                                    # [h, t, d]
        pp = p[b][..., None]
        lim = 2 * tol[b][:, None, :]
        seen_drop[b] = (np.abs(pp * dv / (1 - pp)) > lim).any(axis=2)
        seen_double[b] = (np.abs(pp * dv / (1 + pp)) > lim).any(axis=2)
    return seen_drop, seen_double


@pytest.mark.parametrize("Bq", [1, 8])
def test_full_cache_bound_sees_single_tokens(Bq):
    d = W.decode_layer(batch=1, make_weights=False)
    ks, vs = O.kv_quant_3bit(d["k_cache"], (0,)), O.kv_quant_3bit(d["v_cache"], (0,))
    q = W.normal_bf16(np.random.default_rng(9), (Bq, 32, 128))
    seen_drop, seen_double = _shifts(q, ks, vs, (0,))
    T = seen_drop.shape[2]
    edge = np.zeros(T, bool)
    edge[::256] = True
    edge[255::256] = True
    assert seen_drop.mean() > 0.95 and seen_double.mean() > 0.95
    assert seen_drop[:, :, edge].mean() > 0.93 and seen_double[:, :, edge].mean() > 0.93
    # a slip at a tile edge of a head (either of its two boundary tokens) is seen
    a, b = seen_drop[:, :, 255:T - 1:256], seen_drop[:, :, 256::256]
    assert (a | b).mean() > 0.99


def test_previous_bound_was_blind():
    """For the record: the bound used before (one ulp + 2.5e-4 max|v|) let
    nearly every single-token slip through at this size."""
    d = W.decode_layer(batch=1, make_weights=False)
    ks, vs = O.kv_quant_3bit(d["k_cache"], (0,)), O.kv_quant_3bit(d["v_cache"], (0,))
    q = W.normal_bf16(np.random.default_rng(9), (1, 32, 128))
    o, _ = attention_tolerance(q, ks, vs, (0,))
    rounded = np.abs(O.bf16_to_f32(O.f64_to_bf16(o))).astype(np.float32)
    old = np.spacing(rounded).astype(np.float64) * 2 ** 16 + 2.5e-4 * np.abs(O.kv_dequant(*vs, (0,), 128)).max()
    seen_drop, _ = _shifts(q, ks, vs, (0,), tol=old)
    assert seen_drop.mean() < 0.1
