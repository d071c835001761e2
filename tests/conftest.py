import os
import sys

import numpy as np

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workloads")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA GPU in this environment")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def golden(name):
    """Parse a tests/golden/*.txt fixture: 'key: v v v' lines, '#' comments."""
    out = {}
    with open(os.path.join(ROOT, "tests", "golden", name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            if ":" in line:
                k, v = line.split(":", 1)
                out[k.strip()] = v.split()
            else:
                parts = line.split()
                out.setdefault("_rows", []).append(parts)
    return out


def attention_tolerance(q_bits, k_store, v_store, keep):
    """(o, tol): the fp64 decode attention of the oracle and, per output
    element, the allowed distance of the kernel's bf16 result from it:
    one bf16 ulp of the rounded exact value (the output rounding), plus
    2^-16 (A + |o|) with A = sum_t p_t |v_t| for the fp32 arithmetic.

    The fp32 part: the kernel's scores are D-term dot products and its
    weighted sums run over a few hundred terms per partial sum, so their
    rounding stays near 2^-24 sqrt(n) times those magnitudes: about 2^-18 of
    A with D = 128 and scores of size ~10, a few times below 2^-16; the
    output rounding itself is half an ulp of the one allowed. The bound is
    kept this tight so that one token dropped or counted twice, p_t (v_t - o)
    in size, moves some output of its head by more than twice it for nearly
    every token (checked on the oracle in test_attention_bound_cpu.py)."""
    from oracle import bitlinear_oracle as O
    D = np.asarray(q_bits).shape[2]
    o = O.kv_attention_f64(q_bits, k_store, v_store, keep)
    p = O.kv_attention_probs_f64(q_bits, k_store, keep)
    A = np.einsum("bht,thd->bhd", p, np.abs(O.kv_dequant(*v_store, keep, D)))
    rounded = np.abs(O.bf16_to_f32(O.f64_to_bf16(o))).astype(np.float32)
    ulp = np.spacing(rounded).astype(np.float64) * 2 ** 16  # fp32 spacing -> bf16 spacing
    return o, ulp + 2.0 ** -16 * (A + np.abs(o))
