"""Seeded synthetic inputs for the BitLinear workloads.

This module only draws random numbers and casts them to bf16; it holds none of
the quantisation, packing or GEMM arithmetic. Both the CPU oracle (in tests)
and the CUDA path (in tests and the benchmark) take their inputs from here.

Shapes follow the LLaMA-like layers the pages train (700M to 7B parameters,
"BitNet a4.8: 4-bit Activations for 1-bit LLMs", Telegram review, section
"Эксперименты"), and the value distributions follow that review's section
"Метод": q/k/v/gate/up inputs close to normal, o_proj/down_proj inputs
heavy-tailed. The pages' training data and weights are not used; these draws
stand in for them.

Recipe (every array):
  * activations: ``numpy.random.default_rng(seed)``, drawn in fp32, cast to
    bf16 with round-to-nearest-even (``torch.Tensor.to(torch.bfloat16)``);
  * weights: fp32 ~ N(0, 0.02) from ``default_rng(seed + 1000)``.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

W_STD = 0.02


def to_bf16_bits(x_f32: np.ndarray) -> np.ndarray:
    """fp32 array -> bf16 bit patterns (uint16), round-to-nearest-even via torch."""
    t = torch.from_numpy(np.ascontiguousarray(x_f32, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_torch(bits: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bit patterns -> torch.bfloat16 tensor (CPU), no copy of values."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def weights(rng: np.random.Generator, K: int, N: int) -> np.ndarray:
    """fp32 W [K x N] (in x out) ~ N(0, 0.02)."""
    return rng.normal(0.0, W_STD, size=(K, N)).astype(np.float32)


def normal_bf16(rng: np.random.Generator, shape) -> np.ndarray:
    return to_bf16_bits(rng.standard_normal(size=shape, dtype=np.float32))


def outlier_bf16(rng: np.random.Generator, M: int, K: int, frac=0.01, gain=20.0):
    """N(0,1) with round(frac*K) channels (columns) scaled by `gain` before the cast."""
    x = rng.standard_normal(size=(M, K), dtype=np.float32)
    n_out = int(round(frac * K))
    ch = rng.choice(K, n_out, replace=False)
    x[:, ch] *= np.float32(gain)
    return to_bf16_bits(x), np.sort(ch)


def student_t_bf16(rng: np.random.Generator, M: int, K: int, nu=3.0):
    return to_bf16_bits(rng.standard_t(nu, size=(M, K)).astype(np.float32))


# --------------------------------------------------------------------------
# The five workloads (sizes as stated; the first is the small parity case).
# --------------------------------------------------------------------------

@dataclasses.dataclass
class Projection:
    name: str
    K: int
    group_ends: tuple  # column group ends, one weight scale per group
    W: np.ndarray | None = None  # fp32 [K x N]

    @property
    def N(self):
        return self.group_ends[-1]


def single_w2a4(seed=0):
    """W1.58A4 single layer: X [16 x 256] ~N(0,1), W [256 x 256] ~N(0,0.02)."""
    rng = np.random.default_rng(seed)
    x = normal_bf16(rng, (16, 256))
    W = weights(np.random.default_rng(seed + 1000), 256, 256)
    return dict(x=x, proj=Projection("single", 256, (256,), W))


def input_projection_prefill(seed=1, M=2048, D=2048, ffn=5632, make_weights=True):
    """q/k/v and gate/up inputs: X [M x D] N(0,1) with 1% outlier channels x20;
    fused q|k|v W [D x 3D] (three scale groups) and gate|up W [D x 2*ffn] (two)."""
    rng = np.random.default_rng(seed)
    x, ch = outlier_bf16(rng, M, D)
    wr = np.random.default_rng(seed + 1000)
    qkv = Projection("qkv", D, (D, 2 * D, 3 * D))
    gu = Projection("gate_up", D, (ffn, 2 * ffn))
    if make_weights:
        qkv.W = weights(wr, D, 3 * D)
        gu.W = weights(wr, D, 2 * ffn)
    return dict(x=x, outlier_channels=ch, projs=[qkv, gu])


def o_proj_sparse(seed=2, M=4096, D=4096, make_weights=True):
    """o_proj input: X [M x D] Student-t (nu=3); W [D x D]."""
    rng = np.random.default_rng(seed)
    x = student_t_bf16(rng, M, D)
    p = Projection("o_proj", D, (D,))
    if make_weights:
        p.W = weights(np.random.default_rng(seed + 1000), D, D)
    return dict(x=x, proj=p)


def down_proj_relu2(seed=3, M=4096, D=4096, ffn=11008, make_weights=True):
    """down_proj input pieces: gate, up [M x ffn] N(0,1); W [ffn x D]."""
    rng = np.random.default_rng(seed)
    gate = normal_bf16(rng, (M, ffn))
    up = normal_bf16(rng, (M, ffn))
    p = Projection("down_proj", ffn, (D,))
    if make_weights:
        p.W = weights(np.random.default_rng(seed + 1000), ffn, D)
    return dict(gate=gate, up=up, proj=p)


def decode_layer(seed=4, batch=1, D=4096, ffn=11008, T=4096, H=32, Dh=128,
                 make_weights=True, make_kv=True):
    """One LLaMA-7B-shaped decoder layer at decode time: `batch` tokens through
    q, k, v, o [D x D], gate, up [D x ffn], down [ffn x D]; K and V caches
    [T x H x Dh] ~N(0,1) with the bos token at position 0."""
    rng = np.random.default_rng(seed)
    x = normal_bf16(rng, (batch, D))          # input of q/k/v/gate/up
    xo = student_t_bf16(rng, batch, D)        # input of o_proj
    gate = normal_bf16(rng, (batch, ffn))     # down_proj input pieces
    up = normal_bf16(rng, (batch, ffn))
    wr = np.random.default_rng(seed + 1000)
    projs = [Projection(n, D, (D,)) for n in ("q", "k", "v", "o")]
    projs += [Projection("gate", D, (ffn,)), Projection("up", D, (ffn,)),
              Projection("down", ffn, (D,))]
    if make_weights:
        for p in projs:
            p.W = weights(wr, p.K, p.N)
    out = dict(x=x, xo=xo, gate=gate, up=up, projs=projs, keep4_pos=np.array([0], np.int32))
    if make_kv:
        kr = np.random.default_rng(seed + 2000)
        out["k_cache"] = normal_bf16(kr, (T, H, Dh))
        out["v_cache"] = normal_bf16(kr, (T, H, Dh))
    return out
