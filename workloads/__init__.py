"""Seeded synthetic inputs for the BWTA / BiLLM hot path.

This module only draws random numbers. It holds none of the method's
arithmetic (no binarization, no threshold, no packing, no scales): it returns
latent fp32 weights and fp16 activations, and both the CUDA library and the
CPU oracle start from these same arrays.

Every array comes from ``numpy.random.default_rng([0, config_id, tensor_id,
*extra])`` so that any tensor can be regenerated on its own. Shapes and
distributions follow the workloads the library is measured on:

* tiny linear: M=16, K=256, N=128; W ~ N(0, 0.02); X ~ N(0, 1)
* BERT-base linear layers: M = 32 x 128 = 4096 tokens, (K, N) in
  {(768, 3072), (3072, 768)}; W ~ N(0, 0.02); X ~ Student-t(nu=4)
* LLaMA-7B projections: (K, N) in {(4096, 4096), (4096, 11008), (11008, 4096)}
  at M = 2048 (prefill) and M = 1 (decode); W ~ N(0, 0.02); X ~ Student-t(nu=3)
  with 1% of the entries (Bernoulli per element) multiplied by 20, clipped to
  the fp16 range
* attention: Q, K, V of shape [8, 12, 512, 64] ~ N(0, 1)
* BiLLM-format GEMM at the LLaMA-2-70B FFN shape: K=8192, N=28672,
  W ~ Laplace(0, 0.01), X ~ N(0, 1) at M in {1, 16, 512}
"""
from __future__ import annotations

import numpy as np

FP16_MAX = 65504.0

CFG_TINY, CFG_BERT, CFG_LLAMA, CFG_ATTN, CFG_BILLM, CFG_EDGE = 0, 1, 2, 3, 4, 5

BERT_SHAPES = [(768, 3072), (3072, 768)]            # (K, N)
LLAMA_SHAPES = [(4096, 4096), (4096, 11008), (11008, 4096)]
LLAMA_GROUP = 128
ATTN_SHAPE = (8, 12, 512, 64)                       # batch, heads, seq, head_dim
BILLM_K, BILLM_N, BILLM_BLOCK, BILLM_NSAL = 8192, 28672, 128, 8
BILLM_MS = [1, 16, 512]


def rng(*key: int) -> np.random.Generator:
    return np.random.default_rng([0, *[int(k) for k in key]])


def to_fp16(x: np.ndarray) -> np.ndarray:
    """Clip to the finite fp16 range and round to fp16 (round-to-nearest)."""
    return np.clip(x, -FP16_MAX, FP16_MAX).astype(np.float16)


# ---------------------------------------------------------------- primitives
def latent_normal(shape, std, *key) -> np.ndarray:
    return rng(*key).normal(0.0, std, size=shape).astype(np.float32)


def latent_laplace(shape, scale, *key) -> np.ndarray:
    return rng(*key).laplace(0.0, scale, size=shape).astype(np.float32)


def acts_normal(shape, *key) -> np.ndarray:
    return to_fp16(rng(*key).standard_normal(size=shape))


def acts_student_t(shape, nu, *key, outlier_frac=0.0, outlier_mult=20.0) -> np.ndarray:
    g = rng(*key)
    x = g.standard_t(nu, size=shape)
    if outlier_frac > 0.0:
        hit = g.random(size=shape) < outlier_frac
        x = np.where(hit, x * outlier_mult, x)
    return to_fp16(x)


# ---------------------------------------------------------------- workloads
def tiny():
    M, K, N = 16, 256, 128
    W = latent_normal((N, K), 0.02, CFG_TINY, 0)
    X = acts_normal((M, K), CFG_TINY, 1)
    return dict(M=M, K=K, N=N, group=0, W=W, X=X)


def bert(shape_idx: int, M: int = 4096):
    K, N = BERT_SHAPES[shape_idx]
    W = latent_normal((N, K), 0.02, CFG_BERT, 0, shape_idx)
    X = acts_student_t((M, K), 4, CFG_BERT, 1, shape_idx, M)
    return dict(M=M, K=K, N=N, group=0, W=W, X=X)


def llama_weights(shape_idx: int):
    K, N = LLAMA_SHAPES[shape_idx]
    return latent_normal((N, K), 0.02, CFG_LLAMA, 0, shape_idx)


def llama_acts(shape_idx: int, M: int, stream: int = 0):
    """``stream`` selects an independent batch (another rank or another step)."""
    K, _ = LLAMA_SHAPES[shape_idx]
    return acts_student_t((M, K), 3, CFG_LLAMA, 1, shape_idx, M, stream, outlier_frac=0.01)


def llama(shape_idx: int, M: int, stream: int = 0):
    K, N = LLAMA_SHAPES[shape_idx]
    return dict(M=M, K=K, N=N, group=LLAMA_GROUP, W=llama_weights(shape_idx),
                X=llama_acts(shape_idx, M, stream))


def attn(shape=ATTN_SHAPE):
    Q = acts_normal(shape, CFG_ATTN, 0, *shape)
    Kt = acts_normal(shape, CFG_ATTN, 1, *shape)
    return dict(Q=Q, K=Kt)


def attn_v(shape=ATTN_SHAPE):
    """V of the attention workload, [batch, heads, seq, head_dim] ~ N(0, 1)."""
    return acts_normal(shape, CFG_ATTN, 2, *shape)


def billm_weights(N: int = BILLM_N, K: int = BILLM_K):
    return latent_laplace((N, K), 0.01, CFG_BILLM, 0, N, K)


def billm_acts(M: int, K: int = BILLM_K, stream: int = 0):
    return acts_normal((M, K), CFG_BILLM, 1, M, K, stream)


def edge_acts(M: int, K: int, kind: str, tag: int = 0) -> np.ndarray:
    """Activation rows for edge cases, as fp16.

    kind: 'normal' | 'student' | 'zeros' | 'big' (values near +-65504) |
    'subnormal' (fp16 subnormals only) | 'negzero' (mix of -0.0 and 0.0).
    """
    g = rng(CFG_EDGE, 1, M, K, tag)
    if kind == 'normal':
        return to_fp16(g.standard_normal((M, K)))
    if kind == 'student':
        return to_fp16(g.standard_t(3, (M, K)))
    if kind == 'zeros':
        return np.zeros((M, K), np.float16)
    if kind == 'big':
        return to_fp16(g.choice([-1.0, 1.0], (M, K)) * g.uniform(30000.0, FP16_MAX, (M, K)))
    if kind == 'subnormal':
        bits = g.integers(0, 0x400, (M, K), dtype=np.uint16)
        bits |= (g.integers(0, 2, (M, K), dtype=np.uint16) << 15)
        return bits.view(np.float16)
    if kind == 'negzero':
        bits = np.where(g.random((M, K)) < 0.5, 0x8000, 0x0000).astype(np.uint16)
        return bits.view(np.float16)
    raise ValueError(kind)


def edge_weights(N: int, K: int, tag: int = 0) -> np.ndarray:
    return latent_normal((N, K), 0.02, CFG_EDGE, 0, N, K, tag)
