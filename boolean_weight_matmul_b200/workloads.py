"""Seeded synthetic inputs for the MBOK linear layer.

This module only draws random numbers.  It holds none of the method's
arithmetic (no packing, no scaling, no products), so that the CUDA path and the
CPU oracle can both be fed from it without sharing any computation.

Shapes follow the LLaMA-7B / LLaMA-13B linear layers that the MBOK pages
evaluate ("Highly Efficient and Effective LLMs with Multi-Boolean
Architectures", results section: LLaMA-7B/13B, A100 speed-up on LLaMA-13B
linear layers).  Values follow the recipe of each workload:

* Boolean kernels: every bit is an independent Bernoulli(0.5) draw, produced
  as uniform random 32-bit words, so the draw does not depend on the bit
  layout.
* Scales alpha (fp16, one per kernel k, output row r and 128-column group g):
  either 0.02*|N(0,1)| or a decaying 0.02 * 2^-(k-1) * U(0.5, 1.5).
* Activations: N(0, 1), rounded to bf16 (round-to-nearest-even) unless fp32.
* Dense weights for residual binarisation: N(0, 0.02^2) in fp32.

Storage orders used here are the logical ones the C ABI takes as-is:
alpha is fp16 [M][N/128][K] (kernel index fastest), x is [batch][N],
signs are int8 [K][M][N].  Packed words are only ever drawn as a flat
random array whose length the caller supplies.
"""
from __future__ import annotations

import dataclasses

import numpy as np

GROUP = 128

# Seed streams within one workload.
_BITS, _ALPHA, _X, _W, _SIGNS = 0, 1, 2, 3, 4


def seed_of(workload: int, matrix: int, stream: int) -> int:
    """Seed = 1000*workload + 10*matrix + stream (stream ids above)."""
    return 1000 * workload + 10 * matrix + stream


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def random_words(n_words: int, seed: int) -> np.ndarray:
    """Uniform random uint32 words: every bit is Bernoulli(0.5)."""
    return rng(seed).integers(0, 1 << 32, size=n_words, dtype=np.uint64).astype(np.uint32)


def random_signs(K: int, M: int, N: int, seed: int, p_zero: float = 0.0) -> np.ndarray:
    """int8 [K][M][N] with entries in {-1, +1}; a fraction p_zero is set to 0
    (the packer maps 0 to +1) to exercise that edge."""
    g = rng(seed)
    s = np.where(g.random((K, M, N)) < 0.5, -1, 1).astype(np.int8)
    if p_zero > 0:
        s[g.random((K, M, N)) < p_zero] = 0
    return s


def alpha_abs_normal(K: int, M: int, N: int, seed: int) -> np.ndarray:
    """fp16 [M][N/128][K], alpha = RN16(0.02*|N(0,1)|)."""
    G = N // GROUP
    a = 0.02 * np.abs(rng(seed).standard_normal((M, G, K)))
    return a.astype(np.float16)


def alpha_decaying(K: int, M: int, N: int, seed: int) -> np.ndarray:
    """fp16 [M][N/128][K], alpha_k = RN16(0.02 * 2^-(k-1) * U(0.5, 1.5)) for k=1..K."""
    G = N // GROUP
    u = rng(seed).uniform(0.5, 1.5, size=(M, G, K))
    decay = 0.02 * np.power(2.0, -np.arange(K, dtype=np.float64))
    return (u * decay[None, None, :]).astype(np.float16)


def svid_scales(K: int, M: int, N: int, seed: int):
    """Rank-1 scales: s_in fp16 [K][N] = RN16(U(0.8, 1.2)) and s_out fp16 [K][M] =
    RN16(0.016 * 2^-(k-1) * U(0.8, 1.2)) for k=1..K (so s_out s_in^T is about
    E|W| = 0.016 for W ~ N(0, 0.02^2), halving per kernel)."""
    g = rng(seed)
    s_in = g.uniform(0.8, 1.2, size=(K, N)).astype(np.float16)
    decay = 0.016 * np.power(2.0, -np.arange(K, dtype=np.float64))
    s_out = (g.uniform(0.8, 1.2, size=(K, M)) * decay[:, None]).astype(np.float16)
    return s_in, s_out


def x_normal(batch: int, N: int, seed: int, dtype: str = "bf16") -> np.ndarray:
    """[batch][N] activations ~ N(0,1).  dtype 'f32' gives float32; 'bf16'
    gives the bf16 bit patterns as uint16 (round-to-nearest-even)."""
    x = rng(seed).standard_normal((batch, N)).astype(np.float32)
    if dtype == "f32":
        return x
    if dtype == "bf16":
        return f32_to_bf16_bits(x)
    raise ValueError(dtype)


def w_normal(M: int, N: int, seed: int, std: float = 0.02) -> np.ndarray:
    """fp32 [M][N] dense weight ~ N(0, std^2)."""
    return (std * rng(seed).standard_normal((M, N))).astype(np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest, ties to even) and return the 16-bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    nan = np.isnan(x)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    out = rounded.astype(np.uint16)
    out[nan] = 0x7FC0
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One named workload: shapes and the recipe of its synthetic inputs."""
    name: str
    index: int
    K: int
    M: int
    N: int
    batch: int = 1
    tokens: int = 0
    x_dtype: str = "bf16"
    alpha: str = "decaying"  # 'abs_normal' | 'decaying' | 'residual'


# The five workloads (sizes from the LLaMA-7B / LLaMA-13B linear layers).
TOY_GEMV = Workload("toy_k1_256x512_gemv_b1_f32", 1, K=1, M=256, N=512, batch=1,
                    x_dtype="f32", alpha="abs_normal")
Q_PROJ_7B = Workload("llama7b_q_proj_k3_4096x4096_gemv_b1", 2, K=3, M=4096, N=4096, batch=1)
PREFILL_7B = Workload("llama7b_q_proj_k3_4096x4096_gemm_t2048", 4, K=3, M=4096, N=4096,
                      tokens=2048)


def mlp_7b(K: int, which: str, batch: int) -> Workload:
    """LLaMA-7B MLP: gate/up 11008x4096, down 4096x11008; K in {2,3}; batch in {1,4,16}."""
    M, N = (11008, 4096) if which in ("gate", "up") else (4096, 11008)
    return Workload(f"llama7b_{which}_k{K}_{M}x{N}_gemv_b{batch}", 3, K=K, M=M, N=N,
                    batch=batch, alpha="residual")


# LLaMA-13B decoder layer: q,k,v,o 5120x5120; gate, up 13824x5120; down 5120x13824.
LLAMA13B_LAYER = (("q", 5120, 5120), ("k", 5120, 5120), ("v", 5120, 5120), ("o", 5120, 5120),
                  ("gate", 13824, 5120), ("up", 13824, 5120), ("down", 5120, 13824))
LLAMA13B_LAYERS = 40
SWEEP_K = 4
