"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module holds no arithmetic of the method: it only draws random numbers
(numpy PCG64) and rounds them into the storage types the calls take
(fp32 weights, bf16 activations, fp16 diagonals, random sign words).  16-bit
values are returned as uint16 bit patterns.

Recipes (the pages' workloads stand in by shape; no model or dataset):
  tiny    seed 0: W 512x1024 ~ N(0, 0.02); x 1x1024 bf16 ~ N(0, 1)
  gemv    seed 1: W N x K ~ N(0, 0.02); x B x K bf16 ~ N(0, 1)
  gemm    seed 2: W N x K ~ N(0, 0.02); x M x K bf16 ~ N(0, 1)
  moe     seed 3: x T x H bf16 ~ N(0, 1); logits T x E fp32 ~ N(0, 1);
          expert gate/up I x H and down H x I fp32 ~ N(0, 0.02)
  dbf     seed 4: U (m x r) and V (r x n) uniform random sign bits;
          diagonals fp16 |N(0, 0.05)| + 0.01; x B x n bf16 ~ N(0, 1)
  okt     seed 5: Kronecker factors H (n1 x n1) and R (n2 x n2), each the
          Q factor of a seeded N(0, 1) matrix (columns signed so that the
          triangular factor has a positive diagonal), rounded to fp32;
          weights as stored after the rotation, N x K ~ N(0, 0.02) (an
          orthogonal rotation of i.i.d. Gaussian rows is again i.i.d.
          Gaussian, so these stand for W (H kron R)); x B x K bf16 ~ N(0, 1)
  power   seed 6: power-iteration start vectors, fp32 ~ N(0, 1)
"""
from __future__ import annotations

import numpy as np

SEEDS = {"tiny": 0, "gemv": 1, "gemm": 2, "moe": 3, "dbf": 4, "okt": 5, "power": 6}


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest-even); returns uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def f32_to_fp16_bits(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32).astype(np.float16).view(np.uint16)


def normal_f32(g: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    out = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        out *= np.float32(std)
    return out


def weights(g: np.random.Generator, N: int, K: int, std: float = 0.02) -> np.ndarray:
    return normal_f32(g, (N, K), std)


def activations_bf16(g: np.random.Generator, B: int, K: int) -> np.ndarray:
    return f32_to_bf16_bits(normal_f32(g, (B, K)))


def sign_words(g: np.random.Generator, rows: int, cols: int) -> np.ndarray:
    """rows x cols/32 uint32 words of independent fair sign bits."""
    assert cols % 32 == 0
    return g.integers(0, 2**32, size=(rows, cols // 32), dtype=np.uint64).astype(np.uint32)


def diag_fp16(g: np.random.Generator, n: int) -> np.ndarray:
    return f32_to_fp16_bits(np.abs(normal_f32(g, (n,), 0.05)) + np.float32(0.01))


def tiny_case(seed: int = SEEDS["tiny"]):
    g = rng(seed)
    W = weights(g, 512, 1024)
    x = activations_bf16(g, 1, 1024)
    return W, x


def gemv_case(N: int, K: int, B: int, seed: int = SEEDS["gemv"]):
    g = rng(seed)
    return weights(g, N, K), activations_bf16(g, B, K)


def gemm_case(M: int, N: int, K: int, seed: int = SEEDS["gemm"]):
    g = rng(seed)
    return weights(g, N, K), activations_bf16(g, M, K)


def moe_case(T: int = 512, H: int = 2048, I: int = 1024, E: int = 64, seed: int = SEEDS["moe"]):
    """Returns x bf16 bits [T, H], logits f32 [T, E], gate/up f32 [E, I, H], down f32 [E, H, I]."""
    g = rng(seed)
    x = activations_bf16(g, T, H)
    logits = normal_f32(g, (T, E))
    gate = normal_f32(g, (E, I, H), 0.02)
    up = normal_f32(g, (E, I, H), 0.02)
    down = normal_f32(g, (E, H, I), 0.02)
    return x, logits, gate, up, down


def dbf_case(m: int = 4096, r: int = 4096, n: int = 4096, B: int = 1, seed: int = SEEDS["dbf"]):
    """Returns a [m], B1 words [m, r/32], mid [r], B2 words [r, n/32], b [n], x [B, n]."""
    g = rng(seed)
    B1 = sign_words(g, m, r)
    B2 = sign_words(g, r, n)
    a = diag_fp16(g, m)
    mid = diag_fp16(g, r)
    b = diag_fp16(g, n)
    x = activations_bf16(g, B, n)
    return a, B1, mid, B2, b, x


def orthogonal_f32(g: np.random.Generator, n: int) -> np.ndarray:
    """A random n x n orthogonal matrix rounded to fp32 (Q of a Gaussian)."""
    q, r = np.linalg.qr(g.standard_normal(size=(n, n)))
    q = q * np.where(np.diag(r) < 0, -1.0, 1.0)[None, :]
    return q.astype(np.float32)


def okt_case(N: int, K: int, n1: int, n2: int, B: int, seed: int = SEEDS["okt"]):
    """Returns H f32 [n1, n1], R f32 [n2, n2], rotated weights f32 [N, K], x bf16 [B, K]."""
    assert n1 * n2 == K
    g = rng(seed)
    H = orthogonal_f32(g, n1)
    R = orthogonal_f32(g, n2)
    return H, R, weights(g, N, K), activations_bf16(g, B, K)


def start_vector(n: int, seed: int = SEEDS["power"]) -> np.ndarray:
    """The fixed-seed start vector of a power iteration, fp32 [n] ~ N(0, 1)."""
    return normal_f32(rng(seed), (n,))
