"""Seeded synthetic inputs for the TurboQuant KV-vector hot path.

This module is shared by the CPU oracle tests and the CUDA path. It holds no part of
the method's arithmetic: only the random rotation, the Gaussian sketch and the data
laws of the five workloads, each drawn from numpy's ``default_rng`` with fixed seeds.

Source of the laws (TurboQuant pages):
  * rotation: "the Q factor of the QR decomposition of a Gaussian matrix"
    (a2a-mcp.org, "What is TurboQuant", stage 1, random orthogonal rotation);
  * sketch: "S in R^{m x d} with i.i.d. standard normal entries"
    (blog.hotdry.top, "QJL residual correction");
  * key norms 4-182x value norms (blog.hotdry.top, "engineering configuration list");
  * the recent 128 tokens kept at full precision (same section);
  * GloVe-200-shaped vector search (a2a-mcp.org, benchmark section).

bf16 tensors are carried as uint16 bit patterns (round-to-nearest-even from fp32);
``bf16_to_f64`` returns their exact values.
"""
from __future__ import annotations

import dataclasses
import numpy as np

SEED_PI = 1000
SEED_S = 2000
SEED_DATA = 3000
SEED_QUERY = 4000
SEED_P = 5000


# ----------------------------------------------------------------------------- dtypes
def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    rounded = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_to_f64(b: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(b).astype(np.float64)


# ----------------------------------------------------------------------------- matrices
def haar_rotation(d: int, seed: int) -> np.ndarray:
    """Random orthogonal matrix (fp64): Householder QR of a seeded N(0,1) matrix, with the
    columns' signs fixed by sign(diag R) so that the law is Haar."""
    g = np.random.default_rng(seed).standard_normal((d, d))
    q, r = np.linalg.qr(g)
    return q * np.sign(np.diag(r))[None, :]


def hadamard_signs(d: int, seed: int) -> np.ndarray:
    """The random +-1 diagonal D of a randomized Hadamard rotation (fp64 [d])."""
    return np.where(np.random.default_rng(seed).integers(0, 2, d) == 1, 1.0, -1.0)


def hadamard_rotation(d: int, seed: int) -> np.ndarray:
    """Structured random rotation H D / sqrt(d) (fp64 [d, d]) for d a power of two: H the
    Sylvester Walsh-Hadamard matrix (H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]]), D the
    seeded +-1 diagonal of hadamard_signs. It enters the library as a dense Pi."""
    if d < 1 or d & (d - 1):
        raise ValueError("d must be a power of two")
    h = np.ones((1, 1))
    while h.shape[0] < d:
        h = np.block([[h, h], [h, -h]])
    return h * hadamard_signs(d, seed)[None, :] / np.sqrt(d)


def gaussian_sketch(m: int, d: int, seed: int) -> np.ndarray:
    """QJL projection S (fp64), i.i.d. N(0,1), row-major [m, d]."""
    return np.random.default_rng(seed).standard_normal((m, d))


# ----------------------------------------------------------------------------- configs
@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    d: int
    m: int
    key_bits: tuple  # total bits b for keys (MSE bits = b - 1), or value MSE bits for c3
    pi_seed: int
    s_seed: int

    def pi(self) -> np.ndarray:
        return haar_rotation(self.d, self.pi_seed)

    def s(self) -> np.ndarray:
        return gaussian_sketch(self.m, self.d, self.s_seed)


C1 = Config("c1_tiny", 128, 128, (3,), SEED_PI + 1, SEED_S + 1)
C2 = Config("c2_llama8b_decode", 128, 128, (4, 3), SEED_PI + 2, SEED_S + 2)
C3 = Config("c3_values_128k", 128, 128, (3, 4), SEED_PI + 3, SEED_S + 3)
C4 = Config("c4_batched_decode", 128, 128, (3,), SEED_PI + 4, SEED_S + 4)
C5 = Config("c5_vector_search", 200, 200, (2, 4), SEED_PI + 5, SEED_S + 5)
CONFIGS = {c.name: c for c in (C1, C2, C3, C4, C5)}


def _rng(*key: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence(list(key)))


# c1: 4096 keys x 128, fp32; x = rho * g/|g|, rho log-uniform in [1, 100]; 8 queries ~ N(0, I).
def c1_keys(n: int = 4096, d: int = 128) -> np.ndarray:
    r = _rng(SEED_DATA, 1)
    g = r.standard_normal((n, d))
    rho = np.exp(r.uniform(np.log(1.0), np.log(100.0), size=n))
    return (g / np.linalg.norm(g, axis=1, keepdims=True) * rho[:, None]).astype(np.float32)


def c1_queries(nq: int = 8, d: int = 128) -> np.ndarray:
    return _rng(SEED_QUERY, 1).standard_normal((nq, d)).astype(np.float32)


# c2/c4 key law: per kv-head 4 outlier channels (x20); k_t = rho_t * |v_t| * g/|g|,
# v_t ~ N(0, I_d) a value draw, rho_t log-uniform in [4, 182].
def outlier_channels(cfg_id: int, head: int, d: int = 128, n_out: int = 4) -> np.ndarray:
    return _rng(SEED_DATA, cfg_id, 99, head).choice(d, size=n_out, replace=False)


def key_stream(cfg_id: int, seq: int, head: int, n_tok: int, d: int = 128, tok0: int = 0) -> np.ndarray:
    """Keys of one (sequence, kv-head) stream as bf16 bits [n_tok, d]. Tokens are drawn in
    chunks of 1024 with their own seeds, so any token range can be regenerated alone."""
    out = np.empty((n_tok, d), dtype=np.uint16)
    outl = outlier_channels(cfg_id, head, d)
    c0, c1 = tok0 // 1024, (tok0 + n_tok + 1023) // 1024
    for c in range(c0, c1):
        r = _rng(SEED_DATA, cfg_id, seq, head, c)
        g = r.standard_normal((1024, d)).astype(np.float32)
        g[:, outl] *= 20.0
        v = r.standard_normal((1024, d)).astype(np.float32)
        rho = np.exp(r.uniform(np.log(4.0), np.log(182.0), size=1024)).astype(np.float32)
        k = g / np.linalg.norm(g, axis=1, keepdims=True) * (rho * np.linalg.norm(v, axis=1))[:, None]
        lo, hi = max(tok0, c * 1024), min(tok0 + n_tok, (c + 1) * 1024)
        out[lo - tok0:hi - tok0] = f32_to_bf16_bits(k[lo - c * 1024:hi - c * 1024])
    return out


def decode_queries(cfg_id: int, n_seq: int, n_qh: int, d: int = 128) -> np.ndarray:
    """Query heads ~ N(0, 1) as bf16 bits [n_seq, n_qh, d]."""
    q = _rng(SEED_QUERY, cfg_id).standard_normal((n_seq, n_qh, d)).astype(np.float32)
    return f32_to_bf16_bits(q)


# c3: values ~ N(0, 1) bf16 per kv-head stream; P ~ N(0, 4) fp32 [n_qh, n_tok].
def value_stream(head: int, n_tok: int, d: int = 128, tok0: int = 0, cfg_id: int = 3) -> np.ndarray:
    out = np.empty((n_tok, d), dtype=np.uint16)
    c0, c1 = tok0 // 1024, (tok0 + n_tok + 1023) // 1024
    for c in range(c0, c1):
        v = _rng(SEED_DATA, cfg_id, head, c).standard_normal((1024, d)).astype(np.float32)
        lo, hi = max(tok0, c * 1024), min(tok0 + n_tok, (c + 1) * 1024)
        out[lo - tok0:hi - tok0] = f32_to_bf16_bits(v[lo - c * 1024:hi - c * 1024])
    return out


def logits_p(n_qh: int, n_tok: int, sigma: float = 2.0, cfg_id: int = 3) -> np.ndarray:
    return (sigma * _rng(SEED_P, cfg_id).standard_normal((n_qh, n_tok))).astype(np.float32)


# c5: anisotropic Gaussian, per-dimension std log-uniform in [0.1, 3], rows normalised.
def c5_scales(d: int = 200) -> np.ndarray:
    return np.exp(_rng(SEED_DATA, 5, 7).uniform(np.log(0.1), np.log(3.0), size=d))


def c5_rows(kind: str, r0: int, n: int, d: int = 200) -> np.ndarray:
    """Rows [r0, r0+n) of the database (kind='db') or of the query set (kind='q'), fp32.
    Drawn in chunks of 4096 rows with their own seeds."""
    sig = c5_scales(d)
    tag = 1 if kind == "db" else 2
    out = np.empty((n, d), dtype=np.float32)
    c0, c1 = r0 // 4096, (r0 + n + 4095) // 4096
    for c in range(c0, c1):
        g = _rng(SEED_DATA, 5, tag, c).standard_normal((4096, d)) * sig[None, :]
        g /= np.linalg.norm(g, axis=1, keepdims=True)
        lo, hi = max(r0, c * 4096), min(r0 + n, (c + 1) * 4096)
        out[lo - r0:hi - r0] = g[lo - c * 4096:hi - c * 4096].astype(np.float32)
    return out
