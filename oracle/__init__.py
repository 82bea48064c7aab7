"""fp64 CPU oracle of the TurboQuant KV-vector hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import this package. It shares no code with the CUDA library. The codebook, quantizer,
estimator, reconstruction, P.V and top-k arithmetic lives in ``tq_oracle.c`` (plain C, fp64,
one vector at a time), built into ``liboracle.so`` by ``build()``; the compositions and
variants written here in numpy (decode attention over those functions, sparse values, the
Walsh-Hadamard butterflies, 8-bit keys) use library primitives only (matmul, exp, rint).

Every function here is pinned by a test in ``tests/test_oracle_*.py`` against something
other than itself: closed forms, the printed distortions, brute force on tiny inputs,
exhaustive search, invariants (unbiasedness, orthogonality, rotate-once) and special cases.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile tq_oracle.c (gcc, -O2, OpenMP, no fast-math) into liboracle.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = ctypes.CDLL(_LIB)
    return _lib


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _u8(a):
    return np.ascontiguousarray(a, dtype=np.uint8)


def threads() -> int:
    """OpenMP threads the oracle uses (OMP_NUM_THREADS, else the process's CPU set)."""
    env = os.environ.get("OMP_NUM_THREADS")
    if env:
        return int(env)
    return len(os.sched_getaffinity(0))


# ----------------------------------------------------------------------------- API
def round_half(x) -> np.ndarray:
    """Round to IEEE binary16 (ties to even), returned as fp64."""
    lib = _load()
    a = _f64(x).ravel()
    out = np.empty_like(a)
    lib.orc_round_half_array(ctypes.c_int64(a.size), _p(a), _p(out))
    return out.reshape(np.shape(x))


def codebook(d: int, bits: int, law: str = "beta"):
    """Lloyd-Max codebook for one rotated coordinate: (centroids[L], boundaries[L-1],
    normalised mse, iterations). law='beta' is the exact finite-d law, 'gauss' its limit."""
    lib = _load()
    nl = 1 << bits
    c = np.zeros(nl)
    t = np.zeros(nl - 1)
    mse = ctypes.c_double()
    it = ctypes.c_int()
    st = lib.orc_codebook(d, bits, 0 if law == "beta" else 1, _p(c), _p(t), ctypes.byref(mse), ctypes.byref(it))
    if st != 0:
        raise RuntimeError(f"orc_codebook({d}, {bits}, {law}) -> {st}")
    return c, t, mse.value, it.value


def cell_mass(d: int, bits: int, t, law: str = "beta") -> np.ndarray:
    lib = _load()
    out = np.zeros(1 << bits)
    lib.orc_cell_mass(d, bits, 0 if law == "beta" else 1, _p(_f64(t)), _p(out))
    return out


class Quantized:
    """Unpacked quantizer output: idx [n,d] uint8, sbit [n,m] uint8, nhat/ghat (binary16 values
    as fp64), the exact n and gamma, y [n,d] and z [n,m] for band checks, flags [n]."""

    def __init__(self, **kw):
        self.__dict__.update(kw)


def quantize(x, pi, s, c, t, bits: int, qjl: bool, keep_yz: bool = True, idx_in=None) -> Quantized:
    """Quantize rows of x. With idx_in, the given indices replace the nearest-centroid step."""
    lib = _load()
    x = _f64(x)
    nv, d = x.shape
    pi = _f32(pi)
    m = int(np.shape(s)[0]) if qjl else 0
    s_ = _f32(s) if qjl else np.zeros(1, np.float32)
    idx = np.zeros((nv, d), np.uint8)
    sbit = np.zeros((nv, max(m, 1)), np.uint8)
    nhat, ghat, nex, gex = (np.zeros(nv) for _ in range(4))
    y = np.zeros((nv, d)) if keep_yz else None
    z = np.zeros((nv, max(m, 1))) if (keep_yz and qjl) else None
    flags = np.zeros(nv, np.int32)
    st = lib.orc_quantize(ctypes.c_int64(nv), d, m, bits, int(qjl), _p(x), _p(pi), _p(s_),
                          _p(_f64(c)), _p(_f64(t)), _p(idx), _p(sbit), _p(nhat), _p(ghat),
                          _p(nex), _p(gex), _p(y), _p(z), _p(flags),
                          _p(_u8(idx_in).reshape(nv, d) if idx_in is not None else None))
    if st != 0:
        raise RuntimeError(f"orc_quantize -> {st}")
    return Quantized(idx=idx, sbit=sbit[:, :m], nhat=nhat, ghat=ghat, n_exact=nex, g_exact=gex,
                     y=y, z=(z[:, :m] if z is not None else None), flags=flags)


def logits(idx, sbit, nhat, ghat, pi, s, c, q, qjl: bool, scale: float = 1.0) -> np.ndarray:
    """scale * n^ (<Pi q, c[idx]> + gamma^ sqrt(pi/2)/m <S q, s>) for every (query, key)."""
    lib = _load()
    idx = _u8(idx)
    nk, d = idx.shape
    m = int(np.shape(s)[0]) if qjl else 0
    q = _f64(q).reshape(-1, d)
    out = np.zeros((q.shape[0], nk))
    st = lib.orc_logits(ctypes.c_int64(nk), d, m, 0, int(qjl), _p(idx),
                        _p(_u8(sbit) if qjl else np.zeros(1, np.uint8)), _p(_f64(nhat)),
                        _p(_f64(ghat) if qjl else np.zeros(1)), _p(_f32(pi)),
                        _p(_f32(s) if qjl else np.zeros(1, np.float32)), _p(_f64(c)),
                        ctypes.c_int64(q.shape[0]), _p(q), ctypes.c_double(scale), _p(out))
    if st != 0:
        raise RuntimeError(f"orc_logits -> {st}")
    return out


def exact_dot(keys, q, scale: float = 1.0) -> np.ndarray:
    lib = _load()
    keys = _f64(keys)
    nk, d = keys.shape
    q = _f64(q).reshape(-1, d)
    out = np.zeros((q.shape[0], nk))
    lib.orc_exact_dot(ctypes.c_int64(nk), d, _p(keys), ctypes.c_int64(q.shape[0]), _p(q),
                      ctypes.c_double(scale), _p(out))
    return out


def reconstruct(idx, sbit, nhat, ghat, pi, s, c, qjl: bool) -> np.ndarray:
    lib = _load()
    idx = _u8(idx)
    nv, d = idx.shape
    m = int(np.shape(s)[0]) if qjl else 0
    out = np.zeros((nv, d))
    lib.orc_reconstruct(ctypes.c_int64(nv), d, m, 0, int(qjl), _p(idx),
                        _p(_u8(sbit) if qjl else np.zeros(1, np.uint8)), _p(_f64(nhat)),
                        _p(_f64(ghat) if qjl else np.zeros(1)), _p(_f32(pi)),
                        _p(_f32(s) if qjl else np.zeros(1, np.float32)), _p(_f64(c)), _p(out))
    return out


def pv(idx, nhat, pi, c, P) -> np.ndarray:
    """softmax(P[h]) . V^ for every head h, values reconstructed token by token."""
    lib = _load()
    idx = _u8(idx)
    nt, d = idx.shape
    P = _f32(P)
    nh = P.shape[0]
    out = np.zeros((nh, d))
    st = lib.orc_pv(ctypes.c_int64(nt), d, 0, _p(idx), _p(_f64(nhat)), _p(_f32(pi)), _p(_f64(c)),
                    nh, _p(P), _p(out))
    if st != 0:
        raise RuntimeError(f"orc_pv -> {st}")
    return out


def q8_quantize(x):
    """8-bit keys of the asymmetric K/V configuration (blog.hotdry.top "TurboQuant vector-search
    compression", engineering configuration list: q8_0 keys). Per 32-coordinate chunk:
    s = max|x| / 127 in fp32, codes rint(x / s) in fp32 (round half to even, clamped to
    +-127; the integer decision is taken in the kernel's precision), stored scale = s rounded
    to binary16. x [n, d] with d <= 128 -> (codes int8 [n, d], scales fp64 of binary16
    [n, ceil(d / 32)])."""
    x32 = np.ascontiguousarray(x, dtype=np.float32)
    n, d = x32.shape
    nc = (d + 31) // 32
    xp = np.zeros((n, nc * 32), np.float32)
    xp[:, :d] = x32
    ch = xp.reshape(n, nc, 32)
    am = np.abs(ch).max(axis=2)
    s = (am / np.float32(127.0)).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.where(am[:, :, None] > 0, np.clip(np.rint(ch / s[:, :, None]), -127, 127), 0)
    return q.reshape(n, nc * 32)[:, :d].astype(np.int8), s.astype(np.float16).astype(np.float64)


def q8_logits(codes, scales, q, scale: float = 1.0) -> np.ndarray:
    """scale <q, k~> with k~ = code * scale of its chunk, in fp64, for every (query, key)."""
    codes = np.asarray(codes, dtype=np.float64)
    n, d = codes.shape
    k = codes * np.repeat(np.asarray(scales, dtype=np.float64), 32, axis=1)[:, :d]
    return scale * (_f64(q).reshape(-1, d) @ k.T)


def attention_q8(k_codes, k_scales, v_idx, v_nhat, pi_v, c_v, q, scale: float, tail_k=None,
                 tail_v=None) -> np.ndarray:
    """Decode attention of the asymmetric configuration (blog.hotdry.top, engineering
    configuration list: 8-bit keys, TurboQuant values): softmax over [logits of the 8-bit
    keys, exact logits of the tail keys] times [reconstructed values, tail values], fp64."""
    q = _f64(q)
    q = q.reshape(-1, q.shape[-1])
    lg = [q8_logits(k_codes, k_scales, q, scale)]
    vals = [reconstruct(v_idx, None, v_nhat, None, pi_v, None, c_v, qjl=False)]
    if tail_k is not None and len(tail_k):
        lg.append(exact_dot(tail_k, q, scale))
        vals.append(_f64(tail_v))
    lg = np.concatenate(lg, axis=1)
    w = np.exp(lg - lg.max(axis=1, keepdims=True))
    w /= w.sum(axis=1, keepdims=True)
    return w @ np.concatenate(vals, axis=0)


def fwht_rotate(x, signs) -> np.ndarray:
    """y = H (D x) / sqrt(d) for every row of x, by the O(d log d) butterflies of the fast
    Walsh-Hadamard transform (ai-coding.wiselychen.com "Google TurboQuant KV-cache
    compression", community ports: the rotation as a Walsh-Hadamard transform); d a power of
    two, signs the +-1 diagonal D. The structured counterpart of a dense Pi = H D / sqrt(d)."""
    y = _f64(x) * _f64(signs)[None, :]
    y = y.reshape(-1, y.shape[-1]).copy()
    d = y.shape[1]
    if d & (d - 1):
        raise ValueError("d must be a power of two")
    h = 1
    while h < d:
        for i in range(0, d, 2 * h):
            a = y[:, i:i + h].copy()
            b = y[:, i + h:i + 2 * h].copy()
            y[:, i:i + h] = a + b
            y[:, i + h:i + 2 * h] = a - b
        h *= 2
    return y / np.sqrt(d)


def _attention_parts(k_idx, k_sbit, k_nhat, k_ghat, pi_k, s_k, c_k, v_idx, v_nhat, pi_v, c_v, q, scale,
                     tail_k, tail_v):
    """Logits [nh, n], values [n, d] and the compressed-token count of one kv stream."""
    q = _f64(q)
    q = q.reshape(-1, q.shape[-1])
    lgs, vals, n_comp = [], [], 0
    if k_idx is not None and len(k_idx):
        lgs.append(logits(k_idx, k_sbit, k_nhat, k_ghat, pi_k, s_k, c_k, q, qjl=True, scale=scale))
        vals.append(reconstruct(v_idx, None, v_nhat, None, pi_v, None, c_v, qjl=False))
        n_comp = len(k_idx)
    if tail_k is not None and len(tail_k):
        lgs.append(exact_dot(tail_k, q, scale))
        vals.append(_f64(tail_v))
    if not lgs:
        raise ValueError("attention over no tokens")
    return np.concatenate(lgs, axis=1), np.concatenate(vals, axis=0), n_comp


def attention(k_idx, k_sbit, k_nhat, k_ghat, pi_k, s_k, c_k, v_idx, v_nhat, pi_v, c_v, q, scale: float,
              tail_k=None, tail_v=None, v_skip: float = 0.0) -> np.ndarray:
    """Decode attention of the query heads q [nh, d] of one kv stream, in fp64:
    softmax over [estimated logits of the compressed keys, exact logits of the tail keys]
    times [reconstructed compressed values, tail values] (a2a-mcp.org "What is TurboQuant":
    scores from the codes, the weighted sum over the dequantized values; blog.hotdry.top
    "TurboQuant vector-search compression", engineering configuration list: the recent
    tokens kept at full precision). Either part may be empty (None or zero tokens).

    v_skip > 0: sparse values (ai-coding.wiselychen.com "Google TurboQuant KV-cache
    compression", community extensions, "Sparse V"): a compressed token whose weight relative
    to the largest weight, exp(l_t - max l), is below v_skip drops out of the weighted sum of
    values; the softmax denominator keeps it."""
    lg, vals, n_comp = _attention_parts(k_idx, k_sbit, k_nhat, k_ghat, pi_k, s_k, c_k, v_idx, v_nhat, pi_v, c_v, q,
                                        scale, tail_k, tail_v)
    rel = np.exp(lg - lg.max(axis=1, keepdims=True))
    w = rel / rel.sum(axis=1, keepdims=True)
    if v_skip > 0.0:
        w = w.copy()
        drop = rel < v_skip
        drop[:, n_comp:] = False
        w[drop] = 0.0
    return w @ vals


def attention_skip_mass(k_idx, k_sbit, k_nhat, k_ghat, pi_k, s_k, c_k, v_idx, v_nhat, pi_v, c_v, q, scale: float,
                        tail_k=None, tail_v=None, v_skip: float = 0.0) -> np.ndarray:
    """Per head, sum over the compressed tokens with relative weight below v_skip of w_t |v_t|,
    divided by sum_t w_t |v_t|: a bound on the normalised change any subset of those tokens
    can make when dropped from the value sum (the sparse-value error bound)."""
    lg, vals, n_comp = _attention_parts(k_idx, k_sbit, k_nhat, k_ghat, pi_k, s_k, c_k, v_idx, v_nhat, pi_v, c_v, q,
                                        scale, tail_k, tail_v)
    rel = np.exp(lg - lg.max(axis=1, keepdims=True))
    w = rel / rel.sum(axis=1, keepdims=True)
    wv = w * np.linalg.norm(vals, axis=1)[None, :]
    drop = rel < v_skip
    drop[:, n_comp:] = False
    return (wv * drop).sum(axis=1) / wv.sum(axis=1)


def topk(idx, sbit, nhat, ghat, pi, s, c, q, k: int, qjl: bool = True):
    lib = _load()
    idx = _u8(idx)
    ndb, d = idx.shape
    m = int(np.shape(s)[0]) if qjl else 0
    q = _f64(q).reshape(-1, d)
    oi = np.zeros((q.shape[0], k), np.int64)
    osc = np.zeros((q.shape[0], k))
    st = lib.orc_topk(ctypes.c_int64(ndb), d, m, 0, int(qjl), _p(idx),
                      _p(_u8(sbit) if qjl else np.zeros(1, np.uint8)), _p(_f64(nhat)),
                      _p(_f64(ghat) if qjl else np.zeros(1)), _p(_f32(pi)),
                      _p(_f32(s) if qjl else np.zeros(1, np.float32)), _p(_f64(c)),
                      ctypes.c_int64(q.shape[0]), _p(q), k, _p(oi), _p(osc))
    if st != 0:
        raise RuntimeError(f"orc_topk -> {st}")
    return oi, osc


def exact_topk(xdb, q, k: int):
    lib = _load()
    xdb = _f32(xdb)
    ndb, d = xdb.shape
    q = _f64(q).reshape(-1, d)
    oi = np.zeros((q.shape[0], k), np.int64)
    osc = np.zeros((q.shape[0], k))
    st = lib.orc_exact_topk(ctypes.c_int64(ndb), d, _p(xdb), ctypes.c_int64(q.shape[0]), _p(q), k,
                            _p(oi), _p(osc))
    if st != 0:
        raise RuntimeError(f"orc_exact_topk -> {st}")
    return oi, osc
