"""Pins for the oracle's score functions (CPU only): logits, reconstruction, P.V, top-k.

Each is checked against a different algorithm for the same quantity (reconstruct-then-dot
versus pre-rotated query, rotate-once versus per-token values, a full sort versus the
running top-k) and against special cases with known answers.
"""
import math

import numpy as np
import pytest

import oracle
import tq_inputs as ti


def _setup(d=64, m=64, bits=2, n=200, qjl=True, seed=0):
    c, t, _, _ = oracle.codebook(d, bits)
    pi = ti.haar_rotation(d, seed + 1)
    s = ti.gaussian_sketch(m, d, seed + 2)
    rng = np.random.default_rng(seed + 3)
    x = rng.standard_normal((n, d)) * np.exp(rng.uniform(0, 3, n))[:, None]
    q = oracle.quantize(x, pi, s, c, t, bits, qjl=qjl)
    return c, t, pi, s, x, q


def test_logits_equal_dot_with_reconstruction():
    # <q, x~> computed two ways: pre-rotated query against the codes, and the reconstructed
    # key dotted with q (they agree by linearity of Pi^T and S^T).
    c, t, pi, s, x, q = _setup()
    qs = np.random.default_rng(9).standard_normal((5, 64))
    lg = oracle.logits(q.idx, q.sbit, q.nhat, q.ghat, pi, s, c, qs, qjl=True, scale=0.5)
    xt = oracle.reconstruct(q.idx, q.sbit, q.nhat, q.ghat, pi, s, c, qjl=True)
    assert np.allclose(lg, 0.5 * qs @ xt.T, rtol=1e-12, atol=1e-12)
    # the reconstruction is x_mse + gamma sqrt(pi/2)/m S^T s, rebuilt here from its parts
    pi32 = pi.astype(np.float32).astype(np.float64)
    s32 = s.astype(np.float32).astype(np.float64)
    sg = 2.0 * q.sbit - 1.0
    want = q.nhat[:, None] * (c[q.idx] @ pi32 + (q.ghat * math.sqrt(math.pi / 2) / 64)[:, None] * (sg @ s32))
    assert np.allclose(xt, want, rtol=1e-12, atol=1e-12)


def test_basis_query_returns_reconstruction_coordinate():
    c, t, pi, s, x, q = _setup()
    xt = oracle.reconstruct(q.idx, q.sbit, q.nhat, q.ghat, pi, s, c, qjl=True)
    for i in (0, 17, 63):
        e = np.zeros(64)
        e[i] = 1.0
        lg = oracle.logits(q.idx, q.sbit, q.nhat, q.ghat, pi, s, c, e, qjl=True)
        assert np.allclose(lg[0], xt[:, i], rtol=1e-12, atol=1e-12)


def test_mse_only_logits_and_reconstruction():
    c, t, pi, s, x, q = _setup(qjl=False, bits=3)
    qs = np.random.default_rng(1).standard_normal((3, 64))
    lg = oracle.logits(q.idx, None, q.nhat, None, pi, None, c, qs, qjl=False)
    xh = oracle.reconstruct(q.idx, None, q.nhat, None, pi, None, c, qjl=False)
    assert np.allclose(lg, qs @ xh.T, rtol=1e-12, atol=1e-12)


def test_qjl_term_reduces_logit_error():
    # the 1-bit correction lowers the mean squared logit error versus MSE-only keys of the
    # same MSE bits (its estimate is unbiased; the MSE-only one is not)
    c, t, pi, s, x, q = _setup(n=2000, d=128, m=128, bits=2)
    qs = np.random.default_rng(2).standard_normal((8, 128))
    true = qs @ x.T
    with_qjl = oracle.logits(q.idx, q.sbit, q.nhat, q.ghat, pi, s, c, qs, qjl=True)
    mse_only = oracle.logits(q.idx, None, q.nhat, None, pi, None, c, qs, qjl=False)
    bias_qjl = np.mean(with_qjl - true)
    scale = np.sqrt(np.mean(true ** 2))
    assert abs(bias_qjl) / scale < 0.02
    # MSE-only inner products shrink toward 0 (E<u, x_mse> = 1 - D): regression slope < 1
    slope = np.sum(mse_only * true) / np.sum(true * true)
    assert slope < 0.95


def test_pv_special_cases_and_rotate_once():
    d, bits, nt = 32, 3, 300
    c, t, _, _ = oracle.codebook(d, bits)
    pi = ti.haar_rotation(d, 4)
    v = np.random.default_rng(5).standard_normal((nt, d))
    q = oracle.quantize(v, pi, None, c, t, bits, qjl=False)
    vh = oracle.reconstruct(q.idx, None, q.nhat, None, pi, None, c, qjl=False)
    rng = np.random.default_rng(6)
    P = (2 * rng.standard_normal((3, nt))).astype(np.float32)
    P[1] = 0.0                      # uniform attention -> mean of the values
    P[2] = 0.0
    P[2, 123] = 1e4                 # one-hot -> that value
    o = oracle.pv(q.idx, q.nhat, pi, c, P)
    assert np.allclose(o[1], vh.mean(0), rtol=1e-12, atol=1e-12)
    assert np.allclose(o[2], vh[123], rtol=1e-12, atol=1e-12)
    # rotate once: Pi^T (sum_t w_t n_t c[idx_t]) equals the per-token sum
    w = np.exp(P[0].astype(np.float64) - P[0].max())
    w /= w.sum()
    acc = (w * q.nhat) @ c[q.idx]
    assert np.allclose(o[0], acc @ pi.astype(np.float32).astype(np.float64), rtol=1e-11, atol=1e-12)


def _attention_setup(nt=200, n_tail=7, d=64, seed=20):
    c_k, t_k, _, _ = oracle.codebook(d, 2)
    c_v, t_v, _, _ = oracle.codebook(d, 3)
    pi_k, s_k = ti.haar_rotation(d, seed), ti.gaussian_sketch(d, d, seed + 1)
    pi_v = ti.haar_rotation(d, seed + 2)
    rng = np.random.default_rng(seed + 3)
    keys = rng.standard_normal((nt + n_tail, d)) * np.exp(rng.uniform(0, 2, nt + n_tail))[:, None]
    vals = rng.standard_normal((nt + n_tail, d))
    kq = oracle.quantize(keys[:nt], pi_k, s_k, c_k, t_k, 2, qjl=True)
    vq = oracle.quantize(vals[:nt], pi_v, None, c_v, t_v, 3, qjl=False)
    return dict(k_idx=kq.idx, k_sbit=kq.sbit, k_nhat=kq.nhat, k_ghat=kq.ghat, pi_k=pi_k, s_k=s_k, c_k=c_k,
                v_idx=vq.idx, v_nhat=vq.nhat, pi_v=pi_v, c_v=c_v), keys, vals


def test_attention_composes_logits_and_pv():
    # no tail: the fused result is P.V of the estimated logits (two separately pinned functions)
    a, keys, vals = _attention_setup(n_tail=0)
    qs = np.random.default_rng(21).standard_normal((4, 64))
    o = oracle.attention(**a, q=qs, scale=0.125)
    P = oracle.logits(a["k_idx"], a["k_sbit"], a["k_nhat"], a["k_ghat"], a["pi_k"], a["s_k"], a["c_k"], qs,
                      qjl=True, scale=0.125)
    want = oracle.pv(a["v_idx"], a["v_nhat"], a["pi_v"], a["c_v"], P)
    assert np.allclose(o, want, rtol=1e-5, atol=1e-6 * np.abs(want).max())


def test_attention_uniform_and_one_hot_tail():
    a, keys, vals = _attention_setup()
    nt, d = 200, 64
    vh = oracle.reconstruct(a["v_idx"], None, a["v_nhat"], None, a["pi_v"], None, a["c_v"], qjl=False)
    allv = np.concatenate([vh, vals[nt:]])
    # q = 0: every logit is 0 -> the mean over compressed and tail values together
    o = oracle.attention(**a, q=np.zeros((1, d)), scale=1.0, tail_k=keys[nt:], tail_v=vals[nt:])
    assert np.allclose(o[0], allv.mean(0), rtol=1e-12, atol=1e-12)
    # a tail key far longer than every other, the query along it: all weight on that token
    tk = keys[nt:].copy()
    tk[3] = 1e3 * np.abs(keys).max() * tk[3] / np.linalg.norm(tk[3])
    o = oracle.attention(**a, q=(tk[3] / np.linalg.norm(tk[3]))[None], scale=1.0, tail_k=tk, tail_v=vals[nt:])
    assert np.allclose(o[0], vals[nt + 3], rtol=1e-12, atol=1e-12)
    # tail only and compressed only are the two halves of the same softmax
    qs = np.random.default_rng(22).standard_normal((2, d)) * 0.1
    full = oracle.attention(**a, q=qs, scale=1.0, tail_k=keys[nt:], tail_v=vals[nt:])
    none = {k: None for k in a}
    only_tail = oracle.attention(**none, q=qs, scale=1.0, tail_k=keys[nt:], tail_v=vals[nt:])
    only_comp = oracle.attention(**a, q=qs, scale=1.0)
    assert not np.allclose(full, only_tail) and not np.allclose(full, only_comp)
    lt = qs @ keys[nt:].T
    lc = oracle.logits(a["k_idx"], a["k_sbit"], a["k_nhat"], a["k_ghat"], a["pi_k"], a["s_k"], a["c_k"], qs,
                       qjl=True)
    zt, zc = np.exp(lt).sum(1, keepdims=True), np.exp(lc).sum(1, keepdims=True)
    assert np.allclose(full, (zt * only_tail + zc * only_comp) / (zt + zc), rtol=1e-12, atol=1e-12)


def test_attention_sparse_values():
    a, keys, vals = _attention_setup(n_tail=0)
    qs = np.random.default_rng(23).standard_normal((3, 64)) * 0.3
    dense = oracle.attention(**a, q=qs, scale=1.0)
    # a threshold below every relative weight changes nothing
    assert np.array_equal(oracle.attention(**a, q=qs, scale=1.0, v_skip=1e-300), dense)
    # v_skip = 1 keeps only the largest-weight token in the value sum, the denominator keeps all
    lg = oracle.logits(a["k_idx"], a["k_sbit"], a["k_nhat"], a["k_ghat"], a["pi_k"], a["s_k"], a["c_k"], qs,
                       qjl=True)
    vh = oracle.reconstruct(a["v_idx"], None, a["v_nhat"], None, a["pi_v"], None, a["c_v"], qjl=False)
    top = lg.argmax(axis=1)
    z = np.exp(lg - lg.max(axis=1, keepdims=True)).sum(axis=1)
    assert np.allclose(oracle.attention(**a, q=qs, scale=1.0, v_skip=1.0), vh[top] / z[:, None], rtol=1e-12,
                       atol=1e-14)
    # the change is bounded by the dropped weight mass, which grows with the threshold
    sumwv = (np.exp(lg - lg.max(axis=1, keepdims=True)) / z[:, None]) @ np.linalg.norm(vh, axis=1)
    prev = np.zeros(3)
    for tau in (1e-3, 1e-2, 1e-1, 0.5):
        sp = oracle.attention(**a, q=qs, scale=1.0, v_skip=tau)
        mass = oracle.attention_skip_mass(**a, q=qs, scale=1.0, v_skip=tau)
        assert np.all(mass >= prev) and np.all(mass < 1.0)
        assert np.all(np.max(np.abs(sp - dense), axis=1) <= mass * sumwv * (1 + 1e-12))
        prev = mass
    assert prev.min() > 0.0


def test_topk_matches_full_sort():
    c, t, pi, s, x, q = _setup(n=500)
    qs = np.random.default_rng(7).standard_normal((6, 64))
    oi, osc = oracle.topk(q.idx, q.sbit, q.nhat, q.ghat, pi, s, c, qs, k=10)
    lg = oracle.logits(q.idx, q.sbit, q.nhat, q.ghat, pi, s, c, qs, qjl=True)
    for r in range(6):
        order = np.lexsort((np.arange(500), -lg[r]))[:10]
        assert oi[r].tolist() == order.tolist()
        assert np.array_equal(osc[r], lg[r][order])
    # ties go to the lower index
    dup_idx = np.concatenate([q.idx, q.idx])
    oi2, _ = oracle.topk(dup_idx, np.concatenate([q.sbit, q.sbit]), np.concatenate([q.nhat, q.nhat]),
                         np.concatenate([q.ghat, q.ghat]), pi, s, c, qs[:1], k=4)
    assert oi2[0, 0] < 500 and oi2[0, 1] == oi2[0, 0] + 500


def test_exact_topk_and_exact_dot():
    rng = np.random.default_rng(8)
    xdb = rng.standard_normal((400, 20)).astype(np.float32)
    qs = rng.standard_normal((3, 20))
    oi, osc = oracle.exact_topk(xdb, qs, 7)
    full = qs @ xdb.astype(np.float64).T
    for r in range(3):
        assert oi[r].tolist() == np.argsort(-full[r], kind="stable")[:7].tolist()
    assert np.allclose(oracle.exact_dot(xdb, qs, 2.0), 2.0 * full, rtol=1e-13)
