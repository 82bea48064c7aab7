"""GPU parity at the workloads' full sizes, in the launch configurations the benchmark uses,
checked against the oracle on sampled outputs (tolerances as in test_gpu_parity.py).

  c2: Llama-3.1-8B-shaped decode, 8 kv-heads x 32768 tokens (last 128 kept in bf16), b = 4, 3;
      also fused with the values (tq_attention, b-bit value cache)
  c3: values at 128K context, 8 x 131072, MSE-only 3 and 4 bits, P ~ N(0, 4), 32 q-heads
  c4: batched decode, 64 sequences x 8 kv-heads x 8192 tokens, b = 3, 32 q-heads per sequence
  c5: vector search, 1,000,000 x d=200 database, 10,000 queries, b = 2 and 4, top-10
"""
import math

import numpy as np
import pytest

import oracle
import tq_inputs as ti
from gpu_helpers import (check_attention, compare_codes, gpu_quantize, make_codec, to_dev_bf16, to_dev_f32,
                         torch_cuda, tq, unpack)
from test_gpu_parity import _attention_gpu, _check_logits, _check_pv, _logits_gpu, _pv_gpu, _topk_gpu, check_topk

pytestmark = pytest.mark.gpu
RNG = np.random.default_rng(2026)


def _cb(d, B):
    c, t, _, _ = oracle.codebook(d, B)
    return c, t


@pytest.mark.parametrize("b", [4, 3])
def test_c2_llama_decode(b):
    cfg = ti.C2
    d = m = 128
    B = b - 1
    n_kv, n_all, n_tail, g = 8, 32768, 128, 4
    n_tok = n_all - n_tail
    pi, s = cfg.pi(), cfg.s()
    keys = np.stack([ti.key_stream(2, 0, h, n_all) for h in range(n_kv)])       # [8, 32768, 128] bf16
    qb = ti.decode_queries(2, 1, n_kv * g)
    codec = make_codec(d, m, B, True, pi, s)
    kd = to_dev_bf16(keys)
    packed, st = gpu_quantize(codec, kd, n_kv, n_tok, stride=n_all * d)
    assert st == tq().TQ_OK
    tail = to_dev_bf16(np.ascontiguousarray(keys[:, n_tok:]))
    got = _logits_gpu(codec, packed, 1, n_kv, n_tok, to_dev_bf16(qb), g, tail, n_tail, 1.0 / math.sqrt(d))[0]
    idx, sbit, nhat, ghat = unpack(codec, packed, n_kv, n_tok)
    c, t = _cb(d, B)
    q = ti.bf16_to_f64(qb)[0]
    kf = ti.bf16_to_f64(keys)
    for h in range(n_kv):
        samp = np.sort(RNG.choice(n_tok, 256, replace=False))
        ref = oracle.quantize(kf[h, samp], pi, s, c, t, B, qjl=True)
        compare_codes(idx[h, samp], sbit[h, samp], nhat[h, samp], ghat[h, samp], ref, t, x=kf[h, samp], pi=pi,
                      s=s, c=c, t=t, B=B)
        qh = q[h * g:(h + 1) * g]
        want = oracle.logits(idx[h, samp], sbit[h, samp], nhat[h, samp], ghat[h, samp], pi, s, c, qh, qjl=True,
                             scale=1.0 / math.sqrt(d))
        _check_logits(got[h * g:(h + 1) * g, samp], want, qh, np.linalg.norm(kf[h, samp], axis=1), 1.0 / math.sqrt(d))
        wt = oracle.exact_dot(kf[h, n_tok:], qh, 1.0 / math.sqrt(d))
        _check_logits(got[h * g:(h + 1) * g, n_tok:], wt, qh, np.linalg.norm(kf[h, n_tok:], axis=1), 1.0 / math.sqrt(d))


@pytest.mark.parametrize("b,vs", [(4, 0.0), (3, 0.0), (3, 1e-4)])
def test_c2_fused_attention(b, vs):
    """The c2 decode step fused: keys at b bits (b - 1 MSE + QJL), values at b bits (MSE), the last
    128 tokens in bf16. Two kv-heads are checked against the oracle composition over all 32768
    tokens by the two checks of gpu_helpers.check_attention (the oracle's P.V over the GPU's own
    logits at the P.V tolerance; the full oracle under the capped logit-error bound), plus the
    dropped weight mass when sparse values are on)."""
    d = m = 128
    n_kv, n_all, n_tail, g = 8, 32768, 128, 4
    n_tok = n_all - n_tail
    pik, sk, piv = ti.C2.pi(), ti.C2.s(), ti.C3.pi()
    keys = np.stack([ti.key_stream(2, 0, h, n_all) for h in range(n_kv)])
    vals = np.stack([ti.value_stream(h, n_all) for h in range(n_kv)])
    qb = ti.decode_queries(2, 1, n_kv * g)
    kc = make_codec(d, m, b - 1, True, pik, sk)
    vc = make_codec(d, 0, b, False, piv, None)
    pk, st = gpu_quantize(kc, to_dev_bf16(keys), n_kv, n_tok, stride=n_all * d)
    assert st == tq().TQ_OK
    pvv, st = gpu_quantize(vc, to_dev_bf16(vals), n_kv, n_tok, stride=n_all * d)
    assert st == tq().TQ_OK
    tk = to_dev_bf16(np.ascontiguousarray(keys[:, n_tok:]))
    tv = to_dev_bf16(np.ascontiguousarray(vals[:, n_tok:]))
    scale = 1.0 / math.sqrt(d)
    got = _attention_gpu(kc, vc, pk, pvv, 1, n_kv, n_tok, to_dev_bf16(qb), g, tk, tv, n_tail, scale, vs)[0]
    lg = _logits_gpu(kc, pk, 1, n_kv, n_tok, to_dev_bf16(qb), g, tk, n_tail, scale)[0]
    kidx, ksb, knh, kgh = unpack(kc, pk, n_kv, n_tok)
    vidx, vnh = unpack(vc, pvv, n_kv, n_tok)
    c_k, _ = _cb(d, b - 1)
    c_v, _ = _cb(d, b)
    q = ti.bf16_to_f64(qb)[0]
    kf, vf = ti.bf16_to_f64(keys), ti.bf16_to_f64(vals)
    for h in (0, 5):
        qh = q[h * g:(h + 1) * g]
        want = oracle.attention(kidx[h], ksb[h], knh[h], kgh[h], pik, sk, c_k, vidx[h], vnh[h], piv, c_v, qh, scale,
                                tail_k=kf[h, n_tok:], tail_v=vf[h, n_tok:])
        lo = oracle.logits(kidx[h], ksb[h], knh[h], kgh[h], pik, sk, c_k, qh, qjl=True, scale=scale)
        L = np.concatenate([lo, oracle.exact_dot(kf[h, n_tok:], qh, scale)], axis=1)
        vnorm = np.concatenate([vnh[h], np.linalg.norm(vf[h, n_tok:], axis=1)])
        V = np.concatenate([oracle.reconstruct(vidx[h], None, vnh[h], None, piv, None, c_v, qjl=False),
                            vf[h, n_tok:]])
        skip = None
        if vs > 0.0:
            skip = oracle.attention_skip_mass(kidx[h], ksb[h], knh[h], kgh[h], pik, sk, c_k, vidx[h], vnh[h], piv, c_v,
                                              qh, scale, tail_k=kf[h, n_tok:], tail_v=vf[h, n_tok:], v_skip=vs)
        err, err_c = check_attention(got[h * g:(h + 1) * g], want, L, lg[h * g:(h + 1) * g], n_tok, V, vnorm,
                                     v_skip=vs, skip_mass=skip)
        print(f"c2 attention kv-head {h}: {err.max():.2e} (full), {err_c.max():.2e} (composed)")


@pytest.mark.parametrize("B", [3, 4])
def test_c3_values_128k(B):
    d = 128
    n_kv, n_tok, g = 8, 131072, 4
    pi = ti.C3.pi()
    vals = np.concatenate([ti.value_stream(h, n_tok) for h in range(n_kv)])
    codec = make_codec(d, 0, B, False, pi, None)
    packed, st = gpu_quantize(codec, to_dev_bf16(vals), n_kv, n_tok)
    assert st == tq().TQ_OK
    P = ti.logits_p(n_kv * g, n_tok)
    got = _pv_gpu(codec, packed, 1, n_kv, n_tok, to_dev_f32(P), g)[0]
    assert np.all(np.isfinite(got))
    idx, nhat = unpack(codec, packed, n_kv, n_tok)
    c, t = _cb(d, B)
    vf = ti.bf16_to_f64(vals).reshape(n_kv, n_tok, d)
    for h in (0, 5):   # the whole softmax for two kv-heads (all 131072 tokens)
        Ph = P[h * g:(h + 1) * g]
        want = oracle.pv(idx[h], nhat[h], pi, c, Ph)
        _check_pv(got[h * g:(h + 1) * g], want, Ph.astype(np.float64), nhat[h])
        samp = np.sort(RNG.choice(n_tok, 512, replace=False))
        ref = oracle.quantize(vf[h, samp], pi, None, c, t, B, qjl=False)
        compare_codes(idx[h, samp], None, nhat[h, samp], None, ref, t, qjl=False)


def test_c4_batched_decode():
    cfg = ti.C4
    d = m = 128
    B = 2
    n_seq, n_kv, n_tok, g = 64, 8, 8192, 4
    pi, s = cfg.pi(), cfg.s()
    keys = np.empty((n_seq * n_kv, n_tok, d), np.uint16)
    for sq in range(n_seq):
        for h in range(n_kv):
            keys[sq * n_kv + h] = ti.key_stream(4, sq, h, n_tok)
    qb = ti.decode_queries(4, n_seq, n_kv * g)
    codec = make_codec(d, m, B, True, pi, s)
    packed, st = gpu_quantize(codec, to_dev_bf16(keys), n_seq * n_kv, n_tok)
    assert st == tq().TQ_OK
    got = _logits_gpu(codec, packed, n_seq, n_kv, n_tok, to_dev_bf16(qb), g, None, 0, 1.0 / math.sqrt(d))
    c, t = _cb(d, B)
    raw = packed.cpu().numpy()
    bb = codec.block_bytes()
    from tq_format import unpack_keys
    q = ti.bf16_to_f64(qb)
    for stream in RNG.choice(n_seq * n_kv, 4, replace=False):
        sq, h = divmod(int(stream), n_kv)
        seg = raw[stream * (n_tok // 32) * bb:(stream + 1) * (n_tok // 32) * bb]
        idx, sbit, nhat, ghat = unpack_keys(seg, d, m, B, 1, n_tok)
        samp = np.sort(RNG.choice(n_tok, 128, replace=False))
        kf = ti.bf16_to_f64(keys[stream, samp])
        ref = oracle.quantize(kf, pi, s, c, t, B, qjl=True)
        compare_codes(idx[0, samp], sbit[0, samp], nhat[0, samp], ghat[0, samp], ref, t, x=kf, pi=pi, s=s, c=c, t=t,
                      B=B)
        qh = q[sq, h * g:(h + 1) * g]
        want = oracle.logits(idx[0, samp], sbit[0, samp], nhat[0, samp], ghat[0, samp], pi, s, c, qh, qjl=True,
                             scale=1.0 / math.sqrt(d))
        _check_logits(got[sq][h * g:(h + 1) * g][:, samp], want, qh, np.linalg.norm(kf, axis=1), 1.0 / math.sqrt(d))


@pytest.mark.parametrize("b", [2, 4])
def test_c5_vector_search(b):
    d = m = 200
    B = b - 1
    n_db, n_q, k = 1_000_000, 10_000, 10
    pi, s = ti.C5.pi(), ti.C5.s()
    x = ti.c5_rows("db", 0, n_db)
    qs = ti.c5_rows("q", 0, n_q)
    codec = make_codec(d, m, B, True, pi, s)
    packed, st = gpu_quantize(codec, to_dev_f32(x), 1, n_db)
    assert st == tq().TQ_OK
    gidx, gsc = _topk_gpu(codec, packed, n_db, to_dev_f32(qs), n_q, k)
    idx, sbit, nhat, ghat = unpack(codec, packed, 1, n_db)
    c, t = _cb(d, B)
    samp = np.sort(RNG.choice(n_q, 48, replace=False))
    qsamp = qs[samp].astype(np.float64)
    all_scores = oracle.logits(idx[0], sbit[0], nhat[0], ghat[0], pi, s, c, qsamp, qjl=True)
    xn = np.linalg.norm(x.astype(np.float64), axis=1)
    swaps = check_topk(gidx[samp], gsc[samp], all_scores, qsamp, xn, k)
    # the MSE-only ranking on the same records (no sign K-blocks) against the oracle's first term
    midx, msc = _topk_gpu(codec, packed, n_db, to_dev_f32(qs), n_q, k, estimator=tq().TQ_EST_MSE)
    mse_scores = oracle.logits(idx[0], sbit[0], nhat[0], ghat[0], pi, s, c, qsamp, qjl=False)
    check_topk(midx[samp], msc[samp], mse_scores, qsamp, xn, k)
    # codes of a sample of database vectors
    vs = np.sort(RNG.choice(n_db, 2000, replace=False))
    ref = oracle.quantize(x[vs].astype(np.float64), pi, s, c, t, B, qjl=True)
    compare_codes(idx[0, vs], sbit[0, vs], nhat[0, vs], ghat[0, vs], ref, t, x=x[vs].astype(np.float64), pi=pi, s=s,
                  c=c, t=t, B=B)
    # recall@10 against the exact fp64 top-10 (reported, not pinned)
    ei, _ = oracle.exact_topk(x, qsamp, k)
    recall = np.mean([len(set(gidx[samp][r]) & set(ei[r])) / k for r in range(len(samp))])
    print(f"c5 b={b}: {swaps} near-tie swaps over {len(samp)} sampled queries, recall@10 = {recall:.3f}")
