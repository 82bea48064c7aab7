"""GPU parity of the CUDA hot path against the fp64 oracle (through the C ABI).

Tolerances: indices and sign bits bit-exact except coordinates within 1e-5 of a decision
boundary (at most 1e-4 of all coordinates may differ there); stored |x| and gamma within one
binary16 ulp; logits |dl| / (scale |q| |x|) <= 1e-3; reconstructions |dx~|_inf / |x| <= 1e-3;
P.V |do|_inf / sum_t w_t |v_t| <= 1e-3.
"""
import math

import numpy as np
import pytest

import oracle
import tq_inputs as ti
from gpu_helpers import (TOL, check_attention, compare_codes, gpu_quantize, make_codec, to_dev_bf16, to_dev_f32,
                         torch_cuda, tq, unpack)

pytestmark = pytest.mark.gpu


def _cb(d, B):
    c, t, _, _ = oracle.codebook(d, B)
    return c, t


# ----------------------------------------------------------------------------- quantize
def test_quantize_c1_tiny_keys():
    cfg = ti.C1
    d = m = 128
    B = 2
    pi, s = cfg.pi(), cfg.s()
    x = ti.c1_keys()
    codec = make_codec(d, m, B, True, pi, s)
    packed, st = gpu_quantize(codec, to_dev_f32(x), 1, x.shape[0])
    assert st == tq().TQ_OK
    idx, sbit, nhat, ghat = unpack(codec, packed, 1, x.shape[0])
    c, t = _cb(d, B)
    ref = oracle.quantize(x.astype(np.float64), pi, s, c, t, B, qjl=True)
    nb, nm, na = compare_codes(idx[0], sbit[0], nhat[0], ghat[0], ref, t, x=x.astype(np.float64), pi=pi, s=s,
                               c=c, t=t, B=B)
    print(f"c1: {nb} coordinates in the band, {nm} differ, of {na}")


@pytest.mark.parametrize("B", [1, 2, 3])
def test_quantize_ragged_streams_bf16(B):
    # 3 streams of 77 tokens with a stream stride larger than n_tok*d (a cache with room)
    d = m = 128
    pi, s = ti.haar_rotation(d, 71), ti.gaussian_sketch(m, d, 72)
    n_tok, stride_tok = 77, 90
    bits = np.concatenate([ti.key_stream(2, 0, h, stride_tok) for h in range(3)])
    codec = make_codec(d, m, B, True, pi, s)
    packed, st = gpu_quantize(codec, to_dev_bf16(bits), 3, n_tok, stride_tok * d)
    assert st == tq().TQ_OK
    idx, sbit, nhat, ghat = unpack(codec, packed, 3, n_tok)
    c, t = _cb(d, B)
    x = ti.bf16_to_f64(bits).reshape(3, stride_tok, d)[:, :n_tok]
    for h in range(3):
        ref = oracle.quantize(x[h], pi, s, c, t, B, qjl=True)
        compare_codes(idx[h], sbit[h], nhat[h], ghat[h], ref, t, x=x[h], pi=pi, s=s, c=c, t=t, B=B)
    # unused records of the last block are zero
    raw = packed.cpu().numpy()
    from tq_format import unpack_keys
    i2, s2, n2, g2 = unpack_keys(raw, d, m, B, 3, 96)
    assert not i2[:, n_tok:].any() and not s2[:, n_tok:].any() and not n2[:, n_tok:].any()


@pytest.mark.parametrize("B", [3, 4])
def test_quantize_values(B):
    d = 128
    pi = ti.C3.pi()
    bits = np.concatenate([ti.value_stream(h, 1000) for h in range(2)])
    codec = make_codec(d, 0, B, False, pi, None)
    packed, st = gpu_quantize(codec, to_dev_bf16(bits), 2, 1000)
    assert st == tq().TQ_OK
    idx, nhat = unpack(codec, packed, 2, 1000)
    c, t = _cb(d, B)
    x = ti.bf16_to_f64(bits).reshape(2, 1000, d)
    for h in range(2):
        ref = oracle.quantize(x[h], pi, None, c, t, B, qjl=False)
        compare_codes(idx[h], None, nhat[h], None, ref, t, qjl=False)


@pytest.mark.parametrize("B", [1, 3])
def test_quantize_d200_vector_search(B):
    d = m = 200
    pi, s = ti.C5.pi(), ti.C5.s()
    x = ti.c5_rows("db", 0, 3000)
    codec = make_codec(d, m, B, True, pi, s)
    packed, st = gpu_quantize(codec, to_dev_f32(x), 1, 3000)
    assert st == tq().TQ_OK
    idx, sbit, nhat, ghat = unpack(codec, packed, 1, 3000)
    c, t = _cb(d, B)
    ref = oracle.quantize(x.astype(np.float64), pi, s, c, t, B, qjl=True)
    compare_codes(idx[0], sbit[0], nhat[0], ghat[0], ref, t, x=x.astype(np.float64), pi=pi, s=s, c=c, t=t, B=B)


@pytest.mark.parametrize("d,m,B", [(256, 256, 2), (136, 200, 3), (200, 136, 1)])
def test_quantize_wide_bf16_ragged(d, m, B):
    """Keys with 129..256 coordinates and sketch rows (the 256-wide tensor-core path) from
    bf16 rows: several streams with a ragged last block, padded coordinates and sketch rows."""
    pi, s = ti.haar_rotation(d, 121 + d), ti.gaussian_sketch(m, d, 122 + m)
    n_streams, n_tok = 3, 777
    rng = np.random.default_rng(123 + d)
    x = ti.f32_to_bf16_bits((rng.standard_normal((n_streams * n_tok, d)) * rng.uniform(0.5, 50, (n_streams * n_tok, 1)))
                            .astype(np.float32))
    codec = make_codec(d, m, B, True, pi, s)
    packed, st = gpu_quantize(codec, to_dev_bf16(x), n_streams, n_tok)
    assert st == tq().TQ_OK
    idx, sbit, nhat, ghat = unpack(codec, packed, n_streams, n_tok)
    c, t = _cb(d, B)
    xf = ti.bf16_to_f64(x).reshape(n_streams, n_tok, d)
    for st_i in range(n_streams):
        ref = oracle.quantize(xf[st_i], pi, s, c, t, B, qjl=True)
        compare_codes(idx[st_i], sbit[st_i], nhat[st_i], ghat[st_i], ref, t, x=xf[st_i], pi=pi, s=s, c=c, t=t, B=B)


def test_quantize_range_status_and_zero_vector():
    d = m = 128
    pi, s = ti.haar_rotation(d, 81), ti.gaussian_sketch(m, d, 82)
    x = np.random.default_rng(0).standard_normal((40, d)).astype(np.float32)
    x[3] = 0.0
    x[7] *= 1e5                       # |x| ~ 1.1e6 > 65504
    codec = make_codec(d, m, 2, True, pi, s)
    packed, st = gpu_quantize(codec, to_dev_f32(x), 1, 40)
    assert st == tq().TQ_ERR_RANGE
    idx, sbit, nhat, ghat = unpack(codec, packed, 1, 40)
    assert nhat[0, 3] == 0.0 and math.isinf(nhat[0, 7])
    x[7] = 1.0
    x[9, 5] = np.nan
    packed, st = gpu_quantize(codec, to_dev_f32(x), 1, 40)
    assert st == tq().TQ_ERR_RANGE
    x[9, 5] = 0.0
    packed, st = gpu_quantize(codec, to_dev_f32(x), 1, 40)
    assert st == tq().TQ_OK


# ----------------------------------------------------------------------------- logits
def _logits_gpu(codec, packed, n_seq, n_kv, n_tok, q_dev, g, tail_dev, n_tail, scale):
    torch = torch_cuda()
    m = tq()
    out = torch.full((n_seq, n_kv * g, n_tok + n_tail), float("nan"), dtype=torch.float32, device="cuda")
    ws = m.workspace(codec.workspace_bytes(m.TQ_OP_LOGITS, n_seq, n_kv, g))
    m.tq_logits(codec, packed, n_seq, n_kv, n_tok, q_dev, g, tail_dev, n_tail, scale, out, ws)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


def _check_logits(got, want, q, xnorm, scale):
    err = np.abs(got - want) / (abs(scale) * np.linalg.norm(q, axis=-1)[:, None] * xnorm[None, :])
    assert np.all(np.isfinite(got))
    assert err.max() <= TOL, f"max normalised logit error {err.max():.3e}"
    return err.max()


def test_logits_c1_tiny():
    cfg = ti.C1
    d = m = 128
    B = 2
    pi, s = cfg.pi(), cfg.s()
    x = ti.c1_keys()
    q = ti.c1_queries()
    codec = make_codec(d, m, B, True, pi, s)
    packed, _ = gpu_quantize(codec, to_dev_f32(x), 1, 4096)
    # 8 queries as one sequence with 8 kv heads? No: one kv head, g = 8 query heads
    got = _logits_gpu(codec, packed, 1, 1, 4096, to_dev_f32(q[None]), 8, None, 0, 1.0)[0]
    idx, sbit, nhat, ghat = unpack(codec, packed, 1, 4096)
    c, t = _cb(d, B)
    want = oracle.logits(idx[0], sbit[0], nhat[0], ghat[0], pi, s, c, q.astype(np.float64), qjl=True)
    _check_logits(got, want, q.astype(np.float64), np.linalg.norm(x.astype(np.float64), axis=1), 1.0)
    # end to end against the oracle's own quantization (the codes agree outside the band)
    ref = oracle.quantize(x.astype(np.float64), pi, s, c, t, B, qjl=True)
    same = np.all(ref.idx == idx[0], axis=1) & np.all(ref.sbit == sbit[0], axis=1)
    want2 = oracle.logits(ref.idx, ref.sbit, ref.nhat, ref.ghat, pi, s, c, q.astype(np.float64), qjl=True)
    _check_logits(got[:, same], want2[:, same], q.astype(np.float64),
                  np.linalg.norm(x.astype(np.float64), axis=1)[same], 1.0)
    assert same.mean() > 0.99


@pytest.mark.parametrize("B,g", [(1, 1), (2, 2), (3, 4), (2, 8), (3, 8)])
def test_logits_gqa_ragged_with_tail(B, g):
    d = m = 128
    pi, s = ti.haar_rotation(d, 91), ti.gaussian_sketch(m, d, 92)
    n_seq, n_kv, n_tok, n_tail = 2, 3, 301, 5
    keys = np.stack([np.stack([ti.key_stream(4, sq, h, n_tok + n_tail) for h in range(n_kv)]) for sq in range(n_seq)])
    comp = np.ascontiguousarray(keys[:, :, :n_tok])
    tail = np.ascontiguousarray(keys[:, :, n_tok:])
    qb = ti.decode_queries(9, n_seq, n_kv * g)
    codec = make_codec(d, m, B, True, pi, s)
    packed, _ = gpu_quantize(codec, to_dev_bf16(comp.reshape(-1, d)), n_seq * n_kv, n_tok)
    scale = 1.0 / math.sqrt(d)
    got = _logits_gpu(codec, packed, n_seq, n_kv, n_tok, to_dev_bf16(qb), g, to_dev_bf16(tail), n_tail, scale)
    idx, sbit, nhat, ghat = unpack(codec, packed, n_seq * n_kv, n_tok)
    c, t = _cb(d, B)
    q = ti.bf16_to_f64(qb)
    kf = ti.bf16_to_f64(keys)
    for sq in range(n_seq):
        for h in range(n_kv):
            st = sq * n_kv + h
            qh = q[sq, h * g:(h + 1) * g]
            want = oracle.logits(idx[st], sbit[st], nhat[st], ghat[st], pi, s, c, qh, qjl=True, scale=scale)
            xn = np.linalg.norm(kf[sq, h, :n_tok], axis=1)
            _check_logits(got[sq, h * g:(h + 1) * g, :n_tok], want, qh, xn, scale)
            wt = oracle.exact_dot(kf[sq, h, n_tok:], qh, scale)
            _check_logits(got[sq, h * g:(h + 1) * g, n_tok:], wt, qh, np.linalg.norm(kf[sq, h, n_tok:], axis=1), scale)


@pytest.mark.parametrize("n_seq,n_kv,g,n_tail,rot", [(40, 4, 4, 20, "haar"), (25, 8, 8, 33, "haar"),
                                                     (37, 5, 4, 0, "hadamard"), (61, 5, 4, 3, "hadamard")])
def test_logits_many_heads(n_seq, n_kv, g, n_tail, rot):
    """640 / 1600 query heads: the prologue takes 8 / 16 heads per CTA; tails of 20 / 33 tokens
    span two / three tail CTAs. 740 / 1220 heads with a Sylvester-ordered Hadamard rotation (the
    query transform by butterflies): 8 / 16 heads per CTA, the last CTA holding 4."""
    d = m = 128
    B = 2
    pi = ti.haar_rotation(d, 93) if rot == "haar" else ti.hadamard_rotation(d, 93)
    s = ti.gaussian_sketch(m, d, 94)
    n_tok = 70
    keys = np.stack([np.stack([ti.key_stream(4, sq, h, n_tok + n_tail) for h in range(n_kv)]) for sq in range(n_seq)])
    comp = np.ascontiguousarray(keys[:, :, :n_tok])
    tail = np.ascontiguousarray(keys[:, :, n_tok:])
    qb = ti.decode_queries(11, n_seq, n_kv * g)
    codec = make_codec(d, m, B, True, pi, s)
    packed, _ = gpu_quantize(codec, to_dev_bf16(comp.reshape(-1, d)), n_seq * n_kv, n_tok)
    scale = 1.0 / math.sqrt(d)
    got = _logits_gpu(codec, packed, n_seq, n_kv, n_tok, to_dev_bf16(qb), g, to_dev_bf16(tail), n_tail, scale)
    idx, sbit, nhat, ghat = unpack(codec, packed, n_seq * n_kv, n_tok)
    c, t = _cb(d, B)
    q = ti.bf16_to_f64(qb)
    kf = ti.bf16_to_f64(keys)
    for sq in sorted(set(range(0, n_seq, 7)) | {n_seq - 1}):   # the last sequence ends in the last CTA
        for h in range(n_kv):
            st = sq * n_kv + h
            qh = q[sq, h * g:(h + 1) * g]
            want = oracle.logits(idx[st], sbit[st], nhat[st], ghat[st], pi, s, c, qh, qjl=True, scale=scale)
            _check_logits(got[sq, h * g:(h + 1) * g, :n_tok], want, qh, np.linalg.norm(kf[sq, h, :n_tok], axis=1), scale)
            if n_tail:
                wt = oracle.exact_dot(kf[sq, h, n_tok:], qh, scale)
                _check_logits(got[sq, h * g:(h + 1) * g, n_tok:], wt, qh, np.linalg.norm(kf[sq, h, n_tok:], axis=1),
                              scale)


def test_logits_d200_codec():
    d = m = 200
    pi, s = ti.C5.pi(), ti.C5.s()
    x = ti.c5_rows("db", 0, 700)
    q = ti.c5_rows("q", 0, 4)
    for B in (1, 3):
        codec = make_codec(d, m, B, True, pi, s)
        packed, _ = gpu_quantize(codec, to_dev_f32(x), 1, 700)
        got = _logits_gpu(codec, packed, 1, 1, 700, to_dev_f32(q[None]), 4, None, 0, 1.0)[0]
        idx, sbit, nhat, ghat = unpack(codec, packed, 1, 700)
        c, t = _cb(d, B)
        want = oracle.logits(idx[0], sbit[0], nhat[0], ghat[0], pi, s, c, q.astype(np.float64), qjl=True)
        _check_logits(got, want, q.astype(np.float64), np.linalg.norm(x.astype(np.float64), axis=1), 1.0)


# ----------------------------------------------------------------------------- P.V
def _pv_gpu(codec, packed, n_seq, n_kv, n_tok, P_dev, g):
    torch = torch_cuda()
    m = tq()
    out = torch.full((n_seq, n_kv * g, codec.c.d), float("nan"), dtype=torch.float32, device="cuda")
    ws = m.workspace(codec.workspace_bytes(m.TQ_OP_PV, n_seq * n_kv, n_tok, g))
    m.tq_pv(codec, packed, n_seq, n_kv, n_tok, P_dev, g, out, ws)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


def _check_pv(got, want, P, nhat):
    w = np.exp(P - P.max(axis=1, keepdims=True))
    w /= w.sum(axis=1, keepdims=True)
    denom = w @ nhat
    err = np.max(np.abs(got - want), axis=1) / denom
    assert np.all(np.isfinite(got))
    assert err.max() <= TOL, f"max normalised P.V error {err.max():.3e}"
    return err.max()


@pytest.mark.parametrize("B,g,n_tok", [(3, 4, 5000), (4, 4, 4097), (2, 1, 100), (4, 8, 777), (1, 2, 64),
                                       (3, 4, 1), (2, 4, 31)])
def test_pv(B, g, n_tok):
    d = 128
    pi = ti.C3.pi()
    n_kv = 2
    bits = np.concatenate([ti.value_stream(h, n_tok) for h in range(n_kv)])
    codec = make_codec(d, 0, B, False, pi, None)
    packed, _ = gpu_quantize(codec, to_dev_bf16(bits), n_kv, n_tok)
    P = ti.logits_p(n_kv * g, n_tok)
    got = _pv_gpu(codec, packed, 1, n_kv, n_tok, to_dev_f32(P), g)[0]
    idx, nhat = unpack(codec, packed, n_kv, n_tok)
    c, t = _cb(d, B)
    for h in range(n_kv):
        Ph = P[h * g:(h + 1) * g]
        want = oracle.pv(idx[h], nhat[h], pi, c, Ph)
        _check_pv(got[h * g:(h + 1) * g], want, Ph.astype(np.float64), nhat[h])


@pytest.mark.parametrize("B,g", [(3, 4), (4, 8)])
def test_pv_d200_values(B, g):
    """d = 200 values pad to 256 coordinates: the 16-tile split kernel and the 256-wide merge."""
    d, n_kv, n_tok = 200, 2, 1000
    pi = ti.haar_rotation(d, 121)
    rng = np.random.default_rng(122)
    bits = ti.f32_to_bf16_bits(rng.standard_normal((n_kv * n_tok, d)).astype(np.float32))
    codec = make_codec(d, 0, B, False, pi, None)
    packed, _ = gpu_quantize(codec, to_dev_bf16(bits), n_kv, n_tok)
    P = ti.logits_p(n_kv * g, n_tok)
    got = _pv_gpu(codec, packed, 1, n_kv, n_tok, to_dev_f32(P), g)[0]
    idx, nhat = unpack(codec, packed, n_kv, n_tok)
    c, _ = _cb(d, B)
    for h in range(n_kv):
        Ph = P[h * g:(h + 1) * g]
        want = oracle.pv(idx[h], nhat[h], pi, c, Ph)
        _check_pv(got[h * g:(h + 1) * g], want, Ph.astype(np.float64), nhat[h])


def test_pv_p_rows_unaligned():
    """P whose rows do not start on a 16-byte boundary (a view one float into its buffer):
    the API takes any 4-byte aligned P; parity against the oracle as for aligned rows."""
    torch = torch_cuda()
    d, B, g, n_tok, n_kv = 128, 3, 4, 2048, 2
    pi = ti.C3.pi()
    bits = np.concatenate([ti.value_stream(h, n_tok) for h in range(n_kv)])
    codec = make_codec(d, 0, B, False, pi, None)
    packed, _ = gpu_quantize(codec, to_dev_bf16(bits), n_kv, n_tok)
    P = ti.logits_p(n_kv * g, n_tok)
    buf = torch.empty(P.size + 1, dtype=torch.float32, device="cuda")
    p_off = buf[1:].view(1, n_kv * g, n_tok)
    p_off.copy_(torch.from_numpy(P.astype(np.float32)).view(1, n_kv * g, n_tok))
    got = _pv_gpu(codec, packed, 1, n_kv, n_tok, p_off, g)[0]
    idx, nhat = unpack(codec, packed, n_kv, n_tok)
    c, _ = _cb(d, B)
    for h in range(n_kv):
        Ph = P[h * g:(h + 1) * g]
        want = oracle.pv(idx[h], nhat[h], pi, c, Ph)
        _check_pv(got[h * g:(h + 1) * g], want, Ph.astype(np.float64), nhat[h])


def test_pv_one_hot_and_uniform():
    d, B, n_tok = 128, 3, 300
    pi = ti.C3.pi()
    bits = ti.value_stream(0, n_tok)
    codec = make_codec(d, 0, B, False, pi, None)
    packed, _ = gpu_quantize(codec, to_dev_bf16(bits), 1, n_tok)
    P = np.zeros((2, n_tok), np.float32)
    P[1, 123] = 1e4
    got = _pv_gpu(codec, packed, 1, 1, n_tok, to_dev_f32(P), 2)[0]
    idx, nhat = unpack(codec, packed, 1, n_tok)
    c, _ = _cb(d, B)
    vh = oracle.reconstruct(idx[0], None, nhat[0], None, pi, None, c, qjl=False)
    assert np.max(np.abs(got[0] - vh.mean(0))) <= TOL * nhat[0].mean()
    assert np.max(np.abs(got[1] - vh[123])) <= TOL * nhat[0, 123]


# ----------------------------------------------------------------------------- fused attention
def _attention_gpu(kc, vc, pk, pvv, n_seq, n_kv, n_tok, q_dev, g, tk_dev, tv_dev, n_tail, scale, v_skip=0.0):
    torch = torch_cuda()
    m = tq()
    out = torch.full((n_seq, n_kv * g, kc.c.d), float("nan"), dtype=torch.float32, device="cuda")
    ws = m.workspace(m.tq_attention_workspace_bytes(kc, vc, n_seq, n_kv, n_tok, g, n_tail))
    m.tq_attention(kc, vc, pk, pvv, n_seq, n_kv, n_tok, q_dev, g, tk_dev, tv_dev, n_tail, scale, out, ws, v_skip=v_skip)
    torch.cuda.synchronize()
    assert m.tq_get_status(ws) == m.TQ_OK
    return out.cpu().numpy().astype(np.float64)


def _normal_stream(seed, seq, head, n):
    """N(0, I) vectors as bf16 bits [n, 128] (the value law, drawn under another seed)."""
    return ti.value_stream(head, n, cfg_id=seed * 1000 + seq)


@pytest.mark.parametrize("Bk,Bv,g,n_seq,n_kv,n_tok,n_tail,law,qs,vs", [
    (2, 3, 4, 2, 3, 301, 5, "normal", 1.0, 0.0),      # several streams, ragged last block
    (3, 4, 4, 1, 2, 5000, 128, "normal", 1.0, 0.0),   # many ranges per stream, a 128-token tail
    (1, 2, 1, 1, 2, 64, 0, "normal", 1.0, 0.0),       # no tail
    (2, 4, 2, 1, 2, 0, 33, "normal", 1.0, 0.0),       # tail only
    (3, 3, 4, 1, 1, 1000, 1, "normal", 8.0, 0.0),     # peaked softmax: the running maximum moves
    (2, 1, 4, 3, 1, 33, 7, "normal", 1.0, 0.0),       # 1-bit values, a block of one valid token
    (3, 4, 4, 1, 2, 3000, 128, "c2", 1.0, 0.0),       # the decode key law (outlier channels, long keys)
    (3, 4, 4, 1, 2, 3000, 128, "c2", 1.0, 1e-4),      # sparse values on the same data
    (2, 3, 4, 2, 2, 2000, 16, "normal", 4.0, 1e-2),   # sparse values, a milder softmax
])
def test_attention(Bk, Bv, g, n_seq, n_kv, n_tok, n_tail, law, qs, vs):
    """softmax(scale q . K) . V against the oracle on the same codes, by the two checks of
    gpu_helpers.check_attention: the oracle's P.V over the GPU's own logits at the P.V
    tolerance (softmax, value decode and merge), and the full oracle composition under the
    logit-error bound capped at ATTN_CEIL. With sparse values (vs > 0) the dropped weight mass
    (tokens whose relative weight is below vs) is added: the kernel drops a subset of them."""
    d = m = 128
    pik, sk, piv = ti.haar_rotation(d, 95), ti.gaussian_sketch(m, d, 96), ti.haar_rotation(d, 97)
    n = n_tok + n_tail
    if law == "c2":
        keys = np.stack([np.stack([ti.key_stream(4, sq, h, n) for h in range(n_kv)]) for sq in range(n_seq)])
    else:
        keys = np.stack([np.stack([_normal_stream(51, sq, h, n) for h in range(n_kv)]) for sq in range(n_seq)])
    vals = np.stack([np.stack([_normal_stream(61, sq, h, n) for h in range(n_kv)]) for sq in range(n_seq)])
    kc = make_codec(d, m, Bk, True, pik, sk)
    vc = make_codec(d, 0, Bv, False, piv, None)
    S = n_seq * n_kv
    pk = pvv = None
    if n_tok:
        pk, _ = gpu_quantize(kc, to_dev_bf16(np.ascontiguousarray(keys[:, :, :n_tok]).reshape(-1, d)), S, n_tok)
        pvv, _ = gpu_quantize(vc, to_dev_bf16(np.ascontiguousarray(vals[:, :, :n_tok]).reshape(-1, d)), S, n_tok)
    tk = to_dev_bf16(np.ascontiguousarray(keys[:, :, n_tok:])) if n_tail else None
    tv = to_dev_bf16(np.ascontiguousarray(vals[:, :, n_tok:])) if n_tail else None
    qb = ti.decode_queries(12, n_seq, n_kv * g)
    scale = qs / math.sqrt(d)
    got = _attention_gpu(kc, vc, pk, pvv, n_seq, n_kv, n_tok, to_dev_bf16(qb), g, tk, tv, n_tail, scale, vs)
    lg = _logits_gpu(kc, pk, n_seq, n_kv, n_tok, to_dev_bf16(qb), g, tk, n_tail, scale)
    if n_tok:
        kidx, ksb, knh, kgh = unpack(kc, pk, S, n_tok)
        vidx, vnh = unpack(vc, pvv, S, n_tok)
    c_k, _ = _cb(d, Bk)
    c_v, _ = _cb(d, Bv)
    q = ti.bf16_to_f64(qb)
    kf, vf = ti.bf16_to_f64(keys), ti.bf16_to_f64(vals)
    for sq in range(n_seq):
        for h in range(n_kv):
            st = sq * n_kv + h
            qh = q[sq, h * g:(h + 1) * g]
            if n_tok:
                a = dict(k_idx=kidx[st], k_sbit=ksb[st], k_nhat=knh[st], k_ghat=kgh[st], pi_k=pik, s_k=sk, c_k=c_k,
                         v_idx=vidx[st], v_nhat=vnh[st], pi_v=piv, c_v=c_v)
                lo = oracle.logits(kidx[st], ksb[st], knh[st], kgh[st], pik, sk, c_k, qh, qjl=True, scale=scale)
                vn = vnh[st]
            else:
                a = dict(k_idx=None, k_sbit=None, k_nhat=None, k_ghat=None, pi_k=None, s_k=None, c_k=None,
                         v_idx=None, v_nhat=None, pi_v=None, c_v=None)
                lo, vn = np.zeros((g, 0)), np.zeros(0)
            tkh, tvh = (kf[sq, h, n_tok:], vf[sq, h, n_tok:]) if n_tail else (None, None)
            want = oracle.attention(**a, q=qh, scale=scale, tail_k=tkh, tail_v=tvh)
            L = np.concatenate([lo, oracle.exact_dot(kf[sq, h, n_tok:], qh, scale)], axis=1)
            vnorm = np.concatenate([vn, np.linalg.norm(vf[sq, h, n_tok:], axis=1)])
            vhat = (oracle.reconstruct(vidx[st], None, vnh[st], None, piv, None, c_v, qjl=False) if n_tok
                    else np.zeros((0, d)))
            V = np.concatenate([vhat, vf[sq, h, n_tok:]])
            xn = np.linalg.norm(kf[sq, h], axis=1)
            dl_norm = np.abs(lg[sq, h * g:(h + 1) * g] - L) / (scale * np.linalg.norm(qh, axis=1)[:, None] * xn)
            assert dl_norm.max() <= TOL
            skip = None
            if vs > 0.0:
                skip = oracle.attention_skip_mass(**a, q=qh, scale=scale, tail_k=tkh, tail_v=tvh, v_skip=vs)
            err, err_c = check_attention(got[sq, h * g:(h + 1) * g], want, L, lg[sq, h * g:(h + 1) * g], n_tok, V,
                                         vnorm, v_skip=vs, skip_mass=skip)
            print(f"attention stream {st}: normalised error {err.max():.2e} (full), {err_c.max():.2e} (composed), "
                  f"logit error {dl_norm.max():.2e}")


def test_attention_narrow_codec():
    """d = 96, m = 64: the zero-padded coordinates and sketch rows of the 128-wide blocks."""
    d, m, g, n_tok, n_tail = 96, 64, 2, 200, 9
    pik, sk, piv = ti.haar_rotation(d, 98), ti.gaussian_sketch(m, d, 99), ti.haar_rotation(d, 100)
    rng = np.random.default_rng(101)
    keys = ti.f32_to_bf16_bits(rng.standard_normal((n_tok + n_tail, d)).astype(np.float32))
    vals = ti.f32_to_bf16_bits(rng.standard_normal((n_tok + n_tail, d)).astype(np.float32))
    qb = ti.f32_to_bf16_bits(rng.standard_normal((1, g, d)).astype(np.float32))
    kc = make_codec(d, m, 2, True, pik, sk)
    vc = make_codec(d, 0, 3, False, piv, None)
    pk, _ = gpu_quantize(kc, to_dev_bf16(keys[:n_tok]), 1, n_tok)
    pvv, _ = gpu_quantize(vc, to_dev_bf16(vals[:n_tok]), 1, n_tok)
    tk, tv = to_dev_bf16(keys[n_tok:]), to_dev_bf16(vals[n_tok:])
    scale = 1.0 / math.sqrt(d)
    got = _attention_gpu(kc, vc, pk, pvv, 1, 1, n_tok, to_dev_bf16(qb), g, tk, tv, n_tail, scale)[0]
    lg = _logits_gpu(kc, pk, 1, 1, n_tok, to_dev_bf16(qb), g, tk, n_tail, scale)[0]
    kidx, ksb, knh, kgh = unpack(kc, pk, 1, n_tok)
    vidx, vnh = unpack(vc, pvv, 1, n_tok)
    c_k, _ = _cb(d, 2)
    c_v, _ = _cb(d, 3)
    q = ti.bf16_to_f64(qb)[0]
    kf, vf = ti.bf16_to_f64(keys), ti.bf16_to_f64(vals)
    want = oracle.attention(kidx[0], ksb[0], knh[0], kgh[0], pik, sk, c_k, vidx[0], vnh[0], piv, c_v, q, scale,
                            tail_k=kf[n_tok:], tail_v=vf[n_tok:])
    lo = oracle.logits(kidx[0], ksb[0], knh[0], kgh[0], pik, sk, c_k, q, qjl=True, scale=scale)
    L = np.concatenate([lo, oracle.exact_dot(kf[n_tok:], q, scale)], axis=1)
    vnorm = np.concatenate([vnh[0], np.linalg.norm(vf[n_tok:], axis=1)])
    V = np.concatenate([oracle.reconstruct(vidx[0], None, vnh[0], None, piv, None, c_v, qjl=False), vf[n_tok:]])
    check_attention(got, want, L, lg, n_tok, V, vnorm)


def test_hadamard_rotation_path():
    """A randomized Walsh-Hadamard rotation H D / sqrt(d) as Pi (dense operand) for keys and
    values: codes against the oracle's quantization, logits and fused attention against the
    oracle on the same codes."""
    d = m = 128
    pik, piv = ti.hadamard_rotation(d, 31), ti.hadamard_rotation(d, 32)
    sk = ti.gaussian_sketch(m, d, 33)
    n_kv, n_tok, n_tail, g, B = 2, 700, 6, 4, 2
    keys = np.stack([ti.key_stream(4, 0, h, n_tok + n_tail) for h in range(n_kv)])
    vals = np.stack([_normal_stream(71, 0, h, n_tok + n_tail) for h in range(n_kv)])
    kc = make_codec(d, m, B, True, pik, sk)
    vc = make_codec(d, 0, 3, False, piv, None)
    pk, st = gpu_quantize(kc, to_dev_bf16(np.ascontiguousarray(keys[:, :n_tok]).reshape(-1, d)), n_kv, n_tok)
    assert st == tq().TQ_OK
    pvv, _ = gpu_quantize(vc, to_dev_bf16(np.ascontiguousarray(vals[:, :n_tok]).reshape(-1, d)), n_kv, n_tok)
    kidx, ksb, knh, kgh = unpack(kc, pk, n_kv, n_tok)
    vidx, vnh = unpack(vc, pvv, n_kv, n_tok)
    c_k, t_k = _cb(d, B)
    c_v, _ = _cb(d, 3)
    kf, vf = ti.bf16_to_f64(keys), ti.bf16_to_f64(vals)
    for h in range(n_kv):
        ref = oracle.quantize(kf[h, :n_tok], pik, sk, c_k, t_k, B, qjl=True)
        compare_codes(kidx[h], ksb[h], knh[h], kgh[h], ref, t_k, x=kf[h, :n_tok], pi=pik, s=sk, c=c_k, t=t_k, B=B)
    qb = ti.decode_queries(13, 1, n_kv * g)
    scale = 1.0 / math.sqrt(d)
    tk = to_dev_bf16(np.ascontiguousarray(keys[:, n_tok:]))
    tv = to_dev_bf16(np.ascontiguousarray(vals[:, n_tok:]))
    lg = _logits_gpu(kc, pk, 1, n_kv, n_tok, to_dev_bf16(qb), g, tk, n_tail, scale)[0]
    got = _attention_gpu(kc, vc, pk, pvv, 1, n_kv, n_tok, to_dev_bf16(qb), g, tk, tv, n_tail, scale)[0]
    q = ti.bf16_to_f64(qb)[0]
    for h in range(n_kv):
        qh = q[h * g:(h + 1) * g]
        lo = oracle.logits(kidx[h], ksb[h], knh[h], kgh[h], pik, sk, c_k, qh, qjl=True, scale=scale)
        _check_logits(lg[h * g:(h + 1) * g, :n_tok], lo, qh, np.linalg.norm(kf[h, :n_tok], axis=1), scale)
        want = oracle.attention(kidx[h], ksb[h], knh[h], kgh[h], pik, sk, c_k, vidx[h], vnh[h], piv, c_v, qh, scale,
                                tail_k=kf[h, n_tok:], tail_v=vf[h, n_tok:])
        L = np.concatenate([lo, oracle.exact_dot(kf[h, n_tok:], qh, scale)], axis=1)
        vnorm = np.concatenate([vnh[h], np.linalg.norm(vf[h, n_tok:], axis=1)])
        V = np.concatenate([oracle.reconstruct(vidx[h], None, vnh[h], None, piv, None, c_v, qjl=False),
                            vf[h, n_tok:]])
        check_attention(got[h * g:(h + 1) * g], want, L, lg[h * g:(h + 1) * g], n_tok, V, vnorm)


@pytest.mark.parametrize("d,kind,qf32", [(128, "sylvester", False), (64, "sylvester", False), (128, "xor_rows", False),
                                         (128, "permuted_rows", False), (128, "haar", False), (128, "sylvester", True),
                                         (128, "haar", True)])
def test_rotation_flags_and_wht_logits(d, kind, qf32):
    """The prepared header marks Pi = H D / sqrt(d) with H in Sylvester order (the logits
    prologue then rotates the query by a fast Walsh-Hadamard transform and reads no Pi tile):
    also with rows permuted by i -> i ^ c (H's rows multiply as their indices XOR, so that is
    H D' / sqrt(d) again), not with a generic row permutation (+-1 flag alone) nor for a Haar
    rotation (neither). Logits against the oracle on the same codes in every case, for bf16
    queries and for fp32 queries (whose rows carry a nonzero fp16 lo part: the third pass)."""
    m_ = 128
    if kind == "haar":
        pik = ti.haar_rotation(d, 61)
    else:
        pik = ti.hadamard_rotation(d, 61)
        if kind == "xor_rows":
            pik = pik[np.arange(d) ^ 37]
        elif kind == "permuted_rows":
            pik = pik[np.random.default_rng(62).permutation(d)]
    want_flags = {"sylvester": 3, "xor_rows": 3, "permuted_rows": 1, "haar": 0}[kind]
    sk = ti.gaussian_sketch(m_, d, 63)
    n_kv, n_tok, n_tail, g, B = 2, 333, 3, 4, 2
    kc = make_codec(d, m_, B, True, pik, sk)
    flags = int(kc.prep[:4].cpu().numpy().view(np.uint32)[0])
    assert flags == want_flags, (kind, flags)
    keys = np.stack([ti.key_stream(4, 1, h, n_tok + n_tail, d) for h in range(n_kv)])
    pk, st = gpu_quantize(kc, to_dev_bf16(np.ascontiguousarray(keys[:, :n_tok]).reshape(-1, d)), n_kv, n_tok)
    assert st == tq().TQ_OK
    kidx, ksb, knh, kgh = unpack(kc, pk, n_kv, n_tok)
    c_k, _ = _cb(d, B)
    kf = ti.bf16_to_f64(keys)
    scale = 1.0 / math.sqrt(d)
    tk = to_dev_bf16(np.ascontiguousarray(keys[:, n_tok:]))
    if qf32:
        qf = np.random.default_rng(64).standard_normal((1, n_kv * g, d)).astype(np.float32)
        lg = _logits_gpu(kc, pk, 1, n_kv, n_tok, to_dev_f32(qf), g, tk, n_tail, scale)[0]
        q = qf.astype(np.float64)[0]
    else:
        qb = ti.decode_queries(14, 1, n_kv * g, d)
        lg = _logits_gpu(kc, pk, 1, n_kv, n_tok, to_dev_bf16(qb), g, tk, n_tail, scale)[0]
        q = ti.bf16_to_f64(qb)[0]
    for h in range(n_kv):
        qh = q[h * g:(h + 1) * g]
        lo = oracle.logits(kidx[h], ksb[h], knh[h], kgh[h], pik, sk, c_k, qh, qjl=True, scale=scale)
        _check_logits(lg[h * g:(h + 1) * g, :n_tok], lo, qh, np.linalg.norm(kf[h, :n_tok], axis=1), scale)
        tail = oracle.exact_dot(kf[h, n_tok:], qh, scale)
        _check_logits(lg[h * g:(h + 1) * g, n_tok:], tail, qh, np.linalg.norm(kf[h, n_tok:], axis=1), scale)


def test_wht_prologue_matches_dense_product():
    """The Walsh-Hadamard query transform against the dense mma.sync product on the same
    rotation: a Hadamard Pi with one entry's magnitude moved by one fp32 ulp keeps the +-1 flag
    but not the Sylvester one, so its logits take the dense path; both codecs score the same
    packed keys (quantized under the exact Hadamard Pi) with the same queries."""
    d = m_ = 128
    pik = ti.hadamard_rotation(d, 71).astype(np.float32)
    pid = pik.copy()
    pid[5, 7] = np.nextafter(pid[5, 7], np.float32(2.0) * pid[5, 7])
    sk = ti.gaussian_sketch(m_, d, 72)
    kh, kd = make_codec(d, m_, 2, True, pik, sk), make_codec(d, m_, 2, True, pid, sk)
    assert int(kh.prep[:4].cpu().numpy().view(np.uint32)[0]) == 3
    assert int(kd.prep[:4].cpu().numpy().view(np.uint32)[0]) == 1
    n_kv, n_tok, g = 4, 500, 4
    keys = np.stack([ti.key_stream(4, 2, h, n_tok) for h in range(n_kv)])
    pk, st = gpu_quantize(kh, to_dev_bf16(np.ascontiguousarray(keys).reshape(-1, d)), n_kv, n_tok)
    assert st == tq().TQ_OK
    qb = ti.decode_queries(15, 1, n_kv * g)
    scale = 1.0 / math.sqrt(d)
    lw = _logits_gpu(kh, pk, 1, n_kv, n_tok, to_dev_bf16(qb), g, None, 0, scale)[0]
    ld = _logits_gpu(kd, pk, 1, n_kv, n_tok, to_dev_bf16(qb), g, None, 0, scale)[0]
    q = ti.bf16_to_f64(qb)[0]
    kn = np.linalg.norm(ti.bf16_to_f64(keys), axis=2)
    for h in range(n_kv):
        qh = q[h * g:(h + 1) * g]
        err = np.abs(lw[h * g:(h + 1) * g] - ld[h * g:(h + 1) * g]) / (
            scale * np.linalg.norm(qh, axis=1)[:, None] * kn[h][None, :])
        assert err.max() <= 5e-4, err.max()


def _unpack_q8(packed_dev, d, n_streams, n_tok):
    """Decode the 8-bit key blocks as the header describes them: codes [column][token][16 B],
    then binary16 scales [chunk][token]."""
    nb = (n_tok + 31) // 32
    raw = packed_dev.cpu().numpy().reshape(n_streams * nb, 4352)
    codes = raw[:, :4096].reshape(-1, 8, 32, 16).transpose(0, 2, 1, 3).reshape(n_streams, nb * 32, 128)
    scales = np.ascontiguousarray(raw[:, 4096:]).view(np.float16).reshape(-1, 4, 32).transpose(0, 2, 1)
    scales = scales.reshape(n_streams, nb * 32, 4).astype(np.float64)
    return codes.view(np.int8)[:, :n_tok, :d], scales[:, :n_tok, :(d + 31) // 32], codes.view(np.int8)[:, :, d:]


@pytest.mark.parametrize("d,g,n_seq,n_kv,n_tok,n_tail", [(128, 4, 1, 3, 301, 5), (96, 2, 2, 2, 64, 0),
                                                        (128, 1, 1, 2, 0, 9), (128, 4, 1, 2, 4100, 128)])
def test_q8_keys(d, g, n_seq, n_kv, n_tok, n_tail):
    """8-bit keys: codes and scales bit-exact against the oracle (the integer decisions are
    taken in fp32 on both sides), logits within sqrt(d)/32766 of scale |q| |k~| (the query's
    int16 rounding) under the 1e-3 tolerance."""
    torch = torch_cuda()
    m = tq()
    n = n_tok + n_tail
    keys = np.stack([np.stack([ti.key_stream(4, sq, h, n, d) for h in range(n_kv)]) for sq in range(n_seq)])
    S = n_seq * n_kv
    kd = to_dev_bf16(np.ascontiguousarray(keys[:, :, :n_tok]).reshape(-1, d)) if n_tok else None
    packed = torch.zeros(max(m.tq_q8_packed_bytes(d, S, n_tok), 16), dtype=torch.uint8, device="cuda")
    ws = m.workspace(256)
    if n_tok:
        m.tq_q8_quantize(kd, d, S, n_tok, n_tok * d, packed, ws)
        assert m.tq_get_status(ws) == m.TQ_OK
    kf = ti.bf16_to_f64(keys)
    if n_tok:
        codes, scales, pad = _unpack_q8(packed, d, S, n_tok)
        assert not pad.any()
        for st in range(S):
            want_c, want_s = oracle.q8_quantize(kf.reshape(S, n, d)[st, :n_tok])
            assert np.array_equal(codes[st], want_c)
            assert np.array_equal(scales[st], want_s)
    qb = ti.decode_queries(15, n_seq, n_kv * g, d)
    out = torch.full((n_seq, n_kv * g, n), float("nan"), dtype=torch.float32, device="cuda")
    tail = to_dev_bf16(np.ascontiguousarray(keys[:, :, n_tok:])) if n_tail else None
    scale = 1.0 / math.sqrt(d)
    m.tq_q8_logits(packed, d, n_seq, n_kv, n_tok, to_dev_bf16(qb), g, tail, n_tail, scale, out)
    torch.cuda.synchronize()
    got = out.cpu().numpy().astype(np.float64)
    q = ti.bf16_to_f64(qb)
    for sq in range(n_seq):
        for h in range(n_kv):
            st = sq * n_kv + h
            qh = q[sq, h * g:(h + 1) * g]
            if n_tok:
                c_, s_ = oracle.q8_quantize(kf[sq, h, :n_tok])
                want = oracle.q8_logits(c_, s_, qh, scale)
                rec = c_.astype(np.float64) * np.repeat(s_, 32, axis=1)[:, :d]
                err = np.abs(got[sq, h * g:(h + 1) * g, :n_tok] - want) / (
                    scale * np.linalg.norm(qh, axis=1)[:, None] * np.linalg.norm(rec, axis=1)[None, :])
                assert err.max() <= min(TOL, math.sqrt(d) / 32766 * 1.01), err.max()
            if n_tail:
                wt = oracle.exact_dot(kf[sq, h, n_tok:], qh, scale)
                _check_logits(got[sq, h * g:(h + 1) * g, n_tok:], wt, qh, np.linalg.norm(kf[sq, h, n_tok:], axis=1),
                              scale)


@pytest.mark.parametrize("Bv,g,n_seq,n_kv,n_tok,n_tail,law,vs", [
    (3, 4, 1, 2, 3000, 128, "c2", 0.0),     # the decode key law, a 128-token tail
    (4, 2, 2, 2, 301, 5, "normal", 0.0),    # several streams, ragged last block
    (2, 1, 1, 1, 64, 0, "normal", 0.0),     # no tail
    (3, 4, 1, 2, 2000, 16, "c2", 1e-4),     # sparse values
])
def test_attention_q8_keys(Bv, g, n_seq, n_kv, n_tok, n_tail, law, vs):
    """Decode attention over 8-bit keys and TurboQuant values (the asymmetric configuration)
    against the oracle's attention_q8 on the GPU's own codes, by the two checks of
    gpu_helpers.check_attention: the oracle's P.V over the logits of tq_q8_logits (softmax,
    value decode, merge) and the full oracle composition."""
    torch = torch_cuda()
    m = tq()
    d = 128
    n = n_tok + n_tail
    piv = ti.haar_rotation(d, 131)
    if law == "c2":
        keys = np.stack([np.stack([ti.key_stream(4, sq, h, n) for h in range(n_kv)]) for sq in range(n_seq)])
    else:
        keys = np.stack([np.stack([_normal_stream(81, sq, h, n) for h in range(n_kv)]) for sq in range(n_seq)])
    vals = np.stack([np.stack([_normal_stream(82, sq, h, n) for h in range(n_kv)]) for sq in range(n_seq)])
    S = n_seq * n_kv
    vc = make_codec(d, 0, Bv, False, piv, None)
    pk8 = torch.zeros(m.tq_q8_packed_bytes(d, S, n_tok), dtype=torch.uint8, device="cuda")
    ws0 = m.workspace(256)
    m.tq_q8_quantize(to_dev_bf16(np.ascontiguousarray(keys[:, :, :n_tok]).reshape(-1, d)), d, S, n_tok, n_tok * d,
                     pk8, ws0)
    assert m.tq_get_status(ws0) == m.TQ_OK
    pvv, _ = gpu_quantize(vc, to_dev_bf16(np.ascontiguousarray(vals[:, :, :n_tok]).reshape(-1, d)), S, n_tok)
    tk = to_dev_bf16(np.ascontiguousarray(keys[:, :, n_tok:])) if n_tail else None
    tv = to_dev_bf16(np.ascontiguousarray(vals[:, :, n_tok:])) if n_tail else None
    qb = ti.decode_queries(16, n_seq, n_kv * g)
    scale = 1.0 / math.sqrt(d)
    out = torch.full((n_seq, n_kv * g, d), float("nan"), dtype=torch.float32, device="cuda")
    ws = m.workspace(m.tq_attention_q8_workspace_bytes(vc, n_seq, n_kv, n_tok, g, n_tail))
    m.tq_attention_q8(vc, pk8, pvv, n_seq, n_kv, n_tok, to_dev_bf16(qb), g, tk, tv, n_tail, scale, out, ws, v_skip=vs)
    torch.cuda.synchronize()
    assert m.tq_get_status(ws) == m.TQ_OK
    got = out.cpu().numpy().astype(np.float64)
    lgt = torch.full((n_seq, n_kv * g, n), float("nan"), dtype=torch.float32, device="cuda")
    m.tq_q8_logits(pk8, d, n_seq, n_kv, n_tok, to_dev_bf16(qb), g, tk, n_tail, scale, lgt)
    torch.cuda.synchronize()
    lg = lgt.cpu().numpy().astype(np.float64)
    codes, scales, _ = _unpack_q8(pk8, d, S, n_tok)
    vidx, vnh = unpack(vc, pvv, S, n_tok)
    c_v, _ = _cb(d, Bv)
    q = ti.bf16_to_f64(qb)
    kf, vf = ti.bf16_to_f64(keys), ti.bf16_to_f64(vals)
    for sq in range(n_seq):
        for h in range(n_kv):
            st = sq * n_kv + h
            qh = q[sq, h * g:(h + 1) * g]
            tkh, tvh = (kf[sq, h, n_tok:], vf[sq, h, n_tok:]) if n_tail else (None, None)
            want = oracle.attention_q8(codes[st], scales[st], vidx[st], vnh[st], piv, c_v, qh, scale, tail_k=tkh,
                                       tail_v=tvh)
            L = np.concatenate([oracle.q8_logits(codes[st], scales[st], qh, scale),
                                oracle.exact_dot(kf[sq, h, n_tok:], qh, scale)], axis=1)
            vhat = oracle.reconstruct(vidx[st], None, vnh[st], None, piv, None, c_v, qjl=False)
            V = np.concatenate([vhat, vf[sq, h, n_tok:]])
            vnorm = np.concatenate([vnh[st], np.linalg.norm(vf[sq, h, n_tok:], axis=1)])
            skip = None
            if vs > 0.0:
                rel = np.exp(L - L.max(axis=1, keepdims=True))
                wv = rel / rel.sum(axis=1, keepdims=True) * vnorm[None, :]
                drop = rel < vs
                drop[:, n_tok:] = False
                skip = (wv * drop).sum(axis=1) / wv.sum(axis=1)
            err, err_c = check_attention(got[sq, h * g:(h + 1) * g], want, L, lg[sq, h * g:(h + 1) * g], n_tok, V,
                                         vnorm, v_skip=vs, skip_mass=skip)
            print(f"q8 attention stream {st}: {err.max():.2e} (full), {err_c.max():.2e} (composed)")


def test_attention_rejects_unsupported():
    torch = torch_cuda()
    m = tq()
    d = 128
    kc = make_codec(d, d, 2, True, ti.haar_rotation(d, 1), ti.gaussian_sketch(d, d, 2))
    vc = make_codec(d, 0, 3, False, ti.haar_rotation(d, 3), None)
    q = torch.zeros((1, 8, d), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((1, 8, d), dtype=torch.float32, device="cuda")
    pk = torch.zeros(kc.packed_bytes(1, 64), dtype=torch.uint8, device="cuda")
    pv_ = torch.zeros(vc.packed_bytes(1, 64), dtype=torch.uint8, device="cuda")
    ws = m.workspace(1 << 20)
    with pytest.raises(m.TQError) as e:   # g = 8 is outside the fused kernel's head tile
        m.tq_attention(kc, vc, pk, pv_, 1, 1, 64, q, 8, None, None, 0, 1.0, out, ws)
    assert e.value.status == m.TQ_ERR_UNSUPPORTED
    with pytest.raises(m.TQError) as e:   # a softmax over no tokens
        m.tq_attention(kc, vc, pk, pv_, 1, 1, 0, q, 4, None, None, 0, 1.0, out, ws)
    assert e.value.status == m.TQ_ERR_ARG
    with pytest.raises(m.TQError) as e:   # key and value codecs swapped
        m.tq_attention(vc, kc, pk, pv_, 1, 1, 64, q, 4, None, None, 0, 1.0, out, ws)
    assert e.value.status == m.TQ_ERR_ARG
    assert m.tq_attention_workspace_bytes(kc, vc, 1, 1, 64, 8, 0) == 0


# ----------------------------------------------------------------------------- reconstruction
@pytest.mark.parametrize("qjl,B", [(True, 2), (True, 3), (False, 4)])
def test_dequantize_reconstruction(qjl, B):
    d = m = 128
    pi, s = ti.haar_rotation(d, 61), ti.gaussian_sketch(m, d, 62)
    x = ti.c1_keys(500)
    codec = make_codec(d, m, B, qjl, pi, s if qjl else None)
    packed, _ = gpu_quantize(codec, to_dev_f32(x), 1, 500)
    torch = torch_cuda()
    out = torch.zeros((500, d), dtype=torch.float32, device="cuda")
    tq().tq_dequantize(codec, packed, 1, 500, out)
    got = out.cpu().numpy().astype(np.float64)
    c, t = _cb(d, B)
    if qjl:
        idx, sbit, nhat, ghat = unpack(codec, packed, 1, 500)
        want = oracle.reconstruct(idx[0], sbit[0], nhat[0], ghat[0], pi, s, c, qjl=True)
    else:
        idx, nhat = unpack(codec, packed, 1, 500)
        want = oracle.reconstruct(idx[0], None, nhat[0], None, pi, None, c, qjl=False)
    err = np.max(np.abs(got - want), axis=1) / np.linalg.norm(x.astype(np.float64), axis=1)
    assert err.max() <= TOL


# ----------------------------------------------------------------------------- top-k
def _topk_gpu(codec, packed, n_db, q_dev, n_q, k, estimator=None):
    torch = torch_cuda()
    m = tq()
    idx = torch.full((n_q, k), -7, dtype=torch.int64, device="cuda")
    score = torch.full((n_q, k), float("nan"), dtype=torch.float32, device="cuda")
    ws = m.workspace(codec.workspace_bytes(m.TQ_OP_TOPK, n_q, n_db, k))
    m.tq_topk(codec, packed, n_db, q_dev, n_q, k, idx, score, ws, estimator=estimator)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), score.cpu().numpy().astype(np.float64)


def check_topk(gidx, gsc, all_scores, q, xnorm, k):
    """The GPU set equals the oracle's top-k except for members whose oracle score is within
    1e-3 |q| |x| of the oracle's k-th score; returned scores match the oracle's."""
    swaps = 0
    for r in range(gidx.shape[0]):
        sc = all_scores[r]
        order = np.lexsort((np.arange(sc.size), -sc))
        want = order[:k]
        kth = sc[want[-1]]
        tol = TOL * np.linalg.norm(q[r]) * xnorm
        assert len(set(gidx[r].tolist())) == k and gidx[r].min() >= 0
        diff = set(gidx[r].tolist()) ^ set(want.tolist())
        for i in diff:
            assert abs(sc[i] - kth) <= tol[i], f"query {r}: {i} differs beyond the near-tie band"
        swaps += len(diff) // 2
        assert np.all(np.abs(gsc[r] - sc[gidx[r]]) <= tol[gidx[r]])
        # best first
        assert np.all(np.diff(gsc[r]) <= 1e-6 * np.abs(gsc[r]).max())
    return swaps


@pytest.mark.parametrize("B,n_db,n_q,k", [(1, 5000, 37, 10), (3, 3001, 70, 10), (2, 777, 5, 1), (1, 4096, 33, 32)])
def test_topk_against_oracle(B, n_db, n_q, k):
    d = m = 200
    pi, s = ti.C5.pi(), ti.C5.s()
    x = ti.c5_rows("db", 0, n_db)
    q = ti.c5_rows("q", 0, n_q)
    codec = make_codec(d, m, B, True, pi, s)
    packed, _ = gpu_quantize(codec, to_dev_f32(x), 1, n_db)
    gidx, gsc = _topk_gpu(codec, packed, n_db, to_dev_f32(q), n_q, k)
    idx, sbit, nhat, ghat = unpack(codec, packed, 1, n_db)
    c, t = _cb(d, B)
    all_scores = oracle.logits(idx[0], sbit[0], nhat[0], ghat[0], pi, s, c, q.astype(np.float64), qjl=True)
    xn = np.linalg.norm(x.astype(np.float64), axis=1)
    swaps = check_topk(gidx, gsc, all_scores, q.astype(np.float64), xn, k)
    # the oracle's own top-k routine agrees with the full sort used above
    oi, _ = oracle.topk(idx[0][:500], sbit[0][:500], nhat[0][:500], ghat[0][:500], pi, s, c, q[:3].astype(np.float64),
                        k=min(k, 500))
    assert oi.shape == (3, min(k, 500))
    print(f"top-{k}: {swaps} near-tie swaps over {n_q} queries")


def test_mse_only_estimator():
    """TQ_EST_MSE on QJL key records: logits and top-k equal the oracle's MSE-stage estimate
    |x| <Pi q, c[idx]> on the same codes (signs and gamma unused)."""
    torch = torch_cuda()
    m = tq()
    d = mm = 128
    pi, s = ti.haar_rotation(d, 111), ti.gaussian_sketch(mm, d, 112)
    n_kv, n_tok, g, B = 2, 333, 4, 3
    keys = np.stack([ti.key_stream(4, 1, h, n_tok) for h in range(n_kv)])
    codec = make_codec(d, mm, B, True, pi, s)
    packed, _ = gpu_quantize(codec, to_dev_bf16(keys.reshape(-1, d)), n_kv, n_tok)
    qb = ti.decode_queries(14, 1, n_kv * g)
    out = torch.full((1, n_kv * g, n_tok), float("nan"), dtype=torch.float32, device="cuda")
    ws = m.workspace(codec.workspace_bytes(m.TQ_OP_LOGITS, 1, n_kv, g))
    m.tq_logits(codec, packed, 1, n_kv, n_tok, to_dev_bf16(qb), g, None, 0, 0.5, out, ws, estimator=m.TQ_EST_MSE)
    got = out.cpu().numpy().astype(np.float64)[0]
    idx, sbit, nhat, ghat = unpack(codec, packed, n_kv, n_tok)
    c, _ = _cb(d, B)
    q = ti.bf16_to_f64(qb)[0]
    kf = ti.bf16_to_f64(keys)
    for h in range(n_kv):
        qh = q[h * g:(h + 1) * g]
        want = oracle.logits(idx[h], sbit[h], nhat[h], ghat[h], pi, s, c, qh, qjl=False, scale=0.5)
        _check_logits(got[h * g:(h + 1) * g], want, qh, np.linalg.norm(kf[h], axis=1), 0.5)
        full = oracle.logits(idx[h], sbit[h], nhat[h], ghat[h], pi, s, c, qh, qjl=True, scale=0.5)
        assert np.max(np.abs(want - full)) > 1e-2   # the QJL term is really gone
    with pytest.raises(m.TQError):
        m.tq_logits(codec, packed, 1, n_kv, n_tok, to_dev_bf16(qb), g, None, 0, 0.5, out, ws, estimator=7)
    # top-k with the MSE-only score
    dd = 200
    pi5, s5 = ti.C5.pi(), ti.C5.s()
    x = ti.c5_rows("db", 0, 3000)
    qs = ti.c5_rows("q", 0, 21)
    c5 = make_codec(dd, dd, 2, True, pi5, s5)
    pk5, _ = gpu_quantize(c5, to_dev_f32(x), 1, 3000)
    gidx, gsc = _topk_gpu(c5, pk5, 3000, to_dev_f32(qs), 21, 10, estimator=m.TQ_EST_MSE)
    i5, sb5, nh5, gh5 = unpack(c5, pk5, 1, 3000)
    cc5, _ = _cb(dd, 2)
    all_scores = oracle.logits(i5[0], sb5[0], nh5[0], gh5[0], pi5, s5, cc5, qs.astype(np.float64), qjl=False)
    check_topk(gidx, gsc, all_scores, qs.astype(np.float64), np.linalg.norm(x.astype(np.float64), axis=1), 10)


def test_topk_ties_and_query_tiles():
    """Three tiles of 128 queries, several key ranges each, and every database record stored
    twice: equal scores keep the lower index first, so a duplicate enters the top-k only with
    its original, right after it."""
    torch = torch_cuda()
    d = m = 200
    n, n_q, k = 1600, 300, 8
    pi, s = ti.C5.pi(), ti.C5.s()
    x = ti.c5_rows("db", 4096, n)
    q = ti.c5_rows("q", 4096, n_q)
    codec = make_codec(d, m, 2, True, pi, s)
    packed, _ = gpu_quantize(codec, to_dev_f32(x), 1, n)
    twice = torch.cat([packed, packed])
    gidx, gsc = _topk_gpu(codec, twice, 2 * n, to_dev_f32(q), n_q, k)
    idx, sbit, nhat, ghat = unpack(codec, packed, 1, n)
    c, _ = _cb(d, 2)
    sc = oracle.logits(idx[0], sbit[0], nhat[0], ghat[0], pi, s, c, q.astype(np.float64), qjl=True)
    xn = np.linalg.norm(x.astype(np.float64), axis=1)
    check_topk(gidx, gsc, np.concatenate([sc, sc], axis=1), q.astype(np.float64), np.concatenate([xn, xn]), k)
    for r in range(n_q):
        row = gidx[r].tolist()
        for pos, i in enumerate(row):
            if i >= n:
                assert pos > 0 and row[pos - 1] == i - n and gsc[r][pos] == gsc[r][pos - 1], (r, row)


def test_topk_d128_codec():
    d = m = 128
    pi, s = ti.haar_rotation(d, 111), ti.gaussian_sketch(m, d, 112)
    x = ti.c1_keys(2000)
    q = ti.c1_queries(9)
    codec = make_codec(d, m, 2, True, pi, s)
    packed, _ = gpu_quantize(codec, to_dev_f32(x), 1, 2000)
    gidx, gsc = _topk_gpu(codec, packed, 2000, to_dev_f32(q), 9, 10)
    idx, sbit, nhat, ghat = unpack(codec, packed, 1, 2000)
    c, t = _cb(d, 2)
    all_scores = oracle.logits(idx[0], sbit[0], nhat[0], ghat[0], pi, s, c, q.astype(np.float64), qjl=True)
    check_topk(gidx, gsc, all_scores, q.astype(np.float64), np.linalg.norm(x.astype(np.float64), axis=1), 10)


def test_logits_timeout_status():
    """The timeout path of the bounded waits: with the TQ_TEST_STALL hook every warp of the
    stream kernel waits on a barrier nothing arrives at; the wait runs out, the status word
    reads TQ_ERR_TIMEOUT, the copies in flight are drained, and the next call on the same
    stream and context is correct."""
    torch = torch_cuda()
    m = tq()
    d = 128
    pi, s = ti.haar_rotation(d, 111), ti.gaussian_sketch(d, d, 112)
    n_kv, n_tok, g, B = 4, 5000, 4, 2
    codec = make_codec(d, d, B, True, pi, s)
    keys = np.concatenate([ti.key_stream(4, 0, h, n_tok) for h in range(n_kv)])
    packed, st = gpu_quantize(codec, to_dev_bf16(keys), n_kv, n_tok)
    assert st == m.TQ_OK
    qb = ti.decode_queries(40, 1, n_kv * g)
    q = to_dev_bf16(qb)
    out = torch.full((1, n_kv * g, n_tok), float("nan"), dtype=torch.float32, device="cuda")
    ws = m.workspace(codec.workspace_bytes(m.TQ_OP_LOGITS, 1, n_kv, g))
    m.tq_logits(codec, packed, 1, n_kv, n_tok, q, g, None, 0, 1.0, out, ws, estimator=m.TQ_EST_QJL | m.TQ_TEST_STALL)
    assert m.tq_get_status(ws) == m.TQ_ERR_TIMEOUT
    assert torch.isnan(out).all()          # the stalled call wrote no logits
    assert m.tq_get_status(ws) == m.TQ_OK  # reading the word cleared it
    m.tq_logits(codec, packed, 1, n_kv, n_tok, q, g, None, 0, 1.0, out, ws)
    assert m.tq_get_status(ws) == m.TQ_OK
    got = out.cpu().numpy().astype(np.float64)[0]
    idx, sbit, nhat, ghat = unpack(codec, packed, n_kv, n_tok)
    c, _ = _cb(d, B)
    qf = ti.bf16_to_f64(qb)[0]
    kf = ti.bf16_to_f64(keys).reshape(n_kv, n_tok, d)
    for h in range(n_kv):
        qh = qf[h * g:(h + 1) * g]
        want = oracle.logits(idx[h], sbit[h], nhat[h], ghat[h], pi, s, c, qh, qjl=True)
        _check_logits(got[h * g:(h + 1) * g], want, qh, np.linalg.norm(kf[h], axis=1), 1.0)
