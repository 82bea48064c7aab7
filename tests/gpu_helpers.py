"""Helpers of the GPU parity tests: run the CUDA library through its C ABI and compare with
the oracle under the tolerances of the method's readings."""
from __future__ import annotations

import numpy as np

import oracle
import tq_inputs as ti
from tq_format import unpack_keys, unpack_values

BAND = 1e-5          # decision band, unit-vector domain
MAX_BAND_MISMATCH = 1e-4
TOL = 1e-3           # normalised tolerance of logits, reconstructions and P.V


def torch_cuda():
    import torch
    assert torch.cuda.is_available(), "GPU test run without a CUDA device"
    return torch


def tq():
    import kv_cache_vector_03_b200 as m
    return m


def to_dev_bf16(bits: np.ndarray):
    torch = torch_cuda()
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def to_dev_f32(a: np.ndarray):
    torch = torch_cuda()
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def make_codec(d, m, B, qjl, pi, s):
    torch = torch_cuda()
    return tq().Codec(d, m, B, qjl, torch.from_numpy(pi.astype(np.float32)),
                      torch.from_numpy(s.astype(np.float32)) if qjl else None)


def gpu_quantize(codec, x_dev, n_streams, n_tok, stride=None):
    torch = torch_cuda()
    m = tq()
    packed = torch.zeros(codec.packed_bytes(n_streams, n_tok), dtype=torch.uint8, device="cuda")
    ws = m.workspace(codec.workspace_bytes(m.TQ_OP_QUANTIZE))
    m.tq_quantize(codec, x_dev, n_streams, n_tok, stride if stride is not None else n_tok * codec.c.d, packed, ws)
    status = m.tq_get_status(ws)
    return packed, status


def half_ulp_ok(a, b):
    """|a - b| <= one binary16 ulp at the larger magnitude."""
    mag = np.maximum(np.abs(a), np.abs(b))
    e = np.floor(np.log2(np.maximum(mag, 2.0 ** -24)))
    ulp = np.where(mag >= 2.0 ** -14, 2.0 ** (e - 10), 2.0 ** -24)
    return np.abs(a - b) <= ulp * (1 + 1e-9)


def compare_codes(idx, sbit, nhat, ghat, ref, bounds, qjl=True, x=None, pi=None, s=None, c=None, t=None, B=None):
    """Codes bit-exact outside the decision band; norms within one binary16 ulp.
    A vector whose index was decided differently inside the band has a different residual,
    so its gamma and signs are checked against the oracle's sketch of the GPU's indices
    (x, pi, s, c, t, B are needed for that).
    Returns (in-band coordinate count, in-band mismatch count, total coordinates)."""
    dist = np.min(np.abs(ref.y[..., None] - bounds[None, None, :]), axis=-1)
    in_band = dist < BAND
    mism = idx != ref.idx
    assert not np.any(mism & ~in_band), f"{int(np.sum(mism & ~in_band))} index mismatches outside the band"
    n_band, n_mis, n_all = int(in_band.sum()), int(mism.sum()), mism.size
    assert np.all(half_ulp_ok(nhat, ref.nhat)), "|x|^ differs by more than one binary16 ulp"
    if qjl:
        rz, rs, rg = ref.z, ref.sbit, ref.ghat
        flipped = np.any(mism, axis=1)
        if flipped.any():
            assert x is not None, "index flips need the inputs to re-check the sketch"
            alt = oracle.quantize(x[flipped], pi, s, c, t, B, qjl=True, idx_in=idx[flipped])
            rz, rs, rg = rz.copy(), rs.copy(), rg.copy()
            rz[flipped], rs[flipped], rg[flipped] = alt.z, alt.sbit, alt.ghat
        zb = np.abs(rz) < BAND
        smis = sbit != rs
        assert not np.any(smis & ~zb), f"{int(np.sum(smis & ~zb))} sign mismatches outside the band"
        n_band += int(zb.sum())
        n_mis += int(smis.sum())
        n_all += smis.size
        assert np.all(half_ulp_ok(ghat, rg)), "gamma^ differs by more than one binary16 ulp"
    assert n_mis <= MAX_BAND_MISMATCH * n_all
    return n_band, n_mis, n_all


def unpack(codec, packed_dev, n_streams, n_tok):
    c = codec.c
    buf = packed_dev.cpu().numpy()
    if c.qjl:
        return unpack_keys(buf, c.d, c.m, c.mse_bits, n_streams, n_tok)
    return unpack_values(buf, c.d, c.mse_bits, n_streams, n_tok)


ATTN_CEIL = 5e-3     # ceiling of the fused-attention error against the full oracle


def _softmax_rows(L):
    w = np.exp(L - L.max(axis=1, keepdims=True))
    return w / w.sum(axis=1, keepdims=True)


def check_attention(got, want, L, lg, n_tok, V, vnorm, v_skip=0.0, skip_mass=None):
    """Fused decode attention of the g heads of one kv stream, two checks.

    got [g, d] GPU output; want [g, d] the oracle's attention; L [g, n] the oracle's logits
    (estimator on the compressed keys, exact on the tail); lg [g, n] the GPU's tq_logits on the
    same codes and queries; V [n, d] the oracle's reconstructed compressed values followed by
    the exact tail values; vnorm [n] the stored value norms, then the tail norms.

    1. Composed (the step tolerance of P.V): the oracle's softmax(P) . V with P = the GPU's
       compressed-key logits followed by the exact tail logits. The fused kernel evaluates the
       same logit fragments, so this isolates its softmax, value decode and merge: the error
       is held to TOL of sum_t w_t |v_t| on every workload, whatever the logit scale.
    2. Full oracle: a logit error dl moves every softmax weight by a factor within
       exp(+-2 dl), so the error is at most (expm1(2 dl) + TOL) sum_t w_t |v_t|; the bound is
       capped by the fixed ATTN_CEIL, so a large logit scale cannot widen it.
    With sparse values the dropped weight mass (tokens whose relative weight is below v_skip)
    is added to both bounds. Returns (full error, composed error), per head."""
    assert np.all(np.isfinite(got))
    Lc = np.concatenate([lg[:, :n_tok], L[:, n_tok:]], axis=1)
    wc = _softmax_rows(Lc)
    comp = wc @ V
    skip_c = np.zeros(len(got))
    if v_skip > 0.0:
        rel = np.exp(Lc - Lc.max(axis=1, keepdims=True))
        drop = rel < v_skip
        drop[:, n_tok:] = False
        wv = wc * vnorm[None, :]
        skip_c = (wv * drop).sum(axis=1) / wv.sum(axis=1)
    err_c = np.max(np.abs(got - comp), axis=1) / (wc @ vnorm)
    assert np.all(err_c <= TOL + skip_c), f"composed check: normalised error {err_c} above {TOL + skip_c}"
    w = _softmax_rows(L)
    dl = np.abs(lg - L).max(axis=1)
    err = np.max(np.abs(got - want), axis=1) / (w @ vnorm)
    bound = np.minimum(TOL + np.expm1(2 * dl) + 1e-5, ATTN_CEIL)
    if skip_mass is not None:
        bound = bound + skip_mass
    assert np.all(err <= bound), f"full oracle: normalised error {err} above {bound}"
    return err, err_c
