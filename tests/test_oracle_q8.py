"""Pins for the oracle's 8-bit keys (CPU only): exact cases, rounding, the error bound and a
brute-force logit."""
import numpy as np

import oracle


def test_exact_when_codes_fit():
    # integer values with a chunk maximum of 127 x 2^k: the scale is exactly 2^k (also in
    # binary16), every code is the value / 2^k and the key reads back exactly
    rng = np.random.default_rng(1)
    q = rng.integers(-127, 128, size=(5, 96)).astype(np.float64)
    q[:, ::32] = 127.0                       # each chunk's maximum
    x = q * 2.0 ** np.array([-3, 0, 2, 5, -8])[:, None]
    codes, scales = oracle.q8_quantize(x)
    assert codes.shape == (5, 96) and scales.shape == (5, 3)
    assert np.array_equal(codes, q.astype(np.int8))
    assert np.array_equal(scales, np.repeat(2.0 ** np.array([-3, 0, 2, 5, -8])[:, None], 3, axis=1))


def test_rounding_half_to_even_and_extremes():
    x = np.zeros((1, 32))
    x[0, 0] = 127.0                          # scale 1
    x[0, 1:5] = [2.5, 3.5, -2.5, -0.5]
    x[0, 5] = -127.0
    codes, scales = oracle.q8_quantize(x)
    assert scales[0, 0] == 1.0
    assert list(codes[0, :6]) == [127, 2, 4, -2, 0, -127]
    z, zs = oracle.q8_quantize(np.zeros((2, 64)))
    assert not z.any() and not zs.any()


def test_error_bound_and_chunk_maximum():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((200, 128)) * np.exp(rng.uniform(-3, 3, (200, 1)))
    x[:, :4] *= 20.0                          # outlier channels in chunk 0
    codes, scales = oracle.q8_quantize(x)
    x32 = x.astype(np.float32).astype(np.float64)
    s32 = (np.abs(x32.reshape(200, 4, 32)).max(axis=2).astype(np.float32) / np.float32(127)).astype(np.float64)
    rec = codes.astype(np.float64) * np.repeat(scales, 32, axis=1)
    bound = np.repeat(s32 / 2 + 127 * np.abs(s32 - scales), 32, axis=1) * (1 + 1e-6)
    assert np.all(np.abs(rec - x32) <= bound)
    # the largest magnitude of every chunk takes code +-127
    assert np.all(np.abs(codes.reshape(200, 4, 32)).max(axis=2) == 127)


def test_logits_brute_force():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((7, 40))
    q = rng.standard_normal((3, 40))
    codes, scales = oracle.q8_quantize(x)
    got = oracle.q8_logits(codes, scales, q, scale=0.25)
    for a in range(3):
        for b in range(7):
            want = 0.0
            for i in range(40):
                want += q[a, i] * float(codes[b, i]) * scales[b, i // 32]
            assert abs(got[a, b] - 0.25 * want) <= 1e-12 * max(1.0, abs(want))


def test_attention_over_8bit_keys():
    # no tail: P.V of the 8-bit-key logits (separately pinned functions); q = 0: the mean of
    # the compressed and tail values together
    rng = np.random.default_rng(4)
    d, nt = 64, 150
    keys = rng.standard_normal((nt + 5, d)) * 3.0
    vals = rng.standard_normal((nt + 5, d))
    c_v, t_v, _, _ = oracle.codebook(d, 3)
    pi_v = np.linalg.qr(rng.standard_normal((d, d)))[0]
    vq = oracle.quantize(vals[:nt], pi_v, None, c_v, t_v, 3, qjl=False)
    kc, ks = oracle.q8_quantize(keys[:nt])
    qs = rng.standard_normal((3, d)) * 0.2
    o = oracle.attention_q8(kc, ks, vq.idx, vq.nhat, pi_v, c_v, qs, 0.5)
    want = oracle.pv(vq.idx, vq.nhat, pi_v, c_v, oracle.q8_logits(kc, ks, qs, 0.5))
    assert np.allclose(o, want, rtol=1e-5, atol=1e-6 * np.abs(want).max())
    vh = oracle.reconstruct(vq.idx, None, vq.nhat, None, pi_v, None, c_v, qjl=False)
    o0 = oracle.attention_q8(kc, ks, vq.idx, vq.nhat, pi_v, c_v, np.zeros((1, d)), 1.0, tail_k=keys[nt:],
                             tail_v=vals[nt:])
    assert np.allclose(o0[0], np.concatenate([vh, vals[nt:]]).mean(0), rtol=1e-12, atol=1e-12)
