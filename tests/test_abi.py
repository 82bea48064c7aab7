"""CPU checks of the C-ABI library: it loads, exports every entry point include/tq.h declares,
its host codebook agrees with the oracle's independent one, and argument checks fail before
any device work (no GPU needed)."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def tq():
    import __graft_entry__
    __graft_entry__.build()
    import kv_cache_vector_03_b200 as m
    return m


def header_functions():
    src = open(os.path.join(ROOT, "include", "tq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z_0-9]+)\s*\(", src)))


def test_exports_every_declared_symbol(tq):
    names = header_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(tq.lib, n), f"libtq.so does not export {n}"
    assert set(names) == set(tq.EXPORTED)
    assert tq.lib.tq_abi_version() == 1


@pytest.mark.parametrize("d,B", [(3, 2), (64, 1), (128, 1), (128, 2), (128, 3), (128, 4), (200, 1), (200, 2),
                                 (200, 3), (200, 4), (256, 4)])
def test_codebook_matches_oracle(tq, d, B):
    c, t, mse = tq.tq_make_codebook(d, B)
    oc, ot, omse, _ = oracle.codebook(d, B)
    assert np.max(np.abs(c - oc)) < 1e-12
    assert np.max(np.abs(t - ot)) < 1e-12
    assert abs(mse - omse) < 1e-12
    assert np.array_equal(c, -c[::-1]) and t[len(t) // 2] == 0.0


def _codec(tq, d=128, m=128, B=2, qjl=1, centroids=None, prep=None, prep_bytes=0):
    cent = centroids if centroids is not None else tq.tq_make_codebook(d, B)[0]
    c = tq.tq_codec(d, m, B, qjl, 0x1000, 0x2000 if qjl else None, cent.ctypes.data, prep, prep_bytes)
    return c, cent


def test_sizes(tq):
    c, keep = _codec(tq)
    assert tq.lib.tq_block_bytes(ctypes.byref(c)) == 32 * 52
    assert tq.lib.tq_record_bytes(ctypes.byref(c)) == 52
    c, keep = _codec(tq, B=3)
    assert tq.lib.tq_record_bytes(ctypes.byref(c)) == 68
    for B, rec in ((3, 50), (4, 66)):
        c, keep = _codec(tq, B=B, qjl=0, m=0)
        assert tq.lib.tq_record_bytes(ctypes.byref(c)) == rec
    c, keep = _codec(tq, d=200, m=200, B=1)
    assert tq.lib.tq_block_bytes(ctypes.byref(c)) == 512 * 4 + 128
    assert tq.lib.tq_packed_bytes(ctypes.byref(c), 3, 33) == 3 * 2 * (512 * 4 + 128)


def test_argument_checks_fail_before_device_work(tq):
    c, keep = _codec(tq)
    # unprepared codec
    assert tq.lib.tq_quantize(ctypes.byref(c), 0x10, 0, 1, 32, 32 * 128, 0x100, 0x200, 256, None) == tq.TQ_ERR_ARG
    prep = tq.lib.tq_prep_bytes(ctypes.byref(c))
    assert prep > 0
    c.prep, c.prep_bytes = 0x100000, prep - 1
    assert tq.lib.tq_prepare(ctypes.byref(c), None) == tq.TQ_ERR_WORKSPACE
    c.prep_bytes = prep
    # bad shapes
    for d, m, B in ((12, 128, 2), (264, 128, 2), (128, 4, 2), (128, 128, 4)):
        cent = tq.tq_make_codebook(128, min(B, 3))[0] if B <= 3 else tq.tq_make_codebook(128, 4)[0]
        cc = tq.tq_codec(d, m, B, 1, 0x1000, 0x2000, cent.ctypes.data, 0x100000, 1 << 30)
        assert tq.lib.tq_quantize(ctypes.byref(cc), 0x10, 0, 1, 32, 4096, 0x100, 0x200, 256, None) == \
            tq.TQ_ERR_UNSUPPORTED
    # misaligned packed buffer, bad dtype, small workspace, g not supported, values to logits
    assert tq.lib.tq_quantize(ctypes.byref(c), 0x10, 0, 1, 32, 4096, 0x104, 0x200, 256, None) == tq.TQ_ERR_ARG
    assert tq.lib.tq_quantize(ctypes.byref(c), 0x10, 7, 1, 32, 4096, 0x100, 0x200, 256, None) == tq.TQ_ERR_ARG
    assert tq.lib.tq_quantize(ctypes.byref(c), 0x10, 0, 1, 32, 4096, 0x100, 0x200, 8, None) == tq.TQ_ERR_WORKSPACE
    assert tq.lib.tq_logits(ctypes.byref(c), 0x100, 1, 1, 32, 0x200, 0, 3, None, 0, 1.0, 0x300, 0x400, 1 << 20,
                            None) == tq.TQ_ERR_UNSUPPORTED
    v, keep2 = _codec(tq, qjl=0, m=0, B=3)
    v.prep, v.prep_bytes = 0x100000, 1 << 30
    assert tq.lib.tq_logits(ctypes.byref(v), 0x100, 1, 1, 32, 0x200, 0, 4, None, 0, 1.0, 0x300, 0x400, 1 << 20,
                            None) == tq.TQ_ERR_ARG
    assert tq.lib.tq_pv(ctypes.byref(c), 0x100, 1, 1, 32, 0x200, 4, 0x300, 0x400, 1 << 20, None) == tq.TQ_ERR_ARG
    # asymmetric codebook rejected
    bad = np.array([-0.1, -0.02, 0.03, 0.1])
    cb, keep3 = _codec(tq, centroids=bad)
    cb.prep, cb.prep_bytes = 0x100000, 1 << 30
    assert tq.lib.tq_quantize(ctypes.byref(cb), 0x10, 0, 1, 32, 4096, 0x100, 0x200, 256, None) == tq.TQ_ERR_ARG
    # empty work is a no-op
    assert tq.lib.tq_quantize(ctypes.byref(c), 0x10, 0, 0, 32, 4096, 0x100, 0x200, 256, None) == tq.TQ_OK
    assert tq.lib.tq_make_codebook(2, 2, np.zeros(4).ctypes.data, np.zeros(3).ctypes.data, None) == \
        tq.TQ_ERR_UNSUPPORTED
    assert tq.lib.tq_status_string(tq.TQ_ERR_RANGE).decode().startswith("norm")


def test_attention_host_checks(tq):
    """tq_attention: workspace sizing and argument checks, all before any device work."""
    k, keep_k = _codec(tq, B=3)
    v, keep_v = _codec(tq, qjl=0, m=0, B=4)
    for c in (k, v):
        c.prep, c.prep_bytes = 0x100000, 1 << 30
    K, V = ctypes.byref(k), ctypes.byref(v)
    ws = tq.lib.tq_attention_workspace_bytes
    w0 = ws(K, V, 1, 8, 32640, 4, 0)
    w1 = ws(K, V, 1, 8, 32640, 4, 128)
    assert w0 > 0 and w0 % 256 == 0
    assert w1 - w0 >= 8 * 4 * 128 * 4          # one fp32 tail logit per (query head, tail token)
    assert ws(K, V, 1, 8, 320, 4, 128) < w1    # two ranges per stream instead of about one per SM
    assert ws(K, V, 1, 8, 32640, 8, 0) == 0    # g = 8: outside the fused head tile
    assert ws(V, K, 1, 8, 32640, 4, 0) == 0    # key and value codecs swapped
    wide, keep_w = _codec(tq, d=200, m=200, B=2)
    wide.prep, wide.prep_bytes = 0x100000, 1 << 30
    assert ws(ctypes.byref(wide), V, 1, 8, 320, 4, 0) == 0   # d > 128

    def call(n_seq=1, n_tok=320, g=4, tail_k=0x5000, tail_v=0x6000, n_tail=8, scale=0.125, v_skip=0.0,
             wsb=1 << 24, packed_k=0x1000, q_dtype=tq.TQ_BF16):
        return tq.lib.tq_attention(K, V, packed_k, 0x2000, n_seq, 8, n_tok, 0x3000, q_dtype, g, tail_k, tail_v,
                                   n_tail, scale, v_skip, 0x4000, 0x100000, wsb, None)
    assert call(n_seq=0) == tq.TQ_OK                                   # nothing to do
    assert call(g=8) == tq.TQ_ERR_UNSUPPORTED
    assert call(n_tok=0, n_tail=0) == tq.TQ_ERR_ARG                    # a softmax over no tokens
    assert call(n_tail=9000) == tq.TQ_ERR_UNSUPPORTED                  # above TQ_ATTN_MAX_TAIL
    assert call(tail_v=0x6004) == tq.TQ_ERR_ARG                        # tail values need 8-byte rows
    assert call(packed_k=0x1008) == tq.TQ_ERR_ARG                      # packed caches are 16-byte aligned
    assert call(v_skip=1.5) == tq.TQ_ERR_ARG
    assert call(v_skip=float("nan")) == tq.TQ_ERR_ARG
    assert call(scale=float("inf")) == tq.TQ_ERR_ARG
    assert call(q_dtype=5) == tq.TQ_ERR_ARG
    assert call(wsb=ws(K, V, 1, 8, 320, 4, 8) - 1) == tq.TQ_ERR_WORKSPACE


def test_q8_host_checks(tq):
    assert tq.lib.tq_q8_packed_bytes(128, 3, 33) == 3 * 2 * 4352
    assert tq.lib.tq_q8_packed_bytes(200, 1, 32) == 0
    assert tq.lib.tq_q8_quantize(0x1000, tq.TQ_BF16, 136, 1, 32, 4352, 0x2000, 0x3000, 256, None) == \
        tq.TQ_ERR_UNSUPPORTED
    assert tq.lib.tq_q8_quantize(0x1000, tq.TQ_BF16, 128, 1, 32, 4096, 0x2008, 0x3000, 256, None) == tq.TQ_ERR_ARG
    assert tq.lib.tq_q8_quantize(0x1000, tq.TQ_BF16, 128, 1, 32, 4096, 0x2000, 0x3000, 8, None) == \
        tq.TQ_ERR_WORKSPACE
    assert tq.lib.tq_q8_quantize(0x1000, tq.TQ_BF16, 128, 0, 32, 4096, 0x2000, 0x3000, 256, None) == tq.TQ_OK
    assert tq.lib.tq_q8_logits(0x2000, 128, 1, 8, 64, 0x3000, tq.TQ_BF16, 8, None, 0, 1.0, 0x4000, None) == \
        tq.TQ_ERR_UNSUPPORTED
    assert tq.lib.tq_q8_logits(0x2000, 128, 1, 8, 64, 0x3000, tq.TQ_BF16, 4, None, 70000, 1.0, 0x4000, None) == \
        tq.TQ_ERR_UNSUPPORTED
    assert tq.lib.tq_q8_logits(0x2000, 128, 1, 8, 64, 0x3000, tq.TQ_BF16, 4, None, 3, 1.0, 0x4000, None) == \
        tq.TQ_ERR_ARG
    assert tq.lib.tq_q8_logits(0x2000, 128, 1, 8, 0, 0x3000, tq.TQ_BF16, 4, None, 0, 1.0, 0x4000, None) == tq.TQ_OK


def test_header_is_plain_c():
    """include/tq.h is a C header: it compiles as C99 and as C++ with no CUDA headers."""
    import subprocess
    hdr = os.path.join(ROOT, "include", "tq.h")
    subprocess.check_call(["gcc", "-fsyntax-only", "-std=c99", "-Wall", "-Werror", "-x", "c", hdr])
    subprocess.check_call(["g++", "-fsyntax-only", "-Wall", "-Werror", "-x", "c++", hdr])
