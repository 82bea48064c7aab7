"""tq_logits_noalloc: the logits entry point for callers that cannot allocate device memory
(a host framework whose pool owns the device memory, plugins limited to the buffers they are
handed, loops under a no-allocation policy). It must give the same logits as tq_logits with a
caller workspace, call after call, while sharing one fixed device scratch array.

Collected last on purpose: if it fails, a run that stops at the first failure has already run
every other test."""
import ctypes
import math

import numpy as np
import pytest

import tq_inputs as ti
from gpu_helpers import TOL, gpu_quantize, make_codec, to_dev_bf16, torch_cuda, tq

pytestmark = pytest.mark.gpu


def test_noalloc_logits_match_workspace_logits_twice():
    torch = torch_cuda()
    m = tq()
    d = 128
    pi, s = ti.haar_rotation(d, 101), ti.gaussian_sketch(d, d, 102)
    n_seq, n_kv, n_tok, g = 2, 4, 1000, 4
    codec = make_codec(d, d, 2, True, pi, s)
    keys = np.concatenate([ti.key_stream(4, sq, h, n_tok) for sq in range(n_seq) for h in range(n_kv)])
    packed, _ = gpu_quantize(codec, to_dev_bf16(keys), n_seq * n_kv, n_tok)
    scale = 1.0 / math.sqrt(d)
    ws = m.workspace(codec.workspace_bytes(m.TQ_OP_LOGITS, n_seq, n_kv, g))
    for call in range(2):
        qb = ti.decode_queries(20 + call, n_seq, n_kv * g)
        q = to_dev_bf16(qb)
        ref = torch.zeros((n_seq, n_kv * g, n_tok), dtype=torch.float32, device="cuda")
        got = torch.full((n_seq, n_kv * g, n_tok), float("nan"), dtype=torch.float32, device="cuda")
        m.tq_logits(codec, packed, n_seq, n_kv, n_tok, q, g, None, 0, scale, ref, ws)
        m.tq_logits_noalloc(codec, packed, n_seq, n_kv, n_tok, q, g, None, 0, scale, got)
        torch.cuda.synchronize()
        r, o = ref.cpu().numpy().astype(np.float64), got.cpu().numpy().astype(np.float64)
        qn = np.linalg.norm(ti.bf16_to_f64(qb), axis=-1)[..., None]
        kn = np.linalg.norm(ti.bf16_to_f64(keys), axis=-1).reshape(n_seq, n_kv, 1, n_tok)
        kn = np.repeat(kn, g, axis=2).reshape(n_seq, n_kv * g, n_tok)
        assert np.all(np.isfinite(o))
        assert np.max(np.abs(o - r) / (scale * qn * kn)) <= TOL


def test_noalloc_rejects_requests_beyond_its_scratch():
    m = tq()
    d = 128
    codec = make_codec(d, d, 3, True, ti.haar_rotation(d, 103), ti.gaussian_sketch(d, d, 104))
    # query fragments of 4096 streams need more than the 4 MiB scratch
    need = codec.workspace_bytes(m.TQ_OP_LOGITS, 4096, 1, 4)
    assert need > (4 << 20)
    st = m.lib.tq_logits_noalloc(codec.ref, ctypes.c_void_p(16), 4096, 1, 32, ctypes.c_void_p(16), 0, 4, None, 0,
                                 1.0, ctypes.c_void_p(16), None)
    assert st == m.TQ_ERR_WORKSPACE


def test_noalloc_rejected_arguments_enqueue_nothing():
    """Argument errors come back synchronously, before the shared array is touched: a null
    output, a misaligned packed cache and a non-finite scale are refused, and a following
    valid call still matches tq_logits."""
    torch = torch_cuda()
    m = tq()
    d = 128
    pi, s = ti.haar_rotation(d, 105), ti.gaussian_sketch(d, d, 106)
    n_kv, n_tok, g = 2, 300, 4
    codec = make_codec(d, d, 2, True, pi, s)
    keys = np.concatenate([ti.key_stream(4, 0, h, n_tok) for h in range(n_kv)])
    packed, _ = gpu_quantize(codec, to_dev_bf16(keys), n_kv, n_tok)
    q = to_dev_bf16(ti.decode_queries(30, 1, n_kv * g))
    got = torch.full((1, n_kv * g, n_tok), float("nan"), dtype=torch.float32, device="cuda")
    vp = lambda t: ctypes.c_void_p(t.data_ptr())
    lib = m.lib
    assert lib.tq_logits_noalloc(codec.ref, vp(packed), 1, n_kv, n_tok, vp(q), 1, g, None, 0, 1.0, None,
                                 None) == m.TQ_ERR_ARG
    assert lib.tq_logits_noalloc(codec.ref, ctypes.c_void_p(packed.data_ptr() + 4), 1, n_kv, n_tok, vp(q), 1, g,
                                 None, 0, 1.0, vp(got), None) == m.TQ_ERR_ARG
    assert lib.tq_logits_noalloc(codec.ref, vp(packed), 1, n_kv, n_tok, vp(q), 1, g, None, 0, float("inf"),
                                 vp(got), None) == m.TQ_ERR_ARG
    torch.cuda.synchronize()
    assert torch.isnan(got).all()
    ref = torch.zeros_like(got)
    ws = m.workspace(codec.workspace_bytes(m.TQ_OP_LOGITS, 1, n_kv, g))
    m.tq_logits(codec, packed, 1, n_kv, n_tok, q, g, None, 0, 1.0, ref, ws)
    m.tq_logits_noalloc(codec, packed, 1, n_kv, n_tok, q, g, None, 0, 1.0, got)
    torch.cuda.synchronize()
    assert torch.equal(ref, got)
