"""Python binding of libtq, the TurboQuant KV-vector hot path for B200 (sm_100a).

Argument marshalling only: every function forwards torch device pointers and sizes to the
C ABI in include/tq.h; all arithmetic runs in the CUDA library. PyTorch provides device
memory and streams. Importing this package fails loudly if libtq.so has not been built
(run ``python kv_cache_vector_03_b200/build.py`` or ``__graft_entry__.build()``).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libtq.so is missing at {LIB_PATH}: build it with python kv_cache_vector_03_b200/build.py")

lib = ctypes.CDLL(LIB_PATH)

TQ_OK, TQ_ERR_ARG, TQ_ERR_UNSUPPORTED, TQ_ERR_CUDA = 0, -1, -2, -3
TQ_ERR_RANGE, TQ_ERR_TIMEOUT, TQ_ERR_NOCONV, TQ_ERR_WORKSPACE = -4, -5, -6, -7
TQ_F32, TQ_BF16 = 0, 1
TQ_OP_QUANTIZE, TQ_OP_LOGITS, TQ_OP_PV, TQ_OP_TOPK, TQ_OP_DEQUANTIZE = 0, 1, 2, 3, 4
TQ_EST_QJL, TQ_EST_MSE = 0, 1
TQ_TEST_STALL = 0x100   # test hook: see include/tq.h
EXPORTED = ["tq_make_codebook", "tq_block_bytes", "tq_record_bytes", "tq_packed_bytes", "tq_prep_bytes",
            "tq_prepare", "tq_workspace_bytes", "tq_quantize", "tq_logits", "tq_pv", "tq_topk",
            "tq_dequantize", "tq_reset_status", "tq_get_status", "tq_status_string", "tq_abi_version",
            "tq_logits_noalloc", "tq_attention", "tq_attention_workspace_bytes", "tq_logits_est", "tq_topk_est",
            "tq_q8_packed_bytes", "tq_q8_quantize", "tq_q8_logits", "tq_attention_q8",
            "tq_attention_q8_workspace_bytes"]


class tq_codec(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int), ("m", ctypes.c_int), ("mse_bits", ctypes.c_int), ("qjl", ctypes.c_int),
                ("pi", ctypes.c_void_p), ("s", ctypes.c_void_p), ("centroids", ctypes.c_void_p),
                ("prep", ctypes.c_void_p), ("prep_bytes", ctypes.c_size_t)]


_P, _I, _I64, _SZ, _F = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
_CP = ctypes.POINTER(tq_codec)
_sig = {
    "tq_make_codebook": (_I, [_I, _I, _P, _P, _P]),
    "tq_block_bytes": (_SZ, [_CP]),
    "tq_record_bytes": (_SZ, [_CP]),
    "tq_packed_bytes": (_SZ, [_CP, _I64, _I64]),
    "tq_prep_bytes": (_SZ, [_CP]),
    "tq_prepare": (_I, [_CP, _P]),
    "tq_workspace_bytes": (_SZ, [_CP, _I, _I64, _I64, _I64]),
    "tq_quantize": (_I, [_CP, _P, _I, _I64, _I64, _I64, _P, _P, _SZ, _P]),
    "tq_logits": (_I, [_CP, _P, _I64, _I, _I64, _P, _I, _I, _P, _I, _F, _P, _P, _SZ, _P]),
    "tq_logits_noalloc": (_I, [_CP, _P, _I64, _I, _I64, _P, _I, _I, _P, _I, _F, _P, _P]),
    "tq_pv": (_I, [_CP, _P, _I64, _I, _I64, _P, _I, _P, _P, _SZ, _P]),
    "tq_attention_workspace_bytes": (_SZ, [_CP, _CP, _I64, _I, _I64, _I, _I]),
    "tq_attention": (_I, [_CP, _CP, _P, _P, _I64, _I, _I64, _P, _I, _I, _P, _P, _I, _F, _F, _P, _P, _SZ, _P]),
    "tq_attention_q8_workspace_bytes": (_SZ, [_CP, _I64, _I, _I64, _I, _I]),
    "tq_attention_q8": (_I, [_CP, _P, _P, _I64, _I, _I64, _P, _I, _I, _P, _P, _I, _F, _F, _P, _P, _SZ, _P]),
    "tq_topk": (_I, [_CP, _P, _I64, _P, _I64, _I, _P, _P, _P, _SZ, _P]),
    "tq_logits_est": (_I, [_CP, _P, _I64, _I, _I64, _P, _I, _I, _P, _I, _F, _P, _P, _SZ, _I, _P]),
    "tq_q8_packed_bytes": (_SZ, [_I, _I64, _I64]),
    "tq_q8_quantize": (_I, [_P, _I, _I, _I64, _I64, _I64, _P, _P, _SZ, _P]),
    "tq_q8_logits": (_I, [_P, _I, _I64, _I, _I64, _P, _I, _I, _P, _I, _F, _P, _P]),
    "tq_topk_est": (_I, [_CP, _P, _I64, _P, _I64, _I, _P, _P, _P, _SZ, _I, _P]),
    "tq_dequantize": (_I, [_CP, _P, _I64, _I64, _P, _P, _SZ, _P]),
    "tq_reset_status": (_I, [_P, _P]),
    "tq_get_status": (_I, [_P, _P]),
    "tq_status_string": (ctypes.c_char_p, [_I]),
    "tq_abi_version": (_I, []),
}
for _name, (_res, _args) in _sig.items():
    _fn = getattr(lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


class TQError(RuntimeError):
    def __init__(self, fn, status):
        super().__init__(f"{fn} -> {status} ({lib.tq_status_string(status).decode()})")
        self.status = status


def _check(fn, st):
    if st != TQ_OK:
        raise TQError(fn, st)
    return st


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype(t):
    import torch
    if t.dtype == torch.float32:
        return TQ_F32
    if t.dtype == torch.bfloat16:
        return TQ_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


# ----------------------------------------------------------------------------- API
def tq_make_codebook(d: int, mse_bits: int):
    """Host Lloyd-Max codebook: (centroids, bounds, normalised mse) as fp64 numpy arrays."""
    nl = 1 << mse_bits
    c = np.zeros(nl)
    t = np.zeros(nl - 1)
    mse = ctypes.c_double()
    _check("tq_make_codebook", lib.tq_make_codebook(d, mse_bits, c.ctypes.data, t.ctypes.data, ctypes.byref(mse)))
    return c, t, mse.value


class Codec:
    """A tq_codec with its device matrices and prepared operands (kept alive here)."""

    def __init__(self, d, m, mse_bits, qjl, pi, s, centroids=None, stream=None):
        import torch
        self.pi = pi.to(device="cuda", dtype=torch.float32).contiguous()
        self.s = s.to(device="cuda", dtype=torch.float32).contiguous() if qjl else None
        if centroids is None:
            centroids = tq_make_codebook(d, mse_bits)[0]
        self.centroids = np.ascontiguousarray(centroids, dtype=np.float64)
        self.c = tq_codec(d, m if qjl else 0, mse_bits, int(qjl), self.pi.data_ptr(),
                          self.s.data_ptr() if qjl else None, self.centroids.ctypes.data, None, 0)
        nprep = lib.tq_prep_bytes(ctypes.byref(self.c))
        if nprep == 0:
            raise TQError("tq_prep_bytes", TQ_ERR_UNSUPPORTED)
        self.prep = torch.empty(nprep, dtype=torch.uint8, device="cuda")
        self.c.prep = self.prep.data_ptr()
        self.c.prep_bytes = nprep
        _check("tq_prepare", lib.tq_prepare(ctypes.byref(self.c), _stream(stream)))

    @property
    def ref(self):
        return ctypes.byref(self.c)

    def block_bytes(self):
        return lib.tq_block_bytes(self.ref)

    def record_bytes(self):
        return lib.tq_record_bytes(self.ref)

    def packed_bytes(self, n_streams, n_tok):
        return lib.tq_packed_bytes(self.ref, n_streams, n_tok)

    def workspace_bytes(self, op, a=0, b=0, c=0):
        return lib.tq_workspace_bytes(self.ref, op, a, b, c)


def workspace(nbytes):
    import torch
    ws = torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device="cuda")
    return ws


def tq_quantize(codec: Codec, x, n_streams, n_tok, x_stream_stride, packed, ws, stream=None):
    return _check("tq_quantize", lib.tq_quantize(codec.ref, _ptr(x), _dtype(x), n_streams, n_tok, x_stream_stride,
                                                 _ptr(packed), _ptr(ws), ws.numel(), _stream(stream)))


def tq_logits(codec: Codec, packed, n_seq, n_kv, n_tok, q, g, tail, n_tail, scale, out, ws, stream=None,
              estimator=None):
    if estimator is None:
        return _check("tq_logits", lib.tq_logits(codec.ref, _ptr(packed), n_seq, n_kv, n_tok, _ptr(q), _dtype(q), g,
                                                 _ptr(tail), n_tail, scale, _ptr(out), _ptr(ws), ws.numel(),
                                                 _stream(stream)))
    return _check("tq_logits_est", lib.tq_logits_est(codec.ref, _ptr(packed), n_seq, n_kv, n_tok, _ptr(q), _dtype(q),
                                                     g, _ptr(tail), n_tail, scale, _ptr(out), _ptr(ws), ws.numel(),
                                                     estimator, _stream(stream)))


def tq_logits_noalloc(codec: Codec, packed, n_seq, n_kv, n_tok, q, g, tail, n_tail, scale, out, stream=None):
    """tq_logits with the library's fixed device scratch instead of a caller workspace."""
    return _check("tq_logits_noalloc", lib.tq_logits_noalloc(codec.ref, _ptr(packed), n_seq, n_kv, n_tok, _ptr(q),
                                                             _dtype(q), g, _ptr(tail), n_tail, scale, _ptr(out),
                                                             _stream(stream)))


def tq_pv(codec: Codec, packed_v, n_seq, n_kv, n_tok, P, g, out, ws, stream=None):
    return _check("tq_pv", lib.tq_pv(codec.ref, _ptr(packed_v), n_seq, n_kv, n_tok, _ptr(P), g, _ptr(out), _ptr(ws),
                                     ws.numel(), _stream(stream)))


def tq_attention_workspace_bytes(kcodec: Codec, vcodec: Codec, n_seq, n_kv, n_tok, g, n_tail):
    return lib.tq_attention_workspace_bytes(kcodec.ref, vcodec.ref, n_seq, n_kv, n_tok, g, n_tail)


def tq_attention(kcodec: Codec, vcodec: Codec, packed_k, packed_v, n_seq, n_kv, n_tok, q, g, tail_k, tail_v, n_tail,
                 scale, out, ws, v_skip=0.0, stream=None):
    return _check("tq_attention", lib.tq_attention(kcodec.ref, vcodec.ref, _ptr(packed_k), _ptr(packed_v), n_seq, n_kv,
                                                   n_tok, _ptr(q), _dtype(q), g, _ptr(tail_k), _ptr(tail_v), n_tail,
                                                   scale, v_skip, _ptr(out), _ptr(ws), ws.numel(), _stream(stream)))


def tq_attention_q8_workspace_bytes(vcodec: Codec, n_seq, n_kv, n_tok, g, n_tail):
    return lib.tq_attention_q8_workspace_bytes(vcodec.ref, n_seq, n_kv, n_tok, g, n_tail)


def tq_attention_q8(vcodec: Codec, packed_k8, packed_v, n_seq, n_kv, n_tok, q, g, tail_k, tail_v, n_tail, scale, out,
                    ws, v_skip=0.0, stream=None):
    return _check("tq_attention_q8", lib.tq_attention_q8(vcodec.ref, _ptr(packed_k8), _ptr(packed_v), n_seq, n_kv,
                                                         n_tok, _ptr(q), _dtype(q), g, _ptr(tail_k), _ptr(tail_v),
                                                         n_tail, scale, v_skip, _ptr(out), _ptr(ws), ws.numel(),
                                                         _stream(stream)))


def tq_topk(codec: Codec, packed_db, n_db, q, n_q, k, idx, score, ws, stream=None, estimator=None):
    if estimator is None:
        return _check("tq_topk", lib.tq_topk(codec.ref, _ptr(packed_db), n_db, _ptr(q), n_q, k, _ptr(idx),
                                             _ptr(score), _ptr(ws), ws.numel(), _stream(stream)))
    return _check("tq_topk_est", lib.tq_topk_est(codec.ref, _ptr(packed_db), n_db, _ptr(q), n_q, k, _ptr(idx),
                                                 _ptr(score), _ptr(ws), ws.numel(), estimator, _stream(stream)))


def tq_q8_packed_bytes(d, n_streams, n_tok):
    return lib.tq_q8_packed_bytes(d, n_streams, n_tok)


def tq_q8_quantize(x, d, n_streams, n_tok, x_stream_stride, packed, ws, stream=None):
    return _check("tq_q8_quantize", lib.tq_q8_quantize(_ptr(x), _dtype(x), d, n_streams, n_tok, x_stream_stride,
                                                       _ptr(packed), _ptr(ws), ws.numel(), _stream(stream)))


def tq_q8_logits(packed, d, n_seq, n_kv, n_tok, q, g, tail, n_tail, scale, out, stream=None):
    return _check("tq_q8_logits", lib.tq_q8_logits(_ptr(packed), d, n_seq, n_kv, n_tok, _ptr(q), _dtype(q), g,
                                                   _ptr(tail), n_tail, scale, _ptr(out), _stream(stream)))


def tq_dequantize(codec: Codec, packed, n_streams, n_tok, out, ws=None, stream=None):
    return _check("tq_dequantize", lib.tq_dequantize(codec.ref, _ptr(packed), n_streams, n_tok, _ptr(out), _ptr(ws),
                                                     0 if ws is None else ws.numel(), _stream(stream)))


def tq_reset_status(ws, stream=None):
    return _check("tq_reset_status", lib.tq_reset_status(_ptr(ws), _stream(stream)))


def tq_get_status(ws, stream=None) -> int:
    """TQ_OK or TQ_ERR_RANGE (data-dependent faults since the last read); clears the word."""
    return lib.tq_get_status(_ptr(ws), _stream(stream))
