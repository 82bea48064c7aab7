"""Independent numpy unpacker of libtq's packed records, written from the storage format
description (blocks of 32 vectors; key blocks = bit planes laid out for the int8 MMA
fragment; value blocks = 2B-bit token-pair fields laid out for the fp16 MMA fragment).
Test infrastructure: shares no code with the library or the oracle."""
from __future__ import annotations

import numpy as np


def _round_up(v, a):
    return (v + a - 1) // a * a


def key_block_bytes(d, m, B):
    GD, GM = _round_up(d, 128) // 128, _round_up(m, 128) // 128
    return 512 * (B * GD + GM) + 128


def value_block_bytes(d, B):
    return 4 * _round_up(d, 128) * B + 64


def unpack_keys(buf: np.ndarray, d: int, m: int, B: int, n_streams: int, n_tok: int):
    """-> idx [S, n_tok, d] u8, sbit [S, n_tok, m] u8, nhat, ghat [S, n_tok] (fp64 of binary16)."""
    D, Mp = _round_up(d, 128), _round_up(m, 128)
    GD, GM = D // 128, Mp // 128
    NPG = B * GD + GM
    bb = 512 * NPG + 128
    nb = (n_tok + 31) // 32
    raw = np.asarray(buf, dtype=np.uint8).reshape(n_streams * nb, bb)
    A = raw[:, :512 * NPG].copy().view(np.uint32).reshape(-1, NPG, 8, 4, 4)  # [blk, pg, gq, tq, u]
    A = A.transpose(0, 4, 2, 1, 3).reshape(-1, 32, NPG, 4)                   # [blk, v=8u+gq, pg, tq]

    def plane_bits(pg0, ngroups, nbits):
        words = A[:, :, pg0:pg0 + ngroups, :].reshape(A.shape[0], 32, 4 * ngroups)  # word 4gr + tq
        bits = np.unpackbits(words.copy().view(np.uint8), axis=-1, bitorder="little")
        return bits[..., :nbits]

    idx = np.zeros((A.shape[0], 32, d), np.uint8)
    for pl in range(B):
        idx |= plane_bits(pl * GD, GD, d) << pl
    sbit = plane_bits(B * GD, GM, m)
    nw = raw[:, 512 * NPG:].copy().view(np.uint32).reshape(-1, 8, 4)         # [blk, gq, u]
    nw = nw.transpose(0, 2, 1).reshape(-1, 32)                                # v = 8u + gq
    nhat = (nw & 0xFFFF).astype(np.uint16).view(np.float16).astype(np.float64)
    ghat = (nw >> 16).astype(np.uint16).view(np.float16).astype(np.float64)

    def per_stream(a):
        return a.reshape(n_streams, nb * 32, *a.shape[2:])[:, :n_tok]

    return per_stream(idx), per_stream(sbit), per_stream(nhat), per_stream(ghat)


def unpack_values(buf: np.ndarray, d: int, B: int, n_streams: int, n_tok: int):
    """-> idx [S, n_tok, d] u8, nhat [S, n_tok] (fp64 of binary16)."""
    D = _round_up(d, 128)
    CH = D * B // 128
    bb = 4 * D * B + 64
    nb = (n_tok + 31) // 32
    raw = np.asarray(buf, dtype=np.uint8).reshape(n_streams * nb, bb)
    A = raw[:, :4 * D * B].reshape(-1, CH, 32, 16).transpose(0, 2, 1, 3).reshape(-1, 32, CH * 16)
    bits = np.unpackbits(A, axis=-1, bitorder="little")                        # [blk, lane, D*B]
    nblk = raw.shape[0]
    idx = np.zeros((nblk, 32, D), np.uint8)
    weights = (1 << np.arange(B)).astype(np.uint8)
    for lane in range(32):
        gq, tq = lane >> 2, lane & 3
        for p in range(4):
            tau = 16 * (p >> 1) + 8 * (p & 1) + 2 * tq
            for a in range(D // 8):
                f = (4 * a + p) * 2 * B
                i = 8 * a + gq
                idx[:, tau, i] = bits[:, lane, f:f + B] @ weights
                idx[:, tau + 1, i] = bits[:, lane, f + B:f + 2 * B] @ weights
    nhat = raw[:, 4 * D * B:].copy().view(np.uint16).view(np.float16).astype(np.float64)
    return (idx.reshape(n_streams, nb * 32, D)[:, :n_tok, :d],
            nhat.reshape(n_streams, nb * 32)[:, :n_tok])
