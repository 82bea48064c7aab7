// C-ABI entry points of libtq: argument checks, codebook-derived constants, workspace
// layout and kernel launches. Every entry point is declared and documented in include/tq.h.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>

#include "tq.h"
#include "tq_device.cuh"


namespace {

// polls of the wait that TQ_TEST_STALL makes run out (a few milliseconds at most)
constexpr uint32_t kTestStallPolls = 2000;

size_t align_up(size_t v) { return (v + TQ_ALIGN - 1) / TQ_ALIGN * TQ_ALIGN; }

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

// shape checks shared by every call
int check_codec(const tq_codec* c, bool need_prep) {
    if (!c) return TQ_ERR_ARG;
    if (c->d < 8 || c->d > TQ_MAX_D || c->d % 8) return TQ_ERR_UNSUPPORTED;
    if (c->qjl != 0 && c->qjl != 1) return TQ_ERR_ARG;
    if (c->qjl && (c->m < 8 || c->m > TQ_MAX_D || c->m % 8)) return TQ_ERR_UNSUPPORTED;
    if (c->mse_bits < 1 || c->mse_bits > (c->qjl ? 3 : 4)) return TQ_ERR_UNSUPPORTED;
    if (!c->pi || !c->centroids || (c->qjl && !c->s)) return TQ_ERR_ARG;
    if (!aligned(c->pi, 4) || (c->qjl && !aligned(c->s, 4))) return TQ_ERR_ARG;
    if (need_prep) {
        if (!c->prep || !aligned(c->prep, 256)) return TQ_ERR_ARG;
        if (c->prep_bytes < tq_prep_bytes(c)) return TQ_ERR_WORKSPACE;
    }
    return TQ_OK;
}

TqDims dims_of(const tq_codec* c) { return tq_dims(c->d, c->m, c->mse_bits, c->qjl); }

// centroids (host, fp64) -> boundaries, fp32 copies, +-1 plane coefficients, binary16 table
int codebook_consts(const tq_codec* c, TqCodebookConsts* k) {
    std::memset(k, 0, sizeof(*k));
    const int B = c->mse_bits, L = 1 << B;
    const double* cc = c->centroids;
    double mx = 0.0;
    for (int i = 0; i < L; ++i) {
        if (!std::isfinite(cc[i])) return TQ_ERR_ARG;
        mx = std::fmax(mx, std::fabs(cc[i]));
        if (i && !(cc[i] > cc[i - 1])) return TQ_ERR_ARG;
    }
    for (int i = 0; i < L; ++i)
        if (std::fabs(cc[i] + cc[L - 1 - i]) > 1e-12 * mx) return TQ_ERR_ARG;  // symmetric
    for (int i = 0; i + 1 < L; ++i) k->bounds[i] = (float)(0.5 * (cc[i] + cc[i + 1]));
    for (int i = 0; i < L; ++i) {
        k->cent[i] = (float)cc[i];
        k->lut_half[i] = __half_as_ushort(__float2half_rn((float)cc[i]));
    }
    // Walsh coefficients a_S = 2^-B sum_idx c[idx] prod_{k in S} s_k(idx), s_k = 2 bit_k - 1,
    // for the odd sets the estimator uses: {0}, {1}, {2}, {0,1,2}
    const int sets[4] = {1, 2, 4, 7};
    const int nplanes = B == 3 ? 4 : B;
    double sum = 0.0;
    for (int pl = 0; pl < nplanes; ++pl) {
        double a = 0.0;
        for (int idx = 0; idx < L; ++idx) {
            double prod = 1.0;
            for (int kb = 0; kb < B; ++kb)
                if (sets[pl] >> kb & 1) prod *= (idx >> kb & 1) ? 1.0 : -1.0;
            a += cc[idx] * prod;
        }
        a /= L;
        k->plane_coef[pl] = (float)a;
        sum += a;
    }
    k->plane_sum = (float)sum;
    if (c->qjl) {  // the odd expansion must reproduce every centroid
        for (int idx = 0; idx < L; ++idx) {
            double v = 0.0;
            for (int pl = 0; pl < nplanes; ++pl) {
                double prod = 1.0;
                for (int kb = 0; kb < B; ++kb)
                    if (sets[pl] >> kb & 1) prod *= (idx >> kb & 1) ? 1.0 : -1.0;
                v += k->plane_coef[pl] * prod;
            }
            if (std::fabs(v - cc[idx]) > 1e-6 * mx) return TQ_ERR_ARG;
        }
    }
    return TQ_OK;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? TQ_OK : TQ_ERR_CUDA; }

// workspace regions after the status word
struct LogitsWs { size_t qfrag, qscale, total; };
LogitsWs logits_ws(const TqDims& t, int64_t n_streams, int g) {
    const int ntiles = g > 4 ? 2 : 1;
    LogitsWs w;
    size_t off = TQ_STATUS_BYTES;
    w.qfrag = off; off = align_up(off + (size_t)n_streams * ntiles * t.nmg * 4 * 64 * 4);
    w.qscale = off; off = align_up(off + (size_t)n_streams * ntiles * 4 * 16);
    w.total = off;
    return w;
}

// tq_topk workspace: fp16 query operand rows of the padded query tiles, 1 / sigma per row,
// then the per-range candidate lists
struct TopkWs { int nsplit, n_qt, kb_mse, kb_sign, kq; int64_t n_tiles, tps; size_t qimg, qinv, psc, pix, total; };
TopkWs topk_ws(const TqDims& t, int64_t n_q, int64_t n_db, int k, bool qjl_terms) {
    TopkWs w;
    w.n_tiles = (n_db + 127) / 128;
    w.n_qt = (int)((n_q + 127) / 128);
    w.kb_mse = (t.d + 63) / 64;
    w.kb_sign = qjl_terms ? (t.m + 63) / 64 : 0;
    w.kq = 64 * (w.kb_mse + w.kb_sign);
    w.nsplit = tq_topk_nsplit(w.n_qt, std::max<int64_t>(1, w.n_tiles));
    w.tps = (w.n_tiles + w.nsplit - 1) / w.nsplit;
    size_t off = TQ_STATUS_BYTES;
    w.qimg = off; off = align_up(off + (size_t)w.n_qt * 128 * (64 * (size_t)((t.d + 63) / 64 + (t.m + 63) / 64)) * 2);
    w.qinv = off; off = align_up(off + (size_t)w.n_qt * 128 * 4);
    w.psc = off; off = align_up(off + (size_t)n_q * w.nsplit * k * 4);
    w.pix = off; off = align_up(off + (size_t)n_q * w.nsplit * k * 4);
    w.total = off;
    return w;
}

struct PvWs { int nsplit, bps; size_t part, ml, total; };
PvWs pv_ws(const TqDims& t, int64_t n_streams, int64_t n_tok, int g) {
    PvWs w;
    const int64_t nb = (n_tok + 31) / 32;
    int64_t bps = (nb * n_streams + 2 * tq_device_sms() - 1) / (2 * tq_device_sms());   // about two CTAs per SM
    if (bps < 8) bps = 8;
    if (bps > nb) bps = nb;
    if (bps < 1) bps = 1;
    w.bps = (int)bps;
    w.nsplit = (int)((nb + bps - 1) / bps);
    size_t off = TQ_STATUS_BYTES;
    w.part = off; off = align_up(off + (size_t)n_streams * g * w.nsplit * t.D * 4);
    w.ml = off; off = align_up(off + (size_t)n_streams * g * w.nsplit * 8);
    w.total = off;
    return w;
}

// fused attention: the logits prologue's fragments, the exact tail logits, split partials.
// One CTA per (stream, range) at about two resident CTAs per SM; ranges of at least 8 blocks
// (one per warp).
struct AttnWs { int nsplit, bps; LogitsWs lg; size_t tl, part, ml, total; };
AttnWs attn_ws(const TqDims& tk, int64_t n_streams, int64_t n_tok, int g, int n_tail) {
    AttnWs w;
    w.lg = logits_ws(tk, n_streams, g);
    const int64_t nb = (n_tok + 31) / 32;
    int64_t bps = (nb * n_streams + 2 * tq_device_sms() - 1) / (2 * tq_device_sms());
    bps = std::max<int64_t>(8, bps);
    bps = std::max<int64_t>(1, std::min<int64_t>(bps, nb));
    w.bps = (int)bps;
    w.nsplit = (int)((nb + bps - 1) / bps);
    size_t off = w.lg.total;
    w.tl = off; off = align_up(off + (size_t)n_streams * g * n_tail * 4);
    w.part = off; off = align_up(off + (size_t)n_streams * g * w.nsplit * 128 * 4);
    w.ml = off; off = align_up(off + (size_t)n_streams * g * w.nsplit * 8);
    w.total = off;
    return w;
}

// attention over 8-bit keys: the tail logits, split partials (no query fragments)
struct AttnQ8Ws { int nsplit, bps; size_t tl, part, ml, total; };
AttnQ8Ws attn_q8_ws(int64_t n_streams, int64_t n_tok, int g, int n_tail, int vbits) {
    AttnQ8Ws w;
    const int64_t nb = (n_tok + 31) / 32;
    const int64_t ctas = (int64_t)tq_attention_q8_ctas_per_sm(vbits) * tq_device_sms();   // one wave
    int64_t bps = (nb * n_streams + ctas - 1) / ctas;
    bps = std::max<int64_t>(8, bps);
    bps = std::max<int64_t>(1, std::min<int64_t>(bps, nb));
    w.bps = (int)bps;
    w.nsplit = (int)((nb + bps - 1) / bps);
    size_t off = TQ_STATUS_BYTES;
    w.tl = off; off = align_up(off + (size_t)n_streams * g * n_tail * 4);
    w.part = off; off = align_up(off + (size_t)n_streams * g * w.nsplit * 128 * 4);
    w.ml = off; off = align_up(off + (size_t)n_streams * g * w.nsplit * 8);
    w.total = off;
    return w;
}

// key codec (qjl = 1, d and m <= 128) and value codec (qjl = 0, the same d) of tq_attention
int check_attention_codecs(const tq_codec* kc, const tq_codec* vc) {
    int st = check_codec(kc, true);
    if (st != TQ_OK) return st;
    if ((st = check_codec(vc, true)) != TQ_OK) return st;
    if (!kc->qjl || vc->qjl || kc->d != vc->d) return TQ_ERR_ARG;
    if (kc->d > 128 || kc->m > 128) return TQ_ERR_UNSUPPORTED;
    return TQ_OK;
}

}  // namespace

extern "C" {

int tq_abi_version(void) { return 1; }

const char* tq_status_string(int s) {
    switch (s) {
        case TQ_OK: return "ok";
        case TQ_ERR_ARG: return "invalid argument";
        case TQ_ERR_UNSUPPORTED: return "unsupported shape";
        case TQ_ERR_CUDA: return "CUDA runtime error";
        case TQ_ERR_RANGE: return "norm overflowed binary16 or input not finite";
        case TQ_ERR_TIMEOUT: return "timeout";
        case TQ_ERR_NOCONV: return "codebook did not converge";
        case TQ_ERR_WORKSPACE: return "workspace or prepared buffer too small";
    }
    return "unknown status";
}

int tq_make_codebook(int d, int mse_bits, double* centroids, double* bounds, double* mse) {
    if (!centroids || !bounds) return TQ_ERR_ARG;
    if (d < 3 || d > 4096 || mse_bits < 1 || mse_bits > 8) return TQ_ERR_UNSUPPORTED;
    const int r = tq_host_codebook(d, mse_bits, centroids, bounds, mse);
    return r == 0 ? TQ_OK : (r == -6 ? TQ_ERR_NOCONV : TQ_ERR_ARG);
}

size_t tq_block_bytes(const tq_codec* c) {
    if (check_codec(c, false) != TQ_OK) return 0;
    return dims_of(c).block_bytes;
}

size_t tq_record_bytes(const tq_codec* c) { return tq_block_bytes(c) / 32; }

size_t tq_packed_bytes(const tq_codec* c, int64_t n_streams, int64_t n_tok) {
    if (n_streams < 0 || n_tok < 0) return 0;
    return tq_block_bytes(c) * (size_t)n_streams * (size_t)((n_tok + 31) / 32);
}

size_t tq_prep_bytes(const tq_codec* c) {
    if (check_codec(c, false) != TQ_OK) return 0;
    return tq_prep_layout(dims_of(c)).total;
}

int tq_prepare(const tq_codec* c, void* stream) {
    int st = check_codec(c, true);
    if (st != TQ_OK) return st;
    const TqDims t = dims_of(c);
    const TqPrepLayout L = tq_prep_layout(t);
    uint8_t* base = static_cast<uint8_t*>(c->prep);
    PrepParams p;
    p.pi = c->pi; p.s = c->s;
    p.piT = reinterpret_cast<float*>(base + L.piT);
    p.sT = reinterpret_cast<float*>(base + L.sT);
    p.mT = reinterpret_cast<float*>(base + L.mT);
    p.pih = reinterpret_cast<uint16_t*>(base + L.pih);
    p.pil = reinterpret_cast<uint16_t*>(base + L.pil);
    p.mh = reinterpret_cast<uint16_t*>(base + L.mh);
    p.ml = reinterpret_cast<uint16_t*>(base + L.ml);
    p.img = L.wimg > L.img ? base + L.img : nullptr;
    p.wimg = L.total > L.wimg ? base + L.wimg : nullptr;
    p.hdr = reinterpret_cast<uint32_t*>(base + L.hdr);
    p.d = t.d; p.m = t.m; p.D = t.D; p.Mp = t.Mp; p.qjl = t.qjl;
    return cuda_status(tq_launch_prepare(p, static_cast<cudaStream_t>(stream)));
}

size_t tq_workspace_bytes(const tq_codec* c, int op, int64_t a, int64_t b, int64_t cc) {
    if (check_codec(c, false) != TQ_OK) return 0;
    const TqDims t = dims_of(c);
    switch (op) {
        case TQ_OP_QUANTIZE:
        case TQ_OP_DEQUANTIZE:
            return TQ_STATUS_BYTES;
        case TQ_OP_LOGITS:
            if (a < 0 || b < 1 || cc < 1 || cc > 8) return 0;
            return logits_ws(t, a * b, (int)cc).total;
        case TQ_OP_PV:
            if (a < 0 || b < 1 || cc < 1 || cc > 8) return 0;
            return pv_ws(t, a, b, (int)cc).total;
        case TQ_OP_TOPK:
            if (!c->qjl || a < 1 || b < 1 || cc < 1 || cc > 32 || cc > b) return 0;
            return topk_ws(t, a, b, (int)cc, true).total;
    }
    return 0;
}

int tq_reset_status(void* ws, void* stream) {
    if (!ws) return TQ_ERR_ARG;
    return cuda_status(cudaMemsetAsync(ws, 0, 4, static_cast<cudaStream_t>(stream)));
}

int tq_get_status(void* ws, void* stream) {
    if (!ws) return TQ_ERR_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t word = 0;
    if (cudaMemcpyAsync(&word, ws, 4, cudaMemcpyDeviceToHost, st) != cudaSuccess) return TQ_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return TQ_ERR_CUDA;
    if (word) {
        if (cudaMemsetAsync(ws, 0, 4, st) != cudaSuccess) return TQ_ERR_CUDA;
        if (cudaStreamSynchronize(st) != cudaSuccess) return TQ_ERR_CUDA;
    }
    if (word & TQ_FLAG_TIMEOUT) return TQ_ERR_TIMEOUT;
    return (word & TQ_FLAG_RANGE) ? TQ_ERR_RANGE : TQ_OK;
}

int tq_quantize(const tq_codec* c, const void* x, tq_dtype dtype, int64_t n_streams, int64_t n_tok,
                int64_t x_stream_stride, void* packed, void* ws, size_t ws_bytes, void* stream) {
    int st = check_codec(c, true);
    if (st != TQ_OK) return st;
    if (dtype != TQ_F32 && dtype != TQ_BF16) return TQ_ERR_ARG;
    if (n_streams < 0 || n_tok < 0) return TQ_ERR_ARG;
    if (n_streams == 0 || n_tok == 0) return TQ_OK;
    if (!x || !packed || !ws) return TQ_ERR_ARG;
    if (!aligned(packed, 16) || !aligned(x, dtype == TQ_F32 ? 4 : 2) || !aligned(ws, 4)) return TQ_ERR_ARG;
    if (n_streams > 1 && x_stream_stride < n_tok * c->d) return TQ_ERR_ARG;
    if (ws_bytes < TQ_STATUS_BYTES) return TQ_ERR_WORKSPACE;
    const TqDims t = dims_of(c);
    const TqPrepLayout L = tq_prep_layout(t);
    QuantParams p;
    p.x = x; p.dtype = dtype;
    p.n_streams = n_streams; p.n_tok = n_tok; p.x_stride = x_stream_stride;
    p.nb = (n_tok + 31) / 32;
    if (p.n_streams * p.nb > 0x7fffffffLL) return TQ_ERR_UNSUPPORTED;
    p.packed = static_cast<uint8_t*>(packed);
    p.piT = reinterpret_cast<const float*>(static_cast<uint8_t*>(c->prep) + L.piT);
    p.mT = reinterpret_cast<const float*>(static_cast<uint8_t*>(c->prep) + L.mT);
    p.pih = reinterpret_cast<const uint16_t*>(static_cast<uint8_t*>(c->prep) + L.pih);
    p.pil = reinterpret_cast<const uint16_t*>(static_cast<uint8_t*>(c->prep) + L.pil);
    p.mh = reinterpret_cast<const uint16_t*>(static_cast<uint8_t*>(c->prep) + L.mh);
    p.ml = reinterpret_cast<const uint16_t*>(static_cast<uint8_t*>(c->prep) + L.ml);
    p.img = L.wimg > L.img ? static_cast<const uint8_t*>(c->prep) + L.img : nullptr;
    p.wimg = L.total > L.wimg ? static_cast<const uint8_t*>(c->prep) + L.wimg : nullptr;
    p.hdr = reinterpret_cast<const uint32_t*>(static_cast<const uint8_t*>(c->prep) + L.hdr);
    p.status = static_cast<uint32_t*>(ws);
    p.vec_ok = aligned(x, dtype == TQ_F32 ? 16 : 8) && x_stream_stride % 4 == 0 && c->d % 4 == 0;
    p.t = t;
    if ((st = codebook_consts(c, &p.cb)) != TQ_OK) return st;
    return cuda_status(tq_launch_quantize(p, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

// tq_logits_est behind its argument checks; with clear_status the status word is cleared on
// the stream once every check has passed (the no-workspace variant shares one scratch array).
int tq_logits_run(const tq_codec* c, const void* packed, int64_t n_seq, int n_kv, int64_t n_tok, const void* q,
                  tq_dtype q_dtype, int g, const void* tail, int n_tail, float scale, float* out, void* ws,
                  size_t ws_bytes, int estimator, int clear_status, void* stream) {
    int st = check_codec(c, true);
    if (st != TQ_OK) return st;
    const bool test_stall = (estimator & TQ_TEST_STALL) != 0;
    estimator &= ~TQ_TEST_STALL;
    if (estimator != TQ_EST_QJL && estimator != TQ_EST_MSE) return TQ_ERR_ARG;
    if (!c->qjl) return TQ_ERR_ARG;
    if (g != 1 && g != 2 && g != 4 && g != 8) return TQ_ERR_UNSUPPORTED;
    if (n_seq < 0 || n_kv < 1 || n_tok < 0 || n_tail < 0) return TQ_ERR_ARG;
    if (q_dtype != TQ_F32 && q_dtype != TQ_BF16) return TQ_ERR_ARG;
    if (n_seq == 0 || n_tok + n_tail == 0) return TQ_OK;
    if (!q || !out || !ws || (n_tok > 0 && !packed) || (n_tail > 0 && !tail)) return TQ_ERR_ARG;
    if ((n_tok > 0 && !aligned(packed, 16)) || !aligned(out, 4) || !aligned(ws, 256) ||
        !aligned(q, q_dtype == TQ_F32 ? 4 : 2) || (n_tail > 0 && !aligned(tail, 2)))
        return TQ_ERR_ARG;
    if (!std::isfinite(scale)) return TQ_ERR_ARG;
    const TqDims t = dims_of(c);
    const int64_t n_streams = n_seq * n_kv;
    const LogitsWs W = logits_ws(t, n_streams, g);
    if (ws_bytes < W.total) return TQ_ERR_WORKSPACE;
    const TqPrepLayout L = tq_prep_layout(t);
    LogitsParams p;
    p.packed = static_cast<const uint8_t*>(packed);
    p.q = q; p.q_dtype = q_dtype;
    p.tail = static_cast<const uint16_t*>(tail);
    p.out = out;
    p.piT = reinterpret_cast<const float*>(static_cast<uint8_t*>(c->prep) + L.piT);
    p.sT = reinterpret_cast<const float*>(static_cast<uint8_t*>(c->prep) + L.sT);
    p.pimg = L.wimg > L.img ? static_cast<uint8_t*>(c->prep) + L.img + kTqProImage * kTqImageBytes : nullptr;
    p.hdr = reinterpret_cast<const uint32_t*>(static_cast<uint8_t*>(c->prep) + L.hdr);
    p.qfrag = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + W.qfrag);
    p.qscale = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + W.qscale);
    p.n_seq = n_seq; p.n_tok = n_tok; p.nb = (n_tok + 31) / 32;
    p.n_kv = n_kv; p.g = g; p.ntiles = g > 4 ? 2 : 1; p.n_tail = n_tail;
    p.scale = scale;
    // the MSE-only estimator drops the QJL term (its constants become zero)
    p.kappa = estimator == TQ_EST_MSE ? 0.f : (float)(std::sqrt(M_PI / 2.0) / c->m);
    p.status = static_cast<uint32_t*>(ws);
    p.n_heads_valid = n_streams * g;
    p.test_stall = test_stall ? kTestStallPolls : 0u;
    // the tail runs on a second grid dimension of 16-token CTAs (at most 65535)
    if (n_streams * g > 0x7fffffffLL || n_streams * p.nb > (1LL << 40) || n_tail > 16 * 65534)
        return TQ_ERR_UNSUPPORTED;
    p.t = t;
    if ((st = codebook_consts(c, &p.cb)) != TQ_OK) return st;
    if (clear_status && cudaMemsetAsync(ws, 0, 4, static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return TQ_ERR_CUDA;
    return cuda_status(tq_launch_logits(p, static_cast<cudaStream_t>(stream)));
}

extern "C" {

int tq_logits_est(const tq_codec* c, const void* packed, int64_t n_seq, int n_kv, int64_t n_tok, const void* q,
                  tq_dtype q_dtype, int g, const void* tail, int n_tail, float scale, float* out, void* ws,
                  size_t ws_bytes, int estimator, void* stream) {
    return tq_logits_run(c, packed, n_seq, n_kv, n_tok, q, q_dtype, g, tail, n_tail, scale, out, ws, ws_bytes,
                         estimator, 0, stream);
}

int tq_logits(const tq_codec* c, const void* packed, int64_t n_seq, int n_kv, int64_t n_tok, const void* q,
              tq_dtype q_dtype, int g, const void* tail, int n_tail, float scale, float* out, void* ws,
              size_t ws_bytes, void* stream) {
    return tq_logits_est(c, packed, n_seq, n_kv, n_tok, q, q_dtype, g, tail, n_tail, scale, out, ws, ws_bytes,
                         TQ_EST_QJL, stream);
}

int tq_pv(const tq_codec* c, const void* packed_v, int64_t n_seq, int n_kv, int64_t n_tok, const float* P, int g,
          float* out, void* ws, size_t ws_bytes, void* stream) {
    int st = check_codec(c, true);
    if (st != TQ_OK) return st;
    if (c->qjl) return TQ_ERR_ARG;
    if (g != 1 && g != 2 && g != 4 && g != 8) return TQ_ERR_UNSUPPORTED;
    if (n_seq < 0 || n_kv < 1 || n_tok < 1) return TQ_ERR_ARG;
    if (n_seq == 0) return TQ_OK;
    if (!packed_v || !P || !out || !ws) return TQ_ERR_ARG;
    if (!aligned(packed_v, 16) || !aligned(P, 4) || !aligned(out, 4) || !aligned(ws, 256)) return TQ_ERR_ARG;
    const TqDims t = dims_of(c);
    const int64_t n_streams = n_seq * n_kv;
    const PvWs W = pv_ws(t, n_streams, n_tok, g);
    if (ws_bytes < W.total) return TQ_ERR_WORKSPACE;
    PvParams p;
    p.packed = static_cast<const uint8_t*>(packed_v);
    p.P = P; p.out = out;
    p.piT = reinterpret_cast<const float*>(static_cast<uint8_t*>(c->prep) + tq_prep_layout(t).piT);
    p.status = static_cast<uint32_t*>(ws);
    p.part = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + W.part);
    p.part_ml = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + W.ml);
    p.n_streams = n_streams; p.n_tok = n_tok; p.nb = (n_tok + 31) / 32;
    p.g = g; p.nsplit = W.nsplit; p.blocks_per_split = W.bps;
    // grid sizes: the split CTAs, and the merge's four CTAs per query head
    if (n_streams * W.nsplit > 0x7fffffffLL || n_streams * g * 4 > 0x7fffffffLL) return TQ_ERR_UNSUPPORTED;
    p.t = t;
    if ((st = codebook_consts(c, &p.cb)) != TQ_OK) return st;
    return cuda_status(tq_launch_pv(p, static_cast<cudaStream_t>(stream)));
}

size_t tq_attention_workspace_bytes(const tq_codec* kcodec, const tq_codec* vcodec, int64_t n_seq, int n_kv,
                                    int64_t n_tok, int g, int n_tail) {
    if (check_attention_codecs(kcodec, vcodec) != TQ_OK) return 0;
    if (n_seq < 0 || n_kv < 1 || n_tok < 0 || n_tail < 0 || g < 1 || g > 4) return 0;
    return attn_ws(dims_of(kcodec), n_seq * n_kv, n_tok, g, n_tail).total;
}

int tq_attention(const tq_codec* kcodec, const tq_codec* vcodec, const void* packed_k, const void* packed_v,
                 int64_t n_seq, int n_kv, int64_t n_tok, const void* q, tq_dtype q_dtype, int g, const void* tail_k,
                 const void* tail_v, int n_tail, float scale, float v_skip, float* out, void* ws, size_t ws_bytes,
                 void* stream) {
    int st = check_attention_codecs(kcodec, vcodec);
    if (st != TQ_OK) return st;
    if (g != 1 && g != 2 && g != 4) return TQ_ERR_UNSUPPORTED;
    if (n_seq < 0 || n_kv < 1 || n_tok < 0 || n_tail < 0) return TQ_ERR_ARG;
    if (q_dtype != TQ_F32 && q_dtype != TQ_BF16) return TQ_ERR_ARG;
    if (n_seq == 0) return TQ_OK;
    if (n_tok + n_tail == 0) return TQ_ERR_ARG;   // softmax over no tokens
    if (n_tail > TQ_ATTN_MAX_TAIL) return TQ_ERR_UNSUPPORTED;
    if (!q || !out || !ws || (n_tok > 0 && (!packed_k || !packed_v)) || (n_tail > 0 && (!tail_k || !tail_v)))
        return TQ_ERR_ARG;
    if ((n_tok > 0 && (!aligned(packed_k, 16) || !aligned(packed_v, 16))) || !aligned(out, 4) ||
        !aligned(ws, 256) || !aligned(q, q_dtype == TQ_F32 ? 4 : 2) ||
        (n_tail > 0 && (!aligned(tail_k, 2) || !aligned(tail_v, 8))))
        return TQ_ERR_ARG;
    if (!std::isfinite(scale) || !(v_skip >= 0.f && v_skip <= 1.f)) return TQ_ERR_ARG;
    const TqDims tk = dims_of(kcodec), tv = dims_of(vcodec);
    const int64_t n_streams = n_seq * n_kv;
    if (n_streams * g > 0x7fffffffLL || n_streams * ((n_tok + 31) / 32) > (1LL << 40)) return TQ_ERR_UNSUPPORTED;
    const AttnWs W = attn_ws(tk, n_streams, n_tok, g, n_tail);
    if (ws_bytes < W.total) return TQ_ERR_WORKSPACE;
    // grid sizes: the split CTAs, and the merge's four CTAs per query head
    if (n_streams * W.nsplit > 0x7fffffffLL || n_streams * g * 4 > 0x7fffffffLL) return TQ_ERR_UNSUPPORTED;
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    const uint8_t* kprep = static_cast<const uint8_t*>(kcodec->prep);
    const TqPrepLayout L = tq_prep_layout(tk);

    // 1. query fragments and exact tail logits: the logits prologue with no compressed tokens
    LogitsParams lp;
    std::memset(&lp, 0, sizeof(lp));
    lp.packed = nullptr;
    lp.q = q; lp.q_dtype = q_dtype;
    lp.tail = static_cast<const uint16_t*>(tail_k);
    lp.out = reinterpret_cast<float*>(wsb + W.tl);
    lp.piT = reinterpret_cast<const float*>(kprep + L.piT);
    lp.sT = reinterpret_cast<const float*>(kprep + L.sT);
    lp.pimg = L.wimg > L.img ? kprep + L.img + kTqProImage * kTqImageBytes : nullptr;
    lp.hdr = reinterpret_cast<const uint32_t*>(kprep + L.hdr);
    lp.qfrag = reinterpret_cast<uint32_t*>(wsb + W.lg.qfrag);
    lp.qscale = reinterpret_cast<float*>(wsb + W.lg.qscale);
    lp.status = static_cast<uint32_t*>(ws);
    lp.n_seq = n_seq; lp.n_tok = 0; lp.nb = 0;
    lp.n_kv = n_kv; lp.g = g; lp.ntiles = 1; lp.n_tail = n_tail;
    lp.scale = scale;
    lp.kappa = (float)(std::sqrt(M_PI / 2.0) / kcodec->m);
    lp.n_heads_valid = n_streams * g;
    lp.t = tk;
    if ((st = codebook_consts(kcodec, &lp.cb)) != TQ_OK) return st;

    // 2. + 3. split pass over the compressed keys and values, merge with the tail
    AttnParams p;
    p.packed_k = static_cast<const uint8_t*>(packed_k);
    p.packed_v = static_cast<const uint8_t*>(packed_v);
    p.qfrag = lp.qfrag;
    p.qscale = lp.qscale;
    p.tail_logit = lp.out;
    p.tail_v = static_cast<const uint16_t*>(tail_v);
    p.piT_v = reinterpret_cast<const float*>(static_cast<const uint8_t*>(vcodec->prep) + tq_prep_layout(tv).piT);
    p.out = out;
    p.part = reinterpret_cast<float*>(wsb + W.part);
    p.part_ml = reinterpret_cast<float*>(wsb + W.ml);
    p.status = static_cast<uint32_t*>(ws);
    p.n_streams = n_streams; p.n_tok = n_tok; p.nb = (n_tok + 31) / 32;
    p.g = g; p.nsplit = p.nb > 0 ? W.nsplit : 0; p.blocks_per_split = W.bps; p.n_tail = n_tail;
    p.v_skip = v_skip;
    p.tk = tk; p.tv = tv;
    if ((st = codebook_consts(vcodec, &p.cbv)) != TQ_OK) return st;

    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    cudaError_t e = tq_launch_logits_prologue(lp, cs);
    if (e != cudaSuccess) return TQ_ERR_CUDA;
    return cuda_status(tq_launch_attention(p, cs));
}

size_t tq_attention_q8_workspace_bytes(const tq_codec* vcodec, int64_t n_seq, int n_kv, int64_t n_tok, int g,
                                       int n_tail) {
    if (check_codec(vcodec, true) != TQ_OK || vcodec->qjl || vcodec->d > 128) return 0;
    if (n_seq < 0 || n_kv < 1 || n_tok < 0 || n_tail < 0 || g < 1 || g > 4) return 0;
    return attn_q8_ws(n_seq * n_kv, n_tok, g, n_tail, vcodec->mse_bits).total;
}

int tq_attention_q8(const tq_codec* vcodec, const void* packed_k8, const void* packed_v, int64_t n_seq, int n_kv,
                    int64_t n_tok, const void* q, tq_dtype q_dtype, int g, const void* tail_k, const void* tail_v,
                    int n_tail, float scale, float v_skip, float* out, void* ws, size_t ws_bytes, void* stream) {
    int st = check_codec(vcodec, true);
    if (st != TQ_OK) return st;
    if (vcodec->qjl) return TQ_ERR_ARG;
    if (vcodec->d > 128) return TQ_ERR_UNSUPPORTED;
    if (g != 1 && g != 2 && g != 4) return TQ_ERR_UNSUPPORTED;
    if (n_seq < 0 || n_kv < 1 || n_tok < 0 || n_tail < 0) return TQ_ERR_ARG;
    if (q_dtype != TQ_F32 && q_dtype != TQ_BF16) return TQ_ERR_ARG;
    if (n_seq == 0) return TQ_OK;
    if (n_tok + n_tail == 0) return TQ_ERR_ARG;   // softmax over no tokens
    if (n_tail > TQ_ATTN_MAX_TAIL) return TQ_ERR_UNSUPPORTED;
    if (!q || !out || !ws || (n_tok > 0 && (!packed_k8 || !packed_v)) || (n_tail > 0 && (!tail_k || !tail_v)))
        return TQ_ERR_ARG;
    if ((n_tok > 0 && (!aligned(packed_k8, 16) || !aligned(packed_v, 16))) || !aligned(out, 4) ||
        !aligned(ws, 256) || !aligned(q, q_dtype == TQ_F32 ? 4 : 2) ||
        (n_tail > 0 && (!aligned(tail_k, 2) || !aligned(tail_v, 8))))
        return TQ_ERR_ARG;
    if (!std::isfinite(scale) || !(v_skip >= 0.f && v_skip <= 1.f)) return TQ_ERR_ARG;
    const TqDims tv = dims_of(vcodec);
    const int64_t n_streams = n_seq * n_kv;
    if (n_streams * g > 0x7fffffffLL || n_streams * ((n_tok + 31) / 32) > (1LL << 40)) return TQ_ERR_UNSUPPORTED;
    const AttnQ8Ws W = attn_q8_ws(n_streams, n_tok, g, n_tail, vcodec->mse_bits);
    if (ws_bytes < W.total) return TQ_ERR_WORKSPACE;
    // grid sizes: the split CTAs, and the merge's four CTAs per query head
    if (n_streams * W.nsplit > 0x7fffffffLL || n_streams * g * 4 > 0x7fffffffLL) return TQ_ERR_UNSUPPORTED;
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    AttnParams p;
    std::memset(&p, 0, sizeof(p));
    p.packed_k8 = static_cast<const uint8_t*>(packed_k8);
    p.packed_v = static_cast<const uint8_t*>(packed_v);
    p.q = q; p.q_dtype = q_dtype;
    p.tail_k = static_cast<const uint16_t*>(tail_k);
    p.tail_logit = reinterpret_cast<float*>(wsb + W.tl);
    p.tail_v = static_cast<const uint16_t*>(tail_v);
    p.piT_v = reinterpret_cast<const float*>(static_cast<const uint8_t*>(vcodec->prep) + tq_prep_layout(tv).piT);
    p.out = out;
    p.part = reinterpret_cast<float*>(wsb + W.part);
    p.part_ml = reinterpret_cast<float*>(wsb + W.ml);
    p.status = static_cast<uint32_t*>(ws);
    p.n_streams = n_streams; p.n_tok = n_tok; p.nb = (n_tok + 31) / 32;
    p.g = g; p.nsplit = p.nb > 0 ? W.nsplit : 0; p.blocks_per_split = W.bps; p.n_tail = n_tail;
    p.v_skip = v_skip;
    p.tv = tv;
    p.scale = scale;
    p.d = vcodec->d;
    if ((st = codebook_consts(vcodec, &p.cbv)) != TQ_OK) return st;
    return cuda_status(tq_launch_attention_q8(p, static_cast<cudaStream_t>(stream)));
}

int tq_topk_est(const tq_codec* c, const void* packed_db, int64_t n_db, const float* q, int64_t n_q, int k,
                int64_t* idx, float* score, void* ws, size_t ws_bytes, int estimator, void* stream) {
    int st = check_codec(c, true);
    if (st != TQ_OK) return st;
    if (estimator != TQ_EST_QJL && estimator != TQ_EST_MSE) return TQ_ERR_ARG;
    if (!c->qjl) return TQ_ERR_ARG;
    if (n_q < 0 || n_db < 1 || n_db > 0x7fffffffLL || k < 1 || k > 32 || k > n_db) return TQ_ERR_ARG;
    if (n_q == 0) return TQ_OK;
    if (!packed_db || !q || !idx || !score || !ws) return TQ_ERR_ARG;
    if (!aligned(packed_db, 16) || !aligned(q, 4) || !aligned(idx, 8) || !aligned(score, 4) || !aligned(ws, 256))
        return TQ_ERR_ARG;
    const TqDims t = dims_of(c);
    const TopkWs W = topk_ws(t, n_q, n_db, k, estimator == TQ_EST_QJL);
    if (ws_bytes < W.total) return TQ_ERR_WORKSPACE;
    if ((int64_t)W.n_qt * W.nsplit > 0x7fffffffLL) return TQ_ERR_UNSUPPORTED;
    const TqPrepLayout L = tq_prep_layout(t);
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    TopkParams p;
    std::memset(&p, 0, sizeof(p));
    p.packed = static_cast<const uint8_t*>(packed_db);
    p.q = q;
    p.piT = reinterpret_cast<const float*>(static_cast<uint8_t*>(c->prep) + L.piT);
    p.sT = reinterpret_cast<const float*>(static_cast<uint8_t*>(c->prep) + L.sT);
    p.qimg = reinterpret_cast<uint16_t*>(wsb + W.qimg);
    p.qinv = reinterpret_cast<float*>(wsb + W.qinv);
    p.part_score = reinterpret_cast<float*>(wsb + W.psc);
    p.part_idx = reinterpret_cast<int*>(wsb + W.pix);
    p.out_idx = idx;
    p.out_score = score;
    p.status = static_cast<uint32_t*>(ws);
    p.n_db = n_db; p.nb = (n_db + 31) / 32; p.n_q = n_q; p.n_tiles = W.n_tiles;
    p.k = k; p.nsplit = W.nsplit; p.tiles_per_split = (int)W.tps; p.n_qt = W.n_qt;
    p.kb_mse = W.kb_mse; p.kb_sign = W.kb_sign; p.kq = W.kq;
    p.d = c->d; p.m = c->m;
    p.kappa = estimator == TQ_EST_MSE ? 0.f : (float)(std::sqrt(M_PI / 2.0) / c->m);
    p.t = t;
    if ((st = codebook_consts(c, &p.cb)) != TQ_OK) return st;
    return cuda_status(tq_launch_topk(p, static_cast<cudaStream_t>(stream)));
}

int tq_topk(const tq_codec* c, const void* packed_db, int64_t n_db, const float* q, int64_t n_q, int k, int64_t* idx,
            float* score, void* ws, size_t ws_bytes, void* stream) {
    return tq_topk_est(c, packed_db, n_db, q, n_q, k, idx, score, ws, ws_bytes, TQ_EST_QJL, stream);
}

size_t tq_q8_packed_bytes(int d, int64_t n_streams, int64_t n_tok) {
    if (d < 8 || d > 128 || d % 8 || n_streams < 0 || n_tok < 0) return 0;
    return (size_t)n_streams * (size_t)((n_tok + 31) / 32) * kQ8Block;
}

int tq_q8_quantize(const void* x, tq_dtype dtype, int d, int64_t n_streams, int64_t n_tok, int64_t x_stream_stride,
                   void* packed, void* ws, size_t ws_bytes, void* stream) {
    if (d < 8 || d > 128 || d % 8) return TQ_ERR_UNSUPPORTED;
    if (dtype != TQ_F32 && dtype != TQ_BF16) return TQ_ERR_ARG;
    if (n_streams < 0 || n_tok < 0) return TQ_ERR_ARG;
    if (n_streams == 0 || n_tok == 0) return TQ_OK;
    if (!x || !packed || !ws || !aligned(packed, 16) || !aligned(x, dtype == TQ_F32 ? 4 : 2) || !aligned(ws, 4))
        return TQ_ERR_ARG;
    if (n_streams > 1 && x_stream_stride < n_tok * d) return TQ_ERR_ARG;
    if (ws_bytes < TQ_STATUS_BYTES) return TQ_ERR_WORKSPACE;
    Q8QuantParams p;
    p.x = x; p.dtype = dtype; p.packed = static_cast<uint8_t*>(packed); p.status = static_cast<uint32_t*>(ws);
    p.n_streams = n_streams; p.n_tok = n_tok; p.nb = (n_tok + 31) / 32; p.x_stride = x_stream_stride; p.d = d;
    return cuda_status(tq_launch_q8_quantize(p, static_cast<cudaStream_t>(stream)));
}

int tq_q8_logits(const void* packed, int d, int64_t n_seq, int n_kv, int64_t n_tok, const void* q, tq_dtype q_dtype,
                 int g, const void* tail, int n_tail, float scale, float* out, void* stream) {
    if (d < 8 || d > 128 || d % 8) return TQ_ERR_UNSUPPORTED;
    if (g != 1 && g != 2 && g != 4) return TQ_ERR_UNSUPPORTED;
    if (n_seq < 0 || n_kv < 1 || n_tok < 0 || n_tail < 0) return TQ_ERR_ARG;
    if (q_dtype != TQ_F32 && q_dtype != TQ_BF16) return TQ_ERR_ARG;
    if (n_seq == 0 || n_tok + n_tail == 0) return TQ_OK;
    if (n_tail > TQ_Q8_MAX_TAIL) return TQ_ERR_UNSUPPORTED;
    if (!q || !out || (n_tok > 0 && !packed) || (n_tail > 0 && !tail)) return TQ_ERR_ARG;
    if ((n_tok > 0 && !aligned(packed, 16)) || !aligned(out, 4) || !aligned(q, q_dtype == TQ_F32 ? 4 : 2) ||
        (n_tail > 0 && !aligned(tail, 2)))
        return TQ_ERR_ARG;
    if (!std::isfinite(scale)) return TQ_ERR_ARG;
    const int64_t n_streams = n_seq * n_kv;
    const int64_t nb = (n_tok + 31) / 32;
    // one CTA per (stream, range), about four CTAs per SM; ranges of at least 8 blocks
    int64_t bps = (nb * n_streams + 4 * tq_device_sms() - 1) / (4 * tq_device_sms());
    bps = std::max<int64_t>(8, bps);
    bps = std::max<int64_t>(1, std::min<int64_t>(bps, nb));
    const int64_t nsplit = nb > 0 ? (nb + bps - 1) / bps : 1;
    if (n_streams * nsplit > 0x7fffffffLL) return TQ_ERR_UNSUPPORTED;
    Q8LogitsParams p;
    p.packed = static_cast<const uint8_t*>(packed);
    p.q = q; p.q_dtype = q_dtype; p.tail = static_cast<const uint16_t*>(tail); p.out = out;
    p.n_streams = n_streams; p.n_tok = n_tok; p.nb = nb;
    p.g = g; p.n_tail = n_tail; p.d = d; p.nsplit = (int)nsplit; p.bps = (int)bps; p.scale = scale;
    return cuda_status(tq_launch_q8_logits(p, static_cast<cudaStream_t>(stream)));
}

int tq_dequantize(const tq_codec* c, const void* packed, int64_t n_streams, int64_t n_tok, float* out, void* ws,
                  size_t ws_bytes, void* stream) {
    int st = check_codec(c, false);
    if (st != TQ_OK) return st;
    if (n_streams < 0 || n_tok < 0) return TQ_ERR_ARG;
    if (n_streams == 0 || n_tok == 0) return TQ_OK;
    if (!packed || !out || !aligned(packed, 16) || !aligned(out, 4)) return TQ_ERR_ARG;
    (void)ws; (void)ws_bytes;
    DequantParams p;
    p.packed = static_cast<const uint8_t*>(packed);
    p.out = out; p.pi = c->pi; p.s = c->s;
    p.n_streams = n_streams; p.n_tok = n_tok; p.nb = (n_tok + 31) / 32;
    p.kappa = c->qjl ? (float)(std::sqrt(M_PI / 2.0) / c->m) : 0.f;
    p.t = dims_of(c);
    if ((st = codebook_consts(c, &p.cb)) != TQ_OK) return st;
    return cuda_status(tq_launch_dequant(p, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
