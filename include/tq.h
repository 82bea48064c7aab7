/*
 * tq.h -- C ABI of the TurboQuant KV-vector hot path on NVIDIA B200 (sm_100a).
 *
 * TurboQuant compresses a KV vector x in two stages:
 *   1. rotate it by a random orthogonal Pi and quantize every coordinate of the rotated
 *      unit vector with a Lloyd-Max codebook built offline for the Beta((d-1)/2,(d-1)/2)
 *      coordinate law (blog.hotdry.top "TurboQuant vector-search compression", section
 *      "Random rotation and scalar quantization"; a2a-mcp.org "What is TurboQuant",
 *      stage 1);
 *   2. for keys, store sign(S r) of the residual r = u - x_mse with a Gaussian S, and
 *      gamma = |r| (blog.hotdry.top, section "QJL residual correction").
 * Scores are evaluated on the packed codes with the query rotated once (a2a-mcp.org,
 * stage 2 and "fused Triton kernel"):
 *   <q, x~> = |x| ( <Pi q, c[idx]> + gamma sqrt(pi/2)/m <S q, sign> ).
 * Values use the MSE stage only (friday-blog-bgf.pages.dev "TurboQuant deep dive II",
 * section 1, step 1) and are accumulated as softmax(P) . V.
 *
 * Conventions for every call:
 *   - Device pointers are CUDA global memory of the current device; host pointers are
 *     marked HOST. The library never allocates or frees memory and keeps no global state.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream). All
 *     device work is stream-ordered; calls return once it is enqueued.
 *   - Arguments are checked before any launch; a failed check returns a negative
 *     tq_status and enqueues nothing. Faults that depend on the data (a norm that
 *     overflows binary16, a non-finite input) are recorded in a status word at the start
 *     of the caller's workspace and read back with tq_get_status.
 *   - Readings of the pages adopted here: the QJL factor is sqrt(pi/2)/m (the pages print
 *     /d; every shipped workload has m = d); gamma is the residual norm of the unit
 *     vector u = x/|x|; a coordinate on a decision boundary takes the lower cell; a zero
 *     sketch value gives sign +1; |x| and gamma are stored as IEEE binary16.
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    TQ_OK = 0,
    TQ_ERR_ARG = -1,          /* bad pointer, size or alignment */
    TQ_ERR_UNSUPPORTED = -2,  /* valid request outside the supported shapes */
    TQ_ERR_CUDA = -3,         /* a CUDA runtime call failed */
    TQ_ERR_RANGE = -4,        /* (status word) a norm overflowed binary16 or an input was not finite */
    TQ_ERR_TIMEOUT = -5,      /* (status word) a bounded wait of a kernel ran out */
    TQ_ERR_NOCONV = -6,       /* codebook iteration did not converge */
    TQ_ERR_WORKSPACE = -7     /* workspace or prepared buffer too small / not prepared */
} tq_status;

typedef enum { TQ_F32 = 0, TQ_BF16 = 1 } tq_dtype;

/* A codec: one rotation, one sketch, one codebook.
 *   d         vector dimension, 8..256, multiple of 8.
 *   m         QJL rows, 8..256, multiple of 8 (ignored when qjl = 0).
 *   mse_bits  B, bits of the Lloyd-Max index per coordinate: 1..3 for keys, 1..4 for values.
 *             A key therefore costs b = B + 1 bits per coordinate (blog.hotdry.top, "QJL
 *             residual correction": (b-1) + 1 = b).
 *   qjl       1: key records (MSE stage + QJL signs + gamma); 0: value records (MSE only).
 *   pi        device fp32 [d, d] row-major, orthogonal; y = Pi u.
 *   s         device fp32 [m, d] row-major, i.i.d. N(0,1); NULL when qjl = 0.
 *   centroids HOST fp64 [2^B], sorted and symmetric, from tq_make_codebook (read by every call).
 *   prep      device buffer of tq_prep_bytes(codec) bytes, filled by tq_prepare and
 *             owned by the caller; it must outlive every call that uses the codec.
 * Pi, s and prep must stay unchanged while calls using the codec are in flight.           */
typedef struct {
    int d;
    int m;
    int mse_bits;
    int qjl;
    const float* pi;
    const float* s;
    const double* centroids;
    void* prep;
    size_t prep_bytes;
} tq_codec;

/* Score estimators for packed keys (tq_logits_est, tq_topk_est):
 *   TQ_EST_QJL  |x| (<Pi q, c[idx]> + gamma sqrt(pi/2)/m <S q, s>), unbiased (the default);
 *   TQ_EST_MSE  |x| <Pi q, c[idx]>, the MSE stage alone: the stored signs and gamma are not
 *               used (blog.hotdry.top, monitoring notes: in some settings the QJL correction
 *               lowers ranking quality and an MSE-only mode is preferred). The key records
 *               are the same; only the estimate changes.                                    */
enum { TQ_EST_QJL = 0, TQ_EST_MSE = 1 };

/* Test hook, OR-ed into the estimator of tq_logits_est: every warp of the logits stream
 * kernel first waits on a barrier that nothing arrives at, with a limit of a few thousand
 * polls. The wait runs out as a lost copy would: the kernel records TQ_ERR_TIMEOUT in the
 * status word, waits (bounded) for the copies it has in flight and returns without writing
 * logits, leaving the context usable. It exists to test that path; it is not for use.     */
#define TQ_TEST_STALL 0x100

/* Operations, for tq_workspace_bytes */
enum { TQ_OP_QUANTIZE = 0, TQ_OP_LOGITS = 1, TQ_OP_PV = 2, TQ_OP_TOPK = 3, TQ_OP_DEQUANTIZE = 4 };

/* Lloyd-Max codebook for one coordinate of a rotated unit vector in R^d
 * (blog.hotdry.top, "Random rotation and scalar quantization"; a2a-mcp.org, stage 1: the
 * Beta((d-1)/2,(d-1)/2) law on [-1,1]). HOST only, fp64.
 *   d in 3..4096, mse_bits in 1..8; centroids: 2^B values, bounds: 2^B - 1 midpoints,
 *   mse: d * E(u_i - q(u_i))^2, the normalised distortion (may be NULL).
 * The fixed point is found by Lloyd iteration to |dc| < 1e-15 and symmetrised, so the
 * middle bound is exactly 0. Returns TQ_ERR_NOCONV if 100000 iterations do not converge. */
int tq_make_codebook(int d, int mse_bits, double* centroids, double* bounds, double* mse);

/* Storage. Records are grouped in blocks of 32 vectors; a stream of n_tok vectors takes
 * ceil(n_tok/32) blocks, the unused records of its last block are zero.
 * tq_record_bytes: bytes per vector (block bytes / 32).                                    */
size_t tq_block_bytes(const tq_codec* codec);
size_t tq_record_bytes(const tq_codec* codec);
size_t tq_packed_bytes(const tq_codec* codec, int64_t n_streams, int64_t n_tok);

/* Derived operands (split-precision copies of Pi and of M = S Pi^T, transposes) computed
 * once per codec into codec->prep. Returns TQ_ERR_WORKSPACE if prep_bytes is too small.   */
size_t tq_prep_bytes(const tq_codec* codec);
int tq_prepare(const tq_codec* codec, void* stream);

/* Workspace for one call. Its first 256 bytes hold the status word; the rest holds
 * per-call scratch (pre-rotated queries, split partials). Sizes:
 *   QUANTIZE / DEQUANTIZE: a, b, c unused;  LOGITS: a = n_seq, b = n_kv, c = g;
 *   PV: a = n_seq * n_kv * g heads, b = n_tok;  TOPK: a = n_q, b = n_db, c = k.          */
size_t tq_workspace_bytes(const tq_codec* codec, int op, int64_t a, int64_t b, int64_t c);

/* Quantize n_streams x n_tok vectors (tq_quantize: rotate, nearest centroid, residual,
 * QJL signs, pack; blog.hotdry.top "Random rotation and scalar quantization" and "QJL
 * residual correction").
 *   x        device, dtype fp32 or bf16; vector t of stream s starts at element
 *            s * x_stream_stride + t * d (vectors are contiguous within a stream).
 *   packed   device, tq_packed_bytes(codec, n_streams, n_tok) bytes; stream s occupies
 *            blocks [s * ceil(n_tok/32), (s+1) * ceil(n_tok/32)). 16-byte aligned.
 *   ws       device workspace of tq_workspace_bytes(codec, TQ_OP_QUANTIZE, 0, 0, 0) bytes.
 * A vector whose norm rounds above 65504 or that holds a non-finite value sets
 * TQ_ERR_RANGE in the status word (its record is still written).                       */
int tq_quantize(const tq_codec* codec, const void* x, tq_dtype dtype, int64_t n_streams,
                int64_t n_tok, int64_t x_stream_stride, void* packed, void* ws, size_t ws_bytes,
                void* stream);

/* Attention logits straight from packed keys (a2a-mcp.org, stage 2 / "fused Triton kernel":
 * the query is rotated once, the indices are never dequantized to a full vector).
 *   packed   device key cache (qjl = 1): n_seq * n_kv streams of n_tok vectors, stream
 *            (s, h) at index s * n_kv + h.
 *   q        device [n_seq, n_kv * g, d], fp32 or bf16; query head j reads kv-head j / g.
 *   g        query heads per kv-head, 1, 2, 4 or 8.
 *   tail     device bf16 [n_seq, n_kv, n_tail, d] full-precision recent keys (blog.hotdry.top,
 *            "engineering configuration list": the most recent 128-256 tokens stay at full
 *            precision), or NULL with n_tail = 0. n_tail <= 1048544, else
 *            TQ_ERR_UNSUPPORTED.
 *   out      device fp32 [n_seq, n_kv * g, n_tok + n_tail]: the n_tok compressed-key logits
 *            scale * |x|(<Pi q, c[idx]> + gamma sqrt(pi/2)/m <S q, s>) followed by the n_tail
 *            exact logits scale * <q, k>.
 *   ws       tq_workspace_bytes(codec, TQ_OP_LOGITS, n_seq, n_kv, g) bytes.                */
int tq_logits(const tq_codec* codec, const void* packed, int64_t n_seq, int n_kv, int64_t n_tok,
              const void* q, tq_dtype q_dtype, int g, const void* tail, int n_tail, float scale,
              float* out, void* ws, size_t ws_bytes, void* stream);
/* tq_logits with the estimator chosen (TQ_EST_QJL or TQ_EST_MSE; else TQ_ERR_ARG); the same
 * workspace and layouts. tq_logits is tq_logits_est with TQ_EST_QJL.                      */
int tq_logits_est(const tq_codec* codec, const void* packed, int64_t n_seq, int n_kv, int64_t n_tok,
                  const void* q, tq_dtype q_dtype, int g, const void* tail, int n_tail, float scale,
                  float* out, void* ws, size_t ws_bytes, int estimator, void* stream);

/* softmax(P) . V over MSE-only packed values (friday-blog-bgf.pages.dev, section 1, step 1;
 * accumulated in the rotated domain and rotated back once by Pi^T).
 *   packed_v device value cache (qjl = 0): n_seq * n_kv streams of n_tok vectors.
 *   P        device fp32 [n_seq, n_kv * g, n_tok] attention logits (before softmax).
 *   out      device fp32 [n_seq, n_kv * g, d].
 *   ws       tq_workspace_bytes(codec, TQ_OP_PV, n_seq * n_kv, n_tok, g) bytes.             */
int tq_pv(const tq_codec* codec, const void* packed_v, int64_t n_seq, int n_kv, int64_t n_tok,
          const float* P, int g, float* out, void* ws, size_t ws_bytes, void* stream);

/* Decode attention in one pass over compressed keys and values:
 *   out_h = sum_t softmax_t(l_h) v_t,  l_h,t = scale <q_h, k_t>
 * with the logits of tq_logits (estimator on the packed keys, exact on the bf16 tail) and
 * the values of tq_pv (MSE codes, rotated back once), the logits never written to memory
 * (a2a-mcp.org "What is TurboQuant": scores computed straight from the indices in a fused
 * kernel; blog.hotdry.top, "engineering configuration list": recent tokens at full precision).
 *   kcodec   key codec, qjl = 1, d <= 128 and m <= 128.
 *   vcodec   value codec, qjl = 0, the same d; both prepared.
 *   packed_k device key cache of n_seq * n_kv streams of n_tok tokens (tq_quantize layout).
 *   packed_v device value cache, the same streams and tokens.
 *   q        device [n_seq, n_kv * g, d], fp32 or bf16; query head j reads kv-head j / g.
 *   g        query heads per kv-head, 1, 2 or 4 (else TQ_ERR_UNSUPPORTED).
 *   tail_k, tail_v  device bf16 [n_seq, n_kv, n_tail, d] recent keys and values, the
 *            tokens that follow the compressed ones (tail_v 8-byte aligned); NULL with
 *            n_tail = 0.
 *            n_tail <= TQ_ATTN_MAX_TAIL, else TQ_ERR_UNSUPPORTED.
 *   v_skip   sparse values (ai-coding.wiselychen.com "Google TurboQuant KV-cache compression",
 *            community extensions: "Sparse V" skips the dequantization of low-weight values),
 *            in [0, 1]: a 32-token block of compressed values is skipped when every softmax
 *            weight in it, relative to the largest weight seen so far, is below v_skip; the
 *            softmax denominator still counts them. 0 = dense. A skipped token's final
 *            relative weight is below v_skip too, so the result differs from the dense one by
 *            at most the weight mass of the tokens whose relative weight is below v_skip.
 *   out      device fp32 [n_seq, n_kv * g, d].
 *   ws       tq_attention_workspace_bytes(kcodec, vcodec, n_seq, n_kv, n_tok, g, n_tail) bytes,
 *            256-byte aligned. n_tok + n_tail = 0 is TQ_ERR_ARG (a softmax over no tokens). */
#define TQ_ATTN_MAX_TAIL 8192
size_t tq_attention_workspace_bytes(const tq_codec* kcodec, const tq_codec* vcodec, int64_t n_seq, int n_kv,
                                    int64_t n_tok, int g, int n_tail);
int tq_attention(const tq_codec* kcodec, const tq_codec* vcodec, const void* packed_k, const void* packed_v,
                 int64_t n_seq, int n_kv, int64_t n_tok, const void* q, tq_dtype q_dtype, int g,
                 const void* tail_k, const void* tail_v, int n_tail, float scale, float v_skip, float* out,
                 void* ws, size_t ws_bytes, void* stream);

/* Decode attention of the asymmetric K/V configuration (blog.hotdry.top "TurboQuant
 * vector-search compression", engineering configuration list: 8-bit keys with TurboQuant
 * values) in one pass over the 8-bit key cache and the compressed values:
 *   out_h = sum_t softmax_t(l_h) v_t,  l_h,t = scale <q_h, k~_t> (k~ = code * scale of its chunk)
 * with the logits of tq_q8_logits (int16 fixed-point query) on the 8-bit tokens and exact on the
 * bf16 tail, and the values of tq_pv; the logits never leave the SM.
 *   vcodec   value codec, qjl = 0, d <= 128 (the keys have the same d), prepared.
 *   packed_k8 device 8-bit key cache of n_seq * n_kv streams of n_tok tokens (tq_q8_quantize).
 *   packed_v device value cache, the same streams and tokens.
 *   q, g, tail_k, tail_v, n_tail, scale, v_skip, out: as tq_attention (g in 1, 2, 4).
 *   ws       tq_attention_q8_workspace_bytes(vcodec, n_seq, n_kv, n_tok, g, n_tail) bytes,
 *            256-byte aligned. n_tok + n_tail = 0 is TQ_ERR_ARG.                          */
size_t tq_attention_q8_workspace_bytes(const tq_codec* vcodec, int64_t n_seq, int n_kv, int64_t n_tok, int g,
                                       int n_tail);
int tq_attention_q8(const tq_codec* vcodec, const void* packed_k8, const void* packed_v, int64_t n_seq, int n_kv,
                    int64_t n_tok, const void* q, tq_dtype q_dtype, int g, const void* tail_k, const void* tail_v,
                    int n_tail, float scale, float v_skip, float* out, void* ws, size_t ws_bytes, void* stream);

/* Top-k inner-product search over a packed database (a2a-mcp.org, benchmark section:
 * GloVe d=200 recall; scores are the same estimator as tq_logits with scale 1).
 *   packed_db device, one stream of n_db key records (qjl = 1).
 *   q        device fp32 [n_q, d].
 *   idx      device int64 [n_q, k], score: device fp32 [n_q, k], best first; equal scores
 *            keep the lower index first. 1 <= k <= 32.
 *   ws       tq_workspace_bytes(codec, TQ_OP_TOPK, n_q, n_db, k) bytes.                   */
int tq_topk(const tq_codec* codec, const void* packed_db, int64_t n_db, const float* q,
            int64_t n_q, int k, int64_t* idx, float* score, void* ws, size_t ws_bytes, void* stream);
/* tq_topk with the estimator chosen (TQ_EST_QJL or TQ_EST_MSE; else TQ_ERR_ARG); tq_topk is
 * tq_topk_est with TQ_EST_QJL.                                                               */
int tq_topk_est(const tq_codec* codec, const void* packed_db, int64_t n_db, const float* q,
                int64_t n_q, int k, int64_t* idx, float* score, void* ws, size_t ws_bytes,
                int estimator, void* stream);

/* tq_logits without a caller workspace, for callers that cannot allocate device memory:
 * code inside a host framework whose pool owns all device memory, plugins that may only use
 * the buffers they are given, latency-critical loops under a no-allocation policy. The pages
 * have no counterpart: this is a deployment convenience, not part of the method.
 *   Arguments and results are those of tq_logits, minus ws / ws_bytes.
 *   Scratch: a fixed TQ_NOALLOC_SCRATCH_BYTES (4 MiB) array in device memory, held by every
 *   GPU that loads the library until the process exits. A request whose
 *   tq_workspace_bytes(codec, TQ_OP_LOGITS, n_seq, n_kv, g) exceeds it returns
 *   TQ_ERR_WORKSPACE and enqueues nothing.
 *   The array's device address belongs to the CUDA context that loaded the library's
 *   module. The first call in a context resolves it (cudaGetSymbolAddress, with that context
 *   current): the first call on a device, and the first after cudaDeviceReset or any other
 *   change of the device's current context. Make such a first call before any stream
 *   capture.
 *   Every call on a device shares the array: calls whose GPU work may overlap (other
 *   streams, other threads) race and must be serialised by the caller. Arguments are
 *   checked first; a rejected call enqueues nothing and leaves the array untouched. An
 *   accepted call clears the status word on the stream before its kernels; data-dependent
 *   faults are not reported by this variant.
 *   Nothing is allocated: no cudaMalloc, cudaFree or allocating library routine.        */
#define TQ_NOALLOC_SCRATCH_BYTES ((size_t)4 << 20)
int tq_logits_noalloc(const tq_codec* codec, const void* packed, int64_t n_seq, int n_kv, int64_t n_tok,
                      const void* q, tq_dtype q_dtype, int g, const void* tail, int n_tail, float scale,
                      float* out, void* stream);

/* 8-bit keys, the key side of the asymmetric K/V configuration (blog.hotdry.top "TurboQuant
 * vector-search compression", engineering configuration list: q8_0 keys with TurboQuant
 * values). No rotation or codebook: per 32-coordinate chunk of a key, scale
 * s = max|x| / 127 (fp32), codes rint(x / s) (fp32 division, round half to even, clamped to
 * +-127), stored scale = s rounded to binary16; the key reads back as code * scale.
 * Record: d <= 128 (multiple of 8) padded to 128 coordinates, 136 bytes per key, in blocks
 * of 32 tokens: codes [column j = 0..7][token][16 B] (coordinates 16j .. 16j+15), then
 * scales [chunk c = 0..3][token] binary16. Stream s occupies blocks
 * [s * ceil(n_tok/32), (s+1) * ceil(n_tok/32)); padding tokens are zero.
 *   tq_q8_packed_bytes: bytes of n_streams x n_tok keys, 0 if d is unsupported.
 *   tq_q8_quantize: x device fp32 or bf16, vector t of stream s at s * x_stream_stride + t * d;
 *            packed 16-byte aligned; ws: TQ_STATUS_BYTES (status word: TQ_ERR_RANGE when a
 *            value is not finite or a scale overflows binary16).
 *   tq_q8_logits: out fp32 [n_seq, n_kv * g, n_tok + n_tail] = scale <q, k~> for the packed
 *            keys followed by the exact scale <q, k> of the bf16 tail ([n_seq, n_kv, n_tail,
 *            d], n_tail <= TQ_Q8_MAX_TAIL); q device [n_seq, n_kv * g, d] fp32 or bf16;
 *            g in {1, 2, 4}. The query is rounded to int16 fixed point per head (step
 *            max|q| / 16383): the error is at most sqrt(d) / 32766 of scale |q| |k~|. No
 *            workspace.                                                                        */
#define TQ_Q8_MAX_TAIL 65536
size_t tq_q8_packed_bytes(int d, int64_t n_streams, int64_t n_tok);
int tq_q8_quantize(const void* x, tq_dtype dtype, int d, int64_t n_streams, int64_t n_tok,
                   int64_t x_stream_stride, void* packed, void* ws, size_t ws_bytes, void* stream);
int tq_q8_logits(const void* packed, int d, int64_t n_seq, int n_kv, int64_t n_tok, const void* q,
                 tq_dtype q_dtype, int g, const void* tail, int n_tail, float scale, float* out,
                 void* stream);

/* Diagnostic reconstruction (not on the hot path): x~ = |x|(Pi^T c[idx] + gamma
 * sqrt(pi/2)/m S^T s) for keys, |x| Pi^T c[idx] for values (blog.hotdry.top, "QJL residual
 * correction"). out: device fp32 [n_streams, n_tok, d].                                  */
int tq_dequantize(const tq_codec* codec, const void* packed, int64_t n_streams, int64_t n_tok,
                  float* out, void* ws, size_t ws_bytes, void* stream);

/* Status word. Data-dependent faults of every call that used `ws` accumulate in its first
 * word until read. tq_reset_status enqueues a clear (do it once on a new workspace);
 * tq_get_status synchronises `stream`, reads the word and clears it, returning TQ_OK,
 * TQ_ERR_TIMEOUT if a bounded wait of a kernel ran out (it takes precedence), TQ_ERR_RANGE,
 * or TQ_ERR_CUDA if the read itself failed.                                              */
int tq_reset_status(void* ws, void* stream);
int tq_get_status(void* ws, void* stream);

const char* tq_status_string(int status);
int tq_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* TQ_H */
