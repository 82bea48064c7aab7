// 8-bit keys for the asymmetric K/V configuration (blog.hotdry.top "TurboQuant vector-search
// compression", engineering configuration list: keys at 8 bits (q8_0) with values under
// TurboQuant at 3 bits often beat 3 bits for both, since key norms run 4-182 times the value
// norms).
//
// Format, per block of 32 tokens (d <= 128; coordinates >= d are zero):
//   codes  [column j = 0..7][token 0..31][16 bytes]: the int8 codes of coordinates
//          16j .. 16j + 15, so that lane t of a warp reads token t's column with one 16-byte
//          load and a warp reads 512 contiguous bytes;
//   scales [chunk c = 0..3][token 0..31]: the binary16 scale of coordinates 32c .. 32c + 31.
// A chunk's scale is s = max|x| / 127 (fp32), its codes rint(x / s) (fp32 division, clamped to
// +-127), the stored scale s rounded to binary16; the key reads back as code * scale.
//
// Logits: one CTA per (stream, block range). Four warps turn the stream's query heads into
// int16 fixed point (step max|q| / 16383) split into int8 hi and lo bytes in shared memory;
// then lane t of every warp scores token t of its blocks with dp4a over each 32-coordinate
// chunk (exact int32), scaled per chunk. Tail CTAs (blockIdx.y > 0) give the exact logits of
// the bf16 tail, one token per warp.
#include <cfloat>

#include "tq_device.cuh"

namespace {

constexpr int kQ8Warps = 8;
constexpr int kQ8TailTok = kQ8Warps;   // tail tokens per tail CTA

__device__ __forceinline__ uint32_t pack4_s8(int a, int b, int c, int d) {
    return (uint32_t)(a & 0xff) | ((uint32_t)(b & 0xff) << 8) | ((uint32_t)(c & 0xff) << 16) |
           ((uint32_t)(d & 0xff) << 24);
}

// one warp per token row, the padding rows of a stream's last block included (written as
// zeros); lane L holds coordinates 4L .. 4L + 3, the 8 lanes of chunk L / 8 share its scale
__global__ void __launch_bounds__(kQ8Warps * 32) k_q8_quantize(Q8QuantParams p) {
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * kQ8Warps + (threadIdx.x >> 5);
    const int64_t per_stream = p.nb * 32;
    if (row >= p.n_streams * per_stream) return;
    const int64_t s = row / per_stream, tok = row - s * per_stream;
    const int64_t blk = tok >> 5;
    const int r = (int)(tok & 31);
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (tok < p.n_tok) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int j = 4 * lane + k;
            if (j < p.d) v[k] = tq_load_elem(p.x, p.dtype, s * p.x_stride + tok * p.d + j);
        }
    }
    const bool finite = isfinite(v[0]) && isfinite(v[1]) && isfinite(v[2]) && isfinite(v[3]);
    const bool nonfinite = __any_sync(0xffffffffu, !finite);
    float am = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 4));
    const float sc = am / 127.f;
    int qv[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
        qv[k] = am > 0.f && finite ? (int)fminf(fmaxf(rintf(v[k] / sc), -127.f), 127.f) : 0;
    uint8_t* b = p.packed + ((size_t)s * p.nb + blk) * kQ8Block;
    *reinterpret_cast<uint32_t*>(b + (lane >> 2) * 512 + r * 16 + (lane & 3) * 4) = pack4_s8(qv[0], qv[1], qv[2], qv[3]);
    const uint32_t hb = tq_half_bits(sc);
    if ((lane & 7) == 0) *reinterpret_cast<uint16_t*>(b + 4096 + ((lane >> 3) * 32 + r) * 2) = (uint16_t)hb;
    const bool over = __any_sync(0xffffffffu, (hb & 0x7fffu) >= 0x7c00u);
    if (lane == 0 && (nonfinite || over)) tq_raise(p.status, TQ_FLAG_RANGE);
}

__global__ void __launch_bounds__(kQ8Warps * 32) k_q8_logits(Q8LogitsParams p) {
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.g, d = p.d;
    const int64_t stream = blockIdx.x / p.nsplit;
    const int split = blockIdx.x % p.nsplit;
    const int64_t row = p.n_tok + p.n_tail;
    if (blockIdx.y > 0) {   // exact logits of the bf16 tail: one token per warp, range 0 only
        const int tt = (blockIdx.y - 1) * kQ8TailTok + w;
        if (split != 0 || tt >= p.n_tail) return;
        const uint16_t* kp = p.tail + ((size_t)stream * p.n_tail + tt) * d;
        float kv[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int j = 4 * lane + k;
            kv[k] = j < d ? __uint_as_float((uint32_t)kp[j] << 16) : 0.f;
        }
        for (int h = 0; h < G; ++h) {
            float a = 0.f;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int j = 4 * lane + k;
                if (j < d) a = fmaf(kv[k], tq_load_elem(p.q, p.q_dtype, (stream * G + h) * d + j), a);
            }
            a = tq_warp_sum(a);
            if (lane == 0) p.out[(stream * G + h) * row + p.n_tok + tt] = p.scale * a;
        }
        return;
    }
    // query heads of this stream as int16 fixed point, hi / lo int8 bytes per 16-coordinate column
    __shared__ uint4 s_q[4][2][8];
    __shared__ float s_qs[4];
    if (w < 4) {
        float v[4] = {0.f, 0.f, 0.f, 0.f};
        if (w < G) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int j = 4 * lane + k;
                if (j < d) v[k] = tq_load_elem(p.q, p.q_dtype, (stream * G + w) * d + j);
            }
        }
        const float am = tq_warp_max(fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3]))));
        const float step = am > 0.f && am <= FLT_MAX ? am / 16383.f : 1.f;
        int hi[4], lo[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int qi = (int)fminf(fmaxf(rintf(v[k] / step), -16383.f), 16383.f);
            hi[k] = (qi + 128) >> 8;
            lo[k] = qi - 256 * hi[k];
        }
        reinterpret_cast<uint32_t*>(&s_q[w][0][lane >> 2])[lane & 3] = pack4_s8(hi[0], hi[1], hi[2], hi[3]);
        reinterpret_cast<uint32_t*>(&s_q[w][1][lane >> 2])[lane & 3] = pack4_s8(lo[0], lo[1], lo[2], lo[3]);
        if (lane == 0) s_qs[w] = p.scale * step;
    }
    __syncthreads();
    const int64_t b0 = (int64_t)split * p.bps, b1 = min(b0 + (int64_t)p.bps, p.nb);
    const uint8_t* base = p.packed + (size_t)stream * p.nb * kQ8Block;
    for (int64_t b = b0 + w; b < b1; b += kQ8Warps) {
        const uint8_t* bp = base + (size_t)b * kQ8Block;
        uint4 kc[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) kc[j] = tq_ldg_stream(bp + j * 512 + lane * 16);
        float sc[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) sc[c] = tq_half_val(reinterpret_cast<const uint16_t*>(bp + 4096)[c * 32 + lane]);
        float res[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            int ah[4] = {0, 0, 0, 0}, al[4] = {0, 0, 0, 0};
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const int j = 2 * c + jj;
                const int kw[4] = {(int)kc[j].x, (int)kc[j].y, (int)kc[j].z, (int)kc[j].w};
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const uint4 qh = s_q[h][0][j], ql = s_q[h][1][j];
                    ah[h] = __dp4a(kw[0], (int)qh.x, ah[h]);
                    ah[h] = __dp4a(kw[1], (int)qh.y, ah[h]);
                    ah[h] = __dp4a(kw[2], (int)qh.z, ah[h]);
                    ah[h] = __dp4a(kw[3], (int)qh.w, ah[h]);
                    al[h] = __dp4a(kw[0], (int)ql.x, al[h]);
                    al[h] = __dp4a(kw[1], (int)ql.y, al[h]);
                    al[h] = __dp4a(kw[2], (int)ql.z, al[h]);
                    al[h] = __dp4a(kw[3], (int)ql.w, al[h]);
                }
            }
            // exact in int32: |256 ah + al| <= 32 (127 * 64 * 256 + 127 * 128) < 2^27
#pragma unroll
            for (int h = 0; h < 4; ++h) res[h] = fmaf(sc[c], (float)(256 * ah[h] + al[h]), res[h]);
        }
        const int64_t tok = b * 32 + lane;
        if (tok < p.n_tok)
            for (int h = 0; h < G; ++h) p.out[(stream * G + h) * row + tok] = s_qs[h] * res[h];
    }
}

}  // namespace

cudaError_t tq_launch_q8_quantize(const Q8QuantParams& p, cudaStream_t st) {
    const int64_t rows = p.n_streams * p.nb * 32;
    const int64_t grid = (rows + kQ8Warps - 1) / kQ8Warps;
    if (grid == 0) return cudaSuccess;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidValue;
    k_q8_quantize<<<(unsigned)grid, kQ8Warps * 32, 0, st>>>(p);
    return cudaGetLastError();
}

cudaError_t tq_launch_q8_logits(const Q8LogitsParams& p, cudaStream_t st) {
    if (p.d > 128 || p.g < 1 || p.g > 4 || p.nsplit < 1) return cudaErrorInvalidValue;
    const int64_t gx = p.n_streams * p.nsplit;
    const int64_t gy = 1 + ((int64_t)p.n_tail + kQ8TailTok - 1) / kQ8TailTok;
    if (gx == 0) return cudaSuccess;
    if (gx > 0x7fffffffLL || gy > 65535) return cudaErrorInvalidValue;
    k_q8_logits<<<dim3((unsigned)gx, (unsigned)gy), kQ8Warps * 32, 0, st>>>(p);
    return cudaGetLastError();
}
