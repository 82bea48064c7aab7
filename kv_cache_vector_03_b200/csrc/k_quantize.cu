// tq_quantize: rotate, nearest Lloyd-Max centroid, residual, QJL sign sketch, pack.
// (blog.hotdry.top "TurboQuant vector-search compression", sections "Random rotation and
// scalar quantization" and "QJL residual correction"; a2a-mcp.org "What is TurboQuant",
// stage 1.)
//
// One CTA of 4 warps quantizes one block of 32 vectors in fp32:
//   u = x / |x|                     (|x| accumulated in fp64)
//   y = Pi u                        (lane l owns rotated coordinates l, l+32, ...)
//   idx_i = #{k : y_i > t_k},  r_i = y_i - c[idx_i]   (rotated-domain residual, |r| = gamma)
//   z = M r with M = S Pi^T         (= S (u - Pi^T c[idx]))
// and packs the bit planes with warp ballots (bit l of a ballot = coordinate 32k + l).
#include <algorithm>

#include "tq_device.cuh"

namespace {

template <int KD, int KM, int B>
__global__ void __launch_bounds__(128) k_quantize_f32(QuantParams p) {
    constexpr int D = KD * 32;
    extern __shared__ float smem[];
    float* us = smem;                                               // [32][D]: u, then r
    uint8_t* cs = reinterpret_cast<uint8_t*>(smem + 32 * D);         // [32][D] codes (values)
    __shared__ float s_norm[32], s_gamma[32];
    __shared__ int s_bad[32];

    const TqDims& T = p.t;
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    const int64_t s = blockIdx.x / p.nb, b = blockIdx.x % p.nb;
    uint8_t* blk = p.packed + (size_t)blockIdx.x * T.block_bytes;
    const int d = T.d;

    // ---- 1. load, norm, normalise
#pragma unroll 1
    for (int j = 0; j < 8; ++j) {
        const int v = w + 4 * j;
        const int64_t tok = b * 32 + v;
        const bool valid = tok < p.n_tok;
        const int64_t base = s * p.x_stride + tok * d;
        float xv[KD];
        double n2 = 0.0;
        int bad = 0;
#pragma unroll
        for (int k = 0; k < KD; ++k) {
            const int i = l + 32 * k;
            xv[k] = (valid && i < d) ? tq_load_elem(p.x, p.dtype, base + i) : 0.f;
            bad |= !isfinite(xv[k]);
            n2 += (double)xv[k] * (double)xv[k];
        }
        n2 = tq_warp_sum_d(n2);
        bad = __any_sync(0xffffffffu, bad);
        const float n = (float)sqrt(n2);
#pragma unroll
        for (int k = 0; k < KD; ++k) us[v * D + l + 32 * k] = n > 0.f ? xv[k] / n : 0.f;
        if (l == 0) { s_norm[v] = n; s_bad[v] = bad; }
    }
    __syncwarp();

    // ---- 2. y = Pi u for the warp's 8 vectors
    float acc[8][KD];
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int k = 0; k < KD; ++k) acc[j][k] = 0.f;
#pragma unroll 2
    for (int jj = 0; jj < d; ++jj) {
        float pv[KD];
#pragma unroll
        for (int k = 0; k < KD; ++k) pv[k] = __ldg(p.piT + (size_t)jj * D + l + 32 * k);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float uv = us[(w + 4 * j) * D + jj];
#pragma unroll
            for (int k = 0; k < KD; ++k) acc[j][k] = fmaf(pv[k], uv, acc[j][k]);
        }
    }
    __syncwarp();

    // ---- 3. nearest centroid, residual, code planes
    constexpr int L = 1 << B;
    const uint32_t sec_a = T.sec_a;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int v = w + 4 * j;
        const bool valid = b * 32 + v < p.n_tok;
        int code[KD];
        float g2 = 0.f;
#pragma unroll
        for (int k = 0; k < KD; ++k) {
            const int i = l + 32 * k;
            const float y = acc[j][k];
            int c = 0;
#pragma unroll
            for (int q = 0; q < L - 1; ++q) c += y > p.cb.bounds[q];
            float r = y - p.cb.cent[c];
            if (i >= d || !valid) { c = 0; r = 0.f; }
            code[k] = c;
            g2 = fmaf(r, r, g2);
            us[v * D + i] = r;
            cs[v * D + i] = (uint8_t)c;
        }
        g2 = tq_warp_sum(g2);
        if (l == 0) s_gamma[v] = sqrtf(g2);
        if (T.qjl) {
            const int gq = v & 7, u = v >> 3;
#pragma unroll
            for (int pl = 0; pl < B; ++pl) {
#pragma unroll
                for (int k = 0; k < KD; ++k) {
                    const uint32_t word = __ballot_sync(0xffffffffu, (code[k] >> pl) & 1);
                    if (l == k) {
                        const int pg = pl * T.GD + (k >> 2);
                        const int lane = 4 * gq + (k & 3);
                        reinterpret_cast<uint32_t*>(blk)[(pg * 32 + lane) * 4 + u] = word;
                    }
                }
            }
        }
    }
    __syncwarp();

    // ---- 4. QJL sketch z = M r and its sign plane
    if constexpr (KM > 0) {
        float z[8][KM];
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int k = 0; k < KM; ++k) z[j][k] = 0.f;
#pragma unroll 2
        for (int ii = 0; ii < d; ++ii) {
            float mv[KM];
#pragma unroll
            for (int k = 0; k < KM; ++k) mv[k] = __ldg(p.mT + (size_t)ii * T.Mp + l + 32 * k);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float rv = us[(w + 4 * j) * D + ii];
#pragma unroll
                for (int k = 0; k < KM; ++k) z[j][k] = fmaf(mv[k], rv, z[j][k]);
            }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int v = w + 4 * j;
            const bool valid = b * 32 + v < p.n_tok;
            const int gq = v & 7, u = v >> 3;
#pragma unroll
            for (int k = 0; k < KM; ++k) {
                const bool bit = valid && (l + 32 * k) < T.m && z[j][k] >= 0.f;
                const uint32_t word = __ballot_sync(0xffffffffu, bit);
                if (l == k) {
                    const int pg = T.B * T.GD + (k >> 2);
                    const int lane = 4 * gq + (k & 3);
                    reinterpret_cast<uint32_t*>(blk)[(pg * 32 + lane) * 4 + u] = word;
                }
            }
        }
    }
    __syncthreads();

    // ---- 5. norms, status, and the value layout
    if (threadIdx.x < 32) {
        const int v = threadIdx.x;
        const bool valid = b * 32 + v < p.n_tok;
        const uint32_t nh = valid ? tq_half_bits(s_norm[v]) : 0u;
        const uint32_t gh = valid ? tq_half_bits(s_gamma[v]) : 0u;
        if (valid && (s_bad[v] || (nh & 0x7fffu) >= 0x7c00u)) tq_raise(p.status, TQ_FLAG_RANGE);
        if (T.qjl) {
            const int gq = v & 7, u = v >> 3;
            reinterpret_cast<uint32_t*>(blk + sec_a)[gq * 4 + u] = nh | (gh << 16);
        } else {
            reinterpret_cast<uint16_t*>(blk + sec_a)[v] = (uint16_t)nh;
        }
    }
    if (!T.qjl) {
        // lane string of lane l = 4 gq + tq: fields (a, p) -> code(tau, i) | code(tau+1, i) << B
        const int fb = 2 * B;
        const int words = D * B / 32;
        for (int e = threadIdx.x; e < 32 * words; e += blockDim.x) {
            const int lane = e % 32, wd = e / 32;
            const int gq = lane >> 2, tq = lane & 3;
            uint32_t val = 0;
            const int f0 = (32 * wd) / fb, f1 = (32 * wd + 31) / fb;
            for (int f = f0; f <= f1; ++f) {
                const int a = f >> 2, pp = f & 3;
                const int i = 8 * a + gq;
                const int tau = 16 * (pp >> 1) + 8 * (pp & 1) + 2 * tq;
                const uint32_t F = (uint32_t)cs[tau * D + i] | ((uint32_t)cs[(tau + 1) * D + i] << B);
                const int pos = f * fb - 32 * wd;
                val |= pos >= 0 ? (F << pos) : (F >> (-pos));
            }
            reinterpret_cast<uint32_t*>(blk)[((wd >> 2) * 32 + lane) * 4 + (wd & 3)] = val;
        }
    }
}

// ---------------------------------------------------------------------------------------
// Tensor-core quantizer for d <= 128 (D = Mp = 128 or values): persistent CTAs of 8 warps,
// 128-vector tiles (four 32-vector blocks); warp w owns tile rows 16w..16w+15.
//   Y = (2^e x) (256 Pi)^T on mma.sync m16n8k16 fp16 -> fp32: x scaled by a power of two so
//       that max |2^e x| is in [2^14, 2^15), split hi/lo (bf16 inputs are exact in the hi
//       part: 2 passes; fp32 inputs: 3 passes); Pi as the prepared hi/lo pair.
//   y = Y / (|x| 2^(e+8)); codes, residual r = y - c[idx] and gamma per row.
//   Z = (2^12 r)(256 M)^T, 3 passes (hi.hi + hi.lo + lo.hi): only its sign is kept.
// Operands live in shared memory with 16-byte chunks XOR-swizzled by (row & 7), read with
// ldmatrix. Pi and M stay resident for the whole kernel.
namespace mma16 {

constexpr int kRowBytes = 256;                   // 128 fp16 per row
constexpr int kMatBytes = 128 * kRowBytes;        // 32 KB

__device__ __forceinline__ uint32_t swz(int row, int chunk) {
    return (uint32_t)(row * kRowBytes + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
    return (uint32_t)__half_as_ushort(__float2half_rn(lo)) | ((uint32_t)__half_as_ushort(__float2half_rn(hi)) << 16);
}

}  // namespace mma16

template <bool kF32, int B>
__global__ void __launch_bounds__(256, 1) k_quantize_mma(QuantParams p) {
    using namespace mma16;
    extern __shared__ __align__(1024) uint8_t qsm[];
    uint8_t* PH = qsm;
    uint8_t* PL = PH + kMatBytes;
    uint8_t* MH = PL + kMatBytes;
    uint8_t* ML = MH + kMatBytes;
    uint8_t* AH = ML + kMatBytes;
    uint8_t* AL = AH + kMatBytes;
    uint8_t* CS = AL + kMatBytes;                  // [128][128] codes (value layout only)
    __shared__ float s_norm[128], s_inv[128], s_gamma[128];
    __shared__ int s_bad[128], s_valid[128];

    const TqDims& T = p.t;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    constexpr int L = 1 << B;
    const int d = T.d;
    const int64_t total_blocks = p.n_streams * p.nb;
    const int64_t n_tiles = (total_blocks + 3) / 4;
    const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(qsm);

    // resident operands: Pi (and M) hi/lo, swizzled
    {
        const int nmat = T.qjl ? 4 : 2;
        const uint16_t* srcs[4] = {p.pih, p.pil, p.mh, p.ml};
        for (int e = tid; e < nmat * 128 * 16; e += blockDim.x) {
            const int m = e >> 11, row = (e >> 4) & 127, ch = e & 15;
            const uint4 v = *reinterpret_cast<const uint4*>(srcs[m] + row * 128 + ch * 8);
            *reinterpret_cast<uint4*>(qsm + m * kMatBytes + swz(row, ch)) = v;
        }
        __syncthreads();
    }

    for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
        const int r_base = 16 * warp;             // tile rows of this warp
        // ---- 1. load 16 rows (all loads issued first), then per row: norm, power-of-two
        //         scale, fp16 hi (lo) into the A tile. Lane l holds columns 4l..4l+3.
        float xr[16][4];
        bool vrow[16];
        // all 16 rows of a warp lie in one 32-vector block
        const int64_t wgb = tile * 4 + (r_base >> 5);
        const int64_t ws_ = wgb / p.nb, wtok0 = (wgb % p.nb) * 32 + (r_base & 31);
        const bool wblk = wgb < total_blocks;
        const int64_t wbase = ws_ * p.x_stride + wtok0 * d + 4 * lane;
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) {
            vrow[rr] = wblk && wtok0 + rr < p.n_tok;
            const int64_t base = wbase + (int64_t)rr * d;
            const bool in = vrow[rr] && 4 * lane < d;
            if (kF32) {
                if (p.vec_ok) {
                    const float4 v = in ? __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(p.x) + base))
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
                    xr[rr][0] = v.x; xr[rr][1] = v.y; xr[rr][2] = v.z; xr[rr][3] = v.w;
                } else {
#pragma unroll
                    for (int k = 0; k < 4; ++k) xr[rr][k] = in ? static_cast<const float*>(p.x)[base + k] : 0.f;
                }
            } else {
                uint2 v = make_uint2(0u, 0u);
                if (in) {
                    if (p.vec_ok) {
                        v = __ldg(reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(p.x) + base));
                    } else {
                        const uint16_t* xp = static_cast<const uint16_t*>(p.x) + base;
                        v = make_uint2((uint32_t)xp[0] | ((uint32_t)xp[1] << 16), (uint32_t)xp[2] | ((uint32_t)xp[3] << 16));
                    }
                }
                xr[rr][0] = __uint_as_float(v.x << 16);
                xr[rr][1] = __uint_as_float(v.x & 0xffff0000u);
                xr[rr][2] = __uint_as_float(v.y << 16);
                xr[rr][3] = __uint_as_float(v.y & 0xffff0000u);
            }
        }
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) {
            const int row = r_base + rr;
            float ss = 0.f, mx = 0.f;
            int bad = 0;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                ss = fmaf(xr[rr][k], xr[rr][k], ss);
                mx = fmaxf(mx, fabsf(xr[rr][k]));
                bad |= !isfinite(xr[rr][k]);
            }
            ss = tq_warp_sum(ss);
            mx = tq_warp_max(mx);
            bad = __any_sync(0xffffffffu, bad);
            // power of two 2^ex with max * 2^ex in [2^14, 2^15), from the exponent field of max
            int ex = 0;
            if (mx > 0.f && isfinite(mx)) ex = min(max(14 - (((__float_as_int(mx) >> 23) & 0xff) - 127), -126), 126);
            const float sc2 = __int_as_float((127 + ex) << 23);
            uint32_t h2[2], l2[2];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const float a = xr[rr][2 * k] * sc2, c = xr[rr][2 * k + 1] * sc2;
                h2[k] = pack_half2(a, c);
                if (kF32) {
                    const __half2 hh = *reinterpret_cast<const __half2*>(&h2[k]);
                    l2[k] = pack_half2(a - __low2float(hh), c - __high2float(hh));
                }
            }
            const uint32_t off = swz(row, lane >> 1) + (lane & 1) * 8;
            *reinterpret_cast<uint2*>(AH + off) = make_uint2(h2[0], h2[1]);
            if (kF32) *reinterpret_cast<uint2*>(AL + off) = make_uint2(l2[0], l2[1]);
            if (lane == 0) {
                const float n = sqrtf(ss);
                s_norm[row] = vrow[rr] ? n : 0.f;
                s_inv[row] = n > 0.f ? 1.f / (n * 256.f * sc2) : 0.f;
                s_bad[row] = vrow[rr] && bad;
                s_valid[row] = vrow[rr];
            }
        }
        __syncwarp();

        // ---- 2. Y = A Pi^T over this warp's 16 rows, all 128 output columns
        float acc[16][4];
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
        const int mi = lane >> 3, rr8 = lane & 7;
        const int a_row = r_base + (mi & 1) * 8 + rr8, a_chk = mi >> 1;     // A: matrices (r0-7,k0),(r8-15,k0),(r0-7,k8),(r8-15,k8)
        const int b_row = (mi >> 1) * 8 + rr8, b_chk = mi & 1;               // B: (n0-7,k0),(n0-7,k8),(n8-15,k0),(n8-15,k8)
#pragma unroll 1
        for (int kc = 0; kc < 8; ++kc) {
            uint32_t ah[4], al[4];
            ldsm_x4(sbase + (uint32_t)(AH - qsm) + swz(a_row, 2 * kc + a_chk), ah[0], ah[1], ah[2], ah[3]);
            if (kF32) ldsm_x4(sbase + (uint32_t)(AL - qsm) + swz(a_row, 2 * kc + a_chk), al[0], al[1], al[2], al[3]);
#pragma unroll
            for (int np2 = 0; np2 < 8; ++np2) {
                uint32_t bh[4], bl[4];
                ldsm_x4(sbase + (uint32_t)(PH - qsm) + swz(16 * np2 + b_row, 2 * kc + b_chk), bh[0], bh[1], bh[2], bh[3]);
                ldsm_x4(sbase + (uint32_t)(PL - qsm) + swz(16 * np2 + b_row, 2 * kc + b_chk), bl[0], bl[1], bl[2], bl[3]);
                tq_hmma(acc[2 * np2], ah[0], ah[1], ah[2], ah[3], bh[0], bh[1]);
                tq_hmma(acc[2 * np2 + 1], ah[0], ah[1], ah[2], ah[3], bh[2], bh[3]);
                tq_hmma(acc[2 * np2], ah[0], ah[1], ah[2], ah[3], bl[0], bl[1]);
                tq_hmma(acc[2 * np2 + 1], ah[0], ah[1], ah[2], ah[3], bl[2], bl[3]);
                if (kF32) {
                    tq_hmma(acc[2 * np2], al[0], al[1], al[2], al[3], bh[0], bh[1]);
                    tq_hmma(acc[2 * np2 + 1], al[0], al[1], al[2], al[3], bh[2], bh[3]);
                }
            }
        }
        __syncwarp();

        // ---- 3. codes, residual, gamma, code planes; thread (g, t): rows g, g + 8,
        //         columns 8 nt + 2t + e
        const int rows[2] = {r_base + g, r_base + 8 + g};
        uint32_t cw[B][2][4];
#pragma unroll
        for (int pl = 0; pl < B; ++pl)
#pragma unroll
            for (int h = 0; h < 2; ++h) cw[pl][h][0] = cw[pl][h][1] = cw[pl][h][2] = cw[pl][h][3] = 0u;
        float g2[2] = {0.f, 0.f};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int row = rows[h];
            const float inv = s_inv[row];
            const bool rvalid = s_valid[row];
#pragma unroll
            for (int nt = 0; nt < 16; ++nt) {
                float rv[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int col = 8 * nt + 2 * t + e;
                    const float y = acc[nt][2 * h + e] * inv;
                    int c = 0;
#pragma unroll
                    for (int q = 0; q < L - 1; ++q) c += y > p.cb.bounds[q];
                    float r = y - p.cb.cent[c];
                    if (col >= d || !rvalid) { c = 0; r = 0.f; }
                    g2[h] = fmaf(r, r, g2[h]);
                    rv[e] = r;
                    if (T.qjl) {
#pragma unroll
                        for (int pl = 0; pl < B; ++pl)
                            cw[pl][h][nt >> 2] |= (uint32_t)((c >> pl) & 1) << (8 * (nt & 3) + 2 * t + e);
                    } else {
                        CS[row * 128 + col] = (uint8_t)c;
                    }
                }
                if (T.qjl) {   // residual back into the A tile (scaled by 2^12), hi and lo
                    const float a = rv[0] * 4096.f, c2 = rv[1] * 4096.f;
                    const uint32_t hv = pack_half2(a, c2);
                    const __half2 hh = *reinterpret_cast<const __half2*>(&hv);
                    const uint32_t off = swz(row, nt) + 4 * t;
                    *reinterpret_cast<uint32_t*>(AH + off) = hv;
                    *reinterpret_cast<uint32_t*>(AL + off) = pack_half2(a - __low2float(hh), c2 - __high2float(hh));
                }
            }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            g2[h] += __shfl_xor_sync(0xffffffffu, g2[h], 1);
            g2[h] += __shfl_xor_sync(0xffffffffu, g2[h], 2);
            if (t == 0) s_gamma[rows[h]] = sqrtf(g2[h]);
        }
        if (T.qjl) {
            // plane words: OR over the 4 threads of a row group, thread t stores word t
#pragma unroll
            for (int pl = 0; pl < B; ++pl) {
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        cw[pl][h][w] |= __shfl_xor_sync(0xffffffffu, cw[pl][h][w], 1);
                        cw[pl][h][w] |= __shfl_xor_sync(0xffffffffu, cw[pl][h][w], 2);
                    }
            }
            const int64_t gb = tile * 4 + (r_base >> 5);
            if (gb < total_blocks) {
                uint8_t* blk = p.packed + (size_t)gb * T.block_bytes;
                const int u0 = (r_base & 31) >> 3;   // rows g, g + 8 -> u0, u0 + 1
#pragma unroll
                for (int pl = 0; pl < B; ++pl) {
                    const uint32_t w0 = t == 0 ? cw[pl][0][0] : t == 1 ? cw[pl][0][1] : t == 2 ? cw[pl][0][2] : cw[pl][0][3];
                    const uint32_t w1 = t == 0 ? cw[pl][1][0] : t == 1 ? cw[pl][1][1] : t == 2 ? cw[pl][1][2] : cw[pl][1][3];
                    *reinterpret_cast<uint2*>(blk + ((pl * 32 + 4 * g + t) * 4 + u0) * 4) = make_uint2(w0, w1);
                }
            }
            __syncwarp();

            // ---- 4. Z = R M^T (3 passes), sign plane
#pragma unroll
            for (int i = 0; i < 16; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
#pragma unroll 1
            for (int kc = 0; kc < 8; ++kc) {
                uint32_t ah[4], al[4];
                ldsm_x4(sbase + (uint32_t)(AH - qsm) + swz(a_row, 2 * kc + a_chk), ah[0], ah[1], ah[2], ah[3]);
                ldsm_x4(sbase + (uint32_t)(AL - qsm) + swz(a_row, 2 * kc + a_chk), al[0], al[1], al[2], al[3]);
#pragma unroll
                for (int np2 = 0; np2 < 8; ++np2) {
                    uint32_t bh[4], bl[4];
                    ldsm_x4(sbase + (uint32_t)(MH - qsm) + swz(16 * np2 + b_row, 2 * kc + b_chk), bh[0], bh[1], bh[2], bh[3]);
                    ldsm_x4(sbase + (uint32_t)(ML - qsm) + swz(16 * np2 + b_row, 2 * kc + b_chk), bl[0], bl[1], bl[2], bl[3]);
                    tq_hmma(acc[2 * np2], ah[0], ah[1], ah[2], ah[3], bh[0], bh[1]);
                    tq_hmma(acc[2 * np2 + 1], ah[0], ah[1], ah[2], ah[3], bh[2], bh[3]);
                    tq_hmma(acc[2 * np2], ah[0], ah[1], ah[2], ah[3], bl[0], bl[1]);
                    tq_hmma(acc[2 * np2 + 1], ah[0], ah[1], ah[2], ah[3], bl[2], bl[3]);
                    tq_hmma(acc[2 * np2], al[0], al[1], al[2], al[3], bh[0], bh[1]);
                    tq_hmma(acc[2 * np2 + 1], al[0], al[1], al[2], al[3], bh[2], bh[3]);
                }
            }
            uint32_t sw[2][4] = {{0u, 0u, 0u, 0u}, {0u, 0u, 0u, 0u}};
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const bool rvalid = s_valid[rows[h]];
#pragma unroll
                for (int nt = 0; nt < 16; ++nt)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int col = 8 * nt + 2 * t + e;
                        const bool bit = rvalid && col < T.m && acc[nt][2 * h + e] >= 0.f;
                        sw[h][nt >> 2] |= (uint32_t)bit << (8 * (nt & 3) + 2 * t + e);
                    }
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    sw[h][w] |= __shfl_xor_sync(0xffffffffu, sw[h][w], 1);
                    sw[h][w] |= __shfl_xor_sync(0xffffffffu, sw[h][w], 2);
                }
            }
            if (gb < total_blocks) {
                uint8_t* blk = p.packed + (size_t)gb * T.block_bytes;
                const int u0 = (r_base & 31) >> 3;
                const uint32_t w0 = t == 0 ? sw[0][0] : t == 1 ? sw[0][1] : t == 2 ? sw[0][2] : sw[0][3];
                const uint32_t w1 = t == 0 ? sw[1][0] : t == 1 ? sw[1][1] : t == 2 ? sw[1][2] : sw[1][3];
                *reinterpret_cast<uint2*>(blk + ((B * 32 + 4 * g + t) * 4 + u0) * 4) = make_uint2(w0, w1);
                // norms of rows g, g + 8
                if (t == 0) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int row = rows[h];
                        const bool valid = s_valid[row];
                        const uint32_t nh = valid ? tq_half_bits(s_norm[row]) : 0u;
                        const uint32_t gh = valid ? tq_half_bits(s_gamma[row]) : 0u;
                        if (valid && (s_bad[row] || (nh & 0x7fffu) >= 0x7c00u)) tq_raise(p.status, TQ_FLAG_RANGE);
                        reinterpret_cast<uint32_t*>(blk + T.sec_a)[g * 4 + u0 + h] = nh | (gh << 16);
                    }
                }
            }
        }
        if (!T.qjl) {
            // value layout: norms, then the lane strings of the tile's blocks from the codes
            __syncthreads();
            if (tid < 128) {
                const int row = tid;
                const int64_t gb = tile * 4 + (row >> 5);
                if (gb < total_blocks) {
                    const uint32_t nh = s_valid[row] ? tq_half_bits(s_norm[row]) : 0u;
                    if (s_valid[row] && (s_bad[row] || (nh & 0x7fffu) >= 0x7c00u)) tq_raise(p.status, TQ_FLAG_RANGE);
                    reinterpret_cast<uint16_t*>(p.packed + (size_t)gb * T.block_bytes + T.sec_a)[row & 31] = (uint16_t)nh;
                }
            }
            const int fb = 2 * B, words = 128 * B / 32;
            for (int e = tid; e < 4 * 32 * words; e += blockDim.x) {
                const int bl = e / (32 * words), rem = e % (32 * words);
                const int64_t gb = tile * 4 + bl;
                if (gb >= total_blocks) continue;
                const int ln = rem % 32, wd = rem / 32;
                const int gq = ln >> 2, tq = ln & 3;
                uint32_t val = 0;
                const int f0 = (32 * wd) / fb, f1 = (32 * wd + 31) / fb;
                for (int f = f0; f <= f1; ++f) {
                    const int a = f >> 2, pp = f & 3;
                    const int i = 8 * a + gq;
                    const int tau = 16 * (pp >> 1) + 8 * (pp & 1) + 2 * tq;
                    const uint8_t* crow = CS + (bl * 32) * 128;
                    const uint32_t F = (uint32_t)crow[tau * 128 + i] | ((uint32_t)crow[(tau + 1) * 128 + i] << B);
                    const int pos = f * fb - 32 * wd;
                    val |= pos >= 0 ? (F << pos) : (F >> (-pos));
                }
                reinterpret_cast<uint32_t*>(p.packed + (size_t)gb * T.block_bytes)[((wd >> 2) * 32 + ln) * 4 + (wd & 3)] = val;
            }
        }
        __syncthreads();
    }
}

template <int KD, int KM, int B>
cudaError_t launch(const QuantParams& p, cudaStream_t st) {
    const size_t smem_bytes = (size_t)32 * KD * 32 * 4 + (size_t)32 * KD * 32;
    auto kern = k_quantize_f32<KD, KM, B>;
    static TqLaunchCache cache;
    cudaError_t e = tq_kernel_setup(kern, 128, smem_bytes, cache, nullptr, nullptr);
    if (e != cudaSuccess) return e;
    const int64_t nblocks = p.n_streams * p.nb;
    kern<<<(unsigned)nblocks, 128, smem_bytes, st>>>(p);
    return cudaGetLastError();
}

}  // namespace

template <int KD, int KM>
cudaError_t launch_b(const QuantParams& p, cudaStream_t st) {
    switch (p.t.B) {
        case 1: return launch<KD, KM, 1>(p, st);
        case 2: return launch<KD, KM, 2>(p, st);
        case 3: return launch<KD, KM, 3>(p, st);
        case 4: return launch<KD, KM, 4>(p, st);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_kd(const QuantParams& p, cudaStream_t st, int kd, int km) {
    if (kd == 4 && km == 0) return launch_b<4, 0>(p, st);
    if (kd == 4 && km == 4) return launch_b<4, 4>(p, st);
    if (kd == 4 && km == 8) return launch_b<4, 8>(p, st);
    if (kd == 8 && km == 0) return launch_b<8, 0>(p, st);
    if (kd == 8 && km == 4) return launch_b<8, 4>(p, st);
    if (kd == 8 && km == 8) return launch_b<8, 8>(p, st);
    return cudaErrorInvalidValue;
}

template <bool kF32, int B>
cudaError_t launch_mma(const QuantParams& p, cudaStream_t st) {
    const size_t smem = 6 * (size_t)mma16::kMatBytes + 128 * 128;
    auto kern = k_quantize_mma<kF32, B>;
    static TqLaunchCache cache;
    int sms = 0;
    cudaError_t e = tq_kernel_setup(kern, 256, smem, cache, &sms, nullptr);
    if (e != cudaSuccess) return e;
    const int64_t tiles = (p.n_streams * p.nb + 3) / 4;
    const int64_t grid = std::min<int64_t>(tiles, sms);
    if (grid > 0) kern<<<(unsigned)grid, 256, smem, st>>>(p);
    return cudaGetLastError();
}

cudaError_t tq_launch_quantize(const QuantParams& p, cudaStream_t st) {
    if (p.t.D == 128 && (p.t.Mp == 128 || !p.t.qjl)) return tq_launch_quantize_tc(p, st);
    if (false) {
        const bool f32 = p.dtype == 0;
        switch (p.t.B) {
            case 1: return f32 ? launch_mma<true, 1>(p, st) : launch_mma<false, 1>(p, st);
            case 2: return f32 ? launch_mma<true, 2>(p, st) : launch_mma<false, 2>(p, st);
            case 3: return f32 ? launch_mma<true, 3>(p, st) : launch_mma<false, 3>(p, st);
            case 4: return f32 ? launch_mma<true, 4>(p, st) : launch_mma<false, 4>(p, st);
        }
        return cudaErrorInvalidValue;
    }
    const int kd = p.t.D / 32, km = p.t.Mp / 32;
    return launch_kd(p, st, kd, km);
}
