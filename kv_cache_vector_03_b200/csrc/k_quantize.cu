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

// one CTA of 4 warps per 32-vector block
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

cudaError_t tq_launch_quantize(const QuantParams& p, cudaStream_t st) {
    // d <= 128 with m <= 128 (or no sketch): tensor cores (k_quantize_tc.cu, k_quantize_ws.cu);
    // keys with d, m in 129..256: tensor cores (k_quantize_wide.cu); otherwise fp32
    if (p.t.D == 128 && (p.t.Mp == 128 || !p.t.qjl)) return tq_launch_quantize_tc(p, st);
    if (p.t.qjl && p.t.D == 256 && p.t.Mp == 256 && p.wimg && p.t.B <= 3) return tq_launch_quantize_wide(p, st);
    const int kd = p.t.D / 32, km = p.t.Mp / 32;
    return launch_kd(p, st, kd, km);
}
