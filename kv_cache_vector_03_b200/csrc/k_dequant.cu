// tq_dequantize (diagnostic, not on the hot path): rebuild x~ from a packed record
// (blog.hotdry.top "TurboQuant vector-search compression", section "QJL residual
// correction": x~ = x_mse + gamma sqrt(pi/2)/m S^T sign(S r), scaled by the stored |x|).
#include "tq_device.cuh"

namespace {

__device__ uint32_t key_bit(const uint8_t* blk, const TqDims& T, int pg, int v, int i) {
    const int gq = v & 7, u = v >> 3, w = i >> 5, tq = w & 3;
    const uint32_t word = reinterpret_cast<const uint32_t*>(blk)[((pg + (w >> 2)) * 32 + 4 * gq + tq) * 4 + u];
    return (word >> (i & 31)) & 1u;
}

__device__ uint32_t value_code(const uint8_t* blk, const TqDims& T, int tau, int i) {
    const int B = T.B;
    const int p = 2 * (tau >> 4) + ((tau >> 3) & 1), tq = (tau & 7) >> 1, e2 = tau & 1;
    const int a = i >> 3, gq = i & 7, lane = 4 * gq + tq;
    const int bit = (4 * a + p) * 2 * B + e2 * B;
    uint32_t val = 0;
    for (int k = 0; k < B; ++k) {
        const int bb = bit + k, wd = bb >> 5;
        const uint32_t word = reinterpret_cast<const uint32_t*>(blk)[((wd >> 2) * 32 + lane) * 4 + (wd & 3)];
        val |= ((word >> (bb & 31)) & 1u) << k;
    }
    return val;
}

__global__ void __launch_bounds__(128) k_dequant(DequantParams p) {
    const TqDims& T = p.t;
    __shared__ float s_c[32][TQ_MAX_D];   // centroid values
    __shared__ signed char s_s[32][TQ_MAX_D];   // +-1 signs
    __shared__ float s_n[32], s_g[32];
    const int64_t blkid = blockIdx.x;
    const int64_t s = blkid / p.nb, b = blkid % p.nb;
    const uint8_t* blk = p.packed + (size_t)blkid * T.block_bytes;
    const uint32_t sec_a = T.sec_a;
    for (int e = threadIdx.x; e < 32 * T.D; e += blockDim.x) {
        const int v = e / T.D, i = e % T.D;
        uint32_t code = 0;
        if (T.qjl) {
            for (int pl = 0; pl < T.B; ++pl) code |= key_bit(blk, T, pl * T.GD, v, i) << pl;
        } else {
            code = value_code(blk, T, v, i);
        }
        s_c[v][i] = p.cb.cent[code];
    }
    if (T.qjl)
        for (int e = threadIdx.x; e < 32 * T.Mp; e += blockDim.x) {
            const int v = e / T.Mp, k = e % T.Mp;
            s_s[v][k] = key_bit(blk, T, T.B * T.GD, v, k) ? 1 : -1;
        }
    if (threadIdx.x < 32) {
        const int v = threadIdx.x;
        if (T.qjl) {
            const uint32_t nw = reinterpret_cast<const uint32_t*>(blk + sec_a)[(v & 7) * 4 + (v >> 3)];
            s_n[v] = tq_half_val(nw & 0xffffu);
            s_g[v] = tq_half_val(nw >> 16);
        } else {
            s_n[v] = tq_half_val(reinterpret_cast<const uint16_t*>(blk + sec_a)[v]);
            s_g[v] = 0.f;
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < 32 * T.d; e += blockDim.x) {
        const int v = e / T.d, j = e % T.d;
        const int64_t tok = b * 32 + v;
        if (tok >= p.n_tok) continue;
        float a = 0.f;
        for (int i = 0; i < T.d; ++i) a = fmaf(__ldg(p.pi + (size_t)i * T.d + j), s_c[v][i], a);
        if (T.qjl) {
            float q = 0.f;
            for (int k = 0; k < T.m; ++k) q = fmaf(__ldg(p.s + (size_t)k * T.d + j), (float)s_s[v][k], q);
            a = fmaf(s_g[v] * p.kappa, q, a);
        }
        p.out[((size_t)s * p.n_tok + tok) * T.d + j] = s_n[v] * a;
    }
}

}  // namespace

cudaError_t tq_launch_dequant(const DequantParams& p, cudaStream_t st) {
    k_dequant<<<(unsigned)(p.n_streams * p.nb), 128, 0, st>>>(p);
    return cudaGetLastError();
}
