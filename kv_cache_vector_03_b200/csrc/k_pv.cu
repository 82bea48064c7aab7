// tq_pv: softmax(P) . V over MSE-only packed values (friday-blog-bgf.pages.dev "TurboQuant
// deep dive II", section 1, step 1: values use the rotation + scalar quantizer only).
//
//   o_h = sum_t w_t |v_t| Pi^T c[idx_t] = Pi^T ( sum_t w_t |v_t| c[idx_t] )
// so the weighted sum is accumulated in the rotated domain and rotated back once.
//
// Kernel 1 (split): one CTA of 4 warps per (stream, token range). The range's softmax
// maximum is found first; then each 32-token block is dequantized straight into fp16 MMA
// A fragments (rows = coordinates, K = tokens) through a per-lane shared-memory table that
// maps a 2B-bit field (two tokens' codes of one coordinate) to a half2 of centroids, and
// multiplied on the tensor cores by B = weights exp(P - m) |v| split into fp16 hi + lo
// columns. Partial sums, maxima and softmax denominators go to the workspace.
// Kernel 2 (merge): one CTA per query head combines the partials (log-sum-exp rescale) and
// rotates by Pi^T.
#include "tq_device.cuh"

namespace {

template <int B, int KT, int NT>  // KT = D/16 coordinate tiles, NT = n-tiles of 4 heads
__global__ void __launch_bounds__(128) k_pv_split(PvParams p) {
    constexpr int E = 1 << (2 * B);          // table entries
    constexpr int CH = KT * B / 8;           // 16-byte chunks per lane per block (D*B/128)
    constexpr int NW = 4 * CH;               // 32-bit words per lane per block
    extern __shared__ uint32_t lut[];        // [E][32]
    __shared__ float s_acc[8][KT * 16];
    __shared__ float s_m[8], s_l[8];

    const TqDims& T = p.t;
    const int G = p.g;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int64_t stream = blockIdx.x / p.nsplit;
    const int split = blockIdx.x % p.nsplit;
    const int64_t b0 = (int64_t)split * p.blocks_per_split;
    const int64_t b1 = min(b0 + p.blocks_per_split, p.nb);
    const int64_t t0 = b0 * 32, t1 = min(b1 * 32, p.n_tok);
    const float* Pst = p.P + (size_t)stream * G * p.n_tok;

    for (int e = threadIdx.x; e < E * 32; e += blockDim.x) {
        const int ent = e >> 5;
        lut[e] = p.cb.lut_half[ent & ((1 << B) - 1)] | (p.cb.lut_half[ent >> B] << 16);
    }
    for (int e = threadIdx.x; e < 8 * KT * 16; e += blockDim.x) (&s_acc[0][0])[e] = 0.f;
    // pass 1: per-head maximum over the range
    for (int h = w; h < G; h += 4) {
        float mx = -INFINITY;
        for (int64_t tok = t0 + lane; tok < t1; tok += 32) mx = fmaxf(mx, Pst[(size_t)h * p.n_tok + tok]);
        mx = tq_warp_max(mx);
        if (lane == 0) { s_m[h] = mx; s_l[h] = 0.f; }
    }
    __syncthreads();

    float acc[KT][NT][4];
#pragma unroll
    for (int k = 0; k < KT; ++k)
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int r = 0; r < 4; ++r) acc[k][n][r] = 0.f;
    float lsum[NT];
#pragma unroll
    for (int n = 0; n < NT; ++n) lsum[n] = 0.f;
    float mh[NT];
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        const int head = n * 4 + (g >> 1);
        mh[n] = head < G ? s_m[head] : 0.f;
    }

    const uint8_t* sbase = p.packed + (size_t)stream * p.nb * T.block_bytes;
    const uint32_t sec_a = T.sec_a;
#pragma unroll 1
    for (int64_t bi = b0 + w; bi < b1; bi += 4) {
        const uint8_t* bp = sbase + (size_t)bi * T.block_bytes;
        uint32_t W[NW + 1];
#pragma unroll
        for (int c = 0; c < CH; ++c) {
            const uint4 v = tq_ldg_stream(bp + (size_t)(c * 32 + lane) * 16);
            W[4 * c] = v.x; W[4 * c + 1] = v.y; W[4 * c + 2] = v.z; W[4 * c + 3] = v.w;
        }
        W[NW] = 0u;
        const uint16_t* nrm = reinterpret_cast<const uint16_t*>(bp + sec_a);
        // weights for the 8 tokens this thread feeds: chunk c, pair (2t, 2t+1) and (8+2t, 9+2t)
        uint32_t bw[NT][2][2];
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            const int head = n * 4 + (g >> 1);
            const bool part_lo = g & 1;
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
                for (int hv = 0; hv < 2; ++hv) {
                    uint32_t packed2 = 0;
#pragma unroll
                    for (int e2 = 0; e2 < 2; ++e2) {
                        const int tb = 16 * c + 8 * hv + 2 * t + e2;
                        const int64_t tok = bi * 32 + tb;
                        float wt = 0.f;
                        if (head < G && tok < p.n_tok) {
                            const float ex = __expf(Pst[(size_t)head * p.n_tok + tok] - mh[n]);
                            if (!part_lo) lsum[n] += ex;
                            wt = ex * tq_half_val(nrm[tb]);
                        }
                        const __half hi = __float2half_rn(wt);
                        const __half val = part_lo ? __float2half_rn(wt - __half2float(hi)) : hi;
                        packed2 |= (uint32_t)__half_as_ushort(val) << (16 * e2);
                    }
                    bw[n][c][hv] = packed2;
                }
        }
        // A fragments: field (a, pp) at bit (4a + pp) * 2B of the lane string
#pragma unroll
        for (int k = 0; k < KT; ++k)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t a[4];
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    // r: 0 -> (a=2k, pp=2c), 1 -> (2k+1, 2c), 2 -> (2k, 2c+1), 3 -> (2k+1, 2c+1)
                    const int f = 4 * (2 * k + (r & 1)) + 2 * c + (r >> 1);
                    const int bit = f * 2 * B;
                    const int wi = bit >> 5, sh = bit & 31;
                    uint32_t fld = sh == 0 ? W[wi] : __funnelshift_r(W[wi], W[wi + 1], sh);
                    fld &= (uint32_t)(E - 1);
                    a[r] = lut[fld * 32 + lane];
                }
#pragma unroll
                for (int n = 0; n < NT; ++n) tq_hmma(acc[k][n], a[0], a[1], a[2], a[3], bw[n][c][0], bw[n][c][1]);
            }
    }
    // combine hi + lo columns and the 4 warps
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        const int head = n * 4 + t;
        if (head < G) {
#pragma unroll
            for (int k = 0; k < KT; ++k) {
                atomicAdd(&s_acc[head][16 * k + g], acc[k][n][0] + acc[k][n][1]);
                atomicAdd(&s_acc[head][16 * k + 8 + g], acc[k][n][2] + acc[k][n][3]);
            }
        }
        float ls = lsum[n];
        // lanes 8h + t (t = 0..3) hold the exps of head n*4 + h
        ls += __shfl_xor_sync(0xffffffffu, ls, 1);
        ls += __shfl_xor_sync(0xffffffffu, ls, 2);
        const int hh = n * 4 + (g >> 1);
        if ((lane & 7) == 0 && hh < G) atomicAdd(&s_l[hh], ls);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < G * T.D; e += blockDim.x) {
        const int h = e / T.D, i = e % T.D;
        p.part[(((size_t)stream * G + h) * p.nsplit + split) * T.D + i] = s_acc[h][i];
    }
    if (threadIdx.x < G) {
        float2* ml = reinterpret_cast<float2*>(p.part_ml);
        ml[((size_t)stream * G + threadIdx.x) * p.nsplit + split] = make_float2(s_m[threadIdx.x], s_l[threadIdx.x]);
    }
}

__global__ void __launch_bounds__(256) k_pv_merge(PvParams p) {
    const TqDims& T = p.t;
    const int64_t hq = blockIdx.x;  // stream * g + head
    __shared__ float s_o[TQ_MAX_D];
    const float2* ml = reinterpret_cast<const float2*>(p.part_ml) + (size_t)hq * p.nsplit;
    float M = -INFINITY;
    for (int s = 0; s < p.nsplit; ++s) M = fmaxf(M, ml[s].x);
    for (int i = threadIdx.x; i < T.D; i += blockDim.x) {
        float acc = 0.f, den = 0.f;
        for (int s = 0; s < p.nsplit; ++s) {
            const float2 v = ml[s];
            if (v.y > 0.f) {
                const float f = __expf(v.x - M);
                acc += f * p.part[((size_t)hq * p.nsplit + s) * T.D + i];
                den += f * v.y;
            }
        }
        s_o[i] = acc / den;
    }
    __syncthreads();
    for (int j = threadIdx.x; j < T.d; j += blockDim.x) {
        float o = 0.f;
        for (int i = 0; i < T.d; ++i) o = fmaf(__ldg(p.pi + (size_t)i * T.d + j), s_o[i], o);
        p.out[(size_t)hq * T.d + j] = o;
    }
}

template <int B, int KT, int NT>
cudaError_t launch_split(const PvParams& p, cudaStream_t st) {
    const size_t smem = (size_t)(1 << (2 * B)) * 32 * 4;
    auto kern = k_pv_split<B, KT, NT>;
    static TqLaunchCache cache;
    cudaError_t e = tq_kernel_setup(kern, 128, smem, cache, nullptr, nullptr);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(p.n_streams * p.nsplit), 128, smem, st>>>(p);
    return cudaGetLastError();
}

template <int KT, int NT>
cudaError_t launch_b(const PvParams& p, cudaStream_t st) {
    switch (p.t.B) {
        case 1: return launch_split<1, KT, NT>(p, st);
        case 2: return launch_split<2, KT, NT>(p, st);
        case 3: return launch_split<3, KT, NT>(p, st);
        case 4: return launch_split<4, KT, NT>(p, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t tq_launch_pv(const PvParams& p, cudaStream_t st) {
    cudaError_t e;
    const int nt = p.g > 4 ? 2 : 1;
    if (p.t.D == 128) e = nt == 1 ? launch_b<8, 1>(p, st) : launch_b<8, 2>(p, st);
    else if (p.t.D == 256) e = nt == 1 ? launch_b<16, 1>(p, st) : launch_b<16, 2>(p, st);
    else return cudaErrorInvalidValue;
    if (e != cudaSuccess) return e;
    k_pv_merge<<<(unsigned)(p.n_streams * p.g), 256, 0, st>>>(p);
    return cudaGetLastError();
}
