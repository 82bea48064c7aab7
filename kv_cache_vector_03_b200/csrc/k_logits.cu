// tq_logits: attention logits straight from packed keys with a query rotated once
// (a2a-mcp.org "What is TurboQuant", stage 2 and the fused-kernel note; the estimator is
// blog.hotdry.top "TurboQuant vector-search compression", section "QJL residual
// correction"):
//   l = scale |x| ( <q', c[idx]> + gamma sqrt(pi/2)/m <q'', s> ),  q' = Pi q, q'' = S q.
//
// The codebook is symmetric, so c[idx] is an odd multilinear polynomial in the +-1 values
// s_p = 2 bit_p - 1 of the index bits:
//   B=1: a0 s0;  B=2: a0 s0 + a1 s1;  B=3: a0 s0 + a1 s1 + a2 s2 + a3 s0 s1 s2,
// with s0 s1 s2 = 2 (b0 ^ b1 ^ b2) - 1. Hence
//   <q', c[idx]> = sum_p sum_i (2 a_p q'_i) beta_{p,i} - (sum_p a_p) sum_i q'_i,
//   <q'', s>     = 2 sum_j q''_j bit_j - sum_j q''_j,
// two contractions of {0,1} bit planes against fixed vectors. Each is run on the int8
// tensor cores: the planes become 0/1 bytes with one shift+and per 4 coordinates, and the
// query side is a 16-bit fixed-point vector split into two int8 columns (hi, lo) of the
// same MMA, so the int32 accumulation is exact.
//
// Kernel 1 (prologue, one CTA per (sequence, kv-head)): q', q'', fixed-point fragments in
// MMA order, per-head scales, and the exact logits of the full-precision tail.
// Kernel 2 (stream): each warp owns one (stream, n-tile of 4 heads, run of blocks) task,
// keeps the query fragments in registers and streams 32-key blocks with 16-byte loads.
#include "tq_device.cuh"

namespace {

constexpr int kPrologueThreads = 256;

// fragment index of (stream, ntile, mma plane group, chunk, lane, half)
__device__ __forceinline__ size_t qf_index(int64_t stream, int ntile, int ntiles, int nmg, int mg, int c,
                                           int lane, int h) {
    return ((((size_t)stream * ntiles + ntile) * nmg + mg) * 4 + c) * 64 + lane * 2 + h;
}

__global__ void __launch_bounds__(kPrologueThreads) k_logits_prologue(LogitsParams p) {
    const TqDims& T = p.t;
    const int D = T.D, Mp = T.Mp, d = T.d, G = p.g;
    const int64_t stream = blockIdx.x;                 // seq * n_kv + kv
    const int64_t seq = stream / p.n_kv;
    const int kv = (int)(stream % p.n_kv);
    extern __shared__ float sm[];
    float* qs = sm;                    // [G][D] raw query
    float* qp = qs + G * D;            // [G][D] Pi q
    float* qpp = qp + G * D;           // [G][Mp] S q
    int* iv = reinterpret_cast<int*>(qpp + G * Mp);   // [G][nplanes][D] + [G][Mp] fixed point
    __shared__ float s_max[2][8];
    __shared__ double s_sum[2][8];

    const int np = T.nplanes_mma;
    int* ivA = iv;
    int* ivS = iv + G * np * D;

    // query heads of this kv group
    for (int e = threadIdx.x; e < G * D; e += blockDim.x) {
        const int h = e / D, i = e % D;
        const int64_t qh = seq * ((int64_t)p.n_kv * G) + (int64_t)kv * G + h;
        qs[e] = i < d ? tq_load_elem(p.q, p.q_dtype, qh * d + i) : 0.f;
    }
    __syncthreads();
    // q' = Pi q, q'' = S q (fp32 accumulate)
    for (int e = threadIdx.x; e < G * D; e += blockDim.x) {
        const int h = e / D, i = e % D;
        float a = 0.f;
        for (int j = 0; j < d; ++j) a = fmaf(__ldg(p.piT + (size_t)j * D + i), qs[h * D + j], a);
        qp[e] = a;
    }
    for (int e = threadIdx.x; e < G * Mp; e += blockDim.x) {
        const int h = e / Mp, k = e % Mp;
        float a = 0.f;
        for (int j = 0; j < d; ++j) a = fmaf(__ldg(p.sT + (size_t)j * Mp + k), qs[h * D + j], a);
        qpp[e] = a;
    }
    __syncthreads();
    // per-head max |q'| and |q''| (warp h handles head h; G <= 8 = warps per CTA)
    const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (wid < G) {
        float ma = 0.f, ms = 0.f;
        for (int i = lane; i < D; i += 32) ma = fmaxf(ma, fabsf(qp[wid * D + i]));
        for (int k = lane; k < Mp; k += 32) ms = fmaxf(ms, fabsf(qpp[wid * Mp + k]));
        ma = tq_warp_max(ma);
        ms = tq_warp_max(ms);
        if (lane == 0) { s_max[0][wid] = ma; s_max[1][wid] = ms; }
    }
    __syncthreads();
    float amax = 0.f;
    for (int pl = 0; pl < np; ++pl) amax = fmaxf(amax, fabsf(2.f * p.cb.plane_coef[pl]));
    // fixed point: v = round(value / delta), |v| <= 32000
    for (int e = threadIdx.x; e < G * np * D; e += blockDim.x) {
        const int h = e / (np * D), pl = (e / D) % np, i = e % D;
        const float m0 = s_max[0][h] * amax;
        const float delta = m0 > 0.f ? m0 / 32000.f : 1.f;
        ivA[e] = __float2int_rn(2.f * p.cb.plane_coef[pl] * qp[h * D + i] / delta);
    }
    for (int e = threadIdx.x; e < G * Mp; e += blockDim.x) {
        const int h = e / Mp;
        const float m0 = s_max[1][h];
        const float delta = m0 > 0.f ? m0 / 32000.f : 1.f;
        ivS[e] = __float2int_rn(qpp[e] / delta);
    }
    __syncthreads();
    if (wid < G) {
        double sa = 0.0, ss = 0.0;
        for (int e = lane; e < np * D; e += 32) sa += ivA[wid * np * D + e];
        for (int k = lane; k < Mp; k += 32) ss += ivS[wid * Mp + k];
        sa = tq_warp_sum_d(sa);
        ss = tq_warp_sum_d(ss);
        if (lane == 0) { s_sum[0][wid] = sa; s_sum[1][wid] = ss; }
    }
    __syncthreads();
    // per-head scales: l = |x| (dA accA - KA + gamma kappa (2 dS accS - KS))
    if (threadIdx.x < p.ntiles * 4) {
        const int h = threadIdx.x;
        float4 sc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (h < G) {
            const float ma = s_max[0][h] * amax, ms = s_max[1][h];
            const float dA = ma > 0.f ? ma / 32000.f : 1.f;
            const float dS = ms > 0.f ? ms / 32000.f : 1.f;
            sc = make_float4(dA, (float)(0.5 * dA * s_sum[0][h]), 2.f * dS, (float)(dS * s_sum[1][h]));
        }
        reinterpret_cast<float4*>(p.qscale)[stream * p.ntiles * 4 + h] = sc;
    }
    // fragments: lane (g, t), column g = (head g>>1, part g&1); register (mg, c, h) byte b holds
    // coordinate 128 gr + 32 t + 2c + h + 8b of plane group mg
    const int nmg = T.nmg;
    const int total = p.ntiles * nmg * 4 * 64;
    for (int e = threadIdx.x; e < total; e += blockDim.x) {
        const int hh = e & 1, ln = (e >> 1) & 31, c = (e >> 6) & 3;
        const int mg = (e >> 8) % nmg, nt = (e >> 8) / nmg;
        const int g = ln >> 2, t = ln & 3;
        const int head = nt * 4 + (g >> 1), part = g & 1;
        uint32_t word = 0;
        if (head < G) {
            const bool is_code = mg < np * T.GD;
            const int gr = is_code ? mg % T.GD : mg - np * T.GD;
            const int pl = is_code ? mg / T.GD : 0;
#pragma unroll
            for (int bb = 0; bb < 4; ++bb) {
                const int i = 128 * gr + 32 * t + 2 * c + hh + 8 * bb;
                const int v = is_code ? ivA[(head * np + pl) * D + i] : ivS[head * Mp + i];
                const int hi = (v + 128) >> 8;
                const int lo = v - 256 * hi;
                word |= ((uint32_t)(part ? lo : hi) & 0xffu) << (8 * bb);
            }
        }
        p.qfrag[qf_index(stream, nt, p.ntiles, nmg, mg, c, ln, hh)] = word;
    }
    // exact logits of the full-precision tail: scale <q, k>
    if (p.n_tail > 0) {
        const int64_t row = p.n_tok + p.n_tail;
        for (int e = threadIdx.x; e < G * p.n_tail; e += blockDim.x) {
            const int h = e / p.n_tail, tt = e % p.n_tail;
            const uint16_t* kp = p.tail + ((size_t)stream * p.n_tail + tt) * d;
            float a = 0.f;
            for (int i = 0; i < d; ++i) a = fmaf(__uint_as_float((uint32_t)kp[i] << 16), qs[h * D + i], a);
            const int64_t qh = seq * ((int64_t)p.n_kv * G) + (int64_t)kv * G + h;
            p.out[qh * row + p.n_tok + tt] = p.scale * a;
        }
    }
}

// Stream kernel. NP = code planes in the estimator, GD/GM = 128-coordinate groups of the
// code and sign planes, B = stored code planes.
template <int B, int GD, int GM>
__global__ void __launch_bounds__(128) k_logits_stream(LogitsParams p) {
    constexpr int NP = B == 3 ? 4 : B;
    constexpr int NPG = B * GD + GM;       // stored plane groups
    constexpr int NMG = NP * GD + GM;      // MMA plane groups
    const TqDims& T = p.t;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int64_t tasks_per_tile = (p.nb + p.blocks_per_task - 1) / p.blocks_per_task;
    const int64_t task = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
    const int64_t n_tasks = p.n_seq * p.n_kv * p.ntiles * tasks_per_tile;
    if (task >= n_tasks) return;
    const int64_t stream = task / (p.ntiles * tasks_per_tile);
    const int ntile = (int)((task / tasks_per_tile) % p.ntiles);
    const int64_t b0 = (task % tasks_per_tile) * p.blocks_per_task;
    const int64_t b1 = min(b0 + p.blocks_per_task, p.nb);

    // query fragments and scales of this (stream, n-tile)
    uint32_t qf[NMG][4][2];
#pragma unroll
    for (int mg = 0; mg < NMG; ++mg)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const uint2 v = *reinterpret_cast<const uint2*>(
                p.qfrag + qf_index(stream, ntile, p.ntiles, NMG, mg, c, lane, 0));
            qf[mg][c][0] = v.x;
            qf[mg][c][1] = v.y;
        }
    const int head = ntile * 4 + t;
    const bool head_ok = head < p.g;
    const float4 sc = reinterpret_cast<const float4*>(p.qscale)[stream * p.ntiles * 4 + ntile * 4 + t];
    const float kap = p.kappa, scale = p.scale;
    const int64_t seq = stream / p.n_kv;
    const int kv = (int)(stream % p.n_kv);
    const int64_t row = p.n_tok + p.n_tail;
    float* orow = p.out + (seq * ((int64_t)p.n_kv * p.g) + (int64_t)kv * p.g + head) * row;

    const uint8_t* base = p.packed + (size_t)(stream * p.nb) * T.block_bytes;
    uint4 cur[NPG + 1], nxt[NPG + 1];
    auto load_block = [&](int64_t bi, uint4 (&dst)[NPG + 1]) {
        const uint8_t* bp = base + (size_t)bi * T.block_bytes;
#pragma unroll
        for (int pg = 0; pg < NPG; ++pg) dst[pg] = tq_ldg_stream(bp + (size_t)(pg * 32 + lane) * 16);
        dst[NPG] = tq_ldg_stream(bp + (size_t)NPG * 512 + g * 16);
    };
    if (b0 < b1) load_block(b0, cur);
#pragma unroll 1
    for (int64_t bi = b0; bi < b1; ++bi) {
        if (bi + 1 < b1) load_block(bi + 1, nxt);
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            int accA[4] = {0, 0, 0, 0}, accS[4] = {0, 0, 0, 0};
#pragma unroll
            for (int mg = 0; mg < NMG; ++mg) {
                uint32_t w0, w1;  // words of rows g (u = 2mt) and g + 8 (u = 2mt + 1)
                const uint32_t* cw = nullptr;
                if (mg < NP * GD) {
                    const int pl = mg / GD, gr = mg % GD;
                    if (pl < B) {
                        cw = reinterpret_cast<const uint32_t*>(&cur[pl * GD + gr]);
                        w0 = cw[2 * mt];
                        w1 = cw[2 * mt + 1];
                    } else {  // b0 ^ b1 ^ b2
                        const uint32_t* c0 = reinterpret_cast<const uint32_t*>(&cur[0 * GD + gr]);
                        const uint32_t* c1 = reinterpret_cast<const uint32_t*>(&cur[1 * GD + gr]);
                        const uint32_t* c2 = reinterpret_cast<const uint32_t*>(&cur[2 * GD + gr]);
                        w0 = c0[2 * mt] ^ c1[2 * mt] ^ c2[2 * mt];
                        w1 = c0[2 * mt + 1] ^ c1[2 * mt + 1] ^ c2[2 * mt + 1];
                    }
                } else {
                    cw = reinterpret_cast<const uint32_t*>(&cur[B * GD + (mg - NP * GD)]);
                    w0 = cw[2 * mt];
                    w1 = cw[2 * mt + 1];
                }
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint32_t a0 = (w0 >> (2 * c)) & 0x01010101u;
                    const uint32_t a1 = (w1 >> (2 * c)) & 0x01010101u;
                    const uint32_t a2 = (w0 >> (2 * c + 1)) & 0x01010101u;
                    const uint32_t a3 = (w1 >> (2 * c + 1)) & 0x01010101u;
                    if (mg < NP * GD) tq_imma(accA, a0, a1, a2, a3, qf[mg][c][0], qf[mg][c][1]);
                    else tq_imma(accS, a0, a1, a2, a3, qf[mg][c][0], qf[mg][c][1]);
                }
            }
            // epilogue: thread (g, t) -> head t of the tile, rows g and g + 8
            const uint32_t* nrm = reinterpret_cast<const uint32_t*>(&cur[NPG]);
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int u = 2 * mt + r;
                const int64_t tok = bi * 32 + 8 * u + g;
                const uint32_t nw = nrm[u];
                const float nh = tq_half_val(nw & 0xffffu), gh = tq_half_val(nw >> 16);
                const float va = (float)(256 * accA[2 * r] + accA[2 * r + 1]);
                const float vs = (float)(256 * accS[2 * r] + accS[2 * r + 1]);
                const float est = fmaf(sc.x, va, -sc.y) + gh * kap * fmaf(sc.z, vs, -sc.w);
                if (head_ok && tok < p.n_tok) orow[tok] = scale * nh * est;
            }
        }
        if (bi + 1 < b1) {
#pragma unroll
            for (int i = 0; i <= NPG; ++i) cur[i] = nxt[i];
        }
    }
}

template <int B, int GD, int GM>
cudaError_t launch_stream(const LogitsParams& p, cudaStream_t st) {
    const int64_t tpt = (p.nb + p.blocks_per_task - 1) / p.blocks_per_task;
    const int64_t tasks = p.n_seq * p.n_kv * p.ntiles * tpt;
    const int64_t ctas = (tasks + 3) / 4;
    if (ctas > 0) k_logits_stream<B, GD, GM><<<(unsigned)ctas, 128, 0, st>>>(p);
    return cudaGetLastError();
}

}  // namespace

size_t tq_logits_prologue_smem(const TqDims& t, int g) {
    return (size_t)g * (2 * t.D + t.Mp) * 4 + (size_t)g * (t.nplanes_mma * t.D + t.Mp) * 4;
}

cudaError_t tq_launch_logits(const LogitsParams& p, cudaStream_t st) {
    const size_t smem = tq_logits_prologue_smem(p.t, p.g);
    cudaError_t e = cudaFuncSetAttribute(k_logits_prologue, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k_logits_prologue<<<(unsigned)(p.n_seq * p.n_kv), kPrologueThreads, smem, st>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int B = p.t.B, GD = p.t.GD, GM = p.t.GM;
    if (GD == 1 && GM == 1) {
        if (B == 1) return launch_stream<1, 1, 1>(p, st);
        if (B == 2) return launch_stream<2, 1, 1>(p, st);
        if (B == 3) return launch_stream<3, 1, 1>(p, st);
    } else if (GD == 2 && GM == 2) {
        if (B == 1) return launch_stream<1, 2, 2>(p, st);
        if (B == 2) return launch_stream<2, 2, 2>(p, st);
        if (B == 3) return launch_stream<3, 2, 2>(p, st);
    } else if (GD == 1 && GM == 2) {
        if (B == 1) return launch_stream<1, 1, 2>(p, st);
        if (B == 2) return launch_stream<2, 1, 2>(p, st);
        if (B == 3) return launch_stream<3, 1, 2>(p, st);
    } else if (GD == 2 && GM == 1) {
        if (B == 1) return launch_stream<1, 2, 1>(p, st);
        if (B == 2) return launch_stream<2, 2, 1>(p, st);
        if (B == 3) return launch_stream<3, 2, 1>(p, st);
    }
    return cudaErrorInvalidValue;
}
