// tq_pv: softmax(P) . V over MSE-only packed values (friday-blog-bgf.pages.dev "TurboQuant
// deep dive II", section 1, step 1: values use the rotation + scalar quantizer only).
//
//   o_h = sum_t w_t |v_t| Pi^T c[idx_t] = Pi^T ( sum_t w_t |v_t| c[idx_t] )
// so the weighted sum is accumulated in the rotated domain and rotated back once.
//
// Kernel 1 (split): one CTA of 8 warps per (stream, block range); warp w takes blocks
// w, w + 8, ... of the range. Each warp keeps a ring of NS stages in shared memory: the packed
// 32-token block arrives by a bulk copy (TMA engine, mbarrier completion) and its P values by
// 4-byte asynchronous copies. Per block and head the warp updates a running maximum (online
// softmax: a new maximum rescales the accumulators), computes one exp per (head, token) and
// stages the weights exp(P - m) |v| as fp16 hi + lo columns. The codes are dequantized
// straight into fp16 MMA A fragments (rows = coordinates, K = tokens) through a per-lane
// table that maps a 2B-bit field (two tokens' codes of one coordinate) to a half2 of
// centroids, and multiplied on the tensor cores. The 8 warps meet at the CTA's maximum;
// partial sums, maxima and denominators go to the workspace.
// Kernel 2 (merge): a cluster of four CTAs per query head (one CTA for D = 256) combines the
// partials (log-sum-exp rescale) and rotates by Pi^T.
#include <cooperative_groups.h>

#include "tq_device.cuh"

namespace {

constexpr int kPvWarps = 8;
constexpr int kPvNS = 3;              // ring stages per warp
constexpr uint32_t kWaitLimit = 1u << 22;
constexpr int kPRow = 40;             // floats per staged P row (32 used; 40 spreads the banks)

template <int B, int KT, int NT>
constexpr size_t pv_smem_bytes() {
    return (size_t)(1 << (2 * B)) * 128 + (size_t)kPvWarps * kPvNS * (512 * (KT * B / 8) + 64) +
           (size_t)kPvWarps * kPvNS * 4 * NT * kPRow * 4;
}

template <int B, int KT, int NT>  // KT = D/16 coordinate tiles, NT = n-tiles of 4 heads
__global__ void __launch_bounds__(kPvWarps * 32, KT == 8 ? 2 : 1) k_pv_split(PvParams p) {
    constexpr int NS = kPvNS;
    constexpr int E = 1 << (2 * B);          // table entries
    constexpr int CH = KT * B / 8;           // 16-byte chunks per lane per block (D*B/128)
    constexpr int NW = 4 * CH;               // 32-bit words per lane per block
    constexpr uint32_t SEC_A = 512u * CH;    // codes; 32 fp16 norms follow
    constexpr uint32_t BBYTES = SEC_A + 64u;
    constexpr int HP = 4 * NT;               // heads, padded to whole n-tiles
    extern __shared__ __align__(128) uint8_t smem[];
    uint32_t* lut = reinterpret_cast<uint32_t*>(smem);                              // [E][32]
    uint8_t* ring = smem + (size_t)E * 128;                                          // [warp][NS][BBYTES]
    float* pring = reinterpret_cast<float*>(ring + (size_t)kPvWarps * NS * BBYTES);  // [warp][NS][HP][kPRow]
    __shared__ float s_acc[HP][KT * 16];
    __shared__ float s_m[kPvWarps][HP], s_l[HP];
    __shared__ uint64_t bars[kPvWarps][NS];

    const int G = p.g;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int64_t stream = blockIdx.x / p.nsplit;
    const int split = blockIdx.x % p.nsplit;
    const int64_t b0 = (int64_t)split * p.blocks_per_split;
    const int64_t b1 = min(b0 + p.blocks_per_split, p.nb);
    const float* Pst = p.P + (size_t)stream * G * p.n_tok;
    const uint8_t* sbase = p.packed + (size_t)stream * p.nb * BBYTES;

    for (int e = threadIdx.x; e < E * 8; e += blockDim.x) {   // 32 equal words per entry
        const int ent = e >> 3;
        const uint32_t v = p.cb.lut_half[ent & ((1 << B) - 1)] | (p.cb.lut_half[ent >> B] << 16);
        reinterpret_cast<uint4*>(lut)[e] = make_uint4(v, v, v, v);
    }
    for (int e = threadIdx.x; e < HP * KT * 16; e += blockDim.x) (&s_acc[0][0])[e] = 0.f;
    if (threadIdx.x < HP) s_l[threadIdx.x] = 0.f;
    if (lane == 0)
        for (int s = 0; s < NS; ++s) tq_mbar_init(&bars[w][s], 1);
    tq_fence_mbar_init();
    __syncthreads();

    uint8_t* my_ring = ring + (size_t)w * NS * BBYTES;
    float* my_p = pring + (size_t)w * NS * HP * kPRow;
    const int64_t first = b0 + w;
    const int nmine = first < b1 ? (int)((b1 - first + kPvWarps - 1) / kPvWarps) : 0;
    // block k of this warp (first + 4k) into stage k % NS; every lane commits one copy group.
    // The lane's P pointer (head 0, token 32 (first + 4k) + lane) advances by 128 tokens a block.
    const float* pk = Pst + first * 32 + lane;
    const uint8_t* vk = sbase + (size_t)first * BBYTES;
    auto issue = [&](int k) {
        if (k < nmine) {
            const int s = k % NS;
            if (lane == 0) tq_bulk_load(my_ring + s * BBYTES, vk, BBYTES, &bars[w][s]);
            const bool in = (first + (int64_t)kPvWarps * k) * 32 + lane < p.n_tok;
            float* dst = my_p + s * HP * kPRow + lane;
#pragma unroll
            for (int h = 0; h < HP; ++h)
                if (h < G) tq_cp_async4(dst + h * kPRow, in ? pk + (size_t)h * p.n_tok : p.P, in ? 4u : 0u);
            pk += 32 * kPvWarps;
            vk += (size_t)kPvWarps * BBYTES;
        }
        tq_cp_async_commit();
    };
    for (int k = 0; k < NS; ++k) issue(k);

    float acc[KT][NT][4];
#pragma unroll
    for (int k = 0; k < KT; ++k)
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int r = 0; r < 4; ++r) acc[k][n][r] = 0.f;
    // Thread (g, t) feeds column g of each n-tile n of the B operand: head hb = 4n + g/2, the
    // fp16 hi (g even) or lo (g odd) part of its weights exp(P - m) |v| for the tokens
    // 2t, 2t+1, 2t+8, 2t+9, 16+2t, 17+2t, 24+2t, 25+2t of the block (the K rows of its B
    // fragments). m_run / ml2 / lsum belong to head hb; the accumulator columns 2t, 2t+1 of
    // n-tile n belong to head 4n + t, whose rescale factor comes from lane 8t.
    float m_run[NT], ml2[NT], lsum[NT];
#pragma unroll
    for (int n = 0; n < NT; ++n) { m_run[n] = -INFINITY; ml2[n] = -INFINITY; lsum[n] = 0.f; }
    constexpr float kLog2e = 1.4426950408889634f;
    const uint32_t lane4 = (uint32_t)lane * 4u;
    const bool lo_col = (g & 1) != 0;

    bool ok = true;
    int k = 0;
    for (; k < nmine; ++k) {
        const int s = k % NS;
        tq_cp_async_wait<NS - 1>();   // this lane's P copies of block k have landed
        ok = __all_sync(0xffffffffu, tq_mbar_wait(&bars[w][s], (uint32_t)(k / NS) & 1u, kWaitLimit));
        if (!ok) break;
        __syncwarp();                 // and those of the other lanes are visible
        const uint8_t* bp = my_ring + s * BBYTES;
        const int64_t tok0 = (first + (int64_t)kPvWarps * k) * 32;
        const int64_t rem = p.n_tok - tok0;
        const int nval = rem < 32 ? (int)rem : 32;   // valid tokens of the block
        // norms of the thread's 8 tokens (pairs 2t + 8j, +1)
        float nrm[8];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            const uint32_t nw = reinterpret_cast<const uint32_t*>(bp + SEC_A)[4 * jj + t];
            nrm[2 * jj] = tq_half_val(nw & 0xffffu);
            nrm[2 * jj + 1] = tq_half_val(nw >> 16);
        }
        uint32_t bw[NT][2][2];
        float fac_b[NT];
        bool grew = false;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            const int hb = 4 * n + (g >> 1);
            fac_b[n] = 1.f;
            float pv[8];
            const float* prow = my_p + (s * HP + (hb < G ? hb : 0)) * kPRow + 2 * t;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const float2 v2 = *reinterpret_cast<const float2*>(prow + 8 * jj);
                const int tt = 8 * jj + 2 * t;
                pv[2 * jj] = (hb < G && tt < nval) ? v2.x : -INFINITY;
                pv[2 * jj + 1] = (hb < G && tt + 1 < nval) ? v2.y : -INFINITY;
            }
            float bm = fmaxf(fmaxf(fmaxf(pv[0], pv[1]), fmaxf(pv[2], pv[3])), fmaxf(fmaxf(pv[4], pv[5]), fmaxf(pv[6], pv[7])));
            bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 1));
            bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 2));
            if (bm > m_run[n]) {
                fac_b[n] = tq_exp2((m_run[n] - bm) * kLog2e);   // 0 while the maximum was -inf
                lsum[n] *= fac_b[n];
                m_run[n] = bm;
                ml2[n] = bm * kLog2e;
                grew = true;
            }
            float wv[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float ex = m_run[n] > -INFINITY ? tq_exp2(fmaf(pv[e], kLog2e, -ml2[n])) : 0.f;
                lsum[n] += ex;
                wv[e] = ex * nrm[e];
            }
            // fp16 hi, or the lo remainder, of the weights as the B fragments of both K halves
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const __half2 hi = __floats2half2_rn(wv[2 * q], wv[2 * q + 1]);
                uint32_t v;
                if (lo_col) {
                    const float2 hf = __half22float2(hi);
                    const __half2 lo = __floats2half2_rn(wv[2 * q] - hf.x, wv[2 * q + 1] - hf.y);
                    v = *reinterpret_cast<const uint32_t*>(&lo);
                } else {
                    v = *reinterpret_cast<const uint32_t*>(&hi);
                }
                bw[n][q >> 1][q & 1] = v;
            }
        }
        if (__any_sync(0xffffffffu, grew)) {
            // accumulator columns 2t, 2t + 1 of n-tile n belong to head 4n + t (factor at lane 8t)
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                const float f = __shfl_sync(0xffffffffu, fac_b[n], 8 * t);
#pragma unroll
                for (int kk = 0; kk < KT; ++kk)
#pragma unroll
                    for (int r = 0; r < 4; ++r) acc[kk][n][r] *= f;
            }
        }
        uint32_t W[NW + 1];
#pragma unroll
        for (int c = 0; c < CH; ++c) {
            const uint4 v = *reinterpret_cast<const uint4*>(bp + (c * 32 + lane) * 16);
            W[4 * c] = v.x; W[4 * c + 1] = v.y; W[4 * c + 2] = v.z; W[4 * c + 3] = v.w;
        }
        W[NW] = 0u;
        // A fragments: field (a, pp) at bit (4a + pp) * 2B of the lane string
#pragma unroll
        for (int kk = 0; kk < KT; ++kk)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t a[4];
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    // r: 0 -> (a=2kk, pp=2c), 1 -> (2kk+1, 2c), 2 -> (2kk, 2c+1), 3 -> (2kk+1, 2c+1)
                    const int f = 4 * (2 * kk + (r & 1)) + 2 * c + (r >> 1);
                    const int bit = f * 2 * B;
                    const int wi = bit >> 5, sh = bit & 31;
                    // the field lands at bits 7.., i.e. already times the 128-byte entry stride
                    // (fields start below bit 7 only when they lie inside one word)
                    const uint32_t x = sh >= 7 ? __funnelshift_r(W[wi], W[wi + 1], sh - 7) : W[wi] << (7 - sh);
                    const uint32_t off = (x & ((uint32_t)(E - 1) << 7)) | lane4;
                    a[r] = *reinterpret_cast<const uint32_t*>(reinterpret_cast<const uint8_t*>(lut) + off);
                }
#pragma unroll
                for (int n = 0; n < NT; ++n) tq_hmma(acc[kk][n], a[0], a[1], a[2], a[3], bw[n][c][0], bw[n][c][1]);
            }
        // the stage is consumed: refill it with block k + NS
        __syncwarp();
        if (lane == 0) tq_fence_proxy_async();
        issue(k + NS);
    }
    tq_cp_async_wait<0>();
    if (!ok) {
        // a wait ran out: record it and give the copies in flight a bounded time to land
        if (lane == 0) {
            tq_raise(p.status, TQ_FLAG_TIMEOUT);
            for (int j = k; j < min(k + NS, nmine); ++j)
                tq_mbar_wait(&bars[w][j % NS], (uint32_t)(j / NS) & 1u, kWaitLimit);
        }
        __syncwarp();
    }
    // the CTA's maximum per head; each warp's sums are rescaled to it. Head h's running
    // maximum is held by the lanes whose B column belongs to it (lane 8 (h mod 4) of n-tile h / 4).
    if (t == 0 && (g & 1) == 0)
#pragma unroll
        for (int n = 0; n < NT; ++n) s_m[w][4 * n + (g >> 1)] = m_run[n];
    __syncthreads();
    float scl_b[NT];
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        const int hb = 4 * n + (g >> 1);
        float M = s_m[0][hb];
#pragma unroll
        for (int v = 1; v < kPvWarps; ++v) M = fmaxf(M, s_m[v][hb]);
        scl_b[n] = m_run[n] > -INFINITY ? __expf(m_run[n] - M) : 0.f;
    }
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        const int head = n * 4 + t;
        const float f = __shfl_sync(0xffffffffu, scl_b[n], 8 * t);
        if (head < G) {
#pragma unroll
            for (int kk = 0; kk < KT; ++kk) {
                atomicAdd(&s_acc[head][16 * kk + g], f * (acc[kk][n][0] + acc[kk][n][1]));
                atomicAdd(&s_acc[head][16 * kk + 8 + g], f * (acc[kk][n][2] + acc[kk][n][3]));
            }
        }
    }
    // denominators: the hi lanes of a head (t = 0..3) hold its 32 tokens between them
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        float ls = (g & 1) == 0 ? lsum[n] * scl_b[n] : 0.f;
        ls += __shfl_xor_sync(0xffffffffu, ls, 1);
        ls += __shfl_xor_sync(0xffffffffu, ls, 2);
        const int hb = 4 * n + (g >> 1);
        if (t == 0 && (g & 1) == 0 && hb < G) atomicAdd(&s_l[hb], ls);
    }
    __syncthreads();
    const int D = KT * 16;
    for (int e = threadIdx.x; e < G * D; e += blockDim.x) {
        const int h = e / D, i = e % D;
        p.part[(((size_t)stream * G + h) * p.nsplit + split) * D + i] = s_acc[h][i];
    }
    if (threadIdx.x < G) {
        const int h = threadIdx.x;
        float M = s_m[0][h];
        for (int v = 1; v < kPvWarps; ++v) M = fmaxf(M, s_m[v][h]);
        float2* ml = reinterpret_cast<float2*>(p.part_ml);
        ml[((size_t)stream * G + h) * p.nsplit + split] = make_float2(M, s_l[h]);
    }
}

constexpr int kMergeThreads = 256;

// D = 128: one cluster of four CTAs per query head,
//   out = Pi^T sum_s e^{m_s - M} part_s / sum_s e^{m_s - M} l_s.
// CTA r owns rotated and output coordinates 32 r .. 32 r + 31. Thread (group, quad) folds
// every 32nd range (its quad of the partial) under its own running maximum, every load issued
// before any is used; all four CTAs read every range maximum in the same order, so M and the
// denominator come out identical in each. The quarters of o meet through distributed shared
// memory and CTA r rotates its 32 outputs with its 32 rows of Pi^T (loaded at the start).
constexpr int kMergeCtas = 4;
constexpr int kMergeGroups = 32;   // x 8 coordinate quads = the CTA's 32 coordinates

__global__ void __cluster_dims__(kMergeCtas, 1, 1) __launch_bounds__(kMergeThreads) k_pv_merge4(PvParams p) {
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    const int d = p.t.d, ns = p.nsplit;
    const int r = (int)cluster.block_rank();
    const int64_t hq = blockIdx.x / kMergeCtas;   // stream * g + head
    __shared__ __align__(16) float s_acc[kMergeGroups * 32];
    __shared__ __align__(16) float s_o[128];
    __shared__ float s_w[kMergeGroups], s_gm[kMergeGroups], s_gl[kMergeGroups], s_den;
    const int tid = threadIdx.x, grp = tid >> 3, qd = tid & 7;
    const int c0 = 32 * r + 4 * qd;
    const int jr = 32 * r + (tid >> 3), er = tid & 7;
    float4 wrow[4];
    {
        const float4* rowp = reinterpret_cast<const float4*>(p.piT + (size_t)jr * 128 + er * 16);
#pragma unroll
        for (int k = 0; k < 4; ++k) wrow[k] = __ldg(rowp + k);
    }
    const float2* ml = reinterpret_cast<const float2*>(p.part_ml) + (size_t)hq * ns;
    const float4* src = reinterpret_cast<const float4*>(p.part + (size_t)hq * ns * 128 + c0);
    float m = -INFINITY, l = 0.f;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    constexpr int RB = 8;
    for (int s0 = grp; s0 < ns; s0 += RB * kMergeGroups) {
        float2 v[RB];
        float4 x[RB];
#pragma unroll
        for (int u = 0; u < RB; ++u) {
            const int s = s0 + u * kMergeGroups;
            v[u] = s < ns ? ml[s] : make_float2(-INFINITY, 0.f);
            x[u] = s < ns ? src[(size_t)s * 32] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        float mn = m;
#pragma unroll
        for (int u = 0; u < RB; ++u) mn = v[u].y > 0.f ? fmaxf(mn, v[u].x) : mn;
        if (mn > -INFINITY) {   // a range with weight (every range wrote its partial)
            const float so = __expf(m - mn);
            a.x *= so; a.y *= so; a.z *= so; a.w *= so;
            l *= so;
#pragma unroll
            for (int u = 0; u < RB; ++u) {
                const float sn = v[u].y > 0.f ? __expf(v[u].x - mn) : 0.f;
                a.x = fmaf(sn, x[u].x, a.x); a.y = fmaf(sn, x[u].y, a.y);
                a.z = fmaf(sn, x[u].z, a.z); a.w = fmaf(sn, x[u].w, a.w);
                l = fmaf(sn, v[u].y, l);
            }
            m = mn;
        }
    }
    reinterpret_cast<float4*>(s_acc)[grp * 8 + qd] = a;
    if (qd == 0) { s_gm[grp] = m; s_gl[grp] = l; }
    __syncthreads();
    if (tid < 32) {   // group weights under the common maximum, and the denominator
        const float gm = s_gm[tid];
        float M = gm;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        const float w = gm > -INFINITY ? __expf(gm - M) : 0.f;
        float den = w * s_gl[tid];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
        s_w[tid] = w;
        if (tid == 0) s_den = den;
    }
    __syncthreads();
    if (tid < 32) {   // this CTA's quarter of o
        float v = 0.f;
#pragma unroll 8
        for (int q = 0; q < kMergeGroups; ++q) v = fmaf(s_w[q], s_acc[q * 32 + tid], v);
        s_o[32 * r + tid] = v;
    }
    cluster.sync();   // every quarter of o is written
    if (tid < 128 && (tid >> 5) != r) {
        const float* peer = cluster.map_shared_rank(s_o, (int)(tid >> 5));
        s_o[tid] = peer[tid];
    }
    cluster.sync();   // o is complete here, and no CTA leaves while a peer still reads it
    // out[j] = <row j of Pi^T, o> / den (its columns i >= d are zero); the eight parts of a row
    // meet by shuffles
    float acc = 0.f;
    const float4* op = reinterpret_cast<const float4*>(s_o + er * 16);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float4 w = wrow[k], o = op[k];
        acc = fmaf(w.x, o.x, fmaf(w.y, o.y, fmaf(w.z, o.z, fmaf(w.w, o.w, acc))));
    }
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    acc += __shfl_xor_sync(0xffffffffu, acc, 4);
    if (er == 0 && jr < d) p.out[(size_t)hq * d + jr] = acc / s_den;
}

// D = 256: one CTA per query head: o = sum_s e^{m_s - M} part_s / sum_s e^{m_s - M} l_s,
// then Pi^T o. Every global load of the partials is issued in one round: thread (group,
// coordinate quad) reads the maxima, sums and partial quads of every ngrp-th range and folds
// them under its own running maximum; the groups then meet in shared memory under the common
// one.
__global__ void __launch_bounds__(kMergeThreads) k_pv_merge256(PvParams p) {
    constexpr int D = 256;
    const int d = p.t.d, ns = p.nsplit;
    const int64_t hq = blockIdx.x;   // stream * g + head
    __shared__ __align__(16) float s_acc[kMergeThreads * 4];   // [group][D]
    __shared__ __align__(16) float s_o[256];
    __shared__ float s_gm[8], s_gl[8];
    const int tid = threadIdx.x;
    constexpr int nq = D / 4, ngrp = kMergeThreads / nq;
    const int grp = tid / nq, qd = tid % nq;
    const float2* ml = reinterpret_cast<const float2*>(p.part_ml) + (size_t)hq * ns;
    const float4* src = reinterpret_cast<const float4*>(p.part + (size_t)hq * ns * D) + qd;
    float m = -INFINITY, l = 0.f;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
    // batches whose loads are all issued before any is used; one rescale per batch
    constexpr int RB = 8;
    for (int s0 = grp; s0 < ns; s0 += RB * ngrp) {
        float2 v[RB];
        float4 x[RB];
#pragma unroll
        for (int u = 0; u < RB; ++u) {
            const int s = s0 + u * ngrp;
            v[u] = s < ns ? ml[s] : make_float2(-INFINITY, 0.f);
            x[u] = s < ns ? src[(size_t)s * nq] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        float mn = m;
#pragma unroll
        for (int u = 0; u < RB; ++u) mn = v[u].y > 0.f ? fmaxf(mn, v[u].x) : mn;
        if (mn > -INFINITY) {   // a range with weight (every range wrote its partial)
            const float so = __expf(m - mn);
            a.x *= so; a.y *= so; a.z *= so; a.w *= so;
            l *= so;
#pragma unroll
            for (int u = 0; u < RB; ++u) {
                const float sn = v[u].y > 0.f ? __expf(v[u].x - mn) : 0.f;
                a.x = fmaf(sn, x[u].x, a.x); a.y = fmaf(sn, x[u].y, a.y);
                a.z = fmaf(sn, x[u].z, a.z); a.w = fmaf(sn, x[u].w, a.w);
                l = fmaf(sn, v[u].y, l);
            }
            m = mn;
        }
    }
    reinterpret_cast<float4*>(s_acc)[grp * nq + qd] = a;
    if (qd == 0) { s_gm[grp] = m; s_gl[grp] = l; }
    __syncthreads();
    float M = -INFINITY;
    for (int q = 0; q < ngrp; ++q) M = fmaxf(M, s_gm[q]);
    float den = 0.f;
    for (int q = 0; q < ngrp; ++q) den += s_gm[q] > -INFINITY ? __expf(s_gm[q] - M) * s_gl[q] : 0.f;
    for (int i = tid; i < D; i += kMergeThreads) {
        float v = 0.f;
        for (int q = 0; q < ngrp; ++q)
            if (s_gm[q] > -INFINITY) v = fmaf(__expf(s_gm[q] - M), s_acc[q * D + i], v);
        s_o[i] = v;
    }
    __syncthreads();
    const float inv = 1.f / den;
    // out[j] = sum_i Pi[i][j] o_i = <row j of Pi^T, o> (its columns i >= d are zero): pairs
    // (j, half) with 16-byte loads of the row, the halves joined by a shuffle of neighbouring
    // lanes; the block-uniform trip count keeps warps whole
    const int hl = D / 2;
    for (int e0 = 0; e0 < 2 * d; e0 += kMergeThreads) {
        const int e = e0 + tid, j = e >> 1, hf = e & 1;
        const bool valid = e < 2 * d;
        float acc = 0.f;
        if (valid) {
            const float4* rowp = reinterpret_cast<const float4*>(p.piT + (size_t)j * D + hf * hl);
            const float4* op = reinterpret_cast<const float4*>(s_o + hf * hl);
#pragma unroll 16
            for (int k = 0; k < hl / 4; ++k) {
                const float4 w = __ldg(rowp + k), o = op[k];
                acc = fmaf(w.x, o.x, fmaf(w.y, o.y, fmaf(w.z, o.z, fmaf(w.w, o.w, acc))));
            }
        }
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        if (valid && hf == 0) p.out[(size_t)hq * d + j] = acc * inv;
    }
}

template <int B, int KT, int NT>
cudaError_t launch_split(const PvParams& p, cudaStream_t st) {
    constexpr size_t smem = pv_smem_bytes<B, KT, NT>();
    auto kern = k_pv_split<B, KT, NT>;
    static TqLaunchCache cache;
    cudaError_t e = tq_kernel_setup(kern, kPvWarps * 32, smem, cache, nullptr, nullptr);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(p.n_streams * p.nsplit), kPvWarps * 32, smem, st>>>(p);
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
    if (p.t.D == 128) k_pv_merge4<<<(unsigned)(p.n_streams * p.g * kMergeCtas), kMergeThreads, 0, st>>>(p);
    else k_pv_merge256<<<(unsigned)(p.n_streams * p.g), kMergeThreads, 0, st>>>(p);
    return cudaGetLastError();
}
