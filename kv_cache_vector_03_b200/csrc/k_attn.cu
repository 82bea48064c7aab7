// tq_attention: decode attention softmax(scale q . K) . V in one pass over compressed keys
// and values (a2a-mcp.org "What is TurboQuant", the fused-kernel note: scores straight from the
// indices with the query rotated once; friday-blog-bgf.pages.dev "TurboQuant deep dive II",
// section 1, step 1: values keep the rotation + scalar quantizer; blog.hotdry.top "TurboQuant
// vector-search compression", engineering configuration list: the most recent tokens stay at
// full precision).
//
// The logits never leave the SM. Kernel 1 is the logits prologue (query fragments, exact tail
// logits). Kernel 2 (split): one CTA of 8 warps per (stream, block range); per 32-token block
// a warp receives the key block and the value block in one ring stage (two bulk copies, one
// mbarrier), computes the 32 x 4 logits on the int8 tensor cores (bit planes, as tq_logits),
// keeps a running maximum and sum per head (online softmax), turns exp(l - m) |v| into fp16
// hi + lo MMA columns and accumulates the values, decoded through per-lane half2 tables, on the
// fp16 tensor cores (as tq_pv). Kernel 3 (merge): a cluster of four CTAs per query head combines
// the ranges (log-sum-exp), rotates the value sum by Pi^T once and adds the exact tail.
#include <cooperative_groups.h>

#include <algorithm>
#include <cfloat>

#include "tq_device.cuh"

namespace {

__device__ __forceinline__ uint32_t q8_pack4(int a, int b, int c, int d) {
    return (uint32_t)(a & 0xff) | ((uint32_t)(b & 0xff) << 8) | ((uint32_t)(c & 0xff) << 16) |
           ((uint32_t)(d & 0xff) << 24);
}

constexpr int kAttnWarps = 8;
constexpr int kAttnNS = 2;             // ring stages per warp (key + value block each)
constexpr uint32_t kWaitLimit = 1u << 22;
constexpr int kWCol = 20;              // words per staged weight column (16 used)

template <int BK, int BV>
constexpr uint32_t attn_stage_bytes() {
    return (512u * (BK + 1) + 128u) + (512u * BV + 64u);   // key block (d = m = 128) + value block
}
template <int BK, int BV>
constexpr size_t attn_smem() {
    return (size_t)(1 << (2 * BV)) * 128 + (size_t)kAttnWarps * kAttnNS * attn_stage_bytes<BK, BV>();
}

__device__ __forceinline__ size_t qf_word(int64_t stream, int nmg, int mg, int c, int lane) {
    return (((size_t)stream * nmg + mg) * 4 + c) * 64 + lane * 2;
}

// order-preserving map between floats and ints, for integer atomicMax on float maxima
__device__ __forceinline__ int ord_of(float f) {
    const int i = __float_as_int(f);
    return i >= 0 ? i : i ^ 0x7fffffff;
}
__device__ __forceinline__ float float_of(int i) { return __int_as_float(i >= 0 ? i : i ^ 0x7fffffff); }

// The value side of one 32-token block: B fragments from the staged weights (column g = head
// g/2, hi or lo part; token pairs), A fragments decoded through the per-lane half2 tables from
// the value block's two-token fields, accumulated on the fp16 tensor cores (rows = 128
// rotated coordinates in 8 tiles of 16, K = the 32 tokens).
template <int BV>
__device__ __forceinline__ void attn_values(float (&acc)[8][4], const uint32_t (&wst)[8][kWCol], const uint8_t* vb,
                                            const uint32_t* lut, int lane) {
    constexpr int KT = 8, CH = KT * BV / 8, NW = 4 * CH, E = 1 << (2 * BV);
    const int g = lane >> 2, t = lane & 3;
    const uint32_t lane4 = (uint32_t)lane * 4u;
    uint32_t bw[2][2];
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int hv2 = 0; hv2 < 2; ++hv2) bw[c][hv2] = wst[g][8 * c + 4 * hv2 + t];
    uint32_t W[NW + 1];
#pragma unroll
    for (int c = 0; c < CH; ++c) {
        const uint4 v = *reinterpret_cast<const uint4*>(vb + (c * 32 + lane) * 16);
        W[4 * c] = v.x; W[4 * c + 1] = v.y; W[4 * c + 2] = v.z; W[4 * c + 3] = v.w;
    }
    W[NW] = 0u;
#pragma unroll
    for (int kt = 0; kt < KT; ++kt)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            uint32_t a[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                // field (a, pp) at bit (4a + pp) * 2BV of the lane string; the field lands at
                // bits 7.., i.e. already times the 128-byte entry stride
                const int f = 4 * (2 * kt + (r & 1)) + 2 * c + (r >> 1);
                const int bit = f * 2 * BV;
                const int wi = bit >> 5, sh = bit & 31;
                const uint32_t x = sh >= 7 ? __funnelshift_r(W[wi], W[wi + 1], sh - 7) : W[wi] << (7 - sh);
                const uint32_t off = (x & ((uint32_t)(E - 1) << 7)) | lane4;
                a[r] = *reinterpret_cast<const uint32_t*>(reinterpret_cast<const uint8_t*>(lut) + off);
            }
            tq_hmma(acc[kt], a[0], a[1], a[2], a[3], bw[c][0], bw[c][1]);
        }
}

template <int BK, int BV>   // key MSE bits (1..3), value bits (1..4); d <= 128, m <= 128, g <= 4
__global__ void __launch_bounds__(kAttnWarps * 32, 2) k_attn_split(AttnParams p) {
    constexpr int NS = kAttnNS;
    constexpr int NP = BK == 3 ? 4 : BK;   // estimator code planes
    constexpr int NPG = BK + 1;            // stored key plane groups (one 128-coordinate group each)
    constexpr int NMG = NP + 1;            // MMA plane groups
    constexpr uint32_t BBK = 512u * NPG + 128u;
    constexpr int KT = 8, CH = KT * BV / 8;
    constexpr uint32_t SEC_AV = 512u * CH;
    constexpr uint32_t STG = attn_stage_bytes<BK, BV>();
    constexpr int E = 1 << (2 * BV);
    extern __shared__ __align__(128) uint8_t smem[];
    uint32_t* lut = reinterpret_cast<uint32_t*>(smem);        // [E][32]
    uint8_t* ring = smem + (size_t)E * 128;                    // [warp][NS][STG]
    __shared__ uint32_t wst[kAttnWarps][8][kWCol];             // column 2 head + part: token pairs
    __shared__ float s_acc[4][KT * 16];
    __shared__ float s_m[kAttnWarps][4], s_l[kAttnWarps][4];
    __shared__ int s_cmax[4];   // CTA-wide running maximum per head (order-preserving int image)
    __shared__ uint64_t bars[kAttnWarps][NS];

    const int G = p.g;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;   // MMA fragment coordinates; t is this thread's head
    const int64_t stream = blockIdx.x / p.nsplit;
    const int split = blockIdx.x % p.nsplit;
    const int64_t b0 = (int64_t)split * p.blocks_per_split;
    const int64_t b1 = min(b0 + p.blocks_per_split, p.nb);

    for (int e = threadIdx.x; e < E * 8; e += blockDim.x) {   // 32 equal words per entry
        const int ent = e >> 3;
        const uint32_t v = p.cbv.lut_half[ent & ((1 << BV) - 1)] | (p.cbv.lut_half[ent >> BV] << 16);
        reinterpret_cast<uint4*>(lut)[e] = make_uint4(v, v, v, v);
    }
    for (int e = threadIdx.x; e < 4 * KT * 16; e += blockDim.x) (&s_acc[0][0])[e] = 0.f;
    if (threadIdx.x < 4) s_cmax[threadIdx.x] = ord_of(-INFINITY);
    if (lane == 0)
        for (int s = 0; s < NS; ++s) tq_mbar_init(&bars[w][s], 2);
    tq_fence_mbar_init();
    __syncthreads();

    uint8_t* my_ring = ring + (size_t)w * NS * STG;
    const int64_t first = b0 + w;
    const int nmine = first < b1 ? (int)((b1 - first + kAttnWarps - 1) / kAttnWarps) : 0;
    const uint8_t* kk = p.packed_k + ((size_t)stream * p.nb + first) * BBK;
    const uint8_t* vk = p.packed_v + ((size_t)stream * p.nb + first) * p.tv.block_bytes;
    auto issue = [&](int k) {
        if (k < nmine && lane == 0) {
            const int s = k % NS;
            tq_bulk_load(my_ring + s * STG, kk, BBK, &bars[w][s]);
            tq_bulk_load(my_ring + s * STG + BBK, vk, (uint32_t)p.tv.block_bytes, &bars[w][s]);
        }
        if (k < nmine) {
            kk += (size_t)kAttnWarps * BBK;
            vk += (size_t)kAttnWarps * p.tv.block_bytes;
        }
    };
    for (int k = 0; k < NS; ++k) issue(k);

    // the copies above read only the caches; the query fragments come from the prologue
    tq_pdl_wait();
    uint32_t qf[NMG][4][2];
#pragma unroll
    for (int mg = 0; mg < NMG; ++mg)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const uint2 v = *reinterpret_cast<const uint2*>(p.qfrag + qf_word(stream, NMG, mg, c, lane));
            qf[mg][c][0] = v.x;
            qf[mg][c][1] = v.y;
        }
    const float4 sc = reinterpret_cast<const float4*>(p.qscale)[(size_t)stream * 4 + t];
    const bool hv = t < G;
    constexpr float kLog2e = 1.4426950408889634f;

    float acc[KT][4];
#pragma unroll
    for (int i = 0; i < KT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    float m_run = -INFINITY, lsum = 0.f;   // head t: the same m in the 8 lanes of the head

    bool ok = true;
    int k = 0;
    for (; k < nmine; ++k) {
        const int s = k % NS;
        ok = __all_sync(0xffffffffu, tq_mbar_wait(&bars[w][s], (uint32_t)(k / NS) & 1u, kWaitLimit));
        if (!ok) break;
        const uint8_t* kb = my_ring + s * STG;
        const uint8_t* vb = kb + BBK;
        const int64_t blk = first + (int64_t)kAttnWarps * k;

        // ---- logits of the 32 keys for head t: keys 8u + g, u = 0..3
        const uint4 nrm4 = *reinterpret_cast<const uint4*>(kb + NPG * 512 + g * 16);
        const uint32_t nrm[4] = {nrm4.x, nrm4.y, nrm4.z, nrm4.w};
        float l[4];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            // words of rows g and g + 8 of this m-tile, one pair per stored plane group
            uint2 cur[NPG];
#pragma unroll
            for (int pg = 0; pg < NPG; ++pg)
                cur[pg] = *reinterpret_cast<const uint2*>(kb + (pg * 32 + lane) * 16 + mt * 8);
            int accA[4], accA2[4], accS[4];
#pragma unroll
            for (int mg = 0; mg < NMG; ++mg) {
                uint32_t w0, w1;
                if (mg < NP && mg == 3) {   // b0 ^ b1 ^ b2
                    w0 = cur[0].x ^ cur[1].x ^ cur[2].x;
                    w1 = cur[0].y ^ cur[1].y ^ cur[2].y;
                } else {
                    const int pg = mg < NP ? mg : BK;
                    w0 = cur[pg].x;
                    w1 = cur[pg].y;
                }
                tq_expand_planes(w0, w1, [&](int c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3) {
                    const uint32_t q0 = qf[mg][c][0], q1 = qf[mg][c][1];
                    if (mg < NP) {
                        int(&a)[4] = (c & 1) ? accA : accA2;
                        if (mg == 0 && c >= 2) tq_imma_u8_z(a, a0, a1, a2, a3, q0, q1);
                        else tq_imma_u8(a, a0, a1, a2, a3, q0, q1);
                    } else {
                        if (c == 3) tq_imma_u8_z(accS, a0, a1, a2, a3, q0, q1);
                        else tq_imma_u8(accS, a0, a1, a2, a3, q0, q1);
                    }
                });
            }
#pragma unroll
            for (int r = 0; r < 4; ++r) accA[r] += accA2[r];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int u = 2 * mt + r;
                const uint32_t nw = nrm[u];
                const float nh = tq_half_val(nw & 0xffffu), gh = tq_half_val(nw >> 16);
                const float va = (float)(256 * accA[2 * r] + accA[2 * r + 1]);
                const float vs = (float)(256 * accS[2 * r] + accS[2 * r + 1]);
                const float est = fmaf(sc.x, va, -sc.y) + gh * fmaf(sc.z, vs, -sc.w);
                const bool in = hv && blk * 32 + 8 * u + g < p.n_tok;
                l[u] = in ? nh * est : -INFINITY;
            }
        }
        // ---- online softmax of head t over this block
        float bm = fmaxf(fmaxf(l[0], l[1]), fmaxf(l[2], l[3]));
        bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 4));
        bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 8));
        bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 16));
        // sparse values compare against the largest logit any warp of the CTA has seen (never
        // above the final maximum), so a warp skips from its first block on
        float cmax = bm;
        if (p.v_skip > 0.f) {
            if (g == 0) atomicMax(&s_cmax[t], ord_of(bm));
            cmax = fmaxf(bm, float_of(*reinterpret_cast<volatile int*>(&s_cmax[t])));
        }
        if (bm > m_run) {
            const float fac = tq_exp2((m_run - bm) * kLog2e);   // 0 while the maximum was -inf
#pragma unroll
            for (int i = 0; i < KT; ++i) {
                acc[i][0] *= fac; acc[i][1] *= fac; acc[i][2] *= fac; acc[i][3] *= fac;
            }
            lsum *= fac;
            m_run = bm;
        }
        const float ml2 = m_run * kLog2e;
        const uint16_t* vn = reinterpret_cast<const uint16_t*>(vb + SEC_AV);
        float ev[4];
        bool low = true;
        const float lthr = cmax + __logf(p.v_skip);   // -inf when v_skip = 0
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            ev[u] = m_run > -INFINITY ? tq_exp2(fmaf(l[u], kLog2e, -ml2)) : 0.f;
            lsum += ev[u];
            low = low && (l[u] < lthr || l[u] == -INFINITY);
        }
        // sparse values: every weight of the block is below v_skip relative to the CTA's
        // running maximum (so also to the final one): the softmax sum keeps them, the values
        // are skipped
        if (__all_sync(0xffffffffu, low)) {
            __syncwarp();
            if (lane == 0) tq_fence_proxy_async();
            issue(k + NS);
            continue;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int tok = 8 * u + g;
            const float wt = ev[u] * tq_half_val(vn[tok]);
            const __half hi = __float2half_rn(wt);
            reinterpret_cast<__half*>(&wst[w][2 * t][0])[tok] = hi;
            reinterpret_cast<__half*>(&wst[w][2 * t + 1][0])[tok] = __float2half_rn(wt - __half2float(hi));
        }
        __syncwarp();
        attn_values<BV>(acc, wst[w], vb, lut, lane);
        // the stage is consumed: refill it
        __syncwarp();
        if (lane == 0) tq_fence_proxy_async();
        issue(k + NS);
    }
    if (!ok) {
        if (lane == 0) {
            tq_raise(p.status, TQ_FLAG_TIMEOUT);
            for (int j = k; j < min(k + NS, nmine); ++j)
                tq_mbar_wait(&bars[w][j % NS], (uint32_t)(j / NS) & 1u, kWaitLimit);
        }
        __syncwarp();
    }
    // the 8 lanes of head t hold parts of its sum
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 4);
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 8);
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 16);
    if (g == 0) { s_m[w][t] = m_run; s_l[w][t] = lsum; }
    __syncthreads();
    float M = s_m[0][t];
#pragma unroll
    for (int v = 1; v < kAttnWarps; ++v) M = fmaxf(M, s_m[v][t]);
    const float f = m_run > -INFINITY ? tq_exp2((m_run - M) * kLog2e) : 0.f;
    if (hv) {
#pragma unroll
        for (int kt = 0; kt < KT; ++kt) {
            atomicAdd(&s_acc[t][16 * kt + g], f * (acc[kt][0] + acc[kt][1]));
            atomicAdd(&s_acc[t][16 * kt + 8 + g], f * (acc[kt][2] + acc[kt][3]));
        }
    }
    __syncthreads();
    const int D = KT * 16;
    for (int e = threadIdx.x; e < G * D; e += blockDim.x) {
        const int h = e / D, i = e % D;
        p.part[(((size_t)stream * G + h) * p.nsplit + split) * D + i] = s_acc[h][i];
    }
    if (threadIdx.x < G) {
        const int h = threadIdx.x;
        float Mh = s_m[0][h], L = 0.f;
        for (int v = 1; v < kAttnWarps; ++v) Mh = fmaxf(Mh, s_m[v][h]);
        for (int v = 0; v < kAttnWarps; ++v)
            if (s_m[v][h] > -INFINITY) L += s_l[v][h] * tq_exp2((s_m[v][h] - Mh) * kLog2e);
        reinterpret_cast<float2*>(p.part_ml)[((size_t)stream * G + h) * p.nsplit + split] = make_float2(Mh, L);
    }
}

// One cluster of four CTAs per query head: the ranges and the exact tail under one maximum M,
//   out = (Pi^T sum_s e^{m_s - M} part_s + sum_t e^{l_t - M} v_t) / (sum_s e^{m_s - M} l_s + sum_t e^{l_t - M}).
// CTA r of the cluster owns rotated and output coordinates 32 r .. 32 r + 31. Thread (group,
// quad) folds every 32nd range (its quad of the rotated-domain partial) and every 32nd tail
// token (exact logit, 8-byte load of 4 bf16 value coordinates) under its own running maximum,
// every load issued before any is used. All four CTAs read every range maximum and tail
// logit in the same order, so M and the denominator come out identical in each. The quarters
// of the rotated-domain sum meet through distributed shared memory, and CTA r rotates its 32
// output coordinates with its 32 rows of Pi^T (loaded at the start).
constexpr int kMergeThreads = 256;
constexpr int kMergeCtas = 4;
constexpr int kMergeGroups = 32;   // x 8 coordinate quads = the CTA's 32 coordinates

__global__ void __cluster_dims__(kMergeCtas, 1, 1) __launch_bounds__(kMergeThreads) k_attn_merge(AttnParams p) {
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    const int d = p.tv.d, ns = p.nsplit, nt = p.n_tail;   // D = 128
    const int r = (int)cluster.block_rank();
    const int64_t hq = blockIdx.x / kMergeCtas;   // stream * g + head
    const int64_t stream = hq / p.g;
    __shared__ __align__(16) float s_acc[kMergeGroups * 32], s_tac[kMergeGroups * 32];
    __shared__ __align__(16) float s_o[128];
    __shared__ float s_t[32], s_w[kMergeGroups], s_gm[kMergeGroups], s_gl[kMergeGroups], s_den;
    const int tid = threadIdx.x, grp = tid >> 3, qd = tid & 7;
    const int c0 = 32 * r + 4 * qd;   // this thread's coordinate quad
    // rotation: output jr = 32 r + tid / 8, sixteen coordinates 16 er .. of its row of Pi^T
    const int jr = 32 * r + (tid >> 3), er = tid & 7;
    float4 wrow[4];
    {
        const float4* rowp = reinterpret_cast<const float4*>(p.piT_v + (size_t)jr * 128 + er * 16);
#pragma unroll
        for (int k = 0; k < 4; ++k) wrow[k] = __ldg(rowp + k);
    }
    const float2* ml = reinterpret_cast<const float2*>(p.part_ml) + (size_t)hq * ns;
    const float4* src = reinterpret_cast<const float4*>(p.part + (size_t)hq * ns * 128 + c0);
    float m = -INFINITY, l = 0.f;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = make_float4(0.f, 0.f, 0.f, 0.f);
    constexpr int RB = 4, TB = 4;
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
    const float* tl = p.tail_logit + (size_t)hq * nt;
    const uint2* tv = reinterpret_cast<const uint2*>(p.tail_v + (size_t)stream * nt * d) + c0 / 4;
    const bool qv = c0 / 4 < d / 4;
    for (int t0 = grp; t0 < nt; t0 += TB * kMergeGroups) {
        float lt[TB];
        uint2 vv[TB];
#pragma unroll
        for (int u = 0; u < TB; ++u) {
            const int tt = t0 + u * kMergeGroups;
            lt[u] = tt < nt ? tl[tt] : -INFINITY;
            vv[u] = tt < nt && qv ? __ldg(tv + (size_t)tt * (d / 4)) : make_uint2(0u, 0u);
        }
        float mn = m;
#pragma unroll
        for (int u = 0; u < TB; ++u) mn = fmaxf(mn, lt[u]);
        const float so = __expf(m - mn);   // m = -inf the first time: 0
        a.x *= so; a.y *= so; a.z *= so; a.w *= so;
        b.x *= so; b.y *= so; b.z *= so; b.w *= so;
        l *= so;
#pragma unroll
        for (int u = 0; u < TB; ++u) {
            const float sn = __expf(lt[u] - mn);   // 0 past the tail
            b.x = fmaf(sn, __uint_as_float(vv[u].x << 16), b.x);
            b.y = fmaf(sn, __uint_as_float(vv[u].x & 0xffff0000u), b.y);
            b.z = fmaf(sn, __uint_as_float(vv[u].y << 16), b.z);
            b.w = fmaf(sn, __uint_as_float(vv[u].y & 0xffff0000u), b.w);
            l += sn;
        }
        m = mn;
    }
    reinterpret_cast<float4*>(s_acc)[grp * 8 + qd] = a;
    reinterpret_cast<float4*>(s_tac)[grp * 8 + qd] = b;
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
    if (tid < 64) {   // this CTA's quarter of o (threads 0-31) and of the tail sum (32-63)
        const int i = tid & 31;
        const float* accp = tid < 32 ? s_acc : s_tac;
        float v = 0.f;
#pragma unroll 8
        for (int q = 0; q < kMergeGroups; ++q) v = fmaf(s_w[q], accp[q * 32 + i], v);
        if (tid < 32) s_o[32 * r + i] = v;
        else s_t[i] = v;
    }
    cluster.sync();   // every quarter of o is written
    if (tid < 128 && (tid >> 5) != r) {
        const float* peer = cluster.map_shared_rank(s_o, (int)(tid >> 5));
        s_o[tid] = peer[tid];
    }
    cluster.sync();   // o is complete here, and no CTA leaves while a peer still reads it
    // out[j] = (<row j of Pi^T, o> + t_j) / den; the eight parts of a row meet by shuffles
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
    if (er == 0 && jr < d) p.out[(size_t)hq * d + jr] = (acc + s_t[jr - 32 * r]) / s_den;
}

template <int BK, int BV>
cudaError_t launch_split(const AttnParams& p, cudaStream_t st) {
    constexpr size_t smem = attn_smem<BK, BV>();
    if (p.tk.block_bytes != 512u * (BK + 1) + 128u || p.tv.block_bytes != 512u * BV + 64u) return cudaErrorInvalidValue;
    auto kern = k_attn_split<BK, BV>;
    static TqLaunchCache cache;
    cudaError_t e = tq_kernel_setup(kern, kAttnWarps * 32, smem, cache, nullptr, nullptr);
    if (e != cudaSuccess) return e;
    return tq_launch_pdl(kern, dim3((unsigned)(p.n_streams * p.nsplit)), dim3(kAttnWarps * 32), smem, st, p);
}

template <int BK>
cudaError_t launch_bv(const AttnParams& p, cudaStream_t st) {
    switch (p.tv.B) {
        case 1: return launch_split<BK, 1>(p, st);
        case 2: return launch_split<BK, 2>(p, st);
        case 3: return launch_split<BK, 3>(p, st);
        case 4: return launch_split<BK, 4>(p, st);
    }
    return cudaErrorInvalidValue;
}


// ---------------------------------------------------------------------------------------
// Decode attention over 8-bit keys and TurboQuant values (the asymmetric K/V configuration of
// blog.hotdry.top "TurboQuant vector-search compression", engineering configuration list):
// the split kernel scores each 32-token block with dp4a on the int8 key codes (lane = token,
// the query heads as int16 fixed point in hi / lo bytes, exact int32 per 32-coordinate chunk,
// scaled per chunk, as tq_q8_logits), runs the online softmax of every head across the warp,
// stages exp(l - m) |v| as fp16 hi + lo and accumulates the values as the TurboQuant split
// kernel does; the first range of a stream also writes the exact logits of its bf16 tail.
// The merge is the same kernel.
template <int BV>
constexpr uint32_t q8_stage_bytes() {
    return kQ8Block + (512u * BV + 64u);
}
template <int BV>
constexpr size_t q8_attn_smem() {
    return (size_t)(1 << (2 * BV)) * 128 + (size_t)kAttnWarps * kAttnNS * q8_stage_bytes<BV>();
}

template <int BV>
__global__ void __launch_bounds__(kAttnWarps * 32, 2) k_attn_q8_split(AttnParams p) {
    constexpr int NS = kAttnNS;
    constexpr int KT = 8, CH = KT * BV / 8;
    constexpr uint32_t SEC_AV = 512u * CH;
    constexpr uint32_t STG = q8_stage_bytes<BV>();
    constexpr int E = 1 << (2 * BV);
    extern __shared__ __align__(128) uint8_t smem[];
    uint32_t* lut = reinterpret_cast<uint32_t*>(smem);        // [E][32]
    uint8_t* ring = smem + (size_t)E * 128;                    // [warp][NS][STG]
    __shared__ uint32_t wst[kAttnWarps][8][kWCol];
    __shared__ float s_acc[4][KT * 16];
    __shared__ float s_m[kAttnWarps][4], s_l[kAttnWarps][4];
    __shared__ int s_cmax[4];
    __shared__ uint64_t bars[kAttnWarps][NS];
    __shared__ uint4 s_q[4][2][8];   // per head: hi / lo bytes of the int16 query, per 16-coordinate column
    __shared__ float s_qs[4];        // scale * fixed-point step
    __shared__ __align__(16) float s_qf[4][128];   // the query heads in fp32 (tail logits)

    const int G = p.g, d = p.d;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int64_t stream = blockIdx.x / p.nsplit;
    const int split = blockIdx.x % p.nsplit;
    const int64_t b0 = (int64_t)split * p.blocks_per_split;
    const int64_t b1 = min(b0 + p.blocks_per_split, p.nb);

    for (int e = threadIdx.x; e < E * 8; e += blockDim.x) {
        const int ent = e >> 3;
        const uint32_t v = p.cbv.lut_half[ent & ((1 << BV) - 1)] | (p.cbv.lut_half[ent >> BV] << 16);
        reinterpret_cast<uint4*>(lut)[e] = make_uint4(v, v, v, v);
    }
    for (int e = threadIdx.x; e < 4 * KT * 16; e += blockDim.x) (&s_acc[0][0])[e] = 0.f;
    if (threadIdx.x < 4) s_cmax[threadIdx.x] = ord_of(-INFINITY);
    if (lane == 0)
        for (int s = 0; s < NS; ++s) tq_mbar_init(&bars[w][s], 2);
    tq_fence_mbar_init();
    // query heads as int16 fixed point (step max|q| / 16383), hi / lo int8 bytes
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
        *reinterpret_cast<float4*>(&s_qf[w][4 * lane]) = make_float4(v[0], v[1], v[2], v[3]);
        reinterpret_cast<uint32_t*>(&s_q[w][0][lane >> 2])[lane & 3] = q8_pack4(hi[0], hi[1], hi[2], hi[3]);
        reinterpret_cast<uint32_t*>(&s_q[w][1][lane >> 2])[lane & 3] = q8_pack4(lo[0], lo[1], lo[2], lo[3]);
        if (lane == 0) s_qs[w] = p.scale * step;
    }
    __syncthreads();

    uint8_t* my_ring = ring + (size_t)w * NS * STG;
    const int64_t first = b0 + w;
    const int nmine = first < b1 ? (int)((b1 - first + kAttnWarps - 1) / kAttnWarps) : 0;
    const uint8_t* kk = p.packed_k8 + ((size_t)stream * p.nb + first) * kQ8Block;
    const uint8_t* vk = p.packed_v + ((size_t)stream * p.nb + first) * p.tv.block_bytes;
    auto issue = [&](int k) {
        if (k < nmine && lane == 0) {
            const int s = k % NS;
            tq_bulk_load(my_ring + s * STG, kk, kQ8Block, &bars[w][s]);
            tq_bulk_load(my_ring + s * STG + kQ8Block, vk, (uint32_t)p.tv.block_bytes, &bars[w][s]);
        }
        if (k < nmine) {
            kk += (size_t)kAttnWarps * kQ8Block;
            vk += (size_t)kAttnWarps * p.tv.block_bytes;
        }
    };
    for (int k = 0; k < NS; ++k) issue(k);

    // the exact logits of the stream's bf16 tail (read by the merge), one token per warp of the
    // stream's ranges, against the queries in shared memory
    for (int tt = split * kAttnWarps + w; tt < p.n_tail; tt += p.nsplit * kAttnWarps) {
        const uint16_t* kp = p.tail_k + ((size_t)stream * p.n_tail + tt) * d;
        float kv[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int j = 4 * lane + k;   // d is a multiple of 8: lanes past d hold no coordinates
            kv[k] = j < d ? __uint_as_float((uint32_t)kp[j] << 16) : 0.f;
        }
        for (int h = 0; h < G; ++h) {
            const float4 qv = *reinterpret_cast<const float4*>(&s_qf[h][4 * lane]);
            float a = fmaf(kv[0], qv.x, fmaf(kv[1], qv.y, fmaf(kv[2], qv.z, kv[3] * qv.w)));
            a = tq_warp_sum(a);
            if (lane == 0) p.tail_logit[(stream * G + h) * p.n_tail + tt] = p.scale * a;
        }
    }

    constexpr float kLog2e = 1.4426950408889634f;
    float acc[KT][4];
#pragma unroll
    for (int i = 0; i < KT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    float m_run[4], lsum[4];   // every lane: the running maxima (warp-uniform) and its tokens' sums
#pragma unroll
    for (int h = 0; h < 4; ++h) { m_run[h] = -INFINITY; lsum[h] = 0.f; }

    bool ok = true;
    int k = 0;
    for (; k < nmine; ++k) {
        const int s = k % NS;
        ok = __all_sync(0xffffffffu, tq_mbar_wait(&bars[w][s], (uint32_t)(k / NS) & 1u, kWaitLimit));
        if (!ok) break;
        const uint8_t* kb = my_ring + s * STG;
        const uint8_t* vb = kb + kQ8Block;
        const int64_t blk = first + (int64_t)kAttnWarps * k;
        // ---- logits of token `lane` for the 4 heads: dp4a per 32-coordinate chunk
        uint4 kc[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) kc[j] = *reinterpret_cast<const uint4*>(kb + j * 512 + lane * 16);
        float res[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const float csc = tq_half_val(reinterpret_cast<const uint16_t*>(kb + 4096)[c * 32 + lane]);
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
#pragma unroll
            for (int h = 0; h < 4; ++h) res[h] = fmaf(csc, (float)(256 * ah[h] + al[h]), res[h]);
        }
        const bool tok_in = blk * 32 + lane < p.n_tok;
        float l[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) l[h] = (h < G && tok_in) ? s_qs[h] * res[h] : -INFINITY;
        // ---- online softmax, every head across the warp
        float fac[4];
        bool low = true;
        const float vn = tq_half_val(reinterpret_cast<const uint16_t*>(vb + SEC_AV)[lane]);
        float wt[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const float bm = tq_warp_max(l[h]);
            float cmax = bm;
            if (p.v_skip > 0.f) {
                if (lane == 0) atomicMax(&s_cmax[h], ord_of(bm));
                cmax = fmaxf(bm, float_of(*reinterpret_cast<volatile int*>(&s_cmax[h])));
            }
            fac[h] = 1.f;
            if (bm > m_run[h]) {
                fac[h] = tq_exp2((m_run[h] - bm) * kLog2e);   // 0 while the maximum was -inf
                lsum[h] *= fac[h];
                m_run[h] = bm;
            }
            const float ev = m_run[h] > -INFINITY ? tq_exp2(fmaf(l[h], kLog2e, -m_run[h] * kLog2e)) : 0.f;
            lsum[h] += ev;
            wt[h] = ev * vn;
            low = low && (l[h] < cmax + __logf(p.v_skip) || l[h] == -INFINITY);
        }
        // accumulator columns 2t, 2t + 1 belong to head t
        const float ft = t == 0 ? fac[0] : t == 1 ? fac[1] : t == 2 ? fac[2] : fac[3];
        if (ft != 1.f) {
#pragma unroll
            for (int i = 0; i < KT; ++i) {
                acc[i][0] *= ft; acc[i][1] *= ft; acc[i][2] *= ft; acc[i][3] *= ft;
            }
        }
        if (__all_sync(0xffffffffu, low)) {
            __syncwarp();
            if (lane == 0) tq_fence_proxy_async();
            issue(k + NS);
            continue;
        }
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const __half hi = __float2half_rn(wt[h]);
            reinterpret_cast<__half*>(&wst[w][2 * h][0])[lane] = hi;
            reinterpret_cast<__half*>(&wst[w][2 * h + 1][0])[lane] = __float2half_rn(wt[h] - __half2float(hi));
        }
        __syncwarp();
        attn_values<BV>(acc, wst[w], vb, lut, lane);
        __syncwarp();
        if (lane == 0) tq_fence_proxy_async();
        issue(k + NS);
    }
    if (!ok) {
        if (lane == 0) {
            tq_raise(p.status, TQ_FLAG_TIMEOUT);
            for (int j = k; j < min(k + NS, nmine); ++j)
                tq_mbar_wait(&bars[w][j % NS], (uint32_t)(j / NS) & 1u, kWaitLimit);
        }
        __syncwarp();
    }
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        const float ls = tq_warp_sum(lsum[h]);
        if (lane == 0) { s_m[w][h] = m_run[h]; s_l[w][h] = ls; }
    }
    __syncthreads();
    float M = s_m[0][t];
#pragma unroll
    for (int v = 1; v < kAttnWarps; ++v) M = fmaxf(M, s_m[v][t]);
    const float mt = s_m[w][t];
    const float f = mt > -INFINITY ? tq_exp2((mt - M) * kLog2e) : 0.f;
    if (t < G) {
#pragma unroll
        for (int kt = 0; kt < KT; ++kt) {
            atomicAdd(&s_acc[t][16 * kt + g], f * (acc[kt][0] + acc[kt][1]));
            atomicAdd(&s_acc[t][16 * kt + 8 + g], f * (acc[kt][2] + acc[kt][3]));
        }
    }
    __syncthreads();
    const int D = KT * 16;
    for (int e = threadIdx.x; e < G * D; e += blockDim.x) {
        const int h = e / D, i = e % D;
        p.part[(((size_t)stream * G + h) * p.nsplit + split) * D + i] = s_acc[h][i];
    }
    if (threadIdx.x < G) {
        const int h = threadIdx.x;
        float Mh = s_m[0][h], L = 0.f;
        for (int v = 1; v < kAttnWarps; ++v) Mh = fmaxf(Mh, s_m[v][h]);
        for (int v = 0; v < kAttnWarps; ++v)
            if (s_m[v][h] > -INFINITY) L += s_l[v][h] * tq_exp2((s_m[v][h] - Mh) * kLog2e);
        reinterpret_cast<float2*>(p.part_ml)[((size_t)stream * G + h) * p.nsplit + split] = make_float2(Mh, L);
    }
}

template <int BV>
cudaError_t launch_q8_split(const AttnParams& p, cudaStream_t st) {
    constexpr size_t smem = q8_attn_smem<BV>();
    if (p.tv.block_bytes != 512u * BV + 64u) return cudaErrorInvalidValue;
    auto kern = k_attn_q8_split<BV>;
    static TqLaunchCache cache;
    cudaError_t e = tq_kernel_setup(kern, kAttnWarps * 32, smem, cache, nullptr, nullptr);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(p.n_streams * p.nsplit), kAttnWarps * 32, smem, st>>>(p);
    return cudaGetLastError();
}

// tail-only calls: the tail logits of every stream (one CTA per stream)
__global__ void __launch_bounds__(kAttnWarps * 32) k_attn_q8_tail(AttnParams p) {
    const int G = p.g, d = p.d;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t stream = blockIdx.x;
    for (int tt = w; tt < p.n_tail; tt += kAttnWarps) {
        const uint16_t* kp = p.tail_k + ((size_t)stream * p.n_tail + tt) * d;
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
            if (lane == 0) p.tail_logit[(stream * G + h) * p.n_tail + tt] = p.scale * a;
        }
    }
}
}  // namespace

cudaError_t tq_launch_attention(const AttnParams& p, cudaStream_t st) {
    if (p.tk.D != 128 || p.tk.Mp != 128 || p.tv.D != 128 || p.g < 1 || p.g > 4) return cudaErrorInvalidValue;
    if (p.nsplit > 0) {   // no compressed tokens: the merge sees only the tail
        cudaError_t e = cudaErrorInvalidValue;
        switch (p.tk.B) {
            case 1: e = launch_bv<1>(p, st); break;
            case 2: e = launch_bv<2>(p, st); break;
            case 3: e = launch_bv<3>(p, st); break;
        }
        if (e != cudaSuccess) return e;
    }
    // a plain launch: as a programmatic dependent of the split the merge measured no faster
    k_attn_merge<<<(unsigned)(p.n_streams * p.g * kMergeCtas), kMergeThreads, 0, st>>>(p);
    return cudaGetLastError();
}

// Split CTAs of the 8-bit-key attention that fit one SM: two while the value table and the
// rings take at most half of the 227 KB (values of up to 3 bits), else one (4-bit values: a
// 32 KB table); the key ranges are sized so that the grid is one such wave.
int tq_attention_q8_ctas_per_sm(int bv) {
    constexpr size_t kStaticBound = 8192;   // the kernel's static shared arrays, rounded up
    size_t smem = 0;
    switch (bv) {
        case 1: smem = q8_attn_smem<1>(); break;
        case 2: smem = q8_attn_smem<2>(); break;
        case 3: smem = q8_attn_smem<3>(); break;
        default: smem = q8_attn_smem<4>(); break;
    }
    return smem + kStaticBound <= 232448 / 2 ? 2 : 1;
}

cudaError_t tq_launch_attention_q8(const AttnParams& p, cudaStream_t st) {
    if (p.tv.D != 128 || p.d > 128 || p.g < 1 || p.g > 4) return cudaErrorInvalidValue;
    cudaError_t e = cudaSuccess;
    if (p.nsplit > 0) {
        switch (p.tv.B) {
            case 1: e = launch_q8_split<1>(p, st); break;
            case 2: e = launch_q8_split<2>(p, st); break;
            case 3: e = launch_q8_split<3>(p, st); break;
            case 4: e = launch_q8_split<4>(p, st); break;
            default: e = cudaErrorInvalidValue;
        }
    } else if (p.n_tail > 0) {
        k_attn_q8_tail<<<(unsigned)p.n_streams, kAttnWarps * 32, 0, st>>>(p);
        e = cudaGetLastError();
    }
    if (e != cudaSuccess) return e;
    k_attn_merge<<<(unsigned)(p.n_streams * p.g * kMergeCtas), kMergeThreads, 0, st>>>(p);
    return cudaGetLastError();
}
