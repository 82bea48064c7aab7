// tq_topk: top-k inner-product search over a packed key database (a2a-mcp.org "What is
// TurboQuant", benchmark section: vector search on GloVe d = 200 with recall@k). The score of
// database vector x for query q is the estimator of tq_logits (blog.hotdry.top "TurboQuant
// vector-search compression", section "QJL residual correction"):
//   s(q, x) = |x| ( <Pi q, c[idx]> + gamma sqrt(pi/2)/m <S q, sign> ).
//
// Queries are rotated once by the logits prologue (groups of 4 queries play the role of the
// 4 heads of a kv stream). k_topk_scan: a CTA of 8 warps owns 32 queries (4 per warp) and a
// range of database blocks, which thread 0 streams into a shared ring with bulk copies;
// every warp scores each 32-vector block for its 4 queries on the int8 tensor cores (same
// bit-plane contraction as tq_logits), keeps a per-query threshold (its current k-th best
// score) and appends better candidates to a shared list; a list that fills is merged by a
// warp-wide bitonic sort. Each (query, range) leaves its k best in the workspace and
// k_topk_merge combines the ranges. Order: score descending, ties to the lower index.
#include <algorithm>
#include <climits>

#include "tq_device.cuh"

namespace {

constexpr int kWarps = 8;
constexpr int kList = 128;          // slots per (warp, query) list: k best + candidates
constexpr int kCandBase = 32;       // candidates are appended from this slot
constexpr int kCandMerge = 32;      // merge once this many candidates are waiting
constexpr uint32_t kWaitLimit = 1u << 22;

// "a before b": higher score first, then lower index
__device__ __forceinline__ bool before(float sa, int ia, float sb, int ib) {
    return sa > sb || (sa == sb && ia < ib);
}

// Sort n <= 128 entries of a shared list in "before" order (bitonic, one warp).
__device__ void warp_sort128(float* sc, int* ix, int n, int lane) {
    for (int e = n + lane; e < kList; e += 32) { sc[e] = -INFINITY; ix[e] = INT_MAX; }
    __syncwarp();
    for (int k = 2; k <= kList; k <<= 1)
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int e = lane; e < kList; e += 32) {
                const int pe = e ^ j;
                if (pe > e) {
                    const float sa = sc[e], sb = sc[pe];
                    const int ia = ix[e], ib = ix[pe];
                    const bool a_first = before(sa, ia, sb, ib);
                    if (((e & k) == 0) != a_first) {
                        sc[e] = sb; sc[pe] = sa; ix[e] = ib; ix[pe] = ia;
                    }
                }
            }
            __syncwarp();
        }
}

// Merge the waiting candidates of a list into its k best; returns the new threshold.
__device__ float merge_list(float* sc, int* ix, int& nk, int& ncand, int k, int lane) {
    for (int b = 0; b < ncand; b += 32) {   // compact candidates right after the k best
        const int e = b + lane;
        const float v = e < ncand ? sc[kCandBase + e] : 0.f;
        const int i = e < ncand ? ix[kCandBase + e] : 0;
        __syncwarp();
        if (e < ncand) { sc[nk + e] = v; ix[nk + e] = i; }
        __syncwarp();
    }
    const int n = nk + ncand;
    warp_sort128(sc, ix, n, lane);
    nk = min(n, k);
    ncand = 0;
    return nk == k ? sc[k - 1] : -INFINITY;
}

template <int B, int GD, int GM, int NS>
__global__ void __launch_bounds__(kWarps * 32) k_topk_scan(TopkParams p) {
    constexpr int NP = B == 3 ? 4 : B;
    constexpr int NPG = B * GD + GM;
    constexpr int NMG = NP * GD + GM;
    constexpr uint32_t BB = 512u * NPG + 128u;
    extern __shared__ __align__(128) uint8_t sm[];
    uint8_t* ring = sm;
    float* lsc = reinterpret_cast<float*>(sm + NS * BB);      // [warp][query][kList]
    int* lix = reinterpret_cast<int*>(lsc + kWarps * 4 * kList);
    __shared__ uint64_t bars[NS];
    __shared__ int s_cnt[kWarps][4], s_nk[kWarps][4];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int qg = blockIdx.x / p.nsplit, split = blockIdx.x % p.nsplit;
    const int group = qg * kWarps + warp;
    const bool active = group < p.n_groups;
    const int64_t b0 = (int64_t)split * p.blocks_per_split;
    const int64_t b1 = min(b0 + p.blocks_per_split, p.nb);

    if (tid == 0)
        for (int s = 0; s < NS; ++s) tq_mbar_init(&bars[s], 1);
    if (tid < kWarps * 4) { (&s_cnt[0][0])[tid] = 0; (&s_nk[0][0])[tid] = 0; }
    tq_fence_mbar_init();
    __syncthreads();
    if (tid == 0)
        for (int s = 0; s < NS && b0 + s < b1; ++s)
            tq_bulk_load(ring + s * BB, p.packed + (size_t)(b0 + s) * BB, BB, &bars[s]);

    uint32_t qf[NMG][4][2];
    float4 sc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (active) {
#pragma unroll
        for (int mg = 0; mg < NMG; ++mg)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint2 v = *reinterpret_cast<const uint2*>(
                    p.qfrag + ((((size_t)group * NMG + mg) * 4 + c) * 64 + lane * 2));
                qf[mg][c][0] = v.x;
                qf[mg][c][1] = v.y;
            }
        sc = reinterpret_cast<const float4*>(p.qscale)[(size_t)group * 4 + t];
    }
    float tau = -INFINITY;   // threshold of query t of this warp
    float* my_sc = lsc + (warp * 4) * kList;
    int* my_ix = lix + (warp * 4) * kList;
    bool ok = true;

    for (int64_t bi = b0; bi < b1; ++bi) {
        const int stage = (int)((bi - b0) % NS);
        const uint32_t phase = (uint32_t)(((bi - b0) / NS) & 1);
        ok = __syncthreads_and(tq_mbar_wait(&bars[stage], phase, kWaitLimit));
        if (!ok) break;
        if (active) {
            const uint8_t* bp = ring + stage * BB;
            uint4 cur[NPG + 1];
#pragma unroll
            for (int pg = 0; pg < NPG; ++pg) cur[pg] = *reinterpret_cast<const uint4*>(bp + (pg * 32 + lane) * 16);
            cur[NPG] = *reinterpret_cast<const uint4*>(bp + NPG * 512 + g * 16);
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                int accA[4] = {0, 0, 0, 0}, accS[4] = {0, 0, 0, 0};
#pragma unroll
                for (int mg = 0; mg < NMG; ++mg) {
                    uint32_t w0, w1;
                    if (mg < NP * GD && mg / GD == 3) {
                        const int gr = mg % GD;
                        const uint32_t* c0 = reinterpret_cast<const uint32_t*>(&cur[0 * GD + gr]);
                        const uint32_t* c1 = reinterpret_cast<const uint32_t*>(&cur[1 * GD + gr]);
                        const uint32_t* c2 = reinterpret_cast<const uint32_t*>(&cur[2 * GD + gr]);
                        w0 = c0[2 * mt] ^ c1[2 * mt] ^ c2[2 * mt];
                        w1 = c0[2 * mt + 1] ^ c1[2 * mt + 1] ^ c2[2 * mt + 1];
                    } else {
                        const int pg = mg < NP * GD ? mg : B * GD + (mg - NP * GD);
                        const uint32_t* cw = reinterpret_cast<const uint32_t*>(&cur[pg]);
                        w0 = cw[2 * mt];
                        w1 = cw[2 * mt + 1];
                    }
                    tq_expand_planes(w0, w1, [&](int c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3) {
                        if (mg < NP * GD) tq_imma_u8(accA, a0, a1, a2, a3, qf[mg][c][0], qf[mg][c][1]);
                        else tq_imma_u8(accS, a0, a1, a2, a3, qf[mg][c][0], qf[mg][c][1]);
                    });
                }
                const uint32_t* nrm = reinterpret_cast<const uint32_t*>(&cur[NPG]);
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const int u = 2 * mt + r;
                    const uint32_t nw = nrm[u];
                    const float nh = tq_half_val(nw & 0xffffu), gh = tq_half_val(nw >> 16);
                    const float va = fmaf(256.f, (float)accA[2 * r], (float)accA[2 * r + 1]);
                    const float vs = fmaf(256.f, (float)accS[2 * r], (float)accS[2 * r + 1]);
                    const float score = nh * (fmaf(sc.x, va, -sc.y) + gh * fmaf(sc.z, vs, -sc.w));
                    const int64_t vec = bi * 32 + 8 * u + g;
                    if (vec < p.n_db && (int64_t)group * 4 + t < p.n_q && score >= tau) {
                        const int pos = atomicAdd(&s_cnt[warp][t], 1);
                        my_sc[t * kList + kCandBase + pos] = score;
                        my_ix[t * kList + kCandBase + pos] = (int)vec;
                    }
                }
            }
        }
        __syncthreads();   // every warp is done with this stage and its candidates are visible
        if (tid == 0 && bi + NS < b1) {
            tq_fence_proxy_async();
            tq_bulk_load(ring + stage * BB, p.packed + (size_t)(bi + NS) * BB, BB, &bars[stage]);
        }
        if (active) {
#pragma unroll 1
            for (int qq = 0; qq < 4; ++qq) {
                int nc = s_cnt[warp][qq];
                if (nc >= kCandMerge) {
                    int nk = s_nk[warp][qq];
                    const float th = merge_list(my_sc + qq * kList, my_ix + qq * kList, nk, nc, p.k, lane);
                    if (t == qq) tau = th;
                    __syncwarp();
                    if (lane == 0) { s_nk[warp][qq] = nk; s_cnt[warp][qq] = 0; }
                    __syncwarp();
                }
            }
        }
    }
    if (!ok) {
        if (tid == 0) {
            tq_raise(p.status, TQ_FLAG_TIMEOUT);
            for (int s = 0; s < NS; ++s) tq_mbar_wait(&bars[s], 1u, kWaitLimit);
        }
        return;
    }
    if (active) {
#pragma unroll 1
        for (int qq = 0; qq < 4; ++qq) {
            const int64_t q = (int64_t)group * 4 + qq;
            int nc = s_cnt[warp][qq], nk = s_nk[warp][qq];
            if (nc > 0) merge_list(my_sc + qq * kList, my_ix + qq * kList, nk, nc, p.k, lane);
            if (q < p.n_q)
                for (int e = lane; e < p.k; e += 32) {
                    const size_t o = ((size_t)q * p.nsplit + split) * p.k + e;
                    p.part_score[o] = e < nk ? my_sc[qq * kList + e] : -INFINITY;
                    p.part_idx[o] = e < nk ? my_ix[qq * kList + e] : INT_MAX;
                }
        }
    }
}

// one warp per query: fold the per-range lists two at a time
__global__ void __launch_bounds__(256) k_topk_merge(TopkParams p) {
    __shared__ float s_sc[8][kList];
    __shared__ int s_ix[8][kList];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t q = (int64_t)blockIdx.x * 8 + warp;
    if (q >= p.n_q) return;
    float* sc = s_sc[warp];
    int* ix = s_ix[warp];
    const int k = p.k;
    int nk = 0;
    for (int sp = 0; sp < p.nsplit; ++sp) {
        for (int e = lane; e < k; e += 32) {
            const size_t o = ((size_t)q * p.nsplit + sp) * k + e;
            sc[nk + e] = p.part_score[o];
            ix[nk + e] = p.part_idx[o];
        }
        __syncwarp();
        warp_sort128(sc, ix, nk + k, lane);
        nk = k;
    }
    for (int e = lane; e < k; e += 32) {
        p.out_score[q * k + e] = sc[e];
        p.out_idx[q * k + e] = ix[e] == INT_MAX ? -1 : (int64_t)ix[e];
    }
}

template <int B, int GD, int GM>
cudaError_t launch_scan(const TopkParams& p, cudaStream_t st) {
    constexpr int NS = 4;
    constexpr size_t BB = 512u * (B * GD + GM) + 128u;
    const size_t smem = NS * BB + (size_t)kWarps * 4 * kList * 8;
    auto kern = k_topk_scan<B, GD, GM, NS>;
    static TqLaunchCache cache;
    cudaError_t e = tq_kernel_setup(kern, kWarps * 32, smem, cache, nullptr, nullptr);
    if (e != cudaSuccess) return e;
    const int64_t qgroups = (p.n_groups + kWarps - 1) / kWarps;
    kern<<<(unsigned)(qgroups * p.nsplit), kWarps * 32, smem, st>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t tq_launch_topk(const TopkParams& p, cudaStream_t st) {
    cudaError_t e = cudaErrorInvalidValue;
    const int B = p.t.B, GD = p.t.GD, GM = p.t.GM;
#define TQ_TOPK_CASE(b, gd, gm) \
    if (B == b && GD == gd && GM == gm) e = launch_scan<b, gd, gm>(p, st);
    TQ_TOPK_CASE(1, 1, 1) TQ_TOPK_CASE(2, 1, 1) TQ_TOPK_CASE(3, 1, 1)
    TQ_TOPK_CASE(1, 2, 2) TQ_TOPK_CASE(2, 2, 2) TQ_TOPK_CASE(3, 2, 2)
    TQ_TOPK_CASE(1, 1, 2) TQ_TOPK_CASE(2, 1, 2) TQ_TOPK_CASE(3, 1, 2)
    TQ_TOPK_CASE(1, 2, 1) TQ_TOPK_CASE(2, 2, 1) TQ_TOPK_CASE(3, 2, 1)
#undef TQ_TOPK_CASE
    if (e != cudaSuccess) return e;
    k_topk_merge<<<(unsigned)((p.n_q + 7) / 8), 256, 0, st>>>(p);
    return cudaGetLastError();
}
