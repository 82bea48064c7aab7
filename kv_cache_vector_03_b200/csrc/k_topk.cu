// tq_topk: top-k inner-product search over a packed key database (a2a-mcp.org "What is
// TurboQuant", benchmark section: vector search on GloVe d = 200 with recall@k). The score of
// database vector x for query q is the estimator of tq_logits (blog.hotdry.top "TurboQuant
// vector-search compression", section "QJL residual correction"):
//   s(q, x) = |x| ( <Pi q, c[idx]> + gamma sqrt(pi/2)/m <S q, sign> ).
//
// As a contraction over K = D + Mp coordinates this is one GEMM of the query rows
// a_q = sigma_q [Pi q | kappa S q] with the key columns b_x = [c[idx(x)] | gamma(x) sign(x)],
// scaled per column by |x|: s(q, x) = |x| (a_q . b_x) / sigma_q. It runs on the fifth-generation
// tensor cores in fp16 with fp32 accumulation:
//   k_topk_qprep  one warp per query: Pi q and S q from the prepared transposes in fp32, the
//                 power-of-two sigma_q that puts the row's largest magnitude in [2^13, 2^14),
//                 the fp16 operand row;
//   k_topk_tc     one CTA per (tile of 128 queries, range of key tiles), 14 warps:
//                   warp 0      bulk copies of raw key tiles (4 blocks of 32 records) into a
//                               3-stage ring;
//                   warp 1      one thread issues the MMAs: A = the 128 query rows, resident in
//                               TMEM; B = K-blocks of 64 coordinates x 128 keys from an 8-slot
//                               shared ring; D = 128 x 128 fp32 scores in TMEM, double buffered;
//                               K-steps of 16 coordinates past d (resp. m) are skipped;
//                   warps 2-9   expand each raw tile into the fp16 B operand (128-byte swizzled,
//                               K-major): centroid pairs from a table indexed by the code bits of
//                               two coordinates, sign pairs as gamma with the sign bits set from
//                               a nibble table, |x| as fp32 for the epilogue;
//                   warps 10-13 one thread per query row: scores of 128 keys per tile read from
//                               TMEM, times |x|, against the row's threshold (the worst of its
//                               k best, kept unordered in registers); candidates wait in a
//                               per-row buffer and replace the worst entry, the warp's lanes in
//                               step, once the tile's accumulator is released;
//   k_topk_merge  one warp per query folds the ranges' lists.
// Order: score descending, ties to the lower index. Rounding: the query row and the centroids
// are rounded to fp16 (relative 2^-11 each; gamma and the signs are exact), so a score differs
// from the fp32 estimator by about 2^-11 sqrt(2 sum_i (q'_i c_i)^2) for independent roundings,
// at most 2^-10 (|Pi q| |c| + kappa gamma |S q|_1) |x|.
#include <algorithm>
#include <climits>

#include "tq_device.cuh"
#include "tq_tc.cuh"

namespace {
using namespace tqtc;

constexpr int kList = 128;          // slots of a merge list (k_topk_merge)
constexpr int kThreads = 448;       // 14 warps
constexpr int kMmaWarp = 1, kExpWarp0 = 2, kEpiWarp0 = 10;
constexpr int kSlots = 8;           // B ring: one K-block (128 keys x 64 fp16) per slot
constexpr int kRaw = 3;             // raw tile stages
constexpr int kMaxK = 32;
constexpr int kCandSlots = 32;      // candidate buffer slots per query row
constexpr uint32_t kSlotBytes = 16384;
constexpr uint32_t kWaitLimit = 1u << 22;

// barriers
enum { bFull = 0, bEmpty = kSlots, bRawFull = 2 * kSlots, bRawEmpty = 2 * kSlots + kRaw,
       bNrm = 2 * kSlots + 2 * kRaw, bAccFull = bNrm + kRaw, bAccEmpty = bAccFull + 2, bAReady = bAccEmpty + 2,
       bDrain = bAReady + 1, kNumBars = bDrain + 1 };

template <int B, int GD, int GM>
struct TopkLayout {
    static constexpr int NPG = B * GD + GM;
    static constexpr uint32_t BB = 512u * NPG + 128u;      // one block of 32 records
    static constexpr uint32_t RAWB = 4 * BB;               // one tile of 128 records
    static constexpr uint32_t oRing = 0;
    static constexpr uint32_t oRaw = kSlots * kSlotBytes;
    static constexpr uint32_t oNrm = oRaw + kRaw * RAWB;   // |x| fp32 [stage][128]
    static constexpr uint32_t oCand = oNrm + kRaw * 512;   // candidate buffers: scores, keys [slot][128]
    static constexpr uint32_t oLut = oCand + kCandSlots * 128 * 8;   // pair table (64 words), nibble table (16 x 8 B)
    static constexpr uint32_t oBar = oLut + 64 * 4 + 16 * 8;
    static constexpr uint32_t used = oBar + 8 * kNumBars + 16;
    static constexpr size_t smem = used + 1024;            // + alignment pad
};

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

// ------------------------------------------------------------------ query operand rows
// One warp per row of the padded query tiles; lane l owns outputs l + 32 a.
__global__ void __launch_bounds__(256) k_topk_qprep(TopkParams p) {
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (row >= (int64_t)p.n_qt * 128) return;
    const int nm = p.kb_mse * 2, ns = p.kb_sign * 2;   // outputs per lane of each part
    const int D = p.t.D, Mp = p.t.Mp;
    float acc[16];
#pragma unroll
    for (int a = 0; a < 16; ++a) acc[a] = 0.f;
    if (row < p.n_q) {
        const float* qr = p.q + row * p.d;
        for (int j = 0; j < p.d; ++j) {
            const float qj = __ldg(qr + j);
#pragma unroll
            for (int a = 0; a < 8; ++a)
                if (a < nm) acc[a] = fmaf(__ldg(p.piT + (size_t)j * D + lane + 32 * a), qj, acc[a]);
#pragma unroll
            for (int a = 0; a < 8; ++a)
                if (a < ns) acc[8 + a] = fmaf(__ldg(p.sT + (size_t)j * Mp + lane + 32 * a), qj, acc[8 + a]);
        }
    }
    float mx = 0.f;
#pragma unroll
    for (int a = 0; a < 8; ++a) {
        acc[8 + a] *= p.kappa;
        mx = fmaxf(mx, fmaxf(fabsf(acc[a]), fabsf(acc[8 + a])));
    }
    mx = tq_warp_max(mx);
    // sigma = 2^(13 - e) with mx in [2^e, 2^(e+1)): scaled magnitudes below 2^14
    float sigma = 1.f;
    if (mx > 0.f && isfinite(mx)) {
        const int e = ((__float_as_int(mx) >> 23) & 0xff) - 127;
        sigma = ldexpf(1.f, 13 - max(e, -100));
    }
    uint16_t* out = p.qimg + row * p.kq;
#pragma unroll
    for (int a = 0; a < 8; ++a)
        if (a < nm) out[lane + 32 * a] = __half_as_ushort(__float2half_rn(acc[a] * sigma));
#pragma unroll
    for (int a = 0; a < 8; ++a)
        if (a < ns) out[64 * p.kb_mse + lane + 32 * a] = __half_as_ushort(__float2half_rn(acc[8 + a] * sigma));
    if (lane == 0) p.qinv[row] = row < p.n_q ? 1.f / sigma : 0.f;
}

// ------------------------------------------------------------------ operand expansion
// 32 coordinates (one plane word per code plane) to four 16-byte chunks of fp16 centroids:
// pair t (coordinates 2t, 2t+1) looks up the table entry sum_p ((w_p >> 2t) & 3) << 2p.
template <int B>
__device__ __forceinline__ void mse_word(const uint32_t (&w)[B], const uint32_t* lut, uint4 (&ch)[4]) {
    uint32_t o[16];
    if constexpr (B == 1) {
#pragma unroll
        for (int t = 0; t < 16; ++t) o[t] = lut[(w[0] >> (2 * t)) & 3u];
    } else {
        // nibble n of E holds the (plane 0, plane 1) bits of pair 2n, of O those of pair 2n + 1
        const uint32_t E = (w[0] & 0x33333333u) | ((w[1] & 0x33333333u) << 2);
        const uint32_t O = ((w[0] >> 2) & 0x33333333u) | (w[1] & 0xCCCCCCCCu);
        if constexpr (B == 2) {
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                o[2 * n] = lut[(E >> (4 * n)) & 15u];
                o[2 * n + 1] = lut[(O >> (4 * n)) & 15u];
            }
        } else {
            const uint32_t E2 = w[2] & 0x33333333u, O2 = (w[2] >> 2) & 0x33333333u;
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                o[2 * n] = lut[((E >> (4 * n)) & 15u) | (((E2 >> (4 * n)) & 3u) << 4)];
                o[2 * n + 1] = lut[((O >> (4 * n)) & 15u) | (((O2 >> (4 * n)) & 3u) << 4)];
            }
        }
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) ch[c] = make_uint4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
}

// 32 sketch signs to four chunks of +-gamma: nws = the complemented sign word (bit set = negative),
// the nibble table gives the sign bits of two fp16 pairs
__device__ __forceinline__ void sign_word(uint32_t nws, uint32_t gbase, const uint2* sgn, uint4 (&ch)[4]) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const uint2 m0 = sgn[(nws >> (8 * c)) & 15u], m1 = sgn[(nws >> (8 * c + 4)) & 15u];
        ch[c] = make_uint4(gbase | m0.x, gbase | m0.y, gbase | m1.x, gbase | m1.y);
    }
}

// ------------------------------------------------------------------ the scan
template <int B, int GD, int GM, int KM>
__global__ void __launch_bounds__(kThreads, 1) k_topk_tc(TopkParams p) {
    using Lay = TopkLayout<B, GD, GM>;
    constexpr int NPG = Lay::NPG;
    constexpr uint32_t BB = Lay::BB, RAWB = Lay::RAWB;
    constexpr uint32_t kIdesc = idesc_f16(128, 128);
    extern __shared__ uint8_t raw_smem[];
    const uint32_t raw = tq_smem_addr(raw_smem);
    const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
    uint8_t* sm = raw_smem + pad;
    const uint32_t sb = raw + pad;
    float* s_nrm = reinterpret_cast<float*>(sm + Lay::oNrm);
    float* s_cand = reinterpret_cast<float*>(sm + Lay::oCand);
    uint32_t* s_lut = reinterpret_cast<uint32_t*>(sm + Lay::oLut);
    uint2* s_sgn = reinterpret_cast<uint2*>(sm + Lay::oLut + 256);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Lay::oBar);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + Lay::oBar + 8 * kNumBars);
    volatile uint32_t* s_abort = s_tmem + 1;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qt = blockIdx.x / p.nsplit, split = blockIdx.x % p.nsplit;
    const int64_t t0 = (int64_t)split * p.tiles_per_split;
    const int64_t t1 = t0 + p.tiles_per_split < p.n_tiles ? t0 + p.tiles_per_split : p.n_tiles;
    const int nt = t1 > t0 ? (int)(t1 - t0) : 0;
    const int nkb = p.kb_mse + p.kb_sign;

    if (tid == 0) {
        for (int i = 0; i < kNumBars; ++i) {
            uint32_t count = 1;
            if (i >= bFull && i < bFull + kSlots) count = 8;            // the expansion warps
            if (i >= bRawEmpty && i < bRawEmpty + kRaw) count = 12;     // expansion + epilogue warps
            if (i == bAccEmpty || i == bAccEmpty + 1 || i == bAReady) count = 4;   // the epilogue warps
            if (i >= bNrm && i < bNrm + kRaw) count = 4;                // the expansion warps of half 0
            tq_mbar_init(&bars[i], count);
        }
        *s_abort = 0u;
        tq_fence_mbar_init();
    }
    // tables: centroid pairs (entry e: c[lo] | c[hi] << 16 with lo, hi the even / odd bits of e
    // regrouped per plane) and sign bits of two fp16 pairs per nibble
    if (tid < (1 << (2 * B))) {
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int pl = 0; pl < B; ++pl) {
            lo |= ((tid >> (2 * pl)) & 1u) << pl;
            hi |= ((tid >> (2 * pl + 1)) & 1u) << pl;
        }
        s_lut[tid] = p.cb.lut_half[lo] | (p.cb.lut_half[hi] << 16);
    }
    if (tid >= 64 && tid < 80) {
        const uint32_t n = tid - 64;
        auto m2 = [](uint32_t x) { return ((x & 1u) ? 0x8000u : 0u) | ((x & 2u) ? 0x80000000u : 0u); };
        s_sgn[n] = make_uint2(m2(n & 3u), m2(n >> 2));
    }
    if (warp == kMmaWarp) tmem_alloc(s_tmem, 512);
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = *s_tmem;

    if (warp == 0) {
        // ------------------------------------------------------------ raw tile loads
        if (lane == 0) {
            int issued = 0;
            for (int i = 0; i < nt; ++i) {
                const int st = i % kRaw;
                if (i >= kRaw && !wait_bar(&bars[bRawEmpty + st], ((i / kRaw) - 1) & 1, s_abort, kWaitLimit)) break;
                const int64_t blk0 = (t0 + i) * 4;
                const uint32_t nvb = p.nb - blk0 < 4 ? (uint32_t)(p.nb - blk0) : 4u;
                mbar_expect_tx(&bars[bRawFull + st], nvb * BB);
                bulk_copy(sb + Lay::oRaw + st * RAWB, p.packed + blk0 * BB, nvb * BB, &bars[bRawFull + st]);
                issued = i + 1;
            }
            // no copy may be in flight at exit (a completed phase returns at once)
            for (int i = max(0, issued - kRaw); i < issued; ++i)
                tq_mbar_wait(&bars[bRawFull + i % kRaw], (i / kRaw) & 1, kWaitLimit);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issue
        if (lane == 0) {
            const int ks_mse = (p.d + 15) >> 4, ks_sign = (p.m + 15) >> 4;   // K-steps that hold coordinates
            uint32_t cc = 0;
            bool ok = wait_bar(&bars[bAReady], 0, s_abort, kWaitLimit);
            for (int i = 0; ok && i < nt; ++i) {
                const int ab = i & 1;
                if (i >= 2 && !wait_bar(&bars[bAccEmpty + ab], ((i >> 1) - 1) & 1, s_abort, kWaitLimit)) break;
                fence_after();
                const uint32_t dacc = tmem + 256u + 128u * ab;
                uint32_t accum = 0;
                for (int kb = 0; kb < nkb; ++kb, ++cc) {
                    const int sl = (int)(cc % kSlots);
                    if (!wait_bar(&bars[bFull + sl], (cc / kSlots) & 1, s_abort, kWaitLimit)) { ok = false; break; }
                    fence_after();
                    const int nks = kb < p.kb_mse ? min(4, ks_mse - 4 * kb) : min(4, ks_sign - 4 * (kb - p.kb_mse));
                    const uint32_t bslot = sb + Lay::oRing + sl * kSlotBytes;
                    for (int k = 0; k < nks; ++k) {
                        mma_ts(dacc, tmem + 32u * kb + 8u * k, sdesc(bslot + 32u * k), kIdesc, accum);
                        accum = 1;
                    }
                    commit(&bars[bEmpty + sl]);
                }
                if (!ok) break;
                commit(&bars[bAccFull + ab]);
            }
            // every MMA has completed before TMEM is released
            commit(&bars[bDrain]);
            tq_mbar_wait(&bars[bDrain], 0, kWaitLimit);
        }
    } else if (warp < kEpiWarp0) {
        // ------------------------------------------------------------ B operand expansion
        const int x = tid - 32 * kExpWarp0;
        const int v = x & 127, h = x >> 7;         // key row of the tile, half of each K-block
        const int bk = v >> 5, j = v & 31, gq = j & 7, u = j >> 3;
        auto warp_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
            return __all_sync(0xffffffffu, wait_bar(bar, parity, s_abort, kWaitLimit)) != 0;
        };
        uint32_t cc = 0;
        bool ok = true;
        for (int i = 0; ok && i < nt; ++i) {
            const int st = i % kRaw;
            if (!warp_wait(&bars[bRawFull + st], (i / kRaw) & 1)) break;
            const uint8_t* rb = sm + Lay::oRaw + st * RAWB + bk * BB;
            const bool valid = (t0 + i) * 128 + v < p.n_db;
            const uint32_t nw = valid ? *reinterpret_cast<const uint32_t*>(rb + 512 * NPG + (gq * 4 + u) * 4) : 0u;
            // |x| for the epilogue; NaN marks a key past the database (never a candidate)
            if (h == 0) {
                s_nrm[st * 128 + v] = valid ? tq_half_val(nw & 0xffffu) : __int_as_float(0x7fc00000);
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[bNrm + st]);
            }
            const uint32_t gbase = (nw >> 16) | (nw & 0xffff0000u);   // gamma in both halves
            for (int kb = 0; kb < nkb; ++kb, ++cc) {
                const int sl = (int)(cc % kSlots);
                if (cc >= (uint32_t)kSlots && !warp_wait(&bars[bEmpty + sl], ((cc / kSlots) - 1) & 1)) { ok = false; break; }
                uint4 ch[4];
                if (kb < p.kb_mse) {
                    const int gr = kb >> 1, tq = 2 * (kb & 1) + h;
                    uint32_t w[B];
#pragma unroll
                    for (int pl = 0; pl < B; ++pl)
                        w[pl] = *reinterpret_cast<const uint32_t*>(rb + (pl * GD + gr) * 512 + (4 * gq + tq) * 16 + u * 4);
                    mse_word<B>(w, s_lut, ch);
                } else {
                    const int kb2 = kb - p.kb_mse, gr = kb2 >> 1, tq = 2 * (kb2 & 1) + h;
                    const uint32_t ws =
                        *reinterpret_cast<const uint32_t*>(rb + (B * GD + gr) * 512 + (4 * gq + tq) * 16 + u * 4);
                    sign_word(~ws, gbase, s_sgn, ch);
                }
                if (!valid) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) ch[c] = make_uint4(0u, 0u, 0u, 0u);
                }
                uint8_t* dst = sm + Lay::oRing + sl * kSlotBytes;
#pragma unroll
                for (int c = 0; c < 4; ++c) *reinterpret_cast<uint4*>(dst + sw128(v, 4 * h + c)) = ch[c];
                tq_fence_proxy_async();   // the tensor cores read the slot through the async proxy
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[bFull + sl]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[bRawEmpty + st]);
        }
    } else {
        // ------------------------------------------------------------ scores and the k best
        const int qd = warp & 3;                      // TMEM lane quarter of this warp
        const int r = 32 * qd + lane;                 // query row of the tile
        const int64_t q = (int64_t)qt * 128 + r;
        const bool qvalid = q < p.n_q;
        const uint32_t lane_base = (uint32_t)(32 * qd) << 16;
        auto warp_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
            return __all_sync(0xffffffffu, wait_bar(bar, parity, s_abort, kWaitLimit)) != 0;
        };
        // the query rows into TMEM columns 0 .. kq/2 - 1 (two fp16 per column)
        {
            const uint4* qrow = reinterpret_cast<const uint4*>(p.qimg + q * p.kq);
            for (int c0 = 0; c0 < p.kq / 2; c0 += 16) {
                uint32_t v16[16];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const uint4 t = __ldg(qrow + c0 / 4 + e);
                    v16[4 * e] = t.x; v16[4 * e + 1] = t.y; v16[4 * e + 2] = t.z; v16[4 * e + 3] = t.w;
                }
                tst16(tmem + lane_base + (uint32_t)c0, v16);
            }
            twait_st();
            fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[bAReady]);
        }
        // this row's k best in registers, unordered: slots 0 .. k-1 start at (-inf, INT_MAX);
        // slots k .. KM-1 hold (+inf, -1), which is never the worst. The worst slot (the last in
        // "before" order) is the threshold and is the one a better score replaces.
        const int k = p.k;
        float bsc[KM];
        int bix[KM];
#pragma unroll
        for (int e = 0; e < KM; ++e) {
            bsc[e] = e < k ? -INFINITY : INFINITY;
            bix[e] = e < k ? INT_MAX : -1;
        }
        float wsc = -INFINITY;
        int wix = INT_MAX, wpos = 0;
        if (!qvalid) wsc = INFINITY;    // a padding row keeps nothing
        auto insert = [&](float sv, int iv) {
#pragma unroll
            for (int e = 0; e < KM; ++e)
                if (e == wpos) { bsc[e] = sv; bix[e] = iv; }
            float w = bsc[0];
            int wi = bix[0], wp = 0;
#pragma unroll
            for (int e = 1; e < KM; ++e) {
                const bool later = before(w, wi, bsc[e], bix[e]);
                w = later ? bsc[e] : w;
                wi = later ? bix[e] : wi;
                wp = later ? e : wp;
            }
            wsc = w; wix = wi; wpos = wp;
        };
        // Candidates (scores at or above the threshold) wait in this row's buffer in shared memory
        // ([slot][row]: a warp's lanes hit consecutive words) and are inserted together, the lanes
        // of the warp in step, once per tile after the accumulator is released, or earlier when a
        // buffer might overflow.
        float* cbs = s_cand;
        int* cbi = reinterpret_cast<int*>(s_cand + kCandSlots * 128);
        int ncb = 0;
        auto flush = [&]() {
            for (int c = 0; __any_sync(0xffffffffu, c < ncb); ++c) {
                if (c < ncb) {
                    const float v = cbs[c * 128 + r];
                    const int iv = cbi[c * 128 + r];
                    if (before(v, iv, wsc, wix)) insert(v, iv);
                }
            }
            ncb = 0;
            __syncwarp();
        };
        auto scan16 = [&](const uint32_t (&va)[16], const float* nrm, int key0) {
            float sv[16];
            bool any = false;
#pragma unroll
            for (int e = 0; e < 16; e += 4) {
                const float4 n4 = *reinterpret_cast<const float4*>(nrm + e);
                sv[e] = __uint_as_float(va[e]) * n4.x;
                sv[e + 1] = __uint_as_float(va[e + 1]) * n4.y;
                sv[e + 2] = __uint_as_float(va[e + 2]) * n4.z;
                sv[e + 3] = __uint_as_float(va[e + 3]) * n4.w;
                any |= (sv[e] >= wsc) | (sv[e + 1] >= wsc) | (sv[e + 2] >= wsc) | (sv[e + 3] >= wsc);
            }
            if (any) {
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    if (sv[e] >= wsc) {
                        cbs[ncb * 128 + r] = sv[e];
                        cbi[ncb * 128 + r] = key0 + e;
                        ++ncb;
                    }
            }
            // room for the next 16 scores
            if (__any_sync(0xffffffffu, ncb > kCandSlots - 16)) flush();
            // the TMEM loads and waits that follow are warp-collective: reconverge first
            __syncwarp();
        };
        for (int i = 0; i < nt; ++i) {
            const int ab = i & 1, st = i % kRaw;
            if (!warp_wait(&bars[bAccFull + ab], (i >> 1) & 1)) break;
            if (!warp_wait(&bars[bNrm + st], (i / kRaw) & 1)) break;
            fence_after();
            const uint32_t acc = tmem + lane_base + 256u + 128u * ab;
            const float* nrm = s_nrm + st * 128;
            const int key0 = (int)((t0 + i) * 128);
            uint32_t va[16], vb[16];
            tld16(acc, va);
            twait(va);
#pragma unroll 1
            for (int c = 0; c < 8; c += 2) {
                tld16(acc + 16u * (c + 1), vb);
                scan16(va, nrm + 16 * c, key0 + 16 * c);
                twait(vb);
                if (c + 2 < 8) tld16(acc + 16u * (c + 2), va);
                scan16(vb, nrm + 16 * (c + 1), key0 + 16 * (c + 1));
                if (c + 2 < 8) twait(va);
            }
            fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars[bAccEmpty + ab]);
                mbar_arrive(&bars[bRawEmpty + st]);
            }
            if (__any_sync(0xffffffffu, ncb > 0)) flush();
        }
        if (qvalid && !*s_abort) {
            const float qi = p.qinv[q];
#pragma unroll
            for (int e = 0; e < KM; ++e)
                if (e < k) {
                    const size_t o = ((size_t)q * p.nsplit + split) * k + e;
                    const bool got = bix[e] != INT_MAX;
                    p.part_score[o] = got ? bsc[e] * qi : -INFINITY;
                    p.part_idx[o] = got ? bix[e] : INT_MAX;
                }
        }
    }
    __syncthreads();
    if (*s_abort && tid == 0) tq_raise(p.status, TQ_FLAG_TIMEOUT);
    if (warp == kMmaWarp) {
        fence_after();
        tmem_dealloc(tmem, 512);
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

template <int B, int GD, int GM, int KM>
cudaError_t launch_scan_k(const TopkParams& p, cudaStream_t st) {
    using Lay = TopkLayout<B, GD, GM>;
    static_assert(Lay::smem <= 232448, "top-k shared memory map too large");
    auto kern = k_topk_tc<B, GD, GM, KM>;
    static TqLaunchCache cache;
    cudaError_t e = tq_kernel_setup(kern, kThreads, Lay::smem, cache, nullptr, nullptr);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)((int64_t)p.n_qt * p.nsplit), kThreads, Lay::smem, st>>>(p);
    return cudaGetLastError();
}

// the row's k best live in registers: 16 slots for k <= 16, 32 otherwise
template <int B, int GD, int GM>
cudaError_t launch_scan(const TopkParams& p, cudaStream_t st) {
    return p.k <= 16 ? launch_scan_k<B, GD, GM, 16>(p, st) : launch_scan_k<B, GD, GM, 32>(p, st);
}

}  // namespace

// Ranges per query tile: the split count in 1 .. 64 (at most one per key tile) whose grid
// fills the SMs' waves best (one CTA per SM), the smallest among equals.
int tq_topk_nsplit(int64_t n_qt, int64_t n_tiles) {
    const int64_t sms = tq_device_sms();
    int best = 1;
    double best_eff = -1.0;
    const int64_t cap = std::max<int64_t>(1, std::min<int64_t>(64, n_tiles));
    for (int64_t s = 1; s <= cap; ++s) {
        const int64_t ctas = n_qt * s;
        const int64_t waves = (ctas + sms - 1) / sms;
        const double eff = (double)ctas / (double)(waves * sms);
        if (eff > best_eff + 0.005) { best_eff = eff; best = (int)s; }
    }
    return best;
}

cudaError_t tq_launch_topk(const TopkParams& p, cudaStream_t st) {
    if (p.k < 1 || p.k > kMaxK) return cudaErrorInvalidValue;
    const int64_t rows = (int64_t)p.n_qt * 128;
    k_topk_qprep<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = cudaErrorInvalidValue;
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
