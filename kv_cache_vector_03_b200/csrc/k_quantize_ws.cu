// tq_quantize for bf16 keys with d, m <= 128: a warp-specialized tcgen05 pipeline (rotate,
// nearest Lloyd-Max centroid, residual, QJL sign sketch, pack; blog.hotdry.top "TurboQuant
// vector-search compression", sections "Random rotation and scalar quantization" and "QJL
// residual correction"; a2a-mcp.org "What is TurboQuant", stage 1).
//
// One persistent CTA per SM walks tiles of 128 vectors (four blocks of 32) with 19 warps:
//   warp 16 (one thread)  TMA: the tile's raw bf16 rows, as four 32-row boxes per 64-column
//                         K-block, straight into the 128-byte-swizzled K-major operand layout
//                         (two stages);
//   warp 17 (one thread)  the rotation Y = X (Pi_1 + Pi_2 + Pi_3)^T on the
//                         tensor cores, three bf16 passes whose sum is the fp32 rotation applied
//                         to the exact bf16 input (one pass when Pi is a +-1/sqrt(d) Hadamard
//                         rotation, whose scaled image is exactly +-1), into TMEM;
//   warp 18 (one thread)  the sketch Z = (R_hi + R_lo)(256 M)^T on fp16 (hi.hi + hi.lo + lo.hi)
//                         with the residual operand R read from TMEM, as soon as the epilogue
//                         has written it;
//   warps 0-15            epilogue: warps 0-7 take even tiles, 8-15 odd ones; in each group
//                         warp w owns rows 32 (w mod 4) .. +31 (one vector per thread) and the
//                         column half (w / 4) mod 2:
//                           |x| from the raw bf16 row in shared memory while Y is computed; per-row
//                           thresholds t_k |x| and centroids; from Y the code planes (sign bits),
//                           the scaled residual r |x| 2^k split into an integer-valued fp16 hi part
//                           and an fp16 lo part written to TMEM, gamma^2; then the sign plane from Z.
// Resident in shared memory: Pi_1..3 (bf16) and 256 M hi/lo (fp16), 160 KB, loaded once by
// bulk copies from the prepared images; two 32 KB stages of X. TMEM (512 columns): per tile
// parity two 128-column regions that trade roles on each use: one takes Y and then Z, the
// other the residual operand (hi 64 | lo 64). So the next Y of a parity starts as soon as Z
// has consumed the residual, while the epilogue still reads the signs from the other region.
#include <cuda.h>

#include <algorithm>
#include <atomic>

#include "tq_device.cuh"
#include "tq_tc.cuh"

namespace {
using namespace tqtc;

constexpr int kWsThreads = 608;
constexpr int kTmaWarp = 16, kMmaWarp = 17;   // warps 0-15: epilogue
constexpr uint32_t kMat = 32768;          // one 128 x 128 16-bit operand
constexpr uint32_t kWaitLimit = 1u << 22;

// shared memory map (from a 1024-aligned base)
constexpr uint32_t oPi = 0;               // Pi_1, Pi_2, Pi_3 (bf16)
constexpr uint32_t oM = 3 * kMat;         // M_hi, M_lo (fp16)
constexpr uint32_t oX = 5 * kMat;         // X stage 0, 1 (bf16)
constexpr uint32_t oG2 = 7 * kMat;        // gamma^2 of the upper column half [tile parity][row]
constexpr uint32_t oBar = oG2 + 2 * 128 * 4;   // barriers, then the TMEM base and the abort flag

// barrier indices: per X stage / tile parity, then per (tile parity, lane quarter)
enum {
    bXFull = 0, bXEmpty = 2, bYFull = 4, bRFull = 6, bZFull = 8, bOps = 10, bDrain = 11, bDrainY = 12,
    bG2Full = 13, bG2Empty = 21, kNumBars = 29
};
constexpr size_t kWsSmemUsed = (size_t)oBar + 8 * kNumBars + 8;
constexpr size_t kWsSmem = 232448;        // the per-CTA maximum: the used bytes plus the alignment pad
static_assert(kWsSmemUsed + 1023 <= kWsSmem, "shared memory map too large");

constexpr uint32_t kIdescF16 = idesc_f16(128, 128);
constexpr uint32_t kIdescBF16 = idesc_bf16(128, 128);

// K-step k (16 elements) of a 128 x 128 operand: K-block k / 4, 32 bytes per step inside it
__device__ __forceinline__ uint32_t kstep(int k) { return (uint32_t)(k >> 2) * 16384u + (uint32_t)(k & 3) * 32u; }

// one box of the 3-D tensor map [stream][token][coordinate] (no multicast)
__device__ __forceinline__ void tma_load3(uint32_t dst, const CUtensorMap* map, int c0, int c1, int c2,
                                          uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(tq_smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ uint32_t low_bits(int n) { return n >= 32 ? ~0u : n <= 0 ? 0u : (1u << n) - 1u; }
__device__ __forceinline__ uint32_t shl_in(uint32_t w, uint32_t v) { return __funnelshift_l(v, w, 1); }

struct WsParams {
    uint8_t* packed;
    const uint8_t* img;        // prepared operand images (Pi_1..3, M_hi, M_lo)
    const uint32_t* hdr;       // prep header: +-1 rotation flag, image scale
    uint32_t* status;
    int64_t n_streams, n_tok, nb;
    int d, m;
    TqDims t;
    TqCodebookConsts cb;
};

// sum of squares of the 128 bf16 coordinates of one row of a swizzled X stage (two K-blocks),
// each scaled by sc; four 16-byte chunks in flight at a time
__device__ __forceinline__ float row_ss(const uint8_t* stage, int row, float sc) {
    float s0 = 0.f, s1 = 0.f;
#pragma unroll 4
    for (int c = 0; c < 16; ++c) {
        const uint4 v = *reinterpret_cast<const uint4*>(stage + (c >> 3) * 16384 + sw128(row, c & 7));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float lo = __uint_as_float(w[e] << 16) * sc, hi = __uint_as_float(w[e] & 0xffff0000u) * sc;
            s0 = fmaf(lo, lo, s0);
            s1 = fmaf(hi, hi, s1);
        }
    }
    return s0 + s1;
}

// One row's worth of the code and residual work on 16 TMEM columns: codes into the low
// 16 bits of pw[] (coordinate e at bit e), the residual operand into hw / lw (two fp16 per
// word), gamma^2 into g2. Column index col0 + e; coordinates beyond d (when !FULL) count zero.
template <int B, bool FULL>
__device__ __forceinline__ void residual16(const uint32_t (&yb)[16], const float (&th)[(1 << B) / 2 > 1 ? (1 << B) / 2 - 1 : 1],
                                           const float (&cs)[(1 << B) / 2], float kap, int col0, int d,
                                           uint32_t (&pw)[B], uint32_t (&hw)[8], uint32_t (&lw)[8], float& g2a,
                                           float& g2b) {
    constexpr int H = (1 << B) / 2;
    float rr[16];
#pragma unroll
    for (int pl = 0; pl < B; ++pl) pw[pl] = 0u;
#pragma unroll
    for (int e = 15; e >= 0; --e) {
        const float yv = __uint_as_float(yb[e]);
        const uint32_t w = __float_as_uint(0.f - yv);      // sign bit: y > 0
        const float ay = fabsf(yv);
        float cm = cs[0];
        uint32_t dbits[H > 1 ? H - 1 : 1];
#pragma unroll
        for (int k = 0; k < H - 1; ++k) {
            const float dk = th[k] - ay;                     // sign bit: |y| above boundary k
            dbits[k] = __float_as_uint(dk);
            cm = dk < 0.f ? cs[k + 1] : cm;
        }
        // the centroid takes the sign of y (negative for y <= 0: the lower cell)
        const float csg = __uint_as_float(__float_as_uint(cm) ^ (~w & 0x80000000u));
        float r = fmaf(yv, kap, -csg);
        if (!FULL && col0 + e >= d) r = 0.f;
        rr[e] = r;
        if (e & 1) g2a = fmaf(r, r, g2a);
        else g2b = fmaf(r, r, g2b);
        // index bits: top bit = [y > 0]; lower bits = level bits XNOR [y > 0]
        pw[B - 1] = shl_in(pw[B - 1], w);
        if constexpr (B == 2) {
            pw[0] = shl_in(pw[0], ~(dbits[0] ^ w));
        } else if constexpr (B == 3) {
            pw[1] = shl_in(pw[1], ~(dbits[1] ^ w));
            pw[0] = shl_in(pw[0], ~(dbits[0] ^ dbits[1] ^ dbits[2] ^ w));
        }
    }
    // residual operand: an integer-valued hi part (|hi| <= 2048, exact in fp16) and the
    // remainder in [-1/2, 1/2] as lo
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const float h0 = (rr[2 * q] + 12582912.f) - 12582912.f;
        const float h1 = (rr[2 * q + 1] + 12582912.f) - 12582912.f;
        hw[q] = pack_half2(h0, h1);
        lw[q] = pack_half2(rr[2 * q] - h0, rr[2 * q + 1] - h1);
    }
}

template <int B, bool FULL>
__global__ void __launch_bounds__(kWsThreads, 1) k_quantize_ws(const __grid_constant__ CUtensorMap xmap, WsParams p) {
    constexpr int L = 1 << B, H = L / 2;
    extern __shared__ uint8_t raw_smem[];
    const uint32_t raw = tq_smem_addr(raw_smem);
    const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
    uint8_t* sm = raw_smem + pad;
    const uint32_t sb = raw + pad;
    float* s_g2 = reinterpret_cast<float*>(sm + oG2);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + oBar);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + oBar + 8 * kNumBars);
    volatile uint32_t* s_abort = s_tmem + 1;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t total_blocks = p.n_streams * p.nb;
    const int64_t n_tiles = (total_blocks + 3) / 4;
    const int n_local = (int)((n_tiles - blockIdx.x + gridDim.x - 1) / gridDim.x);   // tiles of this CTA

    if (tid == 0) {
        for (int i = 0; i < kNumBars; ++i) {
            int count = 1;
            if (i >= bXEmpty && i < bXEmpty + 2) count = 9;       // the Y commit and the 8 warps of a tile
            if (i >= bRFull && i < bRFull + 2) count = 8;         // the 8 warps of a tile
            if (i >= bG2Full && i < bG2Full + 8) count = 32;      // every lane of the upper-half warp
            tq_mbar_init(&bars[i], count);
        }
        *s_abort = 0u;
        tq_fence_mbar_init();
    }
    if (warp == kMmaWarp) tmem_alloc(s_tmem, 512);
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = *s_tmem;
    // TMEM regions of tile i (parity b = i & 1, use j = i >> 1 of that parity): Y then Z in
    // acc(i), the residual operand in res(i); the two regions of a parity trade roles each use
    auto acc_col = [](int i) { return 256u * (uint32_t)(i & 1) + 128u * (uint32_t)((i >> 1) & 1); };
    auto res_col = [](int i) { return 256u * (uint32_t)(i & 1) + 128u * (uint32_t)(((i >> 1) + 1) & 1); };

    if (warp == kTmaWarp) {
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&xmap)) : "memory");
            // resident operands: five 32 KB images
            mbar_expect_tx(&bars[bOps], 5 * kMat);
            for (int i = 0; i < 5; ++i) bulk_copy(sb + oPi + i * kMat, p.img + (size_t)i * kMat, kMat, &bars[bOps]);
            int issued = 0;
            for (int i = 0; i < n_local; ++i) {
                const int xs = i & 1;
                // the stage is free once Y(i - 2) and the epilogue's norm pass have read it
                if (i >= 2 && !wait_bar(&bars[bXEmpty + xs], ((i >> 1) - 1) & 1, s_abort, kWaitLimit)) break;
                const int64_t tile = blockIdx.x + (int64_t)i * gridDim.x;
                const int64_t left = total_blocks - tile * 4;
                const int nvb = left < 4 ? (int)left : 4;
                mbar_expect_tx(&bars[bXFull + xs], (uint32_t)nvb * 8192u);
                for (int jb = 0; jb < nvb; ++jb) {
                    const int64_t gb = tile * 4 + jb;
                    const int s = (int)(gb / p.nb), tok0 = (int)(gb % p.nb) * 32;
#pragma unroll
                    for (int h = 0; h < 2; ++h)
                        tma_load3(sb + oX + xs * kMat + h * 16384 + jb * 4096, &xmap, 64 * h, tok0, s, &bars[bXFull + xs]);
                }
                issued = i + 1;
            }
            // nothing may be in flight when the CTA exits (a completed phase returns at once)
            for (int i = issued - 2 < 0 ? 0 : issued - 2; i < issued; ++i)
                tq_mbar_wait(&bars[bXFull + (i & 1)], (i >> 1) & 1, kWaitLimit);
            tq_mbar_wait(&bars[bOps], 0, kWaitLimit);
        }
    } else if (warp == kMmaWarp) {
        // rotation issue: a +-1/sqrt(d) rotation needs the first (exact +-1) piece only
        if (lane == 0) {
            const int y_passes = (p.hdr[0] & TQ_PREP_PM1) ? 1 : 3;
            bool ok = wait_bar(&bars[bOps], 0, s_abort, kWaitLimit);
            for (int i = 0; ok && i < n_local; ++i) {
                const int b = i & 1;
                if (!wait_bar(&bars[bXFull + b], (i >> 1) & 1, s_abort, kWaitLimit)) break;
                // the region takes Y(i) once Z(i - 2) has consumed the residual held there
                if (i >= 2 && !wait_bar(&bars[bZFull + b], ((i >> 1) - 1) & 1, s_abort, kWaitLimit)) break;
                fence_after();
                const uint32_t d = tmem + acc_col(i), xa = sb + oX + b * kMat;
                for (int ps = 0; ps < y_passes; ++ps)
#pragma unroll
                    for (int k = 0; k < 8; ++k)
                        mma_ss(d, sdesc(xa + kstep(k)), sdesc(sb + oPi + ps * kMat + kstep(k)), kIdescBF16,
                               (ps | k) != 0);
                commit(&bars[bYFull + b]);
                commit(&bars[bXEmpty + b]);
            }
            // every Y has completed before TMEM is released
            commit(&bars[bDrainY]);
            tq_mbar_wait(&bars[bDrainY], 0, kWaitLimit);
        }
    } else if (warp == kMmaWarp + 1) {
        // sketch issue
        if (lane == 0) {
            for (int i = 0; i < n_local; ++i) {
                const int b = i & 1;
                if (!wait_bar(&bars[bRFull + b], (i >> 1) & 1, s_abort, kWaitLimit)) break;
                fence_after();
                const uint32_t d = tmem + acc_col(i), r = tmem + res_col(i);
#pragma unroll
                for (int ps = 0; ps < 3; ++ps) {
                    const uint32_t ra = r + (ps == 2 ? 64u : 0u);
                    const uint32_t mb = sb + oM + (ps == 1 ? kMat : 0u);
#pragma unroll
                    for (int k = 0; k < 8; ++k) mma_ts(d, ra + 8u * k, sdesc(mb + kstep(k)), kIdescF16, (ps | k) != 0);
                }
                commit(&bars[bZFull + b]);
            }
            // every Z has completed before TMEM is released
            commit(&bars[bDrain]);
            tq_mbar_wait(&bars[bDrain], 0, kWaitLimit);
        }
    } else {
        // ------------------------------------------------------------------ epilogue
        const int par = warp >> 3, half = (warp >> 2) & 1, wq = warp & 3;
        const uint32_t lane_base = (uint32_t)(32 * wq) << 16;
        const int row = 32 * wq + lane, u = lane >> 3, gq = lane & 7;
        float* g2x = s_g2 + par * 128 + row;
        uint64_t* g2full = &bars[bG2Full + 4 * par + wq];
        uint64_t* g2empty = &bars[bG2Empty + 4 * par + wq];
        const uint8_t* xst = sm + oX + par * kMat;   // this group's X stage
        // Y rows are the rotation scaled by the Pi_1 image factor (sqrt(d) for a +-1 rotation)
        const float y_scale = reinterpret_cast<const float*>(p.hdr)[1];
        float tb[H > 1 ? H - 1 : 1], cmg[H];
#pragma unroll
        for (int k = 0; k < H - 1; ++k) tb[k] = p.cb.bounds[H + k];
#pragma unroll
        for (int k = 0; k < H; ++k) cmg[k] = p.cb.cent[H + k];
        // every lane waits (and acquires); the warp continues only if all of them succeeded
        auto warp_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
            return __all_sync(0xffffffffu, wait_bar(bar, parity, s_abort, kWaitLimit)) != 0;
        };
        int j = 0;
        for (int i = par; i < n_local; i += 2, ++j) {
            const int64_t tile = blockIdx.x + (int64_t)i * gridDim.x;
            const int64_t gb = tile * 4 + wq;
            const bool blk_ok = gb < total_blocks;
            const int64_t tok = blk_ok ? (gb % p.nb) * 32 + lane : 0;
            const bool rvalid = blk_ok && tok < p.n_tok;
            uint8_t* blk = p.packed + (size_t)(blk_ok ? gb : 0) * p.t.block_bytes;
            const uint32_t tY = tmem + lane_base + acc_col(i);   // Y, then Z
            const uint32_t tR = tmem + lane_base + res_col(i);   // residual operand hi | lo
            // |x| from the raw row (exact bf16 inputs) while the tensor cores rotate it; both
            // column halves take the whole row, in the same order
            if (!warp_wait(&bars[bXFull + par], j & 1)) break;
            float ss = row_ss(xst, row, 1.f);
            const bool tiny = ss < 1e-30f && ss > 0.f;
            if (__any_sync(0xffffffffu, tiny)) {
                // a tiny vector in the warp: its sum of squares again on the whole row scaled by 2^60
                const float acc = row_ss(xst, row, 0x1p60f);
                if (tiny) ss = fmaxf(acc * 0x1p-120f, 0x1p-149f);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[bXEmpty + par]);
            const float n = sqrtf(ss);
            const bool finite = isfinite(n);
            const float ny = n * y_scale;
            const float ne = (ny > 0.f && finite) ? ny : 1.f;
            // kap = 2^(10 - floor(log2 ne)): |residual| * ne * kap < 2^11 (integer hi part exact in fp16)
            const int ex = ((__float_as_int(ne) >> 23) & 0xff) - 127;
            const float kap = __int_as_float((127 + min(max(10 - ex, -126), 127)) << 23);
            float th[H > 1 ? H - 1 : 1], cs[H];
#pragma unroll
            for (int k = 0; k < H - 1; ++k) th[k] = tb[k] * ne;
#pragma unroll
            for (int k = 0; k < H; ++k) cs[k] = cmg[k] * ne * kap;
            if (!warp_wait(&bars[bYFull + par], j & 1)) break;
            fence_after();
            // codes and residual of this warp's 64 columns: two plane words (chunks 2 half, +1)
            float g2a = 0.f, g2b = 0.f;
            {
                uint32_t ya[16], yb[16];
                const uint32_t y0 = tY + 64u * half, r0 = tR + 32u * half;
                tld16(y0, ya);
                twait(ya);
#pragma unroll 1
                for (int q = 0; q < 2; ++q) {
                    const int c = 2 * half + q;      // 32-coordinate chunk = plane word index
                    uint32_t pa[B], pb[B], hw[8], lw[8];
                    tld16(y0 + 32u * q + 16u, yb);
                    residual16<B, FULL>(ya, th, cs, kap, 32 * c, p.d, pa, hw, lw, g2a, g2b);
                    tst8(r0 + 16u * q, hw);
                    tst8(r0 + 64u + 16u * q, lw);
                    twait(yb);
                    if (q == 0) tld16(y0 + 32u, ya);
                    residual16<B, FULL>(yb, th, cs, kap, 32 * c + 16, p.d, pb, hw, lw, g2a, g2b);
                    tst8(r0 + 16u * q + 8u, hw);
                    tst8(r0 + 64u + 16u * q + 8u, lw);
                    if (blk_ok) {
                        const uint32_t keep = rvalid ? low_bits(p.d - 32 * c) : 0u;
#pragma unroll
                        for (int pl = 0; pl < B; ++pl)
                            reinterpret_cast<uint32_t*>(blk)[(pl * 32 + 4 * gq + c) * 4 + u] =
                                ((pb[pl] << 16) | pa[pl]) & keep;
                    }
                    if (q == 0) twait(ya);
                }
            }
            twait_st();
            fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[bRFull + par]);
            // gamma^2: the upper column half hands its partial sum to the lower one
            float g2 = g2a + g2b;
            if (half == 1) {
                if (j > 0 && !warp_wait(g2empty, (j - 1) & 1)) break;
                *g2x = g2;
                mbar_arrive(g2full);
            }
            // signs of Z = R M^T over this warp's columns
            if (!warp_wait(&bars[bZFull + par], j & 1)) break;
            fence_after();
            {
                uint32_t za[16], zb[16];
                const uint32_t z0 = tY + 64u * half;
                tld16(z0, za);
                twait(za);
#pragma unroll 1
                for (int q = 0; q < 2; ++q) {
                    const int c = 2 * half + q;
                    tld16(z0 + 32u * q + 16u, zb);
                    uint32_t sa = 0u, sbw = 0u;
#pragma unroll
                    for (int e = 15; e >= 0; --e) sa = shl_in(sa, za[e]);
                    twait(zb);
                    if (q == 0) tld16(z0 + 32u, za);
#pragma unroll
                    for (int e = 15; e >= 0; --e) sbw = shl_in(sbw, zb[e]);
                    // bit = [z >= 0]: the sign bit inverted (an exact zero has sign bit 0)
                    if (blk_ok)
                        reinterpret_cast<uint32_t*>(blk)[(B * 32 + 4 * gq + c) * 4 + u] =
                            rvalid ? ~((sbw << 16) | sa) & low_bits(p.m - 32 * c) : 0u;
                    if (q == 0) twait(za);
                }
            }
            if (half == 0) {
                if (!warp_wait(g2full, j & 1)) break;
                g2 += *g2x;
                __syncwarp();
                if (lane == 0) mbar_arrive(g2empty);
                if (blk_ok) {
                    const float gam = sqrtf(g2) / (ne * kap);
                    const uint32_t nh = rvalid ? tq_half_bits(n) : 0u;
                    const uint32_t gh = rvalid ? tq_half_bits(gam) : 0u;
                    if (rvalid && (!finite || (nh & 0x7fffu) >= 0x7c00u)) tq_raise(p.status, TQ_FLAG_RANGE);
                    reinterpret_cast<uint32_t*>(blk + p.t.sec_a)[gq * 4 + u] = nh | (gh << 16);
                }
            }
        }
    }
    __syncthreads();
    if (*s_abort) {
        if (tid == 0) tq_raise(p.status, TQ_FLAG_TIMEOUT);
    }
    if (warp == kMmaWarp) {
        fence_after();
        tmem_dealloc(tmem, 512);
    }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                    const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled through the runtime's driver entry point (libtq does not link libcuda)
EncodeTiledFn encode_tiled() {
    static std::atomic<EncodeTiledFn> fn{nullptr};
    EncodeTiledFn f = fn.load(std::memory_order_acquire);
    if (f) return f;
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !ptr) {
        cudaGetLastError();
        return nullptr;
    }
    f = reinterpret_cast<EncodeTiledFn>(ptr);
    fn.store(f, std::memory_order_release);
    return f;
}

template <int B, bool FULL>
cudaError_t launch_ws(const CUtensorMap& map, const WsParams& wp, cudaStream_t st) {
    auto kern = k_quantize_ws<B, FULL>;
    static TqLaunchCache cache;
    int sms = 0;
    cudaError_t e = tq_kernel_setup(kern, kWsThreads, kWsSmem, cache, &sms, nullptr);
    if (e != cudaSuccess) return e;
    const int64_t tiles = (wp.n_streams * wp.nb + 3) / 4;
    const int64_t grid = std::min<int64_t>(tiles, sms);
    if (grid > 0) kern<<<(unsigned)grid, kWsThreads, kWsSmem, st>>>(map, wp);
    return cudaGetLastError();
}

}  // namespace

// Whether the warp-specialized kernel takes this request: bf16 keys with D = Mp = 128, B <= 3,
// the prepared images present, and rows a tensor map can describe (16-byte aligned base, stream
// stride a multiple of 8 elements).
bool tq_quantize_ws_eligible(const QuantParams& p) {
    if (!p.t.qjl || p.dtype != 1 || p.t.D != 128 || p.t.Mp != 128 || !p.img) return false;
    if (p.t.B < 1 || p.t.B > 3) return false;
    if ((reinterpret_cast<uintptr_t>(p.x) & 15) != 0) return false;
    if (p.n_streams > 1 && p.x_stride % 8 != 0) return false;
    if (p.n_tok > 0x7fffffffLL || p.n_streams > 0x7fffffffLL) return false;
    return encode_tiled() != nullptr;
}

cudaError_t tq_launch_quantize_ws(const QuantParams& p, cudaStream_t st) {
    EncodeTiledFn enc = encode_tiled();
    if (!enc) return cudaErrorNotSupported;
    CUtensorMap map;
    const cuuint64_t dims[3] = {(cuuint64_t)p.t.d, (cuuint64_t)p.n_tok, (cuuint64_t)p.n_streams};
    const int64_t stride = p.n_streams > 1 ? p.x_stride : p.n_tok * p.t.d;
    const cuuint64_t strides[2] = {(cuuint64_t)p.t.d * 2, (cuuint64_t)stride * 2};
    const cuuint32_t box[3] = {64, 32, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(p.x), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    WsParams wp;
    wp.packed = p.packed;
    wp.img = p.img;
    wp.hdr = p.hdr;
    wp.status = p.status;
    wp.n_streams = p.n_streams;
    wp.n_tok = p.n_tok;
    wp.nb = p.nb;
    wp.d = p.t.d;
    wp.m = p.t.m;
    wp.t = p.t;
    wp.cb = p.cb;
    const bool full = p.t.d == 128;
    switch (p.t.B) {
        case 1: return full ? launch_ws<1, true>(map, wp, st) : launch_ws<1, false>(map, wp, st);
        case 2: return full ? launch_ws<2, true>(map, wp, st) : launch_ws<2, false>(map, wp, st);
        case 3: return full ? launch_ws<3, true>(map, wp, st) : launch_ws<3, false>(map, wp, st);
    }
    return cudaErrorInvalidValue;
}
