// tq_quantize for keys with D = Mp = 256 (d and m in 129..256, e.g. the d = 200 codec of
// the vector-search workload) on the fifth-generation tensor cores: rotate, nearest
// Lloyd-Max centroid, residual, QJL sign sketch, pack (blog.hotdry.top "TurboQuant
// vector-search compression", sections "Random rotation and scalar quantization" and "QJL
// residual correction"; a2a-mcp.org "What is TurboQuant", stage 1 and the GloVe d = 200
// benchmark).
//
// One persistent CTA of 16 warps per SM walks tiles of 128 vectors in phases:
//   A. warp w converts rows 8w .. 8w + 7 (held in registers, loaded during the previous
//      tile's sketch): |x|, a power-of-two row scale, fp16 hi and lo parts of the scaled row
//      as the A operand (four 64-column K-blocks, 128-byte swizzle, 128 KB);
//   B. one thread issues Y = X (256 Pi)^T (hi.hi + hi.lo + lo.hi) as 128 x 128 x 16 MMAs into
//      TMEM columns 0..255, the B operand streamed from L2 in 32 KB chunks (a K-block of 64
//      columns for one half of the output rows, hi and lo) through a three-slot ring of
//      bulk copies that runs two chunks ahead;
//   C. warp w reads TMEM lanes 32 (w mod 4) .. +31 and columns 64 (w / 4) .. +63: codes
//      (compare-count against the fp32 boundaries), code planes, the residual r scaled by
//      2^12 and split into fp16 hi / lo, written over X as the A operand of the sketch;
//      gamma^2 partials meet in spare TMEM columns;
//   D. Z = R (256 M)^T in the same way (M = S Pi^T), into TMEM columns 0..255;
//   E. sign planes from Z, norms and gamma.
#include "tq_device.cuh"

namespace {

constexpr int kWThreads = 512;
constexpr uint32_t kChunk = 32768;
constexpr int kSlots = 3;
constexpr uint32_t kWaitLimit = 1u << 22;
constexpr uint32_t oA = 0;                         // A operand: hi K-blocks 0..3, then lo K-blocks 0..3
constexpr uint32_t oB = 131072;                    // chunk ring
constexpr uint32_t oSmall = oB + kSlots * kChunk;  // per-row data, barriers
constexpr size_t kWideSmem = 232448;
constexpr size_t kWideUsed = oSmall + 128 * 4 * 2 + 256 + 8 * 8 + 16;
static_assert(kWideUsed + 1023 <= kWideSmem, "shared memory map too large");

constexpr uint32_t kIdesc = (1u << 4) | ((128u >> 3) << 17) | ((128u >> 4) << 24);   // fp16, fp32 D, M = N = 128

__device__ __forceinline__ uint64_t sdesc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
__device__ __forceinline__ void mma(uint32_t d, uint64_t a, uint64_t b, uint32_t acc) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %3, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %4, p;\n}\n" ::"r"(d),
        "l"(a), "l"(b), "r"(acc), "r"(kIdesc));
}
__device__ __forceinline__ void commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     tq_smem_addr(bar))
                 : "memory");
}
__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}
// wait for this thread's TMEM loads; the last load's registers are operands, so no use of
// them is scheduled before the wait
__device__ __forceinline__ void twait(uint32_t (&r)[16]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                   "+r"(r[15])
                 :
                 : "memory");
}
__device__ __forceinline__ void tst1(uint32_t taddr, float v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(__float_as_uint(v)) : "memory");
}
__device__ __forceinline__ void tld4(uint32_t taddr, float (&v)[4]) {
    uint32_t r[4];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr)
                 : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3])::"memory");
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ uint32_t low_bits(int n) { return n >= 32 ? ~0u : n <= 0 ? 0u : (1u << n) - 1u; }
__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
    const __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&h);
}
// byte offset of 16-byte chunk kc (columns 8 kc .. 8 kc + 7) of row r in a 64-column K-block
__device__ __forceinline__ uint32_t kb_off(int r, int kc) {
    return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + (((kc & 7) ^ (r & 7)) << 4));
}

constexpr int kRowsPerWarp = 8;

template <bool kF32>
struct WideRows;
template <>
struct WideRows<true> { float4 v[kRowsPerWarp][2]; };   // lane: columns 4 lane .. +3 and 128 + 4 lane .. +3
template <>
struct WideRows<false> { uint2 v[kRowsPerWarp][2]; };

template <bool kF32, int B>
__global__ void __launch_bounds__(kWThreads, 1) k_quantize_wide(QuantParams p) {
    constexpr int L = 1 << B;
    extern __shared__ uint8_t raw_smem[];
    const uint32_t raw = tq_smem_addr(raw_smem);
    const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
    uint8_t* sm = raw_smem + pad;
    const uint32_t sb = raw + pad;
    float* s_inv = reinterpret_cast<float*>(sm + oSmall);        // [128] 4096 / (|x| 256 sc)
    float* s_norm = s_inv + 128;                                   // [128]
    uint8_t* s_flags = reinterpret_cast<uint8_t*>(s_norm + 128);   // [128] bit 0 valid, bit 1 bad; [128] spare
    uint64_t* bars = reinterpret_cast<uint64_t*>(s_flags + 256);   // full[3], free[3], done
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 8);

    const TqDims& T = p.t;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int d = T.d;
    const int64_t total_blocks = p.n_streams * p.nb;
    const int64_t n_tiles = (total_blocks + 3) / 4;

    if (tid == 0) {
        for (int i = 0; i < 2 * kSlots + 1; ++i) tq_mbar_init(&bars[i], 1);
        tq_fence_mbar_init();
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tq_smem_addr(s_tmem)),
                     "r"(512));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = *s_tmem;

    // chunk ring, driven by thread 0: chunk q of the CTA's sequence (16 per tile: 8 of Pi,
    // then 8 of M, in consumption order) lives in slot q % 3
    uint32_t n_loaded = 0, n_used = 0;
    const int my_tiles = (int)((n_tiles - blockIdx.x + gridDim.x - 1) / gridDim.x);
    const uint32_t n_chunks = 16u * (uint32_t)my_tiles;
    auto load_chunk = [&](uint32_t q) -> bool {
        const uint32_t slot = q % kSlots;
        if (q >= kSlots && !tq_mbar_wait(&bars[kSlots + slot], ((q / kSlots) - 1) & 1u, kWaitLimit)) return false;
        tq_bulk_load(sm + oB + slot * kChunk, p.wimg + (size_t)(q & 15u) * kChunk, kChunk, &bars[slot]);
        return true;
    };
    bool ok = true;
    if (tid == 0)
        for (; n_loaded < 2 && n_loaded < n_chunks; ++n_loaded) ok = ok && load_chunk(n_loaded);
    // thread 0: the 8 chunks of one product (12 MMAs each), keeping the ring two chunks ahead
    auto run_product = [&](uint32_t tmem_d) -> bool {
        for (int c = 0; c < 8; ++c) {
            const uint32_t q = n_used, slot = q % kSlots;
            if (!tq_mbar_wait(&bars[slot], (q / kSlots) & 1u, kWaitLimit)) return false;
            fence_after();
            const int nh = c >> 2, kb = c & 3;
            const uint32_t bslot = sb + oB + slot * kChunk;
#pragma unroll
            for (int ps = 0; ps < 3; ++ps) {
                const uint32_t a = sb + oA + (ps == 2 ? 65536u : 0u) + (uint32_t)kb * 16384u;
                const uint32_t b = bslot + (ps == 1 ? 16384u : 0u);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma(tmem_d + 128u * nh, sdesc(a + 32u * k), sdesc(b + 32u * k), (ps | kb | k) != 0);
            }
            commit(&bars[kSlots + slot]);
            ++n_used;
            if (n_loaded < n_chunks) {
                if (!load_chunk(n_loaded)) return false;
                ++n_loaded;
            }
        }
        commit(&bars[2 * kSlots]);
        return true;
    };
    uint32_t n_prod = 0;
    auto wait_product = [&]() -> bool {
        bool w = true;
        if (tid == 0) w = ok && tq_mbar_wait(&bars[2 * kSlots], n_prod & 1u, kWaitLimit);
        ++n_prod;
        const bool all = __syncthreads_and(w) != 0;
        fence_after();
        return all;
    };

    WideRows<kF32> rg;
    auto load_rows = [&](int64_t tile) {
        const int64_t gb = tile * 4 + (warp >> 2);
        const int64_t s = gb / p.nb, tok0 = (gb % p.nb) * 32 + kRowsPerWarp * (warp & 3);
        const bool blk = gb < total_blocks;
        const int64_t base0 = s * p.x_stride + tok0 * d;
#pragma unroll
        for (int rr = 0; rr < kRowsPerWarp; ++rr) {
            const bool in = blk && tok0 + rr < p.n_tok;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int col = 128 * h + 4 * lane;
                const bool cin = in && col < d;
                const int64_t e0 = base0 + (int64_t)rr * d + col;
                if constexpr (kF32) {
                    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (cin) {
                        const float* xp = static_cast<const float*>(p.x) + e0;
                        v = p.vec_ok ? __ldg(reinterpret_cast<const float4*>(xp)) : make_float4(xp[0], xp[1], xp[2], xp[3]);
                    }
                    rg.v[rr][h] = v;
                } else {
                    uint2 v = make_uint2(0u, 0u);
                    if (cin) {
                        const uint16_t* xp = static_cast<const uint16_t*>(p.x) + e0;
                        v = p.vec_ok ? __ldg(reinterpret_cast<const uint2*>(xp))
                                     : make_uint2((uint32_t)xp[0] | ((uint32_t)xp[1] << 16),
                                                  (uint32_t)xp[2] | ((uint32_t)xp[3] << 16));
                    }
                    rg.v[rr][h] = v;
                }
            }
        }
    };

    // codebook in registers
    float bnd[L - 1], cen[L];
#pragma unroll
    for (int k = 0; k < L - 1; ++k) bnd[k] = p.cb.bounds[k];
#pragma unroll
    for (int k = 0; k < L; ++k) cen[k] = 4096.f * p.cb.cent[k];
    // coordinates >= d read y = 0 (zero rows of Pi); their residual is excluded from gamma^2
    const int wq = warp & 3, cq = warp >> 2;          // epilogue: lane quarter, column quarter
    const uint32_t lane_base = (uint32_t)(32 * wq) << 16;
    const int row = 32 * wq + lane;
    const int vb = row & 31, u = vb >> 3, gq = vb & 7;

    if ((int64_t)blockIdx.x < n_tiles) load_rows(blockIdx.x);
    for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
        // ---- A. rows -> |x|, power-of-two scale, fp16 hi / lo A operand
        {
            float x[kRowsPerWarp][8];
#pragma unroll
            for (int rr = 0; rr < kRowsPerWarp; ++rr)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    if constexpr (kF32) {
                        x[rr][4 * h] = rg.v[rr][h].x; x[rr][4 * h + 1] = rg.v[rr][h].y;
                        x[rr][4 * h + 2] = rg.v[rr][h].z; x[rr][4 * h + 3] = rg.v[rr][h].w;
                    } else {
                        x[rr][4 * h] = __uint_as_float(rg.v[rr][h].x << 16);
                        x[rr][4 * h + 1] = __uint_as_float(rg.v[rr][h].x & 0xffff0000u);
                        x[rr][4 * h + 2] = __uint_as_float(rg.v[rr][h].y << 16);
                        x[rr][4 * h + 3] = __uint_as_float(rg.v[rr][h].y & 0xffff0000u);
                    }
                }
            const int64_t gb = tile * 4 + (warp >> 2);
            const int64_t tok0 = (gb % p.nb) * 32 + kRowsPerWarp * (warp & 3);
#pragma unroll
            for (int rr = 0; rr < kRowsPerWarp; ++rr) {
                float v = 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) v = fmaf(x[rr][e], x[rr][e], v);
                v = tq_warp_sum(v);
                const int r = kRowsPerWarp * warp + rr;
                const bool valid = gb < total_blocks && tok0 + rr < p.n_tok;
                const float n = sqrtf(v);
                // 2^ex with |x| 2^ex in [2^14, 2^15): every element then fits binary16
                int ex = 0;
                if (n > 0.f && isfinite(n)) ex = min(max(14 - (((__float_as_int(n) >> 23) & 0xff) - 127), -126), 126);
                const float sc2 = __int_as_float((127 + ex) << 23);
                if (lane == 0) {
                    s_norm[r] = valid ? n : 0.f;
                    s_inv[r] = n > 0.f ? 4096.f / (n * 256.f * sc2) : 0.f;
                    s_flags[r] = (uint8_t)((valid ? 1u : 0u) | ((valid && !isfinite(n)) ? 2u : 0u));
                }
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float a0 = x[rr][4 * h] * sc2, a1 = x[rr][4 * h + 1] * sc2;
                    const float a2 = x[rr][4 * h + 2] * sc2, a3 = x[rr][4 * h + 3] * sc2;
                    const uint32_t h01 = pack_half2(a0, a1), h23 = pack_half2(a2, a3);
                    const float2 f01 = __half22float2(*reinterpret_cast<const __half2*>(&h01));
                    const float2 f23 = __half22float2(*reinterpret_cast<const __half2*>(&h23));
                    const uint32_t l01 = pack_half2(a0 - f01.x, a1 - f01.y), l23 = pack_half2(a2 - f23.x, a3 - f23.y);
                    // columns 128 h + 4 lane .. +3: K-block kb = 2 h + lane / 16, chunk (lane mod 16) / 2
                    const int kb = 2 * h + (lane >> 4), kc = (lane & 15) >> 1;
                    const uint32_t off = (uint32_t)kb * 16384u + kb_off(r, kc) + (lane & 1) * 8;
                    *reinterpret_cast<uint2*>(sm + oA + off) = make_uint2(h01, h23);
                    *reinterpret_cast<uint2*>(sm + oA + 65536 + off) = make_uint2(l01, l23);
                }
            }
        }
        tq_fence_proxy_async();
        fence_before();
        __syncthreads();
        // the next tile's rows stream in while this one is in the tensor cores
        if (tile + gridDim.x < n_tiles) load_rows(tile + gridDim.x);
        // ---- B. Y = X (256 Pi)^T
        if (tid == 0) {
            fence_after();
            ok = ok && run_product(tmem);
        }
        if (!wait_product()) break;

        // ---- C. codes, residual (scaled by 2^12), gamma^2 partials; R over X
        const int64_t gb = tile * 4 + (row >> 5);
        const bool blk_ok = gb < total_blocks;
        const uint8_t fl = s_flags[row];
        const bool rvalid = (fl & 1u) != 0;
        const float inv = s_inv[row];
        uint8_t* blk = p.packed + (size_t)(blk_ok ? gb : 0) * T.block_bytes;
        float g2 = 0.f;
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {         // 16 columns at a time: 64 cq + 16 q ..
            uint32_t yb[16];
            const int col0 = 64 * cq + 16 * q;
            tld16(tmem + lane_base + (uint32_t)col0, yb);
            twait(yb);
            uint32_t pw[B];
#pragma unroll
            for (int pl = 0; pl < B; ++pl) pw[pl] = 0u;
            float rv[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const float yy = __uint_as_float(yb[e]) * inv;       // y scaled by 2^12
                int c = 0;
#pragma unroll
                for (int k = 0; k < L - 1; ++k) c += yy > 4096.f * bnd[k];
                float cc = cen[0];
#pragma unroll
                for (int k = 1; k < L; ++k) cc = c == k ? cen[k] : cc;
                const float r = col0 + e < d ? yy - cc : 0.f;
                rv[e] = r;
                g2 = fmaf(r, r, g2);
#pragma unroll
                for (int pl = 0; pl < B; ++pl) pw[pl] |= (uint32_t)((c >> pl) & 1) << e;
            }
            // residual operand: hi = fp16(r), lo = fp16(r - hi), K-block cq, chunks 2q, 2q + 1
            uint32_t hw[8], lw[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const uint32_t h2 = pack_half2(rv[2 * e], rv[2 * e + 1]);
                const float2 f2 = __half22float2(*reinterpret_cast<const __half2*>(&h2));
                hw[e] = h2;
                lw[e] = pack_half2(rv[2 * e] - f2.x, rv[2 * e + 1] - f2.y);
            }
#pragma unroll
            for (int hv = 0; hv < 2; ++hv) {
                const uint32_t off = (uint32_t)cq * 16384u + kb_off(row, 2 * q + hv);
                *reinterpret_cast<uint4*>(sm + oA + off) = make_uint4(hw[4 * hv], hw[4 * hv + 1], hw[4 * hv + 2], hw[4 * hv + 3]);
                *reinterpret_cast<uint4*>(sm + oA + 65536 + off) =
                    make_uint4(lw[4 * hv], lw[4 * hv + 1], lw[4 * hv + 2], lw[4 * hv + 3]);
            }
            // code plane words: coordinates 32 w .. +31 of plane group (w / 4), word w mod 4
            const int word = (col0 >> 5), half16 = (col0 >> 4) & 1;
            if (blk_ok) {
                // two 16-column pieces of one 32-bit word: the even piece writes the low half
                const int gr = word >> 2, tq = word & 3;
                const uint32_t keep = rvalid ? low_bits(d - col0) & 0xffffu : 0u;
#pragma unroll
                for (int pl = 0; pl < B; ++pl) {
                    uint16_t* wp = reinterpret_cast<uint16_t*>(blk) +
                                   2 * (((pl * T.GD + gr) * 32 + 4 * gq + tq) * 4 + u) + half16;
                    *wp = (uint16_t)(pw[pl] & keep);
                }
            }
        }
        // gamma^2 partials of the four column quarters meet in TMEM columns 256 .. 259
        tst1(tmem + lane_base + 256u + (uint32_t)cq, g2);
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        tq_fence_proxy_async();
        fence_before();
        __syncthreads();
        // ---- D. Z = R (256 M)^T
        if (tid == 0) {
            fence_after();
            ok = ok && run_product(tmem);
        }
        if (!wait_product()) break;

        // ---- E. signs, norms, gamma
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {
            uint32_t zb[16];
            const int col0 = 64 * cq + 16 * q;
            tld16(tmem + lane_base + (uint32_t)col0, zb);
            twait(zb);
            uint32_t sw = 0u;
#pragma unroll
            for (int e = 0; e < 16; ++e) sw |= (uint32_t)(__uint_as_float(zb[e]) >= 0.f) << e;
            if (blk_ok) {
                const int word = col0 >> 5, half16 = (col0 >> 4) & 1;
                const int gr = word >> 2, tq = word & 3;
                const uint32_t keep = rvalid ? low_bits(T.m - col0) & 0xffffu : 0u;
                uint16_t* wp = reinterpret_cast<uint16_t*>(blk) +
                               2 * (((B * T.GD + gr) * 32 + 4 * gq + tq) * 4 + u) + half16;
                *wp = (uint16_t)(sw & keep);
            }
        }
        if (cq == 0) {
            float g4[4];
            tld4(tmem + lane_base + 256u, g4);
            if (blk_ok) {
                const uint32_t nh = rvalid ? tq_half_bits(s_norm[row]) : 0u;
                // coordinates >= d contribute no residual (masked above); gamma of the unit vector
                const float gam = sqrtf(fmaxf(g4[0] + g4[1] + g4[2] + g4[3], 0.f)) * (1.f / 4096.f);
                const uint32_t gh = rvalid ? tq_half_bits(gam) : 0u;
                if (rvalid && ((fl & 2u) || (nh & 0x7fffu) >= 0x7c00u)) tq_raise(p.status, TQ_FLAG_RANGE);
                reinterpret_cast<uint32_t*>(blk + T.sec_a)[gq * 4 + u] = nh | (gh << 16);
            }
        } else {
            float g4[4];
            tld4(tmem + lane_base + 256u, g4);   // keep the warp-wide TMEM loads uniform
            (void)g4;
        }
        fence_before();
        __syncthreads();
        fence_after();
    }
    if (tid == 0 && !ok) tq_raise(p.status, TQ_FLAG_TIMEOUT);
    // thread 0: every MMA it issued completes and every chunk it loaded lands before exit
    if (tid == 0) {
        commit(&bars[2 * kSlots]);
        tq_mbar_wait(&bars[2 * kSlots], n_prod & 1u, kWaitLimit);
        for (uint32_t q = n_used; q < n_loaded; ++q) tq_mbar_wait(&bars[q % kSlots], (q / kSlots) & 1u, kWaitLimit);
    }
    fence_before();
    __syncthreads();
    if (warp == 0) {
        fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
    }
}

template <bool kF32, int B>
cudaError_t launch_wide(const QuantParams& p, cudaStream_t st) {
    auto kern = k_quantize_wide<kF32, B>;
    static TqLaunchCache cache;
    int sms = 0;
    cudaError_t e = tq_kernel_setup(kern, kWThreads, kWideSmem, cache, &sms, nullptr);
    if (e != cudaSuccess) return e;
    const int64_t tiles = (p.n_streams * p.nb + 3) / 4;
    const int64_t grid = std::min<int64_t>(tiles, sms);
    if (grid > 0) kern<<<(unsigned)grid, kWThreads, kWideSmem, st>>>(p);
    return cudaGetLastError();
}

}  // namespace

// keys with D = Mp = 256 and the prepared chunk images
cudaError_t tq_launch_quantize_wide(const QuantParams& p, cudaStream_t st) {
    const bool f32 = p.dtype == 0;
    switch (p.t.B) {
        case 1: return f32 ? launch_wide<true, 1>(p, st) : launch_wide<false, 1>(p, st);
        case 2: return f32 ? launch_wide<true, 2>(p, st) : launch_wide<false, 2>(p, st);
        case 3: return f32 ? launch_wide<true, 3>(p, st) : launch_wide<false, 3>(p, st);
    }
    return cudaErrorInvalidValue;
}
