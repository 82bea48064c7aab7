// tq_quantize for d <= 128 on the fifth-generation tensor cores (tcgen05.mma with TMEM
// accumulators): rotate, nearest Lloyd-Max centroid, residual, QJL sign sketch, pack
// (blog.hotdry.top "TurboQuant vector-search compression", sections "Random rotation and
// scalar quantization" and "QJL residual correction"; a2a-mcp.org "What is TurboQuant",
// stage 1).
//
// One persistent CTA of 16 warps per SM walks tiles of 128 vectors (4 blocks of 32).
//   A. Each warp loads 8 rows (the next tile's rows are fetched into registers while the
//      current tile is in the tensor cores), forms |x| by a transposed warp reduction, scales
//      each row by a power of two and writes it as fp16 hi (and lo for fp32 input) into the
//      A operand, laid out in shared memory in the canonical K-major 128-byte-swizzled form.
//   B. One thread issues Y = X (256 Pi)^T as 128 x 128 x 16 MMAs over the split operands
//      (X_hi Pi_hi + X_hi Pi_lo [+ X_lo Pi_hi]); fp32 accumulation in TMEM columns 0..127.
//   C. Thread (warp, lane) owns TMEM lane 32 (warp % 4) + lane = one vector and a quarter of
//      its columns (32 coordinates = one word of each plane): y, idx = #{k : y > t_k},
//      r = y - c[idx], gamma^2, code-plane words; the residual goes back into the A operand
//      as fp16 hi and lo (scaled by 2^12).
//   D. Z = R (256 M)^T with M = S Pi^T (three split passes) into TMEM columns 128..255; the
//      sign bits are z >= 0. Planes, norms and gamma are stored in the key block format.
// Values (qjl = 0) stop after C: the codes go through shared memory into the value block's
// two-token fields.
#include "tq_device.cuh"

namespace {

constexpr int kThreads = 512;
constexpr uint32_t kMat = 32768;             // one 128 x 128 fp16 operand
constexpr uint32_t kWaitLimit = 1u << 22;
constexpr uint32_t kTmemCols = 256;

// Byte offset of 16-byte chunk kc (8 fp16 of columns 8kc..8kc+7) of row r in a 128 x 128
// fp16 operand: two K-blocks of 64 columns, each [128 rows][128 B] in atoms of 8 rows
// (1024 B), the chunk index XOR (row mod 8) (128-byte swizzle). Operands start 1024-aligned.
__device__ __forceinline__ uint32_t sw128(int r, int kc) {
    return (uint32_t)((kc >> 3) * 16384 + (r >> 3) * 1024 + (r & 7) * 128 + (((kc & 7) ^ (r & 7)) << 4));
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor, kind::f16: fp16 A and B, fp32 D, both K-major, M = 128, N = 128.
constexpr uint32_t kIdesc = (1u << 4) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t ad, uint64_t bd, uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %3, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %4, p;\n}\n" ::"r"(tmem_d),
        "l"(ad), "l"(bd), "r"(accumulate), "r"(kIdesc));
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     tq_smem_addr(bar))
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 16 consecutive fp32 columns of this thread's TMEM lane
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// hi / lo fp16 pairs of four values (packed conversions: one instruction per pair)
__device__ __forceinline__ uint32_t h2bits(__half2 h) { return *reinterpret_cast<const uint32_t*>(&h); }
__device__ __forceinline__ void split4(const float (&a)[4], uint2& h, uint2& l) {
    const __half2 h0 = __floats2half2_rn(a[0], a[1]), h1 = __floats2half2_rn(a[2], a[3]);
    const float2 f0 = __half22float2(h0), f1 = __half22float2(h1);
    h = make_uint2(h2bits(h0), h2bits(h1));
    l = make_uint2(h2bits(__floats2half2_rn(a[0] - f0.x, a[1] - f0.y)), h2bits(__floats2half2_rn(a[2] - f1.x, a[3] - f1.y)));
}
// hi only (values exactly representable, e.g. scaled bf16)
__device__ __forceinline__ uint2 half4(const float (&a)[4]) {
    return make_uint2(h2bits(__floats2half2_rn(a[0], a[1])), h2bits(__floats2half2_rn(a[2], a[3])));
}

constexpr int kRowsPerWarp = 8;   // 16 warps x 8 rows = one 128-vector tile

template <bool kF32>
struct RowRegs;
template <>
struct RowRegs<false> { uint2 v[kRowsPerWarp]; };   // 4 bf16 per lane and row
template <>
struct RowRegs<true> { float4 v[kRowsPerWarp]; };   // 4 fp32 per lane and row

// bits e < n of a 32-bit word, n clamped to [0, 32]
__device__ __forceinline__ uint32_t low_bits(int n) { return n >= 32 ? ~0u : n <= 0 ? 0u : (1u << n) - 1u; }

template <bool kF32, int B, bool QJL>
__global__ void __launch_bounds__(kThreads, 1) k_quantize_tc(QuantParams p) {
    constexpr int L = 1 << B;
    extern __shared__ uint8_t qraw[];
    __shared__ float s_inv[128], s_norm[128], s_sc[128], s_g2[4][128], s_cent[16];
    __shared__ int s_bad[128], s_valid[128];
    __shared__ uint64_t s_bar;
    __shared__ uint32_t s_tmem;

    const TqDims& T = p.t;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int d = T.d;
    const int64_t total_blocks = p.n_streams * p.nb;
    const int64_t n_tiles = (total_blocks + 3) / 4;

    // operand area, 1024-byte aligned: Pi_hi Pi_lo [M_hi M_lo] X_hi X_lo [codes]
    const uint32_t raw = tq_smem_addr(qraw);
    const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
    uint8_t* sm = qraw + pad;
    const uint32_t sb = raw + pad;
    constexpr uint32_t oXH = QJL ? 4 * kMat : 2 * kMat, oXL = oXH + kMat, oCS = oXL + kMat;

    {   // resident B operands: rows = output coordinate (N), columns = K
        constexpr int nmat = QJL ? 4 : 2;
        for (int e = tid; e < nmat * 128 * 16; e += kThreads) {
            const int m = e >> 11, row = (e >> 4) & 127, ch = e & 15;
            const uint16_t* src = m == 0 ? p.pih : m == 1 ? p.pil : m == 2 ? p.mh : p.ml;
            const uint4 v = *reinterpret_cast<const uint4*>(src + row * 128 + ch * 8);
            *reinterpret_cast<uint4*>(sm + m * kMat + sw128(row, ch)) = v;
        }
    }
    if (tid < L) s_cent[tid] = p.cb.cent[tid];
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tq_smem_addr(&s_tmem)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (tid == 0) {
        tq_mbar_init(&s_bar, 1);
        tq_fence_mbar_init();
    }
    tq_fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    uint32_t n_commit = 0;
    // coordinates >= d read y = 0 (zero rows of Pi): their residual -c[idx(0)] is taken
    // back out of gamma^2 below
    float c0 = 0.f;
    {
        int i0 = 0;
#pragma unroll
        for (int k = 0; k < L - 1; ++k) i0 += 0.f > p.cb.bounds[k];
        c0 = s_cent[i0];
    }

    // rows 8 warp .. 8 warp + 7 of a tile lie in one block
    auto load_rows = [&](int64_t tile, RowRegs<kF32>& rg) {
        const int64_t gb = tile * 4 + (warp >> 2);
        const int64_t s = gb / p.nb, tok0 = (gb % p.nb) * 32 + kRowsPerWarp * (warp & 3);
        const bool blk = gb < total_blocks;
        const int64_t base0 = s * p.x_stride + tok0 * d + 4 * lane;
#pragma unroll
        for (int rr = 0; rr < kRowsPerWarp; ++rr) {
            const bool in = blk && tok0 + rr < p.n_tok && 4 * lane < d;
            const int64_t base = base0 + (int64_t)rr * d;
            if constexpr (kF32) {
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (in) {
                    const float* xp = static_cast<const float*>(p.x) + base;
                    if (p.vec_ok) v = __ldg(reinterpret_cast<const float4*>(xp));
                    else v = make_float4(xp[0], xp[1], xp[2], xp[3]);
                }
                rg.v[rr] = v;
            } else {
                uint2 v = make_uint2(0u, 0u);
                if (in) {
                    const uint16_t* xp = static_cast<const uint16_t*>(p.x) + base;
                    if (p.vec_ok) v = __ldg(reinterpret_cast<const uint2*>(xp));
                    else v = make_uint2((uint32_t)xp[0] | ((uint32_t)xp[1] << 16), (uint32_t)xp[2] | ((uint32_t)xp[3] << 16));
                }
                rg.v[rr] = v;
            }
        }
    };
    // one thread waits for the MMAs; the others wait at the barrier
    auto mma_done = [&]() -> bool {
        bool w = true;
        if (tid == 0) w = tq_mbar_wait(&s_bar, n_commit & 1u, kWaitLimit);
        ++n_commit;
        return __syncthreads_and(w) != 0;
    };

    RowRegs<kF32> rg;
    if ((int64_t)blockIdx.x < n_tiles) load_rows(blockIdx.x, rg);
    bool ok = true;
    for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
        // ---- A. rows -> norms (transposed warp reduction), power-of-two scale, fp16 A operand
        {
            float x[kRowsPerWarp][4], v[kRowsPerWarp];
#pragma unroll
            for (int rr = 0; rr < kRowsPerWarp; ++rr) {
                if constexpr (kF32) {
                    x[rr][0] = rg.v[rr].x; x[rr][1] = rg.v[rr].y; x[rr][2] = rg.v[rr].z; x[rr][3] = rg.v[rr].w;
                } else {
                    x[rr][0] = __uint_as_float(rg.v[rr].x << 16); x[rr][1] = __uint_as_float(rg.v[rr].x & 0xffff0000u);
                    x[rr][2] = __uint_as_float(rg.v[rr].y << 16); x[rr][3] = __uint_as_float(rg.v[rr].y & 0xffff0000u);
                }
                v[rr] = fmaf(x[rr][0], x[rr][0], fmaf(x[rr][1], x[rr][1], fmaf(x[rr][2], x[rr][2], x[rr][3] * x[rr][3])));
            }
            // after the xor-16, -8, -4 exchanges lane l holds row (l >> 2) & 7 summed over 8 lanes
            float a4[4], a2[2], a1;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const bool hi = lane & 16;
                a4[k] = (hi ? v[k + 4] : v[k]) + __shfl_xor_sync(0xffffffffu, hi ? v[k] : v[k + 4], 16);
            }
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const bool hi = lane & 8;
                a2[k] = (hi ? a4[k + 2] : a4[k]) + __shfl_xor_sync(0xffffffffu, hi ? a4[k] : a4[k + 2], 8);
            }
            {
                const bool hi = lane & 4;
                a1 = (hi ? a2[1] : a2[0]) + __shfl_xor_sync(0xffffffffu, hi ? a2[0] : a2[1], 4);
            }
            a1 += __shfl_xor_sync(0xffffffffu, a1, 2);
            a1 += __shfl_xor_sync(0xffffffffu, a1, 1);
            const int64_t gb = tile * 4 + (warp >> 2);
            const int64_t tok0 = (gb % p.nb) * 32 + kRowsPerWarp * (warp & 3);
            if ((lane & 3) == 0) {
                const int rr = (lane >> 2) & 7, row = kRowsPerWarp * warp + rr;
                const bool valid = gb < total_blocks && tok0 + rr < p.n_tok;
                const float n = sqrtf(a1);
                // 2^ex with |x| 2^ex in [2^14, 2^15): every element then fits binary16
                int ex = 0;
                if (n > 0.f && isfinite(n)) ex = min(max(14 - (((__float_as_int(n) >> 23) & 0xff) - 127), -126), 126);
                const float sc2 = __int_as_float((127 + ex) << 23);
                s_sc[row] = sc2;
                s_norm[row] = valid ? n : 0.f;
                s_inv[row] = n > 0.f ? 1.f / (n * 256.f * sc2) : 0.f;
                s_bad[row] = valid && !isfinite(n);
                s_valid[row] = valid;
            }
            __syncwarp();
#pragma unroll
            for (int rr = 0; rr < kRowsPerWarp; ++rr) {
                const int row = kRowsPerWarp * warp + rr;
                const float sc2 = s_sc[row];
                float a[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) a[k] = x[rr][k] * sc2;
                const uint32_t off = sw128(row, lane >> 1) + (lane & 1) * 8;
                if constexpr (kF32) {
                    uint2 h, l;
                    split4(a, h, l);
                    *reinterpret_cast<uint2*>(sm + oXH + off) = h;
                    *reinterpret_cast<uint2*>(sm + oXL + off) = l;
                } else {
                    // a scaled bf16 value is exact in binary16 (8 significant bits)
                    *reinterpret_cast<uint2*>(sm + oXH + off) = half4(a);
                }
            }
        }
        // the next tile's rows stream in while this one is in the tensor cores
        if (tile + gridDim.x < n_tiles) load_rows(tile + gridDim.x, rg);

        // ---- B. Y = X Pi^T (scaled), TMEM columns 0..127
        tq_fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            constexpr int np = kF32 ? 3 : 2;
#pragma unroll
            for (int ps = 0; ps < np; ++ps) {
                const uint32_t oa = ps == 2 ? oXL : oXH, ob = ps == 1 ? kMat : 0u;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t ko = (uint32_t)(k >> 2) * 16384u + (uint32_t)(k & 3) * 32u;
                    umma_f16(tmem, umma_desc(sb + oa + ko), umma_desc(sb + ob + ko), (ps | k) != 0);
                }
            }
            umma_commit(&s_bar);
        }
        ok = mma_done();
        if (!ok) break;
        tc_fence_after();

        // ---- C. codes, residual, gamma; thread -> vector row r, columns 32 qc .. 32 qc + 31
        const int r = 32 * (warp & 3) + lane, qc = warp >> 2;
        const uint32_t tl = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
        const float inv = s_inv[r];
        const bool rvalid = s_valid[r] != 0;
        const int64_t gb = tile * 4 + (r >> 5);
        const int vb = r & 31, u = vb >> 3, gq = vb & 7;
        uint8_t* blk = p.packed + (size_t)gb * T.block_bytes;
        uint32_t cw[B];
#pragma unroll
        for (int pl = 0; pl < B; ++pl) cw[pl] = 0u;
        float g2 = 0.f;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            float y[16];
            tmem_ld16(tl + 32 * qc + 16 * q, y);
            float rv[16];
            uint32_t cb4[4] = {0u, 0u, 0u, 0u};
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const float yy = y[e] * inv;
                int c = 0;
#pragma unroll
                for (int k = 0; k < L - 1; ++k) c += yy > p.cb.bounds[k];
                const float rr = yy - s_cent[c];
                g2 = fmaf(rr, rr, g2);
                if (QJL) {
                    rv[e] = rr * 4096.f;
#pragma unroll
                    for (int pl = 0; pl < B; ++pl) cw[pl] |= (uint32_t)((c >> pl) & 1) << (16 * q + e);
                } else {
                    cb4[e >> 2] |= (uint32_t)c << (8 * (e & 3));
                }
            }
            if (QJL) {
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    uint2 h0, l0, h1, l1;
                    const float a0[4] = {rv[8 * hh], rv[8 * hh + 1], rv[8 * hh + 2], rv[8 * hh + 3]};
                    const float a1[4] = {rv[8 * hh + 4], rv[8 * hh + 5], rv[8 * hh + 6], rv[8 * hh + 7]};
                    split4(a0, h0, l0);
                    split4(a1, h1, l1);
                    const uint32_t off = sw128(r, 4 * qc + 2 * q + hh);
                    *reinterpret_cast<uint4*>(sm + oXH + off) = make_uint4(h0.x, h0.y, h1.x, h1.y);
                    *reinterpret_cast<uint4*>(sm + oXL + off) = make_uint4(l0.x, l0.y, l1.x, l1.y);
                }
            } else {
                *reinterpret_cast<uint4*>(sm + oCS + r * 128 + 32 * qc + 16 * q) = make_uint4(cb4[0], cb4[1], cb4[2], cb4[3]);
            }
        }
        // coordinates >= d: codes 0, residual out of gamma^2
        const int nfake = min(32, max(0, 32 * qc + 32 - d));
        s_g2[qc][r] = g2 - (float)nfake * c0 * c0;
        if (QJL && gb < total_blocks) {
            const uint32_t keep = rvalid ? low_bits(d - 32 * qc) : 0u;
#pragma unroll
            for (int pl = 0; pl < B; ++pl)
                reinterpret_cast<uint32_t*>(blk)[(pl * 32 + 4 * gq + qc) * 4 + u] = cw[pl] & keep;
        }

        if constexpr (QJL) {
            // ---- D. Z = R M^T (scaled), TMEM columns 128..255; signs, norms
            tq_fence_proxy_async();
            tc_fence_before();
            __syncthreads();
            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int ps = 0; ps < 3; ++ps) {
                    const uint32_t oa = ps == 2 ? oXL : oXH, ob = ps == 1 ? 3 * kMat : 2 * kMat;
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint32_t ko = (uint32_t)(k >> 2) * 16384u + (uint32_t)(k & 3) * 32u;
                        umma_f16(tmem + 128, umma_desc(sb + oa + ko), umma_desc(sb + ob + ko), (ps | k) != 0);
                    }
                }
                umma_commit(&s_bar);
            }
            ok = mma_done();
            if (!ok) break;
            tc_fence_after();
            uint32_t sw = 0u;
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                float z[16];
                tmem_ld16(tl + 128 + 32 * qc + 16 * q, z);
#pragma unroll
                for (int e = 0; e < 16; ++e) sw |= (uint32_t)(z[e] >= 0.f) << (16 * q + e);
            }
            if (gb < total_blocks) {
                reinterpret_cast<uint32_t*>(blk)[(B * 32 + 4 * gq + qc) * 4 + u] =
                    rvalid ? sw & low_bits(T.m - 32 * qc) : 0u;
                if (qc == 0) {
                    const uint32_t nh = rvalid ? tq_half_bits(s_norm[r]) : 0u;
                    const float gam = sqrtf(fmaxf(s_g2[0][r] + s_g2[1][r] + s_g2[2][r] + s_g2[3][r], 0.f));
                    const uint32_t gh = rvalid ? tq_half_bits(gam) : 0u;
                    if (rvalid && (s_bad[r] || (nh & 0x7fffu) >= 0x7c00u)) tq_raise(p.status, TQ_FLAG_RANGE);
                    reinterpret_cast<uint32_t*>(blk + T.sec_a)[gq * 4 + u] = nh | (gh << 16);
                }
            }
        } else {
            // value layout: norms, then each lane string of the tile's blocks from the codes
            __syncthreads();
            if (tid < 128) {
                const int row = tid;
                const int64_t gbr = tile * 4 + (row >> 5);
                if (gbr < total_blocks) {
                    const uint32_t nh = s_valid[row] ? tq_half_bits(s_norm[row]) : 0u;
                    if (s_valid[row] && (s_bad[row] || (nh & 0x7fffu) >= 0x7c00u)) tq_raise(p.status, TQ_FLAG_RANGE);
                    reinterpret_cast<uint16_t*>(p.packed + (size_t)gbr * T.block_bytes + T.sec_a)[row & 31] = (uint16_t)nh;
                }
            }
            const uint8_t* CS = sm + oCS;
            constexpr int fb = 2 * B, words = 128 * B / 32;
            for (int e = tid; e < 4 * 32 * words; e += kThreads) {
                const int bl = e / (32 * words), rem = e % (32 * words);
                const int64_t gbw = tile * 4 + bl;
                if (gbw >= total_blocks) continue;
                const int ln = rem % 32, wd = rem / 32;
                const int gq2 = ln >> 2, tq = ln & 3;
                uint32_t val = 0;
                const int f0 = (32 * wd) / fb, f1 = (32 * wd + 31) / fb;
                for (int f = f0; f <= f1; ++f) {
                    const int a = f >> 2, pp = f & 3;
                    const int i = 8 * a + gq2;
                    const int tau = 16 * (pp >> 1) + 8 * (pp & 1) + 2 * tq;
                    const uint8_t* crow = CS + (bl * 32) * 128;
                    uint32_t F = 0;
                    if (i < d && s_valid[bl * 32 + tau]) F |= (uint32_t)crow[tau * 128 + i];
                    if (i < d && s_valid[bl * 32 + tau + 1]) F |= (uint32_t)crow[(tau + 1) * 128 + i] << B;
                    const int pos = f * fb - 32 * wd;
                    val |= pos >= 0 ? (F << pos) : (F >> (-pos));
                }
                reinterpret_cast<uint32_t*>(p.packed + (size_t)gbw * T.block_bytes)[((wd >> 2) * 32 + ln) * 4 + (wd & 3)] = val;
            }
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }
    if (!ok) {
        // an MMA did not complete in time: record it and give it a bounded time to finish
        if (tid == 0) {
            tq_raise(p.status, TQ_FLAG_TIMEOUT);
            tq_mbar_wait(&s_bar, (n_commit - 1) & 1u, kWaitLimit);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
    }
}

// ---------------------------------------------------------------------------------------
// Keys from bf16 rows with the tensor cores overlapped: the residual has its own operand (no
// aliasing with the input tile), so Z of tile t runs while the warps stage tile t + 1, and
// Y of tile t + 1 runs while they finish the signs of tile t. Shared memory holds
// Pi_hi Pi_lo M_hi M_lo X R_hi R_lo (224 KB) plus per-row data; gamma^2 partials wait in
// TMEM columns 256..259. Each tile: 16 + 24 MMAs of 128 x 128 x 16.
__device__ __forceinline__ void tmem_st1(uint32_t taddr, float v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(__float_as_uint(v)) : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_ld4(uint32_t taddr, float (&v)[4]) {
    uint32_t r[4];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(r[i]);
}

constexpr uint32_t kPipeSmall = 512 + 1024 + 64 + 32 + 32 + 16 + 16;   // per-row data, barriers, TMEM base
constexpr size_t kPipeSmem = (size_t)7 * kMat + kPipeSmall + 1024;     // + alignment pad

template <int B>
__global__ void __launch_bounds__(kThreads, 1) k_quantize_tc_pipe(QuantParams p) {
    constexpr int L = 1 << B;
    extern __shared__ uint8_t qraw[];
    const TqDims& T = p.t;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int d = T.d;
    const int64_t total_blocks = p.n_streams * p.nb;
    const int64_t n_tiles = (total_blocks + 3) / 4;

    const uint32_t raw = tq_smem_addr(qraw);
    const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
    uint8_t* sm = qraw + pad;
    const uint32_t sb = raw + pad;
    constexpr uint32_t oX = 4 * kMat, oRH = 5 * kMat, oRL = 6 * kMat, oSmall = 7 * kMat;
    float* s_inv = reinterpret_cast<float*>(sm + oSmall);             // [128] (epilogue 1 of the current tile)
    float* s_norm = s_inv + 128;                                     // [2][128] (tile parity)
    float* s_cent = s_norm + 256;                                    // [16]
    uint8_t* s_valid = reinterpret_cast<uint8_t*>(s_cent + 16);      // [2][16] row bit masks
    uint8_t* s_bad = s_valid + 32;                                   // [2][16]
    uint64_t* bars = reinterpret_cast<uint64_t*>(s_bad + 32);        // Y, Z
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + 2);

    {
        for (int e = tid; e < 4 * 128 * 16; e += kThreads) {
            const int m = e >> 11, row = (e >> 4) & 127, ch = e & 15;
            const uint16_t* src = m == 0 ? p.pih : m == 1 ? p.pil : m == 2 ? p.mh : p.ml;
            const uint4 v = *reinterpret_cast<const uint4*>(src + row * 128 + ch * 8);
            *reinterpret_cast<uint4*>(sm + m * kMat + sw128(row, ch)) = v;
        }
    }
    if (tid < L) s_cent[tid] = p.cb.cent[tid];
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tq_smem_addr(s_tmem)),
                     "r"(512));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (tid == 0) {
        tq_mbar_init(&bars[0], 1);
        tq_mbar_init(&bars[1], 1);
        tq_fence_mbar_init();
    }
    tq_fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    uint32_t n_y = 0, n_z = 0;
    float c0 = 0.f;
    {
        int i0 = 0;
#pragma unroll
        for (int k = 0; k < L - 1; ++k) i0 += 0.f > p.cb.bounds[k];
        c0 = s_cent[i0];
    }

    RowRegs<false> rg;
    auto load_rows = [&](int64_t tile) {
        const int64_t gb = tile * 4 + (warp >> 2);
        const int64_t s = gb / p.nb, tok0 = (gb % p.nb) * 32 + kRowsPerWarp * (warp & 3);
        const bool blk = gb < total_blocks;
        const int64_t base0 = s * p.x_stride + tok0 * d + 4 * lane;
#pragma unroll
        for (int rr = 0; rr < kRowsPerWarp; ++rr) {
            const bool in = blk && tok0 + rr < p.n_tok && 4 * lane < d;
            const uint16_t* xp = static_cast<const uint16_t*>(p.x) + base0 + (int64_t)rr * d;
            uint2 v = make_uint2(0u, 0u);
            if (in) {
                if (p.vec_ok) v = __ldg(reinterpret_cast<const uint2*>(xp));
                else v = make_uint2((uint32_t)xp[0] | ((uint32_t)xp[1] << 16), (uint32_t)xp[2] | ((uint32_t)xp[3] << 16));
            }
            rg.v[rr] = v;
        }
    };
    // A: rows in registers -> norms, scale, binary16 X operand, per-row data of parity slot
    auto phase_a = [&](int64_t tile, int slot) {
        float x[kRowsPerWarp][4], v[kRowsPerWarp];
#pragma unroll
        for (int rr = 0; rr < kRowsPerWarp; ++rr) {
            x[rr][0] = __uint_as_float(rg.v[rr].x << 16); x[rr][1] = __uint_as_float(rg.v[rr].x & 0xffff0000u);
            x[rr][2] = __uint_as_float(rg.v[rr].y << 16); x[rr][3] = __uint_as_float(rg.v[rr].y & 0xffff0000u);
            v[rr] = fmaf(x[rr][0], x[rr][0], fmaf(x[rr][1], x[rr][1], fmaf(x[rr][2], x[rr][2], x[rr][3] * x[rr][3])));
        }
        float a4[4], a2[2], a1;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const bool hi = lane & 16;
            a4[k] = (hi ? v[k + 4] : v[k]) + __shfl_xor_sync(0xffffffffu, hi ? v[k] : v[k + 4], 16);
        }
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const bool hi = lane & 8;
            a2[k] = (hi ? a4[k + 2] : a4[k]) + __shfl_xor_sync(0xffffffffu, hi ? a4[k] : a4[k + 2], 8);
        }
        {
            const bool hi = lane & 4;
            a1 = (hi ? a2[1] : a2[0]) + __shfl_xor_sync(0xffffffffu, hi ? a2[0] : a2[1], 4);
        }
        a1 += __shfl_xor_sync(0xffffffffu, a1, 2);
        a1 += __shfl_xor_sync(0xffffffffu, a1, 1);
        // lane 4 rr holds row rr of this warp
        const int64_t gb = tile * 4 + (warp >> 2);
        const int64_t tok0 = (gb % p.nb) * 32 + kRowsPerWarp * (warp & 3);
        const int rr_me = (lane >> 2) & 7, row_me = kRowsPerWarp * warp + rr_me;
        const bool valid = gb < total_blocks && tok0 + rr_me < p.n_tok;
        const float n = sqrtf(a1);
        int ex = 0;
        if (n > 0.f && isfinite(n)) ex = min(max(14 - (((__float_as_int(n) >> 23) & 0xff) - 127), -126), 126);
        const float sc2 = __int_as_float((127 + ex) << 23);
        const uint32_t vb = __ballot_sync(0xffffffffu, valid), bb = __ballot_sync(0xffffffffu, valid && !isfinite(n));
        if ((lane & 3) == 0) {
            s_norm[slot * 128 + row_me] = valid ? n : 0.f;
            s_inv[row_me] = n > 0.f ? 1.f / (n * 256.f * sc2) : 0.f;
        }
        if (lane == 0) {
            uint32_t mv = 0, mb = 0;
#pragma unroll
            for (int rr = 0; rr < 8; ++rr) {
                mv |= ((vb >> (4 * rr)) & 1u) << rr;
                mb |= ((bb >> (4 * rr)) & 1u) << rr;
            }
            s_valid[slot * 16 + warp] = (uint8_t)mv;
            s_bad[slot * 16 + warp] = (uint8_t)mb;
        }
#pragma unroll
        for (int rr = 0; rr < kRowsPerWarp; ++rr) {
            const float s2 = __shfl_sync(0xffffffffu, sc2, 4 * rr);
            const float a[4] = {x[rr][0] * s2, x[rr][1] * s2, x[rr][2] * s2, x[rr][3] * s2};
            // a scaled bf16 value is exact in binary16
            *reinterpret_cast<uint2*>(sm + oX + sw128(kRowsPerWarp * warp + rr, lane >> 1) + (lane & 1) * 8) = half4(a);
        }
    };
    auto issue_y = [&]() {
        tq_fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ps = 0; ps < 2; ++ps)
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t ko = (uint32_t)(k >> 2) * 16384u + (uint32_t)(k & 3) * 32u;
                    umma_f16(tmem, umma_desc(sb + oX + ko), umma_desc(sb + ps * kMat + ko), (ps | k) != 0);
                }
            umma_commit(&bars[0]);
        }
        ++n_y;
    };
    auto issue_z = [&]() {
        tq_fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ps = 0; ps < 3; ++ps) {
                const uint32_t oa = ps == 2 ? oRL : oRH, ob = ps == 1 ? 3 * kMat : 2 * kMat;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const uint32_t ko = (uint32_t)(k >> 2) * 16384u + (uint32_t)(k & 3) * 32u;
                    umma_f16(tmem + 128, umma_desc(sb + oa + ko), umma_desc(sb + ob + ko), (ps | k) != 0);
                }
            }
            umma_commit(&bars[1]);
        }
        ++n_z;
    };
    auto wait_bar = [&](int b, uint32_t count) -> bool {
        bool w = true;
        if (tid == 0) w = tq_mbar_wait(&bars[b], (count - 1) & 1u, kWaitLimit);
        const bool all = __syncthreads_and(w) != 0;
        tc_fence_after();
        return all;
    };

    const int r = 32 * (warp & 3) + lane, qc = warp >> 2;
    const uint32_t tl = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
    const int vb = r & 31, u = vb >> 3, gq = vb & 7;
    // The codebook is symmetric (t_{L/2-1} = 0, c_{L/2+k} = -c_{L/2-1-k}): idx follows from
    // the sign of y and level = #{positive boundaries below |y|}: idx = L/2 + level for y > 0,
    // L/2 - 1 - level otherwise. Everything in this epilogue is scaled by 2^12 (the residual's
    // binary16 scale). A |y| exactly on a boundary of the negative side takes the upper index
    // (inside the parity band; the oracle takes the lower one).
    constexpr int H = L / 2;
    float mth[H > 1 ? H - 1 : 1], cmag[H];
#pragma unroll
    for (int k = 0; k < H - 1; ++k) mth[k] = 4096.f * p.cb.bounds[H + k];
#pragma unroll
    for (int k = 0; k < H; ++k) cmag[k] = 4096.f * p.cb.cent[H + k];
    const float c0s = 4096.f * c0;
    bool ok = true;
    int slot = 0;
    if ((int64_t)blockIdx.x < n_tiles) {
        load_rows(blockIdx.x);
        phase_a(blockIdx.x, 0);
        if ((int64_t)blockIdx.x + gridDim.x < n_tiles) load_rows((int64_t)blockIdx.x + gridDim.x);
        issue_y();
    }
    for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
        ok = wait_bar(0, n_y);
        if (!ok) break;
        // ---- C. codes, residual, gamma^2 of tile (Y in TMEM columns 0..127)
        const float inv = 4096.f * s_inv[r];
        const bool rvalid = (s_valid[slot * 16 + (r >> 3)] >> (r & 7)) & 1u;
        const int64_t gb = tile * 4 + (r >> 5);
        uint8_t* blk = p.packed + (size_t)gb * T.block_bytes;
        uint32_t cw[B];
#pragma unroll
        for (int pl = 0; pl < B; ++pl) cw[pl] = 0u;
        float g2 = 0.f;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            float y[16];
            tmem_ld16(tl + 32 * qc + 16 * q, y);
            float rv[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const float yy = y[e] * inv;
                const float ay = fabsf(yy);
                const bool pos = yy > 0.f;
                // level bits and magnitude of the centroid
                bool pk[H > 1 ? H - 1 : 1];
#pragma unroll
                for (int k = 0; k < H - 1; ++k) pk[k] = ay > mth[k];
                float cm = cmag[0];
#pragma unroll
                for (int k = 0; k < H - 1; ++k) cm = pk[k] ? cmag[k + 1] : cm;
                const float rr = yy - (pos ? cm : -cm);
                g2 = fmaf(rr, rr, g2);
                rv[e] = rr;
                const int bit = 16 * q + e;
                cw[B - 1] |= (uint32_t)pos << bit;
                if constexpr (B == 2) {
                    cw[0] |= (uint32_t)(pos == pk[0]) << bit;
                } else if constexpr (B == 3) {
                    // low bits = level (y > 0) or 3 - level; level = pk0 + pk1 + pk2
                    const bool l1 = pk[1], l0 = pk[0] ^ pk[1] ^ pk[2];
                    cw[1] |= (uint32_t)(l1 == pos) << bit;
                    cw[0] |= (uint32_t)(l0 == pos) << bit;
                }
            }
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                uint2 h0, l0, h1, l1;
                const float a0[4] = {rv[8 * hh], rv[8 * hh + 1], rv[8 * hh + 2], rv[8 * hh + 3]};
                const float a1[4] = {rv[8 * hh + 4], rv[8 * hh + 5], rv[8 * hh + 6], rv[8 * hh + 7]};
                split4(a0, h0, l0);
                split4(a1, h1, l1);
                const uint32_t off = sw128(r, 4 * qc + 2 * q + hh);
                *reinterpret_cast<uint4*>(sm + oRH + off) = make_uint4(h0.x, h0.y, h1.x, h1.y);
                *reinterpret_cast<uint4*>(sm + oRL + off) = make_uint4(l0.x, l0.y, l1.x, l1.y);
            }
        }
        const int nfake = min(32, max(0, 32 * qc + 32 - d));
        tmem_st1(tl + 256 + qc, g2 - (float)nfake * c0s * c0s);
        if (gb < total_blocks) {
            const uint32_t keep = rvalid ? low_bits(d - 32 * qc) : 0u;
#pragma unroll
            for (int pl = 0; pl < B; ++pl)
                reinterpret_cast<uint32_t*>(blk)[(pl * 32 + 4 * gq + qc) * 4 + u] = cw[pl] & keep;
        }
        // ---- D. Z of this tile runs while the next tile is staged and its Y issued
        issue_z();
        const int64_t next = tile + gridDim.x;
        if (next < n_tiles) {
            phase_a(next, slot ^ 1);
            if (next + gridDim.x < n_tiles) load_rows(next + gridDim.x);
            issue_y();
        }
        ok = wait_bar(1, n_z);
        if (!ok) break;
        uint32_t sw = 0u;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            float z[16];
            tmem_ld16(tl + 128 + 32 * qc + 16 * q, z);
#pragma unroll
            for (int e = 0; e < 16; ++e) sw |= (uint32_t)(z[e] >= 0.f) << (16 * q + e);
        }
        if (gb < total_blocks) {
            reinterpret_cast<uint32_t*>(blk)[(B * 32 + 4 * gq + qc) * 4 + u] = rvalid ? sw & low_bits(T.m - 32 * qc) : 0u;
            if (qc == 0) {
                float g4[4];
                tmem_ld4(tl + 256, g4);
                const uint32_t nh = rvalid ? tq_half_bits(s_norm[slot * 128 + r]) : 0u;
                const uint32_t gh =
                    rvalid ? tq_half_bits(sqrtf(fmaxf(g4[0] + g4[1] + g4[2] + g4[3], 0.f)) * (1.f / 4096.f)) : 0u;
                const bool bad = (s_bad[slot * 16 + (r >> 3)] >> (r & 7)) & 1u;
                if (rvalid && (bad || (nh & 0x7fffu) >= 0x7c00u)) tq_raise(p.status, TQ_FLAG_RANGE);
                reinterpret_cast<uint32_t*>(blk + T.sec_a)[gq * 4 + u] = nh | (gh << 16);
            }
        } else if (qc == 0) {
            float g4[4];
            tmem_ld4(tl + 256, g4);   // keep the warp's collective TMEM loads uniform
            (void)g4;
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        slot ^= 1;
    }
    if (!ok) {
        if (tid == 0) {
            tq_raise(p.status, TQ_FLAG_TIMEOUT);
            if (n_y) tq_mbar_wait(&bars[0], (n_y - 1) & 1u, kWaitLimit);
            if (n_z) tq_mbar_wait(&bars[1], (n_z - 1) & 1u, kWaitLimit);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
    }
}

template <int B>
cudaError_t launch_tc_pipe(const QuantParams& p, cudaStream_t st) {
    auto kern = k_quantize_tc_pipe<B>;
    static TqLaunchCache cache;
    int sms = 0;
    cudaError_t e = tq_kernel_setup(kern, kThreads, kPipeSmem, cache, &sms, nullptr);
    if (e != cudaSuccess) return e;
    const int64_t tiles = (p.n_streams * p.nb + 3) / 4;
    const int64_t grid = std::min<int64_t>(tiles, sms);
    if (grid > 0) kern<<<(unsigned)grid, kThreads, kPipeSmem, st>>>(p);
    return cudaGetLastError();
}

template <bool kF32, int B, bool QJL>
cudaError_t launch_tc(const QuantParams& p, cudaStream_t st) {
    const size_t smem = (size_t)(QJL ? 6 : 5) * kMat + 1024;
    auto kern = k_quantize_tc<kF32, B, QJL>;
    static TqLaunchCache cache;
    int sms = 0;
    cudaError_t e = tq_kernel_setup(kern, kThreads, smem, cache, &sms, nullptr);
    if (e != cudaSuccess) return e;
    const int64_t tiles = (p.n_streams * p.nb + 3) / 4;
    const int64_t grid = std::min<int64_t>(tiles, sms);
    if (grid > 0) kern<<<(unsigned)grid, kThreads, smem, st>>>(p);
    return cudaGetLastError();
}

template <bool kF32, bool QJL>
cudaError_t launch_b(const QuantParams& p, cudaStream_t st) {
    switch (p.t.B) {
        case 1: return launch_tc<kF32, 1, QJL>(p, st);
        case 2: return launch_tc<kF32, 2, QJL>(p, st);
        case 3: return launch_tc<kF32, 3, QJL>(p, st);
        case 4: if constexpr (!QJL) return launch_tc<kF32, 4, QJL>(p, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

// d <= 128 with m <= 128 (or no sketch)
cudaError_t tq_launch_quantize_tc(const QuantParams& p, cudaStream_t st) {
    const bool f32 = p.dtype == 0;
    if (tq_quantize_ws_eligible(p)) return tq_launch_quantize_ws(p, st);
    if (p.t.qjl && !f32) {
        switch (p.t.B) {
            case 1: return launch_tc_pipe<1>(p, st);
            case 2: return launch_tc_pipe<2>(p, st);
            case 3: return launch_tc_pipe<3>(p, st);
        }
        return cudaErrorInvalidValue;
    }
    if (p.t.qjl) return f32 ? launch_b<true, true>(p, st) : launch_b<false, true>(p, st);
    return f32 ? launch_b<true, false>(p, st) : launch_b<false, false>(p, st);
}
