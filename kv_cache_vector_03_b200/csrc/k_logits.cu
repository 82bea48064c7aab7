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
// two contractions of {0,1} bit planes against fixed vectors, run on the int8 tensor cores
// (mma.sync m16n8k32, u8 x s8 -> s32). A bit s of a packed byte is masked in place (one
// and per four coordinates, plus one shift per word for s < 4) and leaves the byte 0 or
// 2^(s mod 4 + 4); the query side is a fixed-point vector (|v| <= 4000, about 12 bits) whose
// entries carry the factor 2^(3 - s mod 4), so every product is 128 * bit * v. Each entry
// is split into two int8 columns (hi, lo) of the same MMA, so accumulation is exact.
//
// Kernel 1 (prologue, 8 query heads per CTA): q', q'' for every query head, fixed-point
// fragments in MMA order, per-head scales, exact logits of the tail.
// Kernel 2 (stream, persistent): each warp walks a list of (stream, block range) tasks and
// keeps a ring of 32-key blocks in shared memory filled by bulk copies (TMA engine,
// mbarrier completion), prefetching across task boundaries.
#include <algorithm>

#include "tq_device.cuh"

namespace {

constexpr int kPrologueThreads = 512;
constexpr int kStreamWarps = 8;
constexpr uint32_t kWaitLimit = 1u << 22;

__device__ __forceinline__ size_t qf_index(int64_t stream, int ntile, int ntiles, int nmg, int mg, int c,
                                           int lane, int h) {
    return ((((size_t)stream * ntiles + ntile) * nmg + mg) * 4 + c) * 64 + lane * 2 + h;
}

// Prologue. Grid (ceil(heads / HPC), 1 + ceil(n_tail / 16)), 512 threads; each CTA owns HPC
// (4, 8 or 16) consecutive query heads (rows s*g + h of q), chosen so that about one CTA per
// SM covers all heads: the kernel is latency-bound and every CTA pays one matrix load.
//   y = 0: 1. q' = Pi q and q'' = S q.
//             D = Mp = 128: both products from one A operand (the 16 query rows, fp16 hi/lo) on
//             mma.sync against the prepared swizzled images of 256 Pi and sigma_S S, which arrive
//             by two bulk copies; for a Sylvester-ordered Hadamard Pi, q' is a fast Walsh-Hadamard
//             transform in registers instead. Row maxima meet in shared memory by atomics.
//             Wider codecs: one [HPC x d] x [d x (D + Mp)] FFMA product against (Pi^T | S^T),
//             whose rows arrive by bulk copies of 32 KB in two stages; thread (row slice, head
//             quad, column quad) keeps 4 heads x 8 columns; row slices add up in shared memory.
//          2. per-head max -> fixed-point steps dA (codes, all planes) and dS (signs).
//          3. one warp per (head, plane group), one fragment word pair per lane: it rounds its
//             four coordinates, packs their hi and lo bytes and stores them; warp sums give
//             the per-head constants.
//   y > 0: exact logits of 16 tail tokens for the CTA's heads, one warp per token.
constexpr int kTailTok = 16;   // tail tokens per tail CTA (one per warp)
// FFMA path (D + Mp > 256): matrix rows per bulk-copied chunk (16 rows of W fp32, at most
// 32 KB) and the two stages they cycle through
constexpr int kProRows = 16, kProStages = 2;

template <int NR, int HPC>   // NR: 256-column groups of (Pi^T | S^T); HPC: heads per CTA
__global__ void __launch_bounds__(kPrologueThreads) k_logits_prologue(LogitsParams p) {
    // the kernel that consumes the fragments may launch now; it waits for this grid's
    // completion before it reads them
    tq_pdl_launch_dependents();
    const TqDims& T = p.t;
    const int D = T.D, Mp = T.Mp, d = T.d, G = p.g, np = T.nplanes_mma, W = D + Mp;
    const int n_heads = (int)(p.n_seq * p.n_kv * G);
    const int h_base = blockIdx.x * HPC;
    const int H = min(HPC, n_heads - h_base);
    extern __shared__ __align__(16) float sm[];
    const int tid = threadIdx.x, wid = tid >> 5, lane = tid & 31;

    if (blockIdx.y > 0) {
        // exact logits of the full-precision tail, scale <q, k>: warp w takes token
        // 16 (y - 1) + w and the key rows of the CTA's streams
        float* qh = sm;   // [HPC][d]
        for (int e = tid; e < HPC * d; e += blockDim.x) {
            const int h = e / d, j = e - h * d;
            qh[e] = h < H ? tq_load_elem(p.q, p.q_dtype, (int64_t)(h_base + h) * d + j) : 0.f;
        }
        __syncthreads();
        const int tt = (blockIdx.y - 1) * kTailTok + wid;
        if (tt >= p.n_tail) return;
        const int64_t row = p.n_tok + p.n_tail;
        const int s0 = h_base / G, s1 = (h_base + H - 1) / G;
        for (int st = s0; st <= s1; ++st) {
            const uint16_t* kp = p.tail + ((size_t)st * p.n_tail + tt) * d;
            float kv[8];   // coordinates lane + 32 i of the key (d <= 256)
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int j = lane + 32 * i;
                kv[i] = j < d ? __uint_as_float((uint32_t)kp[j] << 16) : 0.f;
            }
            const int h0 = max(st * G - h_base, 0), h1 = min((st + 1) * G - h_base, H);
            for (int h = h0; h < h1; ++h) {
                float a = 0.f;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int j = lane + 32 * i;
                    if (j < d) a = fmaf(kv[i], qh[h * d + j], a);
                }
                a = tq_warp_sum(a);
                if (lane == 0) p.out[(int64_t)(h_base + h) * row + p.n_tok + tt] = p.scale * a;
            }
        }
        return;
    }

    // MMA path (D + Mp = 256): qo [16][256] (q' then q''), A hi/lo, the four B images.
    // FFMA path (wide codecs): qT [256][HPC] query transposed, then qo [HPC][W].
    float* qT = sm;
    float* qo = NR == 1 ? sm : qT + 256 * HPC;   // q' (0..D-1) then q'' (D..W-1)
    __shared__ uint32_t s_max[2][HPC];   // max |q'|, max |q''| per head (fp32 bits)
    __shared__ uint64_t s_bar[4];   // matrix chunk stages (two bulk copies each)
    const int nmg = T.nmg;
    if (tid == 0) {
        for (int k = 0; k < 4; ++k) tq_mbar_init(&s_bar[k], 2);
        tq_fence_mbar_init();
    }
    const int frag_words = p.ntiles * nmg * 256;

    // heads beyond g inside an n-tile keep zero fragments (only when g < 4)
    if (G < 4) {
        const int st0 = (h_base + G - 1) / G, st1 = (h_base + H) / G;
        uint4* fz = reinterpret_cast<uint4*>(p.qfrag + (size_t)st0 * frag_words);
        for (int e = tid; e < (st1 - st0) * frag_words / 4; e += blockDim.x) fz[e] = make_uint4(0, 0, 0, 0);
    }
    if (tid < 2 * HPC) s_max[tid / HPC][tid % HPC] = 0u;
    if constexpr (NR == 1) {
        // 1. q' = Pi q and q'' = S q on the fp16 tensor cores (mma.sync m16n8k16, operands split
        //    into fp16 hi + lo, three passes), both from the same A = the 16 query rows; warp w
        //    owns output columns 8w .. 8w + 7 of each product. B = the prepared images of 256 Pi
        //    and sigma_S S (128-byte swizzled, row = output coordinate), one bulk copy each.
        //    A Sylvester-ordered Hadamard Pi = H diag(s) / sqrt(d) skips its images: each warp
        //    applies it to its own head as a fast Walsh-Hadamard transform in registers.
        uint8_t* at = reinterpret_cast<uint8_t*>(sm + 16 * 256);   // A hi, A lo [16][256 B]
        uint8_t* bt = at + 2 * 16 * 256;                            // Pi hi, Pi lo, S hi, S lo
        __shared__ float s_qa[16];
        const uint32_t sat = tq_smem_addr(at), sbt = tq_smem_addr(bt);
        const uint32_t flags = __ldg(p.hdr);
        const bool wht = (flags & (TQ_PREP_PM1 | TQ_PREP_WHT)) == (TQ_PREP_PM1 | TQ_PREP_WHT);
        const float inv_ss = 1.f / __ldg(reinterpret_cast<const float*>(p.hdr) + 3);   // a power of two
        if (tid == 0) {
            if (wht) tq_mbar_arrive(&s_bar[0]);
            else tq_bulk_load(bt, p.pimg, 2 * (uint32_t)kTqImageBytes, &s_bar[0]);
            tq_bulk_load(bt + 2 * kTqImageBytes, p.pimg + 2 * kTqImageBytes, 2 * (uint32_t)kTqImageBytes,
                         &s_bar[0]);
        }
        // the query row of this warp's head: lane l holds coordinates 4l .. 4l + 3
        float xq[4];
        {
            const int h = wid;   // 16 warps, 16 rows
            const bool ok = h < H && (int64_t)(h_base + h) < p.n_heads_valid;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int j = 4 * lane + k;
                xq[k] = ok && j < d ? tq_load_elem(p.q, p.q_dtype, (int64_t)(h_base + h) * d + j) : 0.f;
            }
        }
        // A row: scaled by a power of two (max in [2^14, 2^15)) and split into binary16 hi + lo;
        // a_lo: some lo part is nonzero (a bf16 or fp16 query is exact in the hi part)
        bool a_lo = false;
        {
            float mx = fmaxf(fmaxf(fabsf(xq[0]), fabsf(xq[1])), fmaxf(fabsf(xq[2]), fabsf(xq[3])));
            mx = tq_warp_max(mx);
            int ex = 0;
            if (mx > 0.f && isfinite(mx)) ex = min(max(14 - (((__float_as_int(mx) >> 23) & 0xff) - 127), -126), 126);
            const float sc = __int_as_float((127 + ex) << 23);
            const __half2 h0 = __floats2half2_rn(xq[0] * sc, xq[1] * sc), h1 = __floats2half2_rn(xq[2] * sc, xq[3] * sc);
            const float2 f0 = __half22float2(h0), f1 = __half22float2(h1);
            const __half2 l0 = __floats2half2_rn(xq[0] * sc - f0.x, xq[1] * sc - f0.y);
            const __half2 l1 = __floats2half2_rn(xq[2] * sc - f1.x, xq[3] * sc - f1.y);
            const uint32_t off = tq_swz256(wid, lane >> 1) + (lane & 1) * 8;
            *reinterpret_cast<uint2*>(at + off) = make_uint2(*reinterpret_cast<const uint32_t*>(&h0),
                                                            *reinterpret_cast<const uint32_t*>(&h1));
            *reinterpret_cast<uint2*>(at + 4096 + off) = make_uint2(*reinterpret_cast<const uint32_t*>(&l0),
                                                                   *reinterpret_cast<const uint32_t*>(&l1));
            if (lane == 0) s_qa[wid] = 1.f / sc;
            a_lo = (*reinterpret_cast<const uint32_t*>(&l0) | *reinterpret_cast<const uint32_t*>(&l1)) & 0x7fff7fffu;
        }
        if (wht) {
            // q' = H (s * q) / sqrt(d), s_j = sign(Pi[0][j]) (row 0 of H is all ones), read from row
            // 0 of the Pi hi image. Butterflies of span 1 and 2 in registers, spans 4 .. d/2 between
            // lanes l and l ^ (span / 4); only spans below d run, so the zero coordinates from d on
            // never mix with the first d.
            const uint2 r0 = __ldg(reinterpret_cast<const uint2*>(p.pimg + tq_sw128_offset(0, 4 * lane)));
            const uint32_t sg[4] = {r0.x, r0.x >> 16, r0.y, r0.y >> 16};
            float v[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) v[k] = (sg[k] & 0x8000u) ? -xq[k] : xq[k];
            if (d > 1) {
                const float a0 = v[0], a2 = v[2];
                v[0] = a0 + v[1]; v[1] = a0 - v[1];
                v[2] = a2 + v[3]; v[3] = a2 - v[3];
            }
            if (d > 2) {
                const float a0 = v[0], a1 = v[1];
                v[0] = a0 + v[2]; v[2] = a0 - v[2];
                v[1] = a1 + v[3]; v[3] = a1 - v[3];
            }
#pragma unroll
            for (int sh = 0; sh < 5; ++sh) {
                if ((4 << sh) >= d) break;
                const bool hi = (lane >> sh) & 1;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float o = __shfl_xor_sync(0xffffffffu, v[k], 1 << sh);
                    v[k] = hi ? o - v[k] : v[k] + o;
                }
            }
            const float inv = fabsf(__ldg(p.piT));   // |Pi[0][0]| = 1/sqrt(d) as stored
            float mx = 0.f;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                v[k] *= inv;
                qo[wid * 256 + 4 * lane + k] = v[k];
                mx = fmaxf(mx, fabsf(v[k]));
            }
            mx = tq_warp_max(mx);
            if (lane == 0 && wid < HPC) s_max[0][wid] = __float_as_uint(mx);
        }
        a_lo = __syncthreads_or(a_lo);   // A rows, s_qa (and the barrier's initialisation, before anyone waits)
        const bool landed = __syncthreads_and(tq_mbar_wait(&s_bar[0], 0u, kWaitLimit));
        if (!landed) {
            // the images did not land in time: record it, give the copies a bounded time to
            // finish before the shared memory is released, and leave the fragments unwritten
            if (tid == 0) {
                tq_raise(p.status, TQ_FLAG_TIMEOUT);
                tq_mbar_wait(&s_bar[0], 0u, kWaitLimit);
            }
            return;
        }
        // 16-byte chunk c (0..15) of row r of a 128-byte swizzled image: K-block c / 8
        auto bsw = [](int r, int c) { return (uint32_t)((c >> 3) * 16384 + r * 128 + (((c & 7) ^ (r & 7)) << 4)); };
        if constexpr (HPC <= 8) {
            // up to 8 heads: the products transposed, one 16-output x 8-head tile per warp (warp
            // w: product w / 8, outputs 16 (w mod 8) ..), so no MMA rows are spent on absent
            // heads: A = the image rows (fp16 hi / lo), B = the query rows; hi.hi, lo.hi and,
            // when a query row has a nonzero lo part, hi.lo, in separate accumulators
            const int pw = wid >> 3, o0 = 16 * (wid & 7);
            const int mi = lane >> 3, r8 = lane & 7;
            const int a_row = o0 + (mi & 1) * 8 + r8, a_chk = mi >> 1;
            const int b_row = r8, b_chk = mi & 1;
            const int g = lane >> 2, t = lane & 3;
            const uint32_t img = sbt + (uint32_t)(2 * pw) * (uint32_t)kTqImageBytes;
            float acc[3][4];
#pragma unroll
            for (int x = 0; x < 3; ++x) acc[x][0] = acc[x][1] = acc[x][2] = acc[x][3] = 0.f;
            if (!(wht && pw == 0)) {
#pragma unroll
                for (int kc = 0; kc < 8; ++kc) {
                    uint32_t ih[4], il[4], qh[2], ql[2] = {0u, 0u};
                    const uint32_t ao = bsw(a_row, 2 * kc + a_chk);
                    tq_ldsm_x4(img + ao, ih[0], ih[1], ih[2], ih[3]);
                    tq_ldsm_x4(img + (uint32_t)kTqImageBytes + ao, il[0], il[1], il[2], il[3]);
                    tq_ldsm_x2(sat + tq_swz256(b_row, 2 * kc + b_chk), qh[0], qh[1]);
                    if (a_lo) tq_ldsm_x2(sat + 4096 + tq_swz256(b_row, 2 * kc + b_chk), ql[0], ql[1]);
                    tq_hmma(acc[0], ih[0], ih[1], ih[2], ih[3], qh[0], qh[1]);
                    tq_hmma(acc[1], il[0], il[1], il[2], il[3], qh[0], qh[1]);
                    if (a_lo) tq_hmma(acc[2], ih[0], ih[1], ih[2], ih[3], ql[0], ql[1]);
                }
                // accumulator r: output o0 + g (r < 2) or o0 + g + 8, head 2t + (r & 1)
                const float f0 = pw == 0 ? 1.f / 256.f : inv_ss;
                const float fe = s_qa[2 * t] * f0, fo = s_qa[2 * t + 1] * f0;
                float* qe = qo + (2 * t) * 256 + 128 * pw + o0 + g;
                const float v0 = ((acc[0][0] + acc[1][0]) + acc[2][0]) * fe;
                const float v1 = ((acc[0][1] + acc[1][1]) + acc[2][1]) * fo;
                const float v2 = ((acc[0][2] + acc[1][2]) + acc[2][2]) * fe;
                const float v3 = ((acc[0][3] + acc[1][3]) + acc[2][3]) * fo;
                qe[0] = v0;
                qe[256] = v1;
                qe[8] = v2;
                qe[256 + 8] = v3;
                // head maxima: the eight lanes of a head pair, then one shared atomic per head
                float me = fmaxf(fabsf(v0), fabsf(v2)), mo = fmaxf(fabsf(v1), fabsf(v3));
#pragma unroll
                for (int sft = 4; sft < 32; sft <<= 1) {
                    me = fmaxf(me, __shfl_xor_sync(0xffffffffu, me, sft));
                    mo = fmaxf(mo, __shfl_xor_sync(0xffffffffu, mo, sft));
                }
                if (g == 0) {
                    if (2 * t < HPC) atomicMax(&s_max[pw][2 * t], __float_as_uint(me));
                    if (2 * t + 1 < HPC) atomicMax(&s_max[pw][2 * t + 1], __float_as_uint(mo));
                }
            }
        } else {
        // one 16 x 8 output tile of each product per warp over K = 128: A hi/lo x B hi/lo
        // (hi.hi, hi.lo and, when some A lo part is nonzero, lo.hi, in separate accumulators)
        {
            const int mi = lane >> 3, r8 = lane & 7;
            const int a_row = (mi & 1) * 8 + r8, a_chk = mi >> 1;
            const int b_row = 8 * wid + r8, b_chk = mi & 1;
            const int g = lane >> 2, t = lane & 3;
            float ap[3][4], as[3][4];
#pragma unroll
            for (int x = 0; x < 3; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) ap[x][y] = as[x][y] = 0.f;
#pragma unroll
            for (int kc = 0; kc < 8; ++kc) {
                uint32_t ah[4], al[4] = {0u, 0u, 0u, 0u}, bh[2], bl[2];
                tq_ldsm_x4(sat + tq_swz256(a_row, 2 * kc + a_chk), ah[0], ah[1], ah[2], ah[3]);
                if (a_lo) tq_ldsm_x4(sat + 4096 + tq_swz256(a_row, 2 * kc + a_chk), al[0], al[1], al[2], al[3]);
                const uint32_t bo = bsw(b_row, 2 * kc + b_chk);
                if (!wht) {
                    tq_ldsm_x2(sbt + bo, bh[0], bh[1]);
                    tq_ldsm_x2(sbt + (uint32_t)kTqImageBytes + bo, bl[0], bl[1]);
                    tq_hmma(ap[0], ah[0], ah[1], ah[2], ah[3], bh[0], bh[1]);
                    tq_hmma(ap[1], ah[0], ah[1], ah[2], ah[3], bl[0], bl[1]);
                    if (a_lo) tq_hmma(ap[2], al[0], al[1], al[2], al[3], bh[0], bh[1]);
                }
                tq_ldsm_x2(sbt + 2 * (uint32_t)kTqImageBytes + bo, bh[0], bh[1]);
                tq_ldsm_x2(sbt + 3 * (uint32_t)kTqImageBytes + bo, bl[0], bl[1]);
                tq_hmma(as[0], ah[0], ah[1], ah[2], ah[3], bh[0], bh[1]);
                tq_hmma(as[1], ah[0], ah[1], ah[2], ah[3], bl[0], bl[1]);
                if (a_lo) tq_hmma(as[2], al[0], al[1], al[2], al[3], bh[0], bh[1]);
            }
            // accumulator r: row g (r < 2) or g + 8, column 8w + 2t + (r & 1)
            const float fa[2] = {s_qa[g] * (1.f / 256.f), s_qa[g + 8] * (1.f / 256.f)};
            const float fs[2] = {s_qa[g] * inv_ss, s_qa[g + 8] * inv_ss};
            float mp[2] = {0.f, 0.f}, ms[2] = {0.f, 0.f};
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int row = g + 8 * (r >> 1), col = 8 * wid + 2 * t + (r & 1);
                const float vs = ((as[0][r] + as[1][r]) + as[2][r]) * fs[r >> 1];
                qo[row * 256 + 128 + col] = vs;
                ms[r >> 1] = fmaxf(ms[r >> 1], fabsf(vs));
                if (!wht) {
                    const float vp = ((ap[0][r] + ap[1][r]) + ap[2][r]) * fa[r >> 1];
                    qo[row * 256 + col] = vp;
                    mp[r >> 1] = fmaxf(mp[r >> 1], fabsf(vp));
                }
            }
            // row maxima: the four lanes of a row group, then one shared atomic per row
#pragma unroll
            for (int o = 1; o < 4; o <<= 1)
#pragma unroll
                for (int x = 0; x < 2; ++x) {
                    mp[x] = fmaxf(mp[x], __shfl_xor_sync(0xffffffffu, mp[x], o));
                    ms[x] = fmaxf(ms[x], __shfl_xor_sync(0xffffffffu, ms[x], o));
                }
            if (t == 0) {
#pragma unroll
                for (int x = 0; x < 2; ++x) {
                    if (g + 8 * x >= HPC) continue;
                    if (!wht) atomicMax(&s_max[0][g + 8 * x], __float_as_uint(mp[x]));
                    atomicMax(&s_max[1][g + 8 * x], __float_as_uint(ms[x]));
                }
            }
        }
        }
        __syncthreads();   // qo, s_max
    } else {
    for (int e = tid; e < 256 * HPC; e += blockDim.x) {
        const int j = e / HPC, h = e % HPC;
        const bool ok = h < H && j < d && (int64_t)(h_base + h) < p.n_heads_valid;
        qT[e] = ok ? tq_load_elem(p.q, p.q_dtype, (int64_t)(h_base + h) * d + j) : 0.f;
    }
    for (int e = tid; e < HPC * W; e += blockDim.x) qo[e] = 0.f;
    __syncthreads();

    // 1. product. Thread -> ks (row slice ks of KS), hq (heads 4hq .. 4hq + 3), cq (columns
    //    4cq + 256r). A chunk holds [R][D] rows of Pi^T, then [R][Mp] rows of S^T.
    {
        constexpr int NHQ = HPC / 4, KS = kPrologueThreads / (64 * NHQ);
        const int R = kProRows, NST = kProStages, nchunk = (d + R - 1) / R;
        float* stg = qo + HPC * W;
        auto load_chunk = [&](int c) {   // one thread
            const int j0 = c * R, rows = min(R, d - j0);
            float* dst = stg + (size_t)(c % NST) * R * W;
            tq_bulk_load(dst, p.piT + (size_t)j0 * D, (uint32_t)(rows * D * 4), &s_bar[c % NST]);
            tq_bulk_load(dst + R * D, p.sT + (size_t)j0 * Mp, (uint32_t)(rows * Mp * 4), &s_bar[c % NST]);
        };
        if (tid == 0)
            for (int c = 0; c < min(nchunk, NST); ++c) load_chunk(c);
        const int cq = tid & 63, hq = (tid >> 6) % NHQ, ks = tid / (64 * NHQ);
        int off[NR], rstr[NR];
        bool bv[NR];
#pragma unroll
        for (int r = 0; r < NR; ++r) {
            const int col = 256 * r + 4 * cq;
            bv[r] = col < W;
            off[r] = col < D ? col : R * D + (col - D);
            rstr[r] = col < D ? D : Mp;
        }
        float acc[NR][4][4];
#pragma unroll
        for (int r = 0; r < NR; ++r)
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int y = 0; y < 4; ++y) acc[r][x][y] = 0.f;
        bool ok = true;
        int c = 0;
        for (; c < nchunk; ++c) {
            const int stg_i = c % NST;
            const uint32_t parity = (uint32_t)(c / NST) & 1u;
            ok = __syncthreads_and(ok && tq_mbar_wait(&s_bar[stg_i], parity, kWaitLimit));
            if (!ok) break;
            const int j0 = c * R, rows = min(R, d - j0), slice = (rows + KS - 1) / KS;
            const int jj0 = ks * slice, jj1 = min(rows, jj0 + slice);
            const float* st = stg + (size_t)stg_i * R * W;
#pragma unroll 4
            for (int jj = jj0; jj < jj1; ++jj) {
                const float4 a = *reinterpret_cast<const float4*>(qT + (j0 + jj) * HPC + 4 * hq);
                const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
                for (int r = 0; r < NR; ++r) {
                    if (NR > 1 && !bv[r]) continue;
                    const float4 b = *reinterpret_cast<const float4*>(st + off[r] + jj * rstr[r]);
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        acc[r][x][0] = fmaf(av[x], b.x, acc[r][x][0]);
                        acc[r][x][1] = fmaf(av[x], b.y, acc[r][x][1]);
                        acc[r][x][2] = fmaf(av[x], b.z, acc[r][x][2]);
                        acc[r][x][3] = fmaf(av[x], b.w, acc[r][x][3]);
                    }
                }
            }
            if (c + NST < nchunk) {
                __syncthreads();   // stage c % NST is consumed
                if (tid == 0) {
                    tq_fence_proxy_async();
                    load_chunk(c + NST);
                }
            }
        }
        if (!ok) {
            // a copy did not land in time: record it, give the copies in flight a bounded
            // time, and leave the fragments unwritten
            if (tid == 0) {
                tq_raise(p.status, TQ_FLAG_TIMEOUT);
                for (int k = c; k < min(c + NST, nchunk); ++k)
                    tq_mbar_wait(&s_bar[k % NST], (uint32_t)(k / NST) & 1u, kWaitLimit);
            }
            return;
        }
        // the row slices meet in qo
#pragma unroll
        for (int r = 0; r < NR; ++r)
            if (bv[r])
#pragma unroll
                for (int x = 0; x < 4; ++x)
#pragma unroll
                    for (int y = 0; y < 4; ++y) atomicAdd(qo + (4 * hq + x) * W + 256 * r + 4 * cq + y, acc[r][x][y]);
        __syncthreads();
    }
        // 2. per-head maxima (one head per warp)
        if (wid < H) {
            const int h = wid;
            float ma = 0.f, ms = 0.f;
            for (int i = lane; i < D; i += 32) ma = fmaxf(ma, fabsf(qo[h * W + i]));
            for (int k = lane; k < Mp; k += 32) ms = fmaxf(ms, fabsf(qo[h * W + D + k]));
            ma = tq_warp_max(ma);
            ms = tq_warp_max(ms);
            if (lane == 0) {
                s_max[0][h] = __float_as_uint(ma);
                s_max[1][h] = __float_as_uint(ms);
            }
        }
        __syncthreads();
    }
    // 2. fixed-point steps dA (code planes: max |q'| times the largest plane factor) and dS
    //    (signs), 3. fragment words and 4. per-head scales: kNW = 16 / HPC warps per head, warp
    //    sub of a head taking plane groups sub, sub + kNW, ... Lane -> chunk c, slot t, register
    //    hh of a plane group mg; byte bb of the word is coordinate 128 gr + 32 t + 2c + hh + 8 bb,
    //    in column 2 (head % 4) (hi) or 2 (head % 4) + 1 (lo) of n-tile head / 4.
    constexpr int kNW = kPrologueThreads / 32 / HPC;
    __shared__ int s_sum[2][HPC];
    if constexpr (kNW > 1) {
        if (tid < 2 * HPC) s_sum[tid / HPC][tid % HPC] = 0;
        __syncthreads();
    }
    const int h = wid / kNW, sub = wid % kNW;
    float dA = 1.f, dS = 1.f;
    int stream = 0, head = 0;
    if (h < H) {
        float amax = 0.f;
        for (int pl = 0; pl < np; ++pl) amax = fmaxf(amax, fabsf(2.f * p.cb.plane_coef[pl]));
        const float ma = __uint_as_float(s_max[0][h]) * amax, ms = __uint_as_float(s_max[1][h]);
        dA = ma > 0.f ? ma / (float)kTqQueryMax : 1.f;
        dS = ms > 0.f ? ms / (float)kTqQueryMax : 1.f;
        const float invA = 1.f / dA, invS = 1.f / dS;
        const int gh = h_base + h;
        stream = gh / G;
        head = gh - stream * G;
        const int GDv = NR == 1 ? 1 : T.GD;
        const int c = lane >> 3, t = (lane >> 1) & 3, hh = lane & 1;
        // bit s = 2c + hh of the key bytes meets this register: factor 2^(3 - s mod 4)
        const int f = 8 >> ((2 * c + hh) & 3);
        uint32_t* dst = p.qfrag + ((size_t)stream * p.ntiles + (head >> 2)) * nmg * 256 + c * 64 + 16 * (head & 3) +
                        2 * t + hh;
        int sumA = 0, sumS = 0;
#pragma unroll 2
        for (int mg = sub; mg < nmg; mg += kNW) {
            const bool is_code = mg < np * GDv;
            const int gr = is_code ? mg % GDv : mg - np * GDv;
            const float inv = is_code ? 2.f * p.cb.plane_coef[mg / GDv] * invA : invS;
            const float* src = qo + h * W + (is_code ? 0 : D) + 128 * gr + 32 * t + 2 * c + hh;
            uint32_t whi = 0, wlo = 0;
            int sum = 0;
#pragma unroll
            for (int bb = 0; bb < 4; ++bb) {
                const int v = __float2int_rn(src[8 * bb] * inv);
                sum += v;
                const int vf = v * f, hi = (vf + 128) >> 8, lo = vf - 256 * hi;
                whi |= (uint32_t)(hi & 0xff) << (8 * bb);
                wlo |= (uint32_t)(lo & 0xff) << (8 * bb);
            }
            if (is_code) sumA += sum;
            else sumS += sum;
            dst[mg * 256] = whi;
            dst[mg * 256 + 8] = wlo;   // lane + 4 (column lo) -> word + 8
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            sumA += __shfl_xor_sync(0xffffffffu, sumA, o);
            sumS += __shfl_xor_sync(0xffffffffu, sumS, o);
        }
        if constexpr (kNW > 1) {
            if (lane == 0) {
                atomicAdd(&s_sum[0][h], sumA);
                atomicAdd(&s_sum[1][h], sumS);
            }
        } else if (lane == 0) {
            s_sum[0][h] = sumA;
            s_sum[1][h] = sumS;
        }
    }
    if constexpr (kNW > 1) __syncthreads();   // every warp of a head has added its sums
    // scales, folding the 128 of the u8 bit bytes, the QJL factor kappa and the attention
    // scale: l = |x| (dA/128 accA - KA + gamma (kappa 2 dS/128 accS - kappa KS))
    if (h < H && sub == 0 && lane == 0) {
        const float sa = p.scale;
        reinterpret_cast<float4*>(p.qscale)[(size_t)stream * p.ntiles * 4 + head] =
            make_float4(sa * dA / 128.f, sa * 0.5f * dA * (float)s_sum[0][h], sa * p.kappa * 2.f * dS / 128.f,
                        sa * p.kappa * dS * (float)s_sum[1][h]);
    }
}

// Walks a warp's contiguous range of the flattened (stream, block) index: every warp gets
// the same number of blocks (+-1) and changes stream (reloading its query fragments) at most
// a few times; no divisions after the first.
struct FlatWalk {
    int64_t left;   // blocks still to visit
    int stream, blk;
    __device__ void init(const LogitsParams& p, int64_t b0, int64_t b1) {
        left = b1 - b0;
        stream = (int)(b0 / p.nb);
        blk = (int)(b0 - (int64_t)stream * p.nb);
    }
    __device__ bool valid() const { return left > 0; }
    __device__ void advance(const LogitsParams& p) {
        --left;
        if (++blk == (int)p.nb) {
            blk = 0;
            ++stream;
        }
    }
};

// NP = estimator code planes, GD/GM = 128-coordinate groups of code / sign planes,
// B = stored code planes, NT = n-tiles of 4 query heads, NS = ring stages per warp;
// QJL = false (the MSE-only estimator, kappa = 0) runs no sign-plane MMAs.
template <int B, int GD, int GM, int NT, int NS, bool QJL>
__global__ void __launch_bounds__(kStreamWarps * 32) k_logits_stream(LogitsParams p) {
    constexpr int NP = B == 3 ? 4 : B;
    constexpr int NPG = B * GD + GM;       // stored plane groups
    constexpr int NMG = NP * GD + GM;      // MMA plane groups of the fragments
    constexpr int NMG_RUN = QJL ? NMG : NP * GD;   // the groups this variant multiplies
    constexpr uint32_t BB = 512u * NPG + 128u;
    // exact int32 combination of the hi/lo columns while 128 * 8 kTqQueryMax * K < 2^31
    constexpr bool kIntComb = NP * GD <= 4 && GM <= 4;
    extern __shared__ __align__(128) uint8_t ring[];
    // one barrier per ring stage, plus one that nothing arrives at (the test stall)
    __shared__ uint64_t bars[kStreamWarps][NS + 1];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    uint8_t* my_ring = ring + (size_t)warp * NS * BB;
    if (lane == 0)
        for (int s = 0; s <= NS; ++s) tq_mbar_init(&bars[warp][s], 1);
    tq_fence_mbar_init();
    __syncwarp();

    const int64_t n_blocks = p.n_seq * p.n_kv * p.nb, n_warps = (int64_t)gridDim.x * kStreamWarps;
    const int64_t gw = (int64_t)blockIdx.x * kStreamWarps + warp;
    FlatWalk prod, cons;
    prod.init(p, gw * n_blocks / n_warps, (gw + 1) * n_blocks / n_warps);
    cons = prod;
    uint32_t issued = 0;   // copies issued so far (lane 0): copy k fills stage k % NS
    if (lane == 0) {
        for (int s = 0; s < NS && prod.valid(); ++s) {
            tq_bulk_load(my_ring + s * BB, p.packed + ((size_t)prod.stream * p.nb + prod.blk) * BB, BB, &bars[warp][s]);
            prod.advance(p);
            ++issued;
        }
    }

    // the copies above read only keys; the query fragments come from the prologue
    tq_pdl_wait();
    const int64_t row = p.n_tok + p.n_tail;
    uint32_t qf[NT][NMG_RUN][4][2];
    float4 sc[NT];
    float* orow[NT];
    bool hv[NT];
    int cur_stream = -1;
    uint32_t seq = 0;
    // test stall: a bounded wait on the barrier nothing arrives at runs out, exactly as a
    // copy that never lands would
    bool ok = p.test_stall == 0u || __all_sync(0xffffffffu, tq_mbar_wait(&bars[warp][NS], 0u, p.test_stall));
    while (ok && cons.valid()) {
        if (cons.stream != cur_stream) {
            cur_stream = cons.stream;
#pragma unroll
            for (int n = 0; n < NT; ++n) {
#pragma unroll
                for (int mg = 0; mg < NMG_RUN; ++mg)
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const uint2 v = *reinterpret_cast<const uint2*>(
                            p.qfrag + qf_index(cur_stream, n, NT, NMG, mg, c, lane, 0));
                        qf[n][mg][c][0] = v.x;
                        qf[n][mg][c][1] = v.y;
                    }
                sc[n] = reinterpret_cast<const float4*>(p.qscale)[(size_t)cur_stream * NT * 4 + n * 4 + t];
                hv[n] = n * 4 + t < p.g;
                orow[n] = p.out + ((int64_t)cur_stream * p.g + (hv[n] ? n * 4 + t : 0)) * row;
            }
        }
        const int stage = seq % NS;
        ok = __all_sync(0xffffffffu, tq_mbar_wait(&bars[warp][stage], (seq / NS) & 1u, kWaitLimit));
        if (!ok) break;
        const uint8_t* bp = my_ring + stage * BB;
        uint4 cur[NPG + 1];
#pragma unroll
        for (int pg = 0; pg < NPG; ++pg) cur[pg] = *reinterpret_cast<const uint4*>(bp + (pg * 32 + lane) * 16);
        cur[NPG] = *reinterpret_cast<const uint4*>(bp + NPG * 512 + g * 16);
        const bool full = (int64_t)(cons.blk + 1) * 32 <= p.n_tok;
        const int n_valid = full ? 32 : (int)(p.n_tok - (int64_t)cons.blk * 32);
        const int tok0 = cons.blk * 32 + g;

#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            // code planes accumulate in two chains (chunks c odd / even), the sign plane in one
            int accA[NT][4], accA2[NT][4], accS[NT][4];
            if constexpr (!QJL) {
#pragma unroll
                for (int n = 0; n < NT; ++n) accS[n][0] = accS[n][1] = accS[n][2] = accS[n][3] = 0;
            }
#pragma unroll
            for (int mg = 0; mg < NMG_RUN; ++mg) {
                uint32_t w0, w1;  // words of rows g (u = 2mt) and g + 8 (u = 2mt + 1)
                if (mg < NP * GD && mg / GD == 3) {  // b0 ^ b1 ^ b2
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
#pragma unroll
                    for (int n = 0; n < NT; ++n) {
                        const uint32_t b0 = qf[n][mg][c][0], b1 = qf[n][mg][c][1];
                        if (mg < NP * GD) {
                            int(&acc)[4] = (c & 1) ? accA[n] : accA2[n];
                            if (mg == 0 && c >= 2) tq_imma_u8_z(acc, a0, a1, a2, a3, b0, b1);   // first of its chain
                            else tq_imma_u8(acc, a0, a1, a2, a3, b0, b1);
                        } else {
                            if (mg == NP * GD && c == 3) tq_imma_u8_z(accS[n], a0, a1, a2, a3, b0, b1);
                            else tq_imma_u8(accS[n], a0, a1, a2, a3, b0, b1);
                        }
                    }
                });
            }
#pragma unroll
            for (int n = 0; n < NT; ++n)
#pragma unroll
                for (int r = 0; r < 4; ++r) accA[n][r] += accA2[n][r];
            // epilogue: thread (g, t) -> head t of each n-tile, rows g and g + 8
            const uint32_t* nrm = reinterpret_cast<const uint32_t*>(&cur[NPG]);
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int u = 2 * mt + r;
                const uint32_t nw = nrm[u];
                const float nh = tq_half_val(nw & 0xffffu), gh = tq_half_val(nw >> 16);
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    float va, vs;
                    if (kIntComb) {
                        va = (float)(256 * accA[n][2 * r] + accA[n][2 * r + 1]);
                        vs = (float)(256 * accS[n][2 * r] + accS[n][2 * r + 1]);
                    } else {
                        va = fmaf(256.f, (float)accA[n][2 * r], (float)accA[n][2 * r + 1]);
                        vs = fmaf(256.f, (float)accS[n][2 * r], (float)accS[n][2 * r + 1]);
                    }
                    const float est = fmaf(sc[n].x, va, -sc[n].y) + gh * fmaf(sc[n].z, vs, -sc[n].w);
                    if (hv[n] && (full || 8 * u + g < n_valid)) orow[n][tok0 + 8 * u] = nh * est;
                }
            }
        }
        // the stage's data are consumed (all reads above fed the MMAs): refill it
        __syncwarp();
        if (lane == 0 && prod.valid()) {
            tq_fence_proxy_async();
            tq_bulk_load(my_ring + stage * BB, p.packed + ((size_t)prod.stream * p.nb + prod.blk) * BB, BB,
                         &bars[warp][stage]);
            prod.advance(p);
            ++issued;
        }
        ++seq;
        cons.advance(p);
    }
    if (!ok) {
        // a wait ran out: record it, then give each copy still in flight (copies seq .. issued-1)
        // a bounded time to land before the CTA's shared memory is released
        if (lane == 0) {
            tq_raise(p.status, TQ_FLAG_TIMEOUT);
            for (uint32_t k = seq; k < issued; ++k) tq_mbar_wait(&bars[warp][k % NS], (k / NS) & 1u, kWaitLimit);
        }
        __syncwarp();
    }
}

template <int B, int GD, int GM, int NT, bool QJL>
cudaError_t launch_stream(const LogitsParams& p0, cudaStream_t st) {
    constexpr int NS = 4;
    constexpr int NPG = B * GD + GM;
    constexpr size_t BB = 512u * NPG + 128u;
    const size_t smem = (size_t)kStreamWarps * NS * BB;
    auto kern = k_logits_stream<B, GD, GM, NT, NS, QJL>;
    static TqLaunchCache cache;
    int sms = 0, per_sm = 0;
    cudaError_t e = tq_kernel_setup(kern, kStreamWarps * 32, smem, cache, &sms, &per_sm);
    if (e != cudaSuccess) return e;
    // persistent: as many CTAs as fit, each warp a contiguous equal share of the blocks
    const LogitsParams& p = p0;
    const int64_t n_blocks = p.n_seq * p.n_kv * p.nb;
    const int64_t grid = std::min<int64_t>((n_blocks + kStreamWarps - 1) / kStreamWarps, (int64_t)per_sm * sms);
    if (grid == 0) return cudaSuccess;
    return tq_launch_pdl(kern, dim3((unsigned)grid), dim3(kStreamWarps * 32), smem, st, p);
}

template <int B, int GD, int GM>
cudaError_t launch_nt(const LogitsParams& p, cudaStream_t st) {
    // the MSE-only estimator (kappa = 0) multiplies no sign planes
    if (p.kappa == 0.f)
        return p.ntiles == 1 ? launch_stream<B, GD, GM, 1, false>(p, st) : launch_stream<B, GD, GM, 2, false>(p, st);
    return p.ntiles == 1 ? launch_stream<B, GD, GM, 1, true>(p, st) : launch_stream<B, GD, GM, 2, true>(p, st);
}

}  // namespace

// heads per prologue CTA: about one CTA per SM
static int prologue_hpc(int64_t n_heads) {
    const int64_t sms = tq_device_sms();
    return n_heads <= sms * 4 ? 4 : n_heads <= sms * 8 ? 8 : 16;
}

// MMA path (D + Mp = 256): qo [16][256] fp32 + A hi/lo [16][256 B] + the four 32 KB B images
constexpr size_t kPrologueSmemMma = (size_t)16 * 256 * 4 + 2 * 16 * 256 + 4 * 128 * 256;

size_t tq_logits_prologue_smem(const TqDims& t, int hpc) {
    const int W = t.D + t.Mp;
    if (W <= 256) return kPrologueSmemMma;
    return ((size_t)256 * hpc + (size_t)hpc * W + (size_t)kProStages * kProRows * W) * 4;
}

// largest prologue shared memory over the supported codecs and head counts
constexpr size_t kPrologueSmemWide = ((size_t)256 * 16 + (size_t)16 * 512 + (size_t)2 * 16 * 512) * 4;
constexpr size_t kPrologueMaxSmem = kPrologueSmemWide > kPrologueSmemMma ? kPrologueSmemWide : kPrologueSmemMma;

template <int NR, int HPC>
cudaError_t launch_prologue(const LogitsParams& p, int64_t n_heads, cudaStream_t st) {
    const size_t smem = tq_logits_prologue_smem(p.t, HPC);
    auto kern = k_logits_prologue<NR, HPC>;
    static TqLaunchCache cache;
    cudaError_t e = tq_kernel_setup(kern, kPrologueThreads, kPrologueMaxSmem, cache, nullptr, nullptr);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)((n_heads + HPC - 1) / HPC), 1u + (unsigned)((p.n_tail + kTailTok - 1) / kTailTok));
    kern<<<grid, kPrologueThreads, smem, st>>>(p);
    return cudaGetLastError();
}

cudaError_t tq_launch_logits_prologue(const LogitsParams& p, cudaStream_t st) {
    const int64_t n_heads = p.n_seq * p.n_kv * p.g;
    const bool wide = p.t.D + p.t.Mp > 256;
    if (!wide && (p.pimg == nullptr || p.hdr == nullptr)) return cudaErrorInvalidValue;   // 256-wide: images needed
    switch (prologue_hpc(n_heads)) {
        case 4: return wide ? launch_prologue<2, 4>(p, n_heads, st) : launch_prologue<1, 4>(p, n_heads, st);
        case 8: return wide ? launch_prologue<2, 8>(p, n_heads, st) : launch_prologue<1, 8>(p, n_heads, st);
        default: return wide ? launch_prologue<2, 16>(p, n_heads, st) : launch_prologue<1, 16>(p, n_heads, st);
    }
}

cudaError_t tq_launch_logits(const LogitsParams& p, cudaStream_t st) {
    cudaError_t e = tq_launch_logits_prologue(p, st);
    if (e != cudaSuccess) return e;
    if (p.nb == 0) return cudaSuccess;
    const int B = p.t.B, GD = p.t.GD, GM = p.t.GM;
#define TQ_LOGITS_CASE(b, gd, gm) \
    if (B == b && GD == gd && GM == gm) return launch_nt<b, gd, gm>(p, st);
    TQ_LOGITS_CASE(1, 1, 1) TQ_LOGITS_CASE(2, 1, 1) TQ_LOGITS_CASE(3, 1, 1)
    TQ_LOGITS_CASE(1, 2, 2) TQ_LOGITS_CASE(2, 2, 2) TQ_LOGITS_CASE(3, 2, 2)
    TQ_LOGITS_CASE(1, 1, 2) TQ_LOGITS_CASE(2, 1, 2) TQ_LOGITS_CASE(3, 1, 2)
    TQ_LOGITS_CASE(1, 2, 1) TQ_LOGITS_CASE(2, 2, 1) TQ_LOGITS_CASE(3, 2, 1)
#undef TQ_LOGITS_CASE
    return cudaErrorInvalidValue;
}
