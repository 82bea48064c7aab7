// Device-side helpers and kernel parameter blocks of libtq (sm_100a).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "tq_internal.h"

#include <atomic>
#include <mutex>

#define TQ_DEVICE __device__ __forceinline__

// Per-device launch facts of one kernel, established on its first launch on a device: the
// dynamic shared-memory opt-in (cudaFuncSetAttribute), the SM count and the CTAs that fit
// on one SM. Later launches read them without any CUDA API call.
struct TqLaunchCache {
    static constexpr int kDevices = 64;
    int sms[kDevices];
    int per_sm[kDevices];
    std::atomic<bool> done[kDevices];
    std::mutex mu;
};

template <typename Kernel>
inline cudaError_t tq_kernel_setup(Kernel kern, int threads, size_t max_smem, TqLaunchCache& c, int* sms,
                                   int* per_sm) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= TqLaunchCache::kDevices) return cudaErrorInvalidDevice;
    if (!c.done[dev].load(std::memory_order_acquire)) {
        std::lock_guard<std::mutex> guard(c.mu);
        if (!c.done[dev].load(std::memory_order_relaxed)) {
            if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)max_smem)) !=
                cudaSuccess)
                return e;
            int n = 0, occ = 0;
            if ((e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
            if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, threads, max_smem)) != cudaSuccess)
                return e;
            c.sms[dev] = n;
            c.per_sm[dev] = occ > 0 ? occ : 1;
            c.done[dev].store(true, std::memory_order_release);
        }
    }
    if (sms) *sms = c.sms[dev];
    if (per_sm) *per_sm = c.per_sm[dev];
    return cudaSuccess;
}

// SM count of the current device (cached per device). Split counts, and so workspace sizes,
// follow it; with no usable device (a size query on a machine without a GPU) the B200's 148
// is assumed.
inline int tq_device_sms() {
    constexpr int kDevices = 64;
    static std::atomic<int> cache[kDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kDevices) {
        cudaGetLastError();
        return 148;
    }
    int n = cache[dev].load(std::memory_order_relaxed);
    if (n > 0) return n;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        return 148;
    }
    cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

TQ_DEVICE uint32_t tq_half_bits(float v) { return (uint32_t)__half_as_ushort(__float2half_rn(v)); }
TQ_DEVICE float tq_half_val(uint32_t bits) { return __half2float(__ushort_as_half((unsigned short)bits)); }

TQ_DEVICE float tq_load_elem(const void* p, int dtype, int64_t i) {
    if (dtype == 1) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
    return reinterpret_cast<const float*>(p)[i];
}

TQ_DEVICE void tq_raise(uint32_t* status, uint32_t flag) {
    if (status) atomicOr(status, flag);
}

// Programmatic dependent launch: a kernel launched with programmatic stream serialization may
// start once every CTA of the kernel before it has called launch_dependents (or exited); its
// wait returns when that kernel has completed and its writes are visible. Without the launch
// attribute both are no-ops.
TQ_DEVICE void tq_pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
TQ_DEVICE void tq_pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Launches kern<<<grid, block, smem, st>>>(args...) as a programmatic dependent of the
// previous kernel on st.
template <typename... KArgs, typename... Args>
inline cudaError_t tq_launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                 Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

// 2^x by the hardware approximation (ex2.approx.ftz: relative error about 2^-22)
TQ_DEVICE float tq_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// warp-wide reductions
TQ_DEVICE float tq_warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
TQ_DEVICE double tq_warp_sum_d(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
TQ_DEVICE float tq_warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// int8 tensor-core MMA, 16x8x32, s32 accumulate (legacy warp-level path): A u8, B s8
// Bit planes to u8 MMA operands. Bit s of every byte of a packed word is one coordinate.
// Masking it in place leaves the byte 0 or 2^s; bits 4..7 are masked in the word itself and
// bits 0..3 in the word shifted left by 4, where they sit at 4..7. The weight 2^(s mod 4 + 4)
// this leaves on the A byte is compensated on the query side, whose fixed-point values carry
// the factor 2^(3 - s mod 4) (at most 8 x kTqQueryMax, inside the int16 hi/lo range), so
// every product is 128 * bit * query value. For the words w0 (row g) and w1 (row g + 8) of
// one k-chunk this yields, for c = 3 .. 0, a0, a1 <- bit 2c and a2, a3 <- bit 2c + 1, the A
// fragment of chunk c; f(c, a0, a1, a2, a3) consumes it. One shift and one mask per register
// pair of the old shift-then-mask form is saved.
constexpr int kTqQueryMax = 4000;   // |query fixed-point value| before the 2^(3 - s mod 4) factor

template <typename F>
TQ_DEVICE void tq_expand_planes(uint32_t w0, uint32_t w1, F&& f) {
    const uint32_t u0 = w0 << 4, u1 = w1 << 4;
    f(3, w0 & 0x40404040u, w1 & 0x40404040u, w0 & 0x80808080u, w1 & 0x80808080u);
    f(2, w0 & 0x10101010u, w1 & 0x10101010u, w0 & 0x20202020u, w1 & 0x20202020u);
    f(1, u0 & 0x40404040u, u1 & 0x40404040u, u0 & 0x80808080u, u1 & 0x80808080u);
    f(0, u0 & 0x10101010u, u1 & 0x10101010u, u0 & 0x20202020u, u1 & 0x20202020u);
}

TQ_DEVICE void tq_imma_u8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                          uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// the same MMA with a zero accumulator input (starts a chain without initialising registers)
TQ_DEVICE void tq_imma_u8_z(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                            uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};\n"
        : "=r"(c[0]), "=r"(c[1]), "=r"(c[2]), "=r"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "r"(0));
}

// ldmatrix: four / two 8x8 b16 matrices from shared memory (row addresses from lanes 0-31 / 0-15)
TQ_DEVICE void tq_ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
TQ_DEVICE void tq_ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];\n" : "=r"(r0), "=r"(r1) : "r"(addr));
}
// byte offset of 16-byte chunk `chunk` of row `row` in rows of 256 bytes, XOR-swizzled by
// row mod 8 so that ldmatrix reads of 8 rows hit distinct banks
TQ_DEVICE uint32_t tq_swz256(int row, int chunk) { return (uint32_t)(row * 256 + ((chunk ^ (row & 7)) << 4)); }

// ---------------------------------------------------------------------- mbarrier + bulk copy
// One-dimensional bulk copies global -> shared through the TMA engine, completion tracked
// by a shared-memory mbarrier (transaction bytes). Waits are bounded: a wait that does not
// complete within `limit` polls returns false and the caller records TQ_FLAG_TIMEOUT.
TQ_DEVICE uint32_t tq_smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

TQ_DEVICE void tq_mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(tq_smem_addr(bar)), "r"(count));
}
TQ_DEVICE void tq_fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory"); }
TQ_DEVICE void tq_fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory"); }

TQ_DEVICE void tq_mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(tq_smem_addr(bar)) : "memory");
}

TQ_DEVICE void tq_bulk_load(void* dst_smem, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(tq_smem_addr(bar)), "r"(bytes)
                 : "memory");
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
            tq_smem_addr(dst_smem)),
        "l"(src), "r"(bytes), "r"(tq_smem_addr(bar))
        : "memory");
}

TQ_DEVICE bool tq_mbar_wait(uint64_t* bar, uint32_t phase, uint32_t limit) {
    const uint32_t a = tq_smem_addr(bar);
    for (uint32_t it = 0; it < limit; ++it) {
        uint32_t done;
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
            : "=r"(done)
            : "r"(a), "r"(phase)
            : "memory");
        if (done) return true;
    }
    return false;
}

// int8 tensor-core MMA, 16x8x32, s32 accumulate (legacy warp-level path)
TQ_DEVICE void tq_imma(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                       uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// fp16 tensor-core MMA, 16x8x16, fp32 accumulate
TQ_DEVICE void tq_hmma(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                       uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 16-byte streaming load of data read once (does not allocate in L1)
// 4-byte asynchronous copy global -> shared (zero-filled when src_bytes = 0, which reads
// nothing), grouped per thread by commit / wait_group.
TQ_DEVICE void tq_cp_async4(void* dst_smem, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(tq_smem_addr(dst_smem)), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}
TQ_DEVICE void tq_cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
TQ_DEVICE void tq_cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

TQ_DEVICE uint4 tq_ldg_stream(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// ---------------------------------------------------------------------- kernel params
struct PrepParams {
    const float* pi;
    const float* s;
    float* piT;
    float* sT;
    float* mT;
    uint16_t *pih, *pil, *mh, *ml;
    uint8_t* img;          // operand images of the warp-specialized quantize, or null
    uint8_t* wimg;         // chunked operand images of the 256-wide quantize, or null
    uint32_t* hdr;         // prep header (flags)
    int d, m, D, Mp, qjl;
};

// Byte offset of element (row r, column c) in a 128 x 128 16-bit tensor-core operand laid
// out as two K-blocks of 64 columns, [128 rows][128 B] each, in 8-row atoms of 1024 B with
// the 16-byte chunk index XOR (row mod 8) (the canonical K-major 128-byte swizzle).
TQ_DEVICE uint32_t tq_sw128_offset(int r, int c) {
    const int kc = c >> 3;
    return (uint32_t)((kc >> 3) * 16384 + (r >> 3) * 1024 + (r & 7) * 128 + (((kc & 7) ^ (r & 7)) << 4) + (c & 7) * 2);
}

struct QuantParams {
    const void* x;
    int dtype;
    int64_t n_streams, n_tok, x_stride, nb;  // nb = blocks per stream
    uint8_t* packed;
    const float* piT;
    const float* mT;
    const uint16_t *pih, *pil, *mh, *ml;
    const uint8_t* img;    // operand images of the warp-specialized kernel, or null
    const uint8_t* wimg;   // chunked operand images of the 256-wide kernel, or null
    const uint32_t* hdr;   // prep header (flags)
    uint32_t* status;
    int vec_ok;            // rows can be read 4 elements at a time (alignment of x, stride, d)
    TqDims t;
    TqCodebookConsts cb;
};

struct LogitsParams {
    const uint8_t* packed;
    const void* q;
    int q_dtype;
    const uint16_t* tail;  // bf16 bits
    float* out;
    const float* piT;
    const float* sT;
    const uint8_t* pimg;   // prologue images (256 Pi hi, lo, sigma_S S hi, lo), D = Mp = 128 only
    const uint32_t* hdr;   // prep header (rotation flags, sigma_S), with pimg
    uint32_t* qfrag;       // [stream][ntile][nmg][4][32][2]
    float* qscale;         // [stream][ntile*4][4]: dA/128, KA, 2dS/128, KS
    uint32_t* status;
    int64_t n_seq, n_tok, nb;
    int n_kv, g, ntiles, n_tail;
    float scale, kappa;
    int64_t n_heads_valid;                   // query rows that exist (later heads read as zero)
    uint32_t test_stall;                     // 0, or the poll limit of a wait that is made to run out
    TqDims t;
    TqCodebookConsts cb;
};

struct PvParams {
    const uint8_t* packed;
    const float* P;
    float* out;
    const float* piT;      // prepared Pi^T, fp32 [D][D] (row j = column j of Pi), 256-byte aligned
    uint32_t* status;
    float* part;           // [stream*g heads][nsplit][D]
    float* part_ml;        // [stream*g heads][nsplit][2]: max, sum
    int64_t n_streams, n_tok, nb;
    int g, nsplit, blocks_per_split;
    TqDims t;
    TqCodebookConsts cb;
};

struct TopkParams {
    const uint8_t* packed;      // one stream of n_db key records
    const float* q;             // fp32 [n_q][d] queries
    const float* piT;           // prepared PiT [D][D] and ST [D][Mp] (fp32)
    const float* sT;
    uint16_t* qimg;             // [n_qt * 128][kq] fp16 query operand rows (scaled by sigma)
    float* qinv;                // [n_qt * 128] 1 / sigma
    float* part_score;          // [n_q][nsplit][k]
    int* part_idx;              // [n_q][nsplit][k]
    int64_t* out_idx;
    float* out_score;
    uint32_t* status;
    int64_t n_db, nb, n_q, n_tiles;   // n_tiles: key tiles of 128
    int k, nsplit, tiles_per_split, n_qt;
    int kb_mse, kb_sign, kq;    // K-blocks of 64 of the two parts (kb_sign = 0: MSE-only), kq = 64 (kb_mse + kb_sign)
    int d, m;
    float kappa;                // sqrt(pi/2)/m, or 0 (MSE-only)
    TqDims t;
    TqCodebookConsts cb;
};

struct AttnParams {
    const uint8_t* packed_k;      // key blocks (qjl = 1), d <= 128, m <= 128
    const uint8_t* packed_v;      // value blocks (qjl = 0), same d
    const uint32_t* qfrag;        // query fragments of the key codec (logits prologue)
    const float* qscale;          // per-head constants (attention scale folded in)
    float* tail_logit;            // [stream * g + head][n_tail] exact tail logits (prologue, or the q8 split)
    const uint16_t* tail_v;       // bf16 [stream][n_tail][d] full-precision recent values
    const float* piT_v;           // prepared Pi^T of the value codec, fp32 [D][D]
    float* out;                   // fp32 [stream * g + head][d]
    float* part;                  // [stream * g + head][nsplit][D] rotated-domain partial sums
    float* part_ml;               // [stream * g + head][nsplit][2]: max, sum of weights
    uint32_t* status;
    int64_t n_streams, n_tok, nb;
    int g, nsplit, blocks_per_split, n_tail;
    float v_skip;                 // sparse values: a block whose weights are all below it skips its values
    TqDims tk, tv;
    TqCodebookConsts cbv;         // value codebook (binary16 decode table)
    // 8-bit keys (tq_attention_q8): the key cache, the raw queries and the bf16 tail keys,
    // whose exact logits the split kernel writes to tail_logit
    const uint8_t* packed_k8;
    const void* q;
    int q_dtype;
    const uint16_t* tail_k;
    float scale;
    int d;
};

// 8-bit keys (per 32-coordinate chunk: int8 codes and one binary16 scale), d <= 128
constexpr uint32_t kQ8Block = 4096u + 256u;   // 32 tokens: codes [column 0..7][token][16 B], scales [chunk][token]
struct Q8QuantParams {
    const void* x;
    int dtype;
    uint8_t* packed;
    uint32_t* status;
    int64_t n_streams, n_tok, nb, x_stride;
    int d;
};
struct Q8LogitsParams {
    const uint8_t* packed;
    const void* q;
    int q_dtype;
    const uint16_t* tail;   // bf16 [stream][n_tail][d] or null
    float* out;
    int64_t n_streams, n_tok, nb;
    int g, n_tail, d, nsplit, bps;
    float scale;
};

struct DequantParams {
    const uint8_t* packed;
    float* out;
    const float* pi;
    const float* s;
    int64_t n_streams, n_tok, nb;
    float kappa;
    TqDims t;
    TqCodebookConsts cb;
};

// kernel launchers (one translation unit each)
cudaError_t tq_launch_prepare(const PrepParams& p, cudaStream_t st);
cudaError_t tq_launch_quantize(const QuantParams& p, cudaStream_t st);
cudaError_t tq_launch_logits(const LogitsParams& p, cudaStream_t st);
cudaError_t tq_launch_pv(const PvParams& p, cudaStream_t st);
cudaError_t tq_launch_dequant(const DequantParams& p, cudaStream_t st);
cudaError_t tq_launch_logits_prologue(const LogitsParams& p, cudaStream_t st);
cudaError_t tq_launch_quantize_tc(const QuantParams& p, cudaStream_t st);
bool tq_quantize_ws_eligible(const QuantParams& p);
cudaError_t tq_launch_quantize_wide(const QuantParams& p, cudaStream_t st);
cudaError_t tq_launch_quantize_ws(const QuantParams& p, cudaStream_t st);
cudaError_t tq_launch_attention(const AttnParams& p, cudaStream_t st);
cudaError_t tq_launch_attention_q8(const AttnParams& p, cudaStream_t st);
int tq_attention_q8_ctas_per_sm(int value_bits);
cudaError_t tq_launch_topk(const TopkParams& p, cudaStream_t st);
int tq_topk_nsplit(int64_t n_qt, int64_t n_tiles);   // key ranges per query tile
cudaError_t tq_launch_q8_quantize(const Q8QuantParams& p, cudaStream_t st);
cudaError_t tq_launch_q8_logits(const Q8LogitsParams& p, cudaStream_t st);
