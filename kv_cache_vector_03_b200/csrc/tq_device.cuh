// Device-side helpers and kernel parameter blocks of libtq (sm_100a).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "tq_internal.h"

#define TQ_DEVICE __device__ __forceinline__

TQ_DEVICE uint32_t tq_half_bits(float v) { return (uint32_t)__half_as_ushort(__float2half_rn(v)); }
TQ_DEVICE float tq_half_val(uint32_t bits) { return __half2float(__ushort_as_half((unsigned short)bits)); }

TQ_DEVICE float tq_load_elem(const void* p, int dtype, int64_t i) {
    if (dtype == 1) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
    return reinterpret_cast<const float*>(p)[i];
}

TQ_DEVICE void tq_raise(uint32_t* status, uint32_t flag) {
    if (status) atomicOr(status, flag);
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
    int d, m, D, Mp, qjl;
};

struct QuantParams {
    const void* x;
    int dtype;
    int64_t n_streams, n_tok, x_stride, nb;  // nb = blocks per stream
    uint8_t* packed;
    const float* piT;
    const float* mT;
    uint32_t* status;
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
    uint32_t* qfrag;       // [stream][ntile][nmg][4][32][2]
    float* qscale;         // [stream][ntile*4][4]: dA, KA, 2dS, KS
    int64_t n_seq, n_tok, nb;
    int n_kv, g, ntiles, n_tail;
    float scale, kappa;
    int blocks_per_task;
    TqDims t;
    TqCodebookConsts cb;
};

struct PvParams {
    const uint8_t* packed;
    const float* P;
    float* out;
    const float* pi;
    float* part;           // [stream*g heads][nsplit][D]
    float* part_ml;        // [stream*g heads][nsplit][2]: max, sum
    int64_t n_streams, n_tok, nb;
    int g, nsplit, blocks_per_split;
    TqDims t;
    TqCodebookConsts cb;
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
