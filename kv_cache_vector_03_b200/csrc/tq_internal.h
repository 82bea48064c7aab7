// Internal definitions shared by the host code and the CUDA kernels of libtq.
//
// Storage formats (blocks of 32 vectors, little-endian words):
//
// Key block (qjl = 1). D = d rounded up to 128, Mp = m rounded up to 128, GD = D/128,
// GM = Mp/128. A vector has B code planes (plane p, bit i = bit p of idx_i) and one sign
// plane (bit j = [z_j >= 0]); bits beyond d (resp. m) are 0. Word w of a plane holds the
// plane's bits 32w..32w+31, bit i at position i mod 32. The NPG = B*GD + GM plane groups
// are ordered [code plane 0 groups 0..GD-1, ..., code plane B-1 ..., sign groups 0..GM-1];
// group gr of a plane is its words 4gr..4gr+3.
//   section A: for pg in 0..NPG-1, lane l in 0..31 (l = 4*gq + tq), u in 0..3:
//              word 4*gr(pg) + tq of plane(pg) of vector 8u + gq        (4 bytes each)
//   section B: for gq in 0..7, u in 0..3: vector 8u + gq: |x| then gamma, binary16 each
//   block bytes = 512 * NPG + 128
//
// Value block (qjl = 0). D = d rounded up to 128. Lane l = 4*gq + tq owns coordinates
// i = 8a + gq (a = 0..D/8-1) and token pairs p = 0..3 with tokens
// tau(p) = 16(p>>1) + 8(p&1) + 2tq and tau(p)+1. The field of (a, p) is
// code(tau, i) | code(tau+1, i) << B (2B bits) at bit offset (4a + p) * 2B of the lane's
// bit string (D*B bits = D*B/128 chunks of 16 bytes).
//   section A: for chunk c, lane l: 16 bytes = bits 128c..128c+127 of lane l's string
//   section B: 32 x |x| binary16, token order
//   block bytes = 4 * D * B + 64
#pragma once
#include <stddef.h>
#include <stdint.h>

#define TQ_MAX_D 256
#define TQ_MAX_B 4
#define TQ_STATUS_BYTES 256
#define TQ_ALIGN 256

// status word bits (device, first word of the workspace)
#define TQ_FLAG_RANGE 1u
#define TQ_FLAG_TIMEOUT 2u

struct TqDims {
    int d, m, B, qjl;
    int D, Mp, GD, GM;
    int npg;          // stored plane groups per key (B*GD + GM); 0 for values
    int nplanes_mma;  // code planes used by the estimator: B=1:1, B=2:2, B=3:4 (adds b0^b1^b2)
    int nmg;          // MMA plane groups: nplanes_mma*GD + GM
    uint32_t sec_a;   // bytes of section A (codes); the norms follow it
    size_t block_bytes;
};

static inline int tq_round_up(int v, int a) { return (v + a - 1) / a * a; }

static inline TqDims tq_dims(int d, int m, int B, int qjl) {
    TqDims t;
    t.d = d; t.m = qjl ? m : 0; t.B = B; t.qjl = qjl;
    t.D = tq_round_up(d, 128);
    t.Mp = qjl ? tq_round_up(m, 128) : 0;
    t.GD = t.D / 128;
    t.GM = t.Mp / 128;
    t.npg = qjl ? B * t.GD + t.GM : 0;
    t.nplanes_mma = B == 3 ? 4 : B;
    t.nmg = qjl ? t.nplanes_mma * t.GD + t.GM : 0;
    t.sec_a = qjl ? 512u * (uint32_t)t.npg : 4u * (uint32_t)t.D * (uint32_t)B;
    t.block_bytes = (size_t)t.sec_a + (qjl ? 128 : 64);
    return t;
}

// Prepared (derived) operands, laid out in the caller's prep buffer:
//   header (256 B: word 0 = TQ_PREP_PM1 when every entry of the d x d Pi is +-1/sqrt(d), a
//   scaled Hadamard rotation, plus TQ_PREP_WHT when moreover d is a power of two and
//   Pi = H diag(s) / sqrt(d) with H the Sylvester Hadamard matrix, H[i][j] = (-1)^popcount(i & j);
//   float word 1 = the factor by which the Pi_1 image exceeds Pi; word 2 = max |S| (fp32 bits);
//   float word 3 = sigma_S, the power of two that puts max |S| sigma_S in [128, 256))
//   | PiT fp32 [D][D] | ST fp32 [D][Mp] | MT fp32 [D][Mp]
//   | Pi_hi, Pi_lo fp16 [D][D] | M_hi, M_lo fp16 [Mp][D]     (tensor-core quantize)
//   | images (keys with D = Mp = 128 only): Pi_1, Pi_2, Pi_3 bf16, M_hi, M_lo fp16 (quantize),
//     then 256 Pi hi, lo and sigma_S S hi, lo fp16 (query prologue)
//   | wide images (keys with D = Mp = 256 only): 256 Pi then 256 M, each as 8 chunks of
//     32 KB, chunk 4 nh + kb = rows 128 nh .. +127, columns 64 kb .. +63: fp16 hi (16 KB)
//     then lo (16 KB), each [128 rows][128 B] with the same 128-byte swizzle
// PiT[j][i] = Pi[i][j], ST[j][k] = S[k][j], MT[i][k] = M[k][i] with M = S Pi^T, all zero
// outside the d x d / m x d corners. The fp16 pairs hold 256 Pi and 256 M split as
// hi = half(v), lo = half(v - hi), row-major (row = output coordinate).
// For a +-1/sqrt(d) rotation the Pi_1 image holds sqrt(d) Pi (exactly +-1) and Pi_2 = Pi_3 = 0,
// so one bf16 pass rotates exactly (up to the fp32 rounding of the stored Pi).
// The images are 128 x 128 16-bit operands (row = output coordinate, column = K) stored
// byte for byte as the tensor cores read them from shared memory: two K-blocks of 64
// columns, each [128 rows][128 B] in 8-row atoms of 1024 B, 16-byte chunk index XOR
// (row mod 8) (the 128-byte swizzle). Pi = Pi_1 + Pi_2 + Pi_3 exactly (bf16 pieces of the
// fp32 matrix: 8 + 8 + 8 significant bits); M_hi, M_lo as above.
#define TQ_PREP_PM1 1u
#define TQ_PREP_WHT 2u
constexpr size_t kTqImageBytes = 128 * 128 * 2;
constexpr int kTqNumImages = 9;     // Pi_1..3, M_hi, M_lo, then Pi_hi, Pi_lo, S_hi, S_lo
constexpr int kTqProImage = 5;      // first image of the query prologue
constexpr size_t kTqWideChunk = 32768;
struct TqPrepLayout {
    size_t hdr, piT, sT, mT, pih, pil, mh, ml, img, wimg, total;
};

static inline TqPrepLayout tq_prep_layout(const TqDims& t) {
    TqPrepLayout L;
    size_t off = 0;
    L.hdr = off; off += 256;
    L.piT = off; off += (size_t)t.D * t.D * 4;
    L.sT = off; off += t.qjl ? (size_t)t.D * t.Mp * 4 : 0;
    L.mT = off; off += t.qjl ? (size_t)t.D * t.Mp * 4 : 0;
    L.pih = off; off += (size_t)t.D * t.D * 2;
    L.pil = off; off += (size_t)t.D * t.D * 2;
    L.mh = off; off += t.qjl ? (size_t)t.Mp * t.D * 2 : 0;
    L.ml = off; off += t.qjl ? (size_t)t.Mp * t.D * 2 : 0;
    L.img = off; off += (t.qjl && t.D == 128 && t.Mp == 128) ? kTqNumImages * kTqImageBytes : 0;
    L.wimg = off; off += (t.qjl && t.D == 256 && t.Mp == 256) ? 16 * kTqWideChunk : 0;
    L.total = off;
    return L;
}

// Codebook-derived constants passed to kernels by value.
struct TqCodebookConsts {
    float bounds[16];     // 2^B - 1 decision boundaries (fp32)
    float cent[16];       // 2^B centroids (fp32)
    float plane_coef[4];  // estimator coefficient a_pi of each MMA code plane (+-1 basis)
    float plane_sum;      // sum of plane_coef (constant term of the +-1 expansion)
    uint32_t lut_half[16];// binary16 centroid bit patterns (values)
};

// Host side helpers implemented in tq_codebook.cpp
int tq_host_codebook(int d, int B, double* c, double* t, double* mse);
