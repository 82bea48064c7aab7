// Derived operands of a codec: transposes of Pi and S, and M = S Pi^T (the sketch applied in
// the rotated domain: S r = S Pi^T (y - c[idx]) because Pi^T Pi = I; blog.hotdry.top
// "TurboQuant vector-search compression", section "QJL residual correction").
#include "tq_device.cuh"

__device__ void split_half(double v, uint16_t* hi, uint16_t* lo) {
    const __half h = __double2half(v);
    *hi = __half_as_ushort(h);
    *lo = __half_as_ushort(__double2half(v - (double)__half2float(h)));
}

// fp16 hi/lo pairs of 256 Pi (row = output coordinate i, column = input j) and 256 M
__global__ void k_prepare_split(PrepParams p) {
    const int64_t n_pi = (int64_t)p.D * p.D, n_m = p.qjl ? (int64_t)p.Mp * p.D : 0;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n_pi + n_m;
         e += (int64_t)gridDim.x * blockDim.x) {
        if (e < n_pi) {
            const int i = (int)(e / p.D), j = (int)(e % p.D);
            const double v = (i < p.d && j < p.d) ? 256.0 * (double)p.pi[(int64_t)i * p.d + j] : 0.0;
            split_half(v, p.pih + e, p.pil + e);
        } else {
            const int64_t f = e - n_pi;
            const int k = (int)(f / p.D), i = (int)(f % p.D);  // M[k][i] = sum_j S[k][j] Pi[i][j]
            double acc = 0.0;
            if (k < p.m && i < p.d)
                for (int j = 0; j < p.d; ++j)
                    acc += (double)p.s[(int64_t)k * p.d + j] * (double)p.pi[(int64_t)i * p.d + j];
            split_half(256.0 * acc, p.mh + f, p.ml + f);
        }
    }
}

__global__ void k_prepare(PrepParams p) {
    const int64_t n_pi = (int64_t)p.D * p.D;
    const int64_t n_s = (int64_t)p.D * p.Mp;
    const int64_t total = n_pi + (p.qjl ? 2 * n_s : 0);
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        if (e < n_pi) {
            int j = (int)(e / p.D), i = (int)(e % p.D);          // PiT[j][i] = Pi[i][j]
            p.piT[e] = (i < p.d && j < p.d) ? p.pi[(int64_t)i * p.d + j] : 0.f;
        } else if (e < n_pi + n_s) {
            int64_t f = e - n_pi;
            int j = (int)(f / p.Mp), k = (int)(f % p.Mp);        // ST[j][k] = S[k][j]
            p.sT[f] = (j < p.d && k < p.m) ? p.s[(int64_t)k * p.d + j] : 0.f;
        } else {
            int64_t f = e - n_pi - n_s;
            int i = (int)(f / p.Mp), k = (int)(f % p.Mp);        // MT[i][k] = sum_j S[k][j] Pi[i][j]
            double acc = 0.0;
            if (i < p.d && k < p.m)
                for (int j = 0; j < p.d; ++j)
                    acc += (double)p.s[(int64_t)k * p.d + j] * (double)p.pi[(int64_t)i * p.d + j];
            p.mT[f] = (float)acc;
        }
    }
}

// Operand images of the warp-specialized quantize (D = Mp = 128): Pi as three bf16 pieces
// (Pi_1 = bf16(Pi), Pi_2 = bf16(Pi - Pi_1), Pi_3 = bf16(Pi - Pi_1 - Pi_2): each difference
// is exact in fp32 and the three pieces sum to the fp32 matrix), and the fp16 hi/lo pair of
// 256 M, all in the swizzled shared-memory layout. Runs after k_prepare_split (reads M).
// Header: whether every entry of the d x d Pi is +-1/sqrt(d) (within fp32 rounding), i.e. Pi
// is a scaled Hadamard rotation such as H D / sqrt(d); the flag word starts with the bit set.
__global__ void k_check_pm1(PrepParams p) {
    const double r = sqrt((double)p.d);
    bool ok = true;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < (int64_t)p.d * p.d;
         e += (int64_t)gridDim.x * blockDim.x)
        ok = ok && fabs(fabs((double)p.pi[e]) * r - 1.0) < 1e-6;
    if (!__syncthreads_and(ok) && threadIdx.x == 0) atomicAnd(&p.hdr[0], 0u);
}

// Header: whether Pi is a Sylvester-ordered randomized Hadamard rotation H diag(s) / sqrt(d)
// with one stored magnitude: d is a power of two, every |Pi[i][j]| equals |Pi[0][0]| bit for
// bit, and every sign is (-1)^popcount(i & j) times the sign of row 0 (H[0][j] = 1).
__global__ void k_check_wht(PrepParams p) {
    bool ok = (p.d & (p.d - 1)) == 0;
    const float mag = fabsf(p.pi[0]);
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; ok && e < (int64_t)p.d * p.d;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int i = (int)(e / p.d), j = (int)(e % p.d);
        const bool neg = p.pi[e] < 0.f, neg0 = p.pi[j] < 0.f;
        ok = fabsf(p.pi[e]) == mag && neg == (neg0 != ((__popc((unsigned)(i & j)) & 1) != 0));
    }
    if (!__syncthreads_and(ok) && threadIdx.x == 0) atomicAnd(&p.hdr[0], ~TQ_PREP_WHT);
}

// Header word 2: max |S| (fp32 bits; non-negative floats order as their bit patterns).
__global__ void k_smax(PrepParams p) {
    float mx = 0.f;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < (int64_t)p.m * p.d;
         e += (int64_t)gridDim.x * blockDim.x)
        mx = fmaxf(mx, fabsf(p.s[e]));
    mx = tq_warp_max(mx);
    if ((threadIdx.x & 31) == 0) atomicMax(&p.hdr[2], __float_as_uint(mx));
}

// sigma_S = 2^(7 - floor(log2 max |S|)), so that sigma_S S stays below 256 (the range of the
// fp16 hi/lo split the Pi images use as 256 Pi)
__device__ float s_image_scale(uint32_t max_bits) {
    const float mx = __uint_as_float(max_bits);
    if (!(mx > 0.f) || !isfinite(mx)) return 1.f;
    const int ex = ((__float_as_int(mx) >> 23) & 0xff) - 127;
    return __int_as_float((127 + min(max(7 - ex, -126), 127)) << 23);
}

__global__ void k_prepare_images(PrepParams p) {
    const bool pm1 = (p.hdr[0] & TQ_PREP_PM1) != 0;
    const float up = pm1 ? sqrtf((float)p.d) : 1.f;
    const float ss = s_image_scale(p.hdr[2]);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        reinterpret_cast<float*>(p.hdr)[1] = pm1 ? up : 1.f;
        reinterpret_cast<float*>(p.hdr)[3] = ss;
    }
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < 128 * 128; e += gridDim.x * blockDim.x) {
        const int i = e >> 7, j = e & 127;
        const uint32_t off = tq_sw128_offset(i, j);
        const float v0 = (i < p.d && j < p.d) ? p.pi[(int64_t)i * p.d + j] : 0.f;
        // a +-1/sqrt(d) rotation: the first piece is exactly +-1 and the others vanish
        const float v = pm1 ? (v0 > 0.f ? 1.f : v0 < 0.f ? -1.f : 0.f) : v0;
        const __nv_bfloat16 b1 = __float2bfloat16_rn(v);
        const float r1 = v - __bfloat162float(b1);
        const __nv_bfloat16 b2 = __float2bfloat16_rn(r1);
        const __nv_bfloat16 b3 = __float2bfloat16_rn(r1 - __bfloat162float(b2));
        *reinterpret_cast<__nv_bfloat16*>(p.img + 0 * kTqImageBytes + off) = b1;
        *reinterpret_cast<__nv_bfloat16*>(p.img + 1 * kTqImageBytes + off) = b2;
        *reinterpret_cast<__nv_bfloat16*>(p.img + 2 * kTqImageBytes + off) = b3;
        *reinterpret_cast<uint16_t*>(p.img + 3 * kTqImageBytes + off) = p.mh[e];
        *reinterpret_cast<uint16_t*>(p.img + 4 * kTqImageBytes + off) = p.ml[e];
        // query prologue: 256 Pi (row i = output coordinate) and sigma_S S (row = sketch row)
        uint8_t* pro = p.img + kTqProImage * kTqImageBytes;
        *reinterpret_cast<uint16_t*>(pro + 0 * kTqImageBytes + off) = p.pih[e];
        *reinterpret_cast<uint16_t*>(pro + 1 * kTqImageBytes + off) = p.pil[e];
        const double sv = (i < p.m && j < p.d) ? (double)ss * (double)p.s[(int64_t)i * p.d + j] : 0.0;
        split_half(sv, reinterpret_cast<uint16_t*>(pro + 2 * kTqImageBytes + off),
                   reinterpret_cast<uint16_t*>(pro + 3 * kTqImageBytes + off));
    }
}

// Chunked images of 256 Pi and 256 M for the 256-wide quantize (D = Mp = 256): chunk
// 4 nh + kb holds rows 128 nh .. +127 and columns 64 kb .. +63 as fp16 hi then lo, each in
// the swizzled [128 rows][128 B] layout. Runs after k_prepare_split (reads its hi/lo pairs).
__global__ void k_prepare_wide_images(PrepParams p) {
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < 2 * 256 * 256; e += gridDim.x * blockDim.x) {
        const int mat = e >> 16, r = (e >> 8) & 255, c = e & 255;
        const size_t src = (size_t)r * 256 + c;
        const uint16_t hi = mat == 0 ? p.pih[src] : p.mh[src];
        const uint16_t lo = mat == 0 ? p.pil[src] : p.ml[src];
        uint8_t* chunk = p.wimg + ((size_t)mat * 8 + (r >> 7) * 4 + (c >> 6)) * kTqWideChunk;
        const uint32_t off = tq_sw128_offset(r & 127, c & 63);
        *reinterpret_cast<uint16_t*>(chunk + off) = hi;
        *reinterpret_cast<uint16_t*>(chunk + 16384 + off) = lo;
    }
}

cudaError_t tq_launch_prepare(const PrepParams& p, cudaStream_t st) {
    k_prepare<<<296, 256, 0, st>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    k_prepare_split<<<296, 256, 0, st>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (p.img) {
        // flag word: TQ_PREP_PM1 | TQ_PREP_WHT (low byte 0x03) until an entry disproves them;
        // max |S| from zero
        if ((e = cudaMemsetAsync(p.hdr, 0, 16, st)) != cudaSuccess) return e;
        if ((e = cudaMemsetAsync(p.hdr, TQ_PREP_PM1 | TQ_PREP_WHT, 1, st)) != cudaSuccess) return e;
        k_smax<<<64, 256, 0, st>>>(p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        k_check_pm1<<<64, 256, 0, st>>>(p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        k_check_wht<<<64, 256, 0, st>>>(p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        k_prepare_images<<<64, 256, 0, st>>>(p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (p.wimg) {
        k_prepare_wide_images<<<256, 256, 0, st>>>(p);
        e = cudaGetLastError();
    }
    return e;
}
