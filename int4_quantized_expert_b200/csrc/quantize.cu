// Quantization kernels: int4 groups (of 128, or 64 or 32) and e4m3 rows.
//
// int4_row_quantize, from "1 卡跑通 Llama 4" (discosf.com), section
// "FP8 / Int4 混合量化": per group of 128 consecutive K values,
// scale = max(max|w|, 1e-6) / 8 and q = clamp(round(w / scale), -8, 7).
// Groups of 64 and 32 follow the same rule: "Meta Llama Models Llama 4 单卡
// 量化推理与选型指南" (lshu.cn) names a smaller group_size as the likely next
// step of the int4 path.
// FP8 row quantization, from "Meta Llama Models Llama 4 单卡量化推理与选型指南"
// (lshu.cn), section "量化环节做了什么" (quantize_fp8_per_row).
//
// Both are one pass over HBM: every input byte is read once and every output
// byte written once, so the bound is HBM bandwidth.
#include <cuda_fp8.h>

#include "common.cuh"

namespace moe {

// ---------------------------------------------------------------------------
// int4: a warp takes four consecutive blocks of 128 values (2 KB) per step,
// eight lanes per block.  Load j (0..3) of lane `sub` reads values
// j * 32 + sub * 4 .. + 3 of its block, so each load instruction reads four
// whole 128-byte lines, and a lane holds 16 values of one block: all of its
// group for G = 128, two groups' halves for G = 64, four quarter-groups for
// G = 32.  The group maximum is the lane's own maximum reduced over the
// block's eight lanes (three shuffles).  U steps are loaded before any is
// quantized.  Groups never straddle rows (the row length is a multiple of
// 128), so group g covers elements g * G .. g * G + G - 1 of the flattened
// matrix and its scale is scales[g].
//
// Rounding: q = clamp(rint(w / s), -8, 7) with w / s the IEEE quotient.
// y = w * rn(1 / s) lies within 2^-19 of that quotient (|w / s| <= 8; two
// roundings of at most 2^-24 relative each), so rint(y) is the same code
// unless y is within that distance of a half-integer; a lane holding such a
// value (about 1 in 10^4 lanes) redoes its 16 values with the division
// itself.  rint is an fp32 add of 1.5 * 2^23 (round to nearest even; the sum's
// ulp is 1 for |y| < 2^22), whose low four mantissa bits are then the code in
// two's complement.
// ---------------------------------------------------------------------------
constexpr float kRoundMagic = 12582912.0f;     // 1.5 * 2^23

template <int G>
__global__ void __launch_bounds__(256) quantize_int4_kernel(const float* __restrict__ w,
                                                            int64_t n_blocks,
                                                            uint8_t* __restrict__ codes,
                                                            float* __restrict__ scales) {
    constexpr int NG = 128 / G;        // groups per block
    constexpr int JG = 4 / NG;         // loads of a lane per group
    constexpr int U = 2;               // steps in flight per warp
    const int lane = threadIdx.x & 31;
    const int gi = lane >> 3, sub = lane & 7;
    const int64_t warp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t n_warps = (int64_t(gridDim.x) * blockDim.x) >> 5;
    const int64_t n_steps = (n_blocks + 3) >> 2;

    for (int64_t s0 = warp * U; s0 < n_steps; s0 += n_warps * U) {
        float f[U][16];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t b = (s0 + u) * 4 + gi;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint4 v = make_uint4(0, 0, 0, 0);
                if (b < n_blocks) v = ldg_stream(w + b * 128 + j * 32 + sub * 4);
                f[u][4 * j] = __uint_as_float(v.x);
                f[u][4 * j + 1] = __uint_as_float(v.y);
                f[u][4 * j + 2] = __uint_as_float(v.z);
                f[u][4 * j + 3] = __uint_as_float(v.w);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t b = (s0 + u) * 4 + gi;
            float sc[NG], rc[NG];
#pragma unroll
            for (int g = 0; g < NG; ++g) {
                float m = 0.0f;
#pragma unroll
                for (int e = 16 * g / NG; e < 16 * (g + 1) / NG; ++e) m = fmaxf(m, fabsf(f[u][e]));
#pragma unroll
                for (int o = 4; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                sc[g] = fmaxf(m, 1e-6f) * 0.125f;     // exact: division by 8
                rc[g] = __frcp_rn(sc[g]);
            }
            float t[16];
            bool near_half = false;
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const float y = f[u][e] * rc[e / (4 * JG)];
                t[e] = y + kRoundMagic;
                near_half |= fabsf(y - (t[e] - kRoundMagic)) > 0.5f - 0x1p-18f;
            }
            if (near_half) {
#pragma unroll
                for (int e = 0; e < 16; ++e) t[e] = __fdiv_rn(f[u][e], sc[e / (4 * JG)]) + kRoundMagic;
            }
            if (b < n_blocks) {
                uint16_t* out = reinterpret_cast<uint16_t*>(codes + b * 64);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    uint32_t c[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) c[i] = __float_as_uint(fminf(t[4 * j + i], kRoundMagic + 7.0f));
                    // low byte of c[i] into byte i, then two nibbles per byte
                    const uint32_t q = __byte_perm(__byte_perm(c[0], c[1], 0x0040), __byte_perm(c[2], c[3], 0x4000),
                                                   0x7610) & 0x0F0F0F0Fu;
                    out[j * 8 + sub] = uint16_t(__byte_perm(q | (q >> 4), 0, 0x0020));
                }
                if (sub == 0) {
#pragma unroll
                    for (int g = 0; g < NG; ++g) scales[b * NG + g] = sc[g];
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------
// e4m3 rows: one CTA per row.  Rows longer than 8192 values are read twice
// (amax, then encode; the second read hits L2); shorter ones stay in registers.
// ---------------------------------------------------------------------------
template <typename T>
__device__ __forceinline__ void load8(const T* p, float f[8]);

template <>
__device__ __forceinline__ void load8<bf16>(const bf16* p, float f[8]) {
    uint4 v = *reinterpret_cast<const uint4*>(p);
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) { f[2 * i] = bf16_lo(w[i]); f[2 * i + 1] = bf16_hi(w[i]); }
}

template <>
__device__ __forceinline__ void load8<float>(const float* p, float f[8]) {
    uint4 a = *reinterpret_cast<const uint4*>(p);
    uint4 b = *reinterpret_cast<const uint4*>(p + 4);
    f[0] = __uint_as_float(a.x); f[1] = __uint_as_float(a.y);
    f[2] = __uint_as_float(a.z); f[3] = __uint_as_float(a.w);
    f[4] = __uint_as_float(b.x); f[5] = __uint_as_float(b.y);
    f[6] = __uint_as_float(b.z); f[7] = __uint_as_float(b.w);
}

__device__ __forceinline__ float block_max(float m, float* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) red[warp] = m;
    __syncthreads();
    m = (lane < int(blockDim.x >> 5)) ? red[lane] : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    return m;
}

// e4m3 encode of 8 values (round to nearest even, saturating to +-448).
__device__ __forceinline__ uint2 encode8_e4m3(const float f[8]) {
    uint32_t out[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint32_t word = 0;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            float2 pair = make_float2(f[4 * h + 2 * i], f[4 * h + 2 * i + 1]);
            __nv_fp8x2_storage_t b = __nv_cvt_float2_to_fp8x2(pair, __NV_SATFINITE, __NV_E4M3);
            word |= uint32_t(b) << (16 * i);
        }
        out[h] = word;
    }
    return make_uint2(out[0], out[1]);
}

template <typename T>
__global__ void __launch_bounds__(256) quantize_fp8_rows_kernel(const T* __restrict__ x, int64_t rows,
                                                                int64_t cols, int64_t num_valid,
                                                                float scale_ub, uint8_t* __restrict__ q,
                                                                float* __restrict__ scales) {
    __shared__ float red[32];
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
        uint8_t* qrow = q + r * cols;
        if (r >= num_valid) {
            for (int64_t c = int64_t(threadIdx.x) * 8; c < cols; c += int64_t(blockDim.x) * 8)
                *reinterpret_cast<uint2*>(qrow + c) = make_uint2(0, 0);
            if (threadIdx.x == 0) scales[r] = 0.0f;
            continue;
        }
        const T* xrow = x + r * cols;
        float m = 0.0f;
        for (int64_t c = int64_t(threadIdx.x) * 8; c < cols; c += int64_t(blockDim.x) * 8) {
            float f[8];
            load8<T>(xrow + c, f);
#pragma unroll
            for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(f[i]));
        }
        m = block_max(m, red);
        const float a = fminf(m, scale_ub);
        const float s = __fdiv_rn(fmaxf(a, 1e-12f), 448.0f);
        for (int64_t c = int64_t(threadIdx.x) * 8; c < cols; c += int64_t(blockDim.x) * 8) {
            float f[8];
            load8<T>(xrow + c, f);
#pragma unroll
            for (int i = 0; i < 8; ++i) f[i] = __fdiv_rn(f[i], s);
            *reinterpret_cast<uint2*>(qrow + c) = encode8_e4m3(f);
        }
        if (threadIdx.x == 0) scales[r] = s;
    }
}

// e4m3 of x / s for 8 values, as the IEEE quotient would give.  y = x * rn(1 / s)
// is within 2^-22 relative of the quotient, so the codes of y * (1 - 2^-20) and
// y * (1 + 2^-20) bracket it; the encoding is monotonic, so where the two agree
// they are its code.  Where they differ (y within about 2^-20 of a rounding
// boundary, once in ~10^4 groups of 8) the values are divided outright.
__device__ __forceinline__ uint2 encode8_e4m3_div(const float f[8], float s, float rs) {
    float lo[8], hi[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float y = f[i] * rs;
        lo[i] = y * (1.0f - 0x1p-20f);
        hi[i] = y * (1.0f + 0x1p-20f);
    }
    const uint2 a = encode8_e4m3(lo), b = encode8_e4m3(hi);
    if (a.x == b.x && a.y == b.y) return a;
    float y[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) y[i] = __fdiv_rn(f[i], s);
    return encode8_e4m3(y);
}

// Rows of up to 256 * 8 * CH values: the row stays in registers between the
// amax reduction and the encoding, so it is read once.
template <typename T, int CH>
__global__ void __launch_bounds__(256, 4) quantize_fp8_rows_reg_kernel(const T* __restrict__ x, int64_t rows,
                                                                       int64_t cols, int64_t num_valid,
                                                                       float scale_ub, uint8_t* __restrict__ q,
                                                                       float* __restrict__ scales) {
    __shared__ float red[32];
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
        uint8_t* qrow = q + r * cols;
        if (r >= num_valid) {
            for (int64_t c = int64_t(threadIdx.x) * 8; c < cols; c += int64_t(blockDim.x) * 8)
                *reinterpret_cast<uint2*>(qrow + c) = make_uint2(0, 0);
            if (threadIdx.x == 0) scales[r] = 0.0f;
            continue;
        }
        const T* xrow = x + r * cols;
        float f[CH][8];
        float m = 0.0f;
#pragma unroll
        for (int c = 0; c < CH; ++c) {
            const int64_t col = (int64_t(c) * 256 + threadIdx.x) * 8;
            if (col < cols) {
                load8<T>(xrow + col, f[c]);
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) f[c][i] = 0.0f;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(f[c][i]));
        }
        m = block_max(m, red);
        const float a = fminf(m, scale_ub);
        const float s = __fdiv_rn(fmaxf(a, 1e-12f), 448.0f);
        const float rs = __frcp_rn(s);
#pragma unroll
        for (int c = 0; c < CH; ++c) {
            const int64_t col = (int64_t(c) * 256 + threadIdx.x) * 8;
            if (col < cols) *reinterpret_cast<uint2*>(qrow + col) = encode8_e4m3_div(f[c], s, rs);
        }
        if (threadIdx.x == 0) scales[r] = s;
    }
}

moe_status launch_quantize_int4(const float* w, int64_t rows, int64_t cols, int group_size, uint8_t* codes,
                                float* scales, cudaStream_t stream) {
    const int64_t n_blocks = rows * (cols / 128);
    if (n_blocks == 0) return MOE_OK;
    void (*kern)(const float*, int64_t, uint8_t*, float*) = nullptr;
    switch (group_size) {
        case 128: kern = quantize_int4_kernel<128>; break;
        case 64: kern = quantize_int4_kernel<64>; break;
        case 32: kern = quantize_int4_kernel<32>; break;
        default: return MOE_ERR_UNSUPPORTED_SHAPE;
    }
    // One resident wave (CTAs per SM from the occupancy calculator), grid-stride
    // beyond it: a second partial wave would leave SMs idle at the end.
    int dev = 0, sms = 148, per_sm = 1;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, 0);
    if (per_sm < 1) per_sm = 1;
    const int64_t warps_needed = ceil_div(ceil_div(n_blocks, 4), 2);
    int64_t blocks = ceil_div(warps_needed, 8);
    const int64_t cap = int64_t(sms) * per_sm;
    if (blocks > cap) blocks = cap;
    kern<<<unsigned(blocks), 256, 0, stream>>>(w, n_blocks, codes, scales);
    return launch_status();
}

moe_status launch_quantize_fp8_rows(const void* x, int32_t x_dtype, int64_t rows, int64_t cols,
                                    int64_t num_valid, float scale_ub, uint8_t* q, float* scales,
                                    cudaStream_t stream) {
    if (rows == 0) return MOE_OK;
    const unsigned blocks = unsigned(rows < 65535 * 16 ? rows : 65535 * 16);
    const bool b16 = x_dtype == MOE_DTYPE_BF16;
#define MOE_FP8_ROWS(KERNEL, ...)                                                                        \
    (b16 ? KERNEL<bf16 __VA_ARGS__><<<blocks, 256, 0, stream>>>(static_cast<const bf16*>(x), rows, cols, \
                                                                num_valid, scale_ub, q, scales)          \
         : KERNEL<float __VA_ARGS__><<<blocks, 256, 0, stream>>>(static_cast<const float*>(x), rows, cols, \
                                                                 num_valid, scale_ub, q, scales))
    if (cols <= 2048) MOE_FP8_ROWS(quantize_fp8_rows_reg_kernel, , 1);
    else if (cols <= 4096) MOE_FP8_ROWS(quantize_fp8_rows_reg_kernel, , 2);
    else if (cols <= 8192) MOE_FP8_ROWS(quantize_fp8_rows_reg_kernel, , 4);
    else MOE_FP8_ROWS(quantize_fp8_rows_kernel);
#undef MOE_FP8_ROWS
    return launch_status();
}

}  // namespace moe
