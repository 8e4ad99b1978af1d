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
// int4: one warp quantizes one block of 128 consecutive values per step
// (32 lanes x float4), UNROLL blocks in flight per warp to keep enough bytes
// in flight.  A block holds 128 / G groups of G = 4 * LPG values; the group
// maximum is reduced over its LPG lanes (G = 128, 64 or 32: 32, 16 or 8
// lanes), whose first lane writes the scale.  Groups never straddle rows
// (the row length is a multiple of 128), so group g covers elements
// g * G .. g * G + G - 1 of the flattened matrix and its scale is scales[g].
// ---------------------------------------------------------------------------
template <int UNROLL, int LPG>
__global__ void __launch_bounds__(256) quantize_int4_kernel(const float* __restrict__ w,
                                                            int64_t n_blocks,
                                                            uint8_t* __restrict__ codes,
                                                            float* __restrict__ scales) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t n_warps = (int64_t(gridDim.x) * blockDim.x) >> 5;

    for (int64_t b0 = warp * UNROLL; b0 < n_blocks; b0 += n_warps * UNROLL) {
        uint4 v[UNROLL];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int64_t b = b0 + u;
            if (b < n_blocks) v[u] = ldg_stream(w + b * 128 + lane * 4);
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int64_t b = b0 + u;
            if (b >= n_blocks) break;
            float f[4] = {__uint_as_float(v[u].x), __uint_as_float(v[u].y),
                          __uint_as_float(v[u].z), __uint_as_float(v[u].w)};
            float m = fmaxf(fmaxf(fabsf(f[0]), fabsf(f[1])), fmaxf(fabsf(f[2]), fabsf(f[3])));
#pragma unroll
            for (int o = LPG / 2; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            const float s = fmaxf(m, 1e-6f) * 0.125f;   // exact: division by 8
            // q = clamp(rint(w / s)) with w / s the IEEE quotient.  |w / s| <= 8,
            // and y = w * rn(1 / s) lies within 2^-19 of that quotient (two
            // roundings of at most 2^-24 relative each), so rint gives the same
            // code unless y is within that distance of a half-integer; those
            // elements (about 1 in 10^5) take the division itself.
            const float r = __frcp_rn(s);
            uint32_t packed = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float y = f[i] * r;
                if (fabsf((y - floorf(y)) - 0.5f) < 0x1p-18f) y = __fdiv_rn(f[i], s);
                const float q = fminf(fmaxf(rintf(y), -8.0f), 7.0f);   // half to even
                packed |= (uint32_t(int(q)) & 0xFu) << (4 * i);
            }
            reinterpret_cast<uint16_t*>(codes + b * 64)[lane] = uint16_t(packed);
            if (lane % LPG == 0) scales[b * (32 / LPG) + lane / LPG] = s;
        }
    }
}

// ---------------------------------------------------------------------------
// e4m3 rows: one CTA per row; the row is read twice (amax, then encode); the
// second read hits L2 for the row sizes used here.
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

moe_status launch_quantize_int4(const float* w, int64_t rows, int64_t cols, int group_size, uint8_t* codes,
                                float* scales, cudaStream_t stream) {
    const int64_t n_blocks = rows * (cols / 128);
    if (n_blocks == 0) return MOE_OK;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    constexpr int UNROLL = 4;
    const int64_t warps_needed = ceil_div(n_blocks, UNROLL);
    int64_t blocks = ceil_div(warps_needed, 8);
    const int64_t cap = int64_t(sms) * 8;    // 8 CTAs x 256 threads per SM, grid-stride beyond
    if (blocks > cap) blocks = cap;
    switch (group_size) {
        case 128: quantize_int4_kernel<UNROLL, 32><<<unsigned(blocks), 256, 0, stream>>>(w, n_blocks, codes, scales); break;
        case 64: quantize_int4_kernel<UNROLL, 16><<<unsigned(blocks), 256, 0, stream>>>(w, n_blocks, codes, scales); break;
        case 32: quantize_int4_kernel<UNROLL, 8><<<unsigned(blocks), 256, 0, stream>>>(w, n_blocks, codes, scales); break;
        default: return MOE_ERR_UNSUPPORTED_SHAPE;
    }
    return launch_status();
}

moe_status launch_quantize_fp8_rows(const void* x, int32_t x_dtype, int64_t rows, int64_t cols,
                                    int64_t num_valid, float scale_ub, uint8_t* q, float* scales,
                                    cudaStream_t stream) {
    if (rows == 0) return MOE_OK;
    const unsigned blocks = unsigned(rows < 65535 * 16 ? rows : 65535 * 16);
    if (x_dtype == MOE_DTYPE_BF16)
        quantize_fp8_rows_kernel<bf16><<<blocks, 256, 0, stream>>>(
            static_cast<const bf16*>(x), rows, cols, num_valid, scale_ub, q, scales);
    else
        quantize_fp8_rows_kernel<float><<<blocks, 256, 0, stream>>>(
            static_cast<const float*>(x), rows, cols, num_valid, scale_ub, q, scales);
    return launch_status();
}

}  // namespace moe
