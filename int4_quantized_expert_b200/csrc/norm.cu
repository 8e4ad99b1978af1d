// RMSNorm, the normalization a Llama block applies before its FFN.
//
// "Llama 开源模型系列" (docs.ifdog.com), section "RMSNorm：为什么去掉减均值也能
// 工作": RMSNorm(x) = x / sqrt((1/d) sum_i x_i^2 + eps) * gamma -- only the
// scaling by the root mean square, no mean subtraction.
//
// One CTA of 256 threads per token row.  Pass 1 sums the squares in fp32
// (each thread over its 8-value chunks, then a fixed shuffle tree and a
// fixed order over the 8 warps, so the sum does not depend on timing);
// r = 1 / sqrt(sum / d + eps) with IEEE division and square root.  Pass 2
// writes bf16((x * r) * gamma) (round to nearest even); its second read of
// the row hits L1/L2.  The layer runs it as its first kernel and feeds the
// result to everything after it.  HBM-bound: 4 bytes per element (bf16 in
// and out) plus gamma, once per row from L2.
#include "norm.cuh"

namespace moe {

constexpr int RN_THREADS = 256;

__global__ void __launch_bounds__(RN_THREADS) rmsnorm_kernel(const bf16* __restrict__ x, int D,
                                                             const bf16* __restrict__ gamma, float eps,
                                                             bf16* __restrict__ out) {
    __shared__ float red[RN_THREADS / 32];
    const int64_t r = blockIdx.x;
    const bf16* row = x + r * D;
    const int nblk = D / 8;
    float ss = 0.0f;
    for (int b = threadIdx.x; b < nblk; b += RN_THREADS) {
        const uint4 v = *reinterpret_cast<const uint4*>(row + 8 * b);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float a = bf16_lo(w[i]), c = bf16_hi(w[i]);
            ss = fmaf(a, a, ss);
            ss = fmaf(c, c, ss);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    float tot = 0.0f;
#pragma unroll
    for (int i = 0; i < RN_THREADS / 32; ++i) tot += red[i];
    const float rs = 1.0f / sqrtf(tot / float(D) + eps);
    bf16* orow = out + r * D;
    for (int b = threadIdx.x; b < nblk; b += RN_THREADS) {
        const uint4 v = *reinterpret_cast<const uint4*>(row + 8 * b);
        const uint4 g = *reinterpret_cast<const uint4*>(gamma + 8 * b);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w}, gw[4] = {g.x, g.y, g.z, g.w};
        uint32_t o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            o[i] = pack_bf16x2((bf16_lo(w[i]) * rs) * bf16_lo(gw[i]), (bf16_hi(w[i]) * rs) * bf16_hi(gw[i]));
        *reinterpret_cast<uint4*>(orow + 8 * b) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

moe_status launch_rmsnorm(const bf16* x, int64_t T, int D, const bf16* gamma, float eps, bf16* out,
                          cudaStream_t stream) {
    if (T == 0) return MOE_OK;
    rmsnorm_kernel<<<unsigned(T), RN_THREADS, 0, stream>>>(x, D, gamma, eps, out);
    return launch_status();
}

}  // namespace moe
