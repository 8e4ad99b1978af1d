// Router, top-k, gate and token bucketing.
//
// "1 卡跑通 Llama 4" (discosf.com), section "混合专家路由": MoE.forward scores
// every token against every expert (router_scores), keeps the top-k experts
// (torch.topk) and later adds the score-weighted expert outputs back into
// their tokens.  "Llama 开源模型系列" (docs.ifdog.com), section "MoE 架构详解":
// the router is a linear layer; Scout keeps 1 of 16 experts, Maverick 8 of 128.
//
// Kernels:
//   route_topk_kernel  logits = x W_r^T (+b) on tensor cores (m16n8k16, fp32
//                      accumulate), then per token k passes of a warp argmax
//                      (ties -> lower expert index), then the gate.
//   bucket_kernel      one CTA: per-expert counts, exclusive offsets and the
//                      stable permutation of slots, using warp match/ballot
//                      ranks and a block scan over warps.
#include "common.cuh"

namespace moe {

constexpr int RT_TOK = 64;      // tokens per CTA (4 warps x 16)
constexpr int RT_K = 64;        // K chunk staged in shared memory
constexpr int RT_EPASS = 64;    // experts per accumulator pass (8 n-tiles)
constexpr int RT_LD = RT_K + 8; // padded row length (bf16) -> conflict-free 32-bit reads

__global__ void __launch_bounds__(128) route_topk_kernel(
    const bf16* __restrict__ x, int T, int D, const bf16* __restrict__ wr,
    const float* __restrict__ bias, int E, int k, int32_t* __restrict__ ids,
    float* __restrict__ gates, bf16* __restrict__ x_frag) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    bf16* xs = reinterpret_cast<bf16*>(smem_raw);                 // [RT_TOK][RT_LD]
    bf16* ws = xs + RT_TOK * RT_LD;                               // [RT_EPASS][RT_LD]
    float* logits = reinterpret_cast<float*>(ws + RT_EPASS * RT_LD);  // [RT_TOK][E]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, c = lane & 3;
    const int t0 = blockIdx.x * RT_TOK;

    for (int e0 = 0; e0 < E; e0 += RT_EPASS) {
        float acc[8][4];
#pragma unroll
        for (int n = 0; n < 8; ++n)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[n][i] = 0.0f;

        for (int k0 = 0; k0 < D; k0 += RT_K) {
            __syncthreads();
            // stage x[t0 .. t0+63][k0 .. k0+63] and W_r[e0 .. e0+63][k0 .. k0+63]
            for (int i = tid; i < RT_TOK * (RT_K / 8); i += 128) {
                const int r = i / (RT_K / 8), q = i % (RT_K / 8);
                uint4 v = make_uint4(0, 0, 0, 0);
                const int t = t0 + r;
                if (t < T) {
                    v = *reinterpret_cast<const uint4*>(x + int64_t(t) * D + k0 + q * 8);
                    // The first expert pass also writes x in the layout the
                    // weight-streaming kernels read: every 8 consecutive values
                    // stored as x0 x4 x1 x5 x2 x6 x3 x7.
                    if (x_frag != nullptr && e0 == 0) {
                        uint4 p;
                        p.x = prmt(v.x, v.z, 0x5410);
                        p.y = prmt(v.x, v.z, 0x7632);
                        p.z = prmt(v.y, v.w, 0x5410);
                        p.w = prmt(v.y, v.w, 0x7632);
                        *reinterpret_cast<uint4*>(x_frag + int64_t(t) * D + k0 + q * 8) = p;
                    }
                }
                *reinterpret_cast<uint4*>(xs + r * RT_LD + q * 8) = v;
            }
            for (int i = tid; i < RT_EPASS * (RT_K / 8); i += 128) {
                const int r = i / (RT_K / 8), q = i % (RT_K / 8);
                uint4 v = make_uint4(0, 0, 0, 0);
                if (e0 + r < E) v = *reinterpret_cast<const uint4*>(wr + int64_t(e0 + r) * D + k0 + q * 8);
                *reinterpret_cast<uint4*>(ws + r * RT_LD + q * 8) = v;
            }
            __syncthreads();
            const bf16* xa = xs + (warp * 16) * RT_LD;
#pragma unroll
            for (int kk = 0; kk < RT_K; kk += 16) {
                const uint32_t a0 = *reinterpret_cast<const uint32_t*>(xa + g * RT_LD + kk + 2 * c);
                const uint32_t a1 = *reinterpret_cast<const uint32_t*>(xa + (g + 8) * RT_LD + kk + 2 * c);
                const uint32_t a2 = *reinterpret_cast<const uint32_t*>(xa + g * RT_LD + kk + 2 * c + 8);
                const uint32_t a3 = *reinterpret_cast<const uint32_t*>(xa + (g + 8) * RT_LD + kk + 2 * c + 8);
#pragma unroll
                for (int n = 0; n < 8; ++n) {
                    if (e0 + n * 8 >= E) break;
                    const bf16* wb = ws + (n * 8 + g) * RT_LD + kk + 2 * c;
                    const uint32_t b0 = *reinterpret_cast<const uint32_t*>(wb);
                    const uint32_t b1 = *reinterpret_cast<const uint32_t*>(wb + 8);
                    mma_bf16_16816(acc[n], a0, a1, a2, a3, b0, b1);
                }
            }
        }
        // scatter this pass's logits to shared memory
#pragma unroll
        for (int n = 0; n < 8; ++n) {
            const int e = e0 + n * 8 + 2 * c;
            const int r0 = warp * 16 + g;
            if (e < E) {
                logits[r0 * E + e] = acc[n][0];
                logits[(r0 + 8) * E + e] = acc[n][2];
            }
            if (e + 1 < E) {
                logits[r0 * E + e + 1] = acc[n][1];
                logits[(r0 + 8) * E + e + 1] = acc[n][3];
            }
        }
    }
    __syncthreads();

    // top-k per token: each warp takes 16 tokens; lane holds experts lane + 32 i
    for (int r = warp * 16; r < warp * 16 + 16; ++r) {
        const int t = t0 + r;
        if (t >= T) break;
        float v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = lane + 32 * i;
            v[i] = (e < E) ? logits[r * E + e] + (bias ? bias[e] : 0.0f) : -INFINITY;
        }
        float chosen_val[8];
        int chosen_id[8];
        for (int j = 0; j < k; ++j) {
            // lane-local best (largest value, lowest index among equals)
            float bv = -INFINITY;
            int bi = 0x7fffffff;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int e = lane + 32 * i;
                if (e < E && (v[i] > bv || (v[i] == bv && e < bi))) { bv = v[i]; bi = e; }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
            }
            chosen_val[j] = bv;
            chosen_id[j] = bi;
            // remove the winner: a NaN never compares greater or equal, so it
            // is never selected again
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (lane + 32 * i == bi) v[i] = __int_as_float(0x7fc00000u);
        }
        if (lane == 0) {
            if (k == 1) {
                ids[int64_t(t)] = chosen_id[0];
                gates[int64_t(t)] = 1.0f / (1.0f + expf(-chosen_val[0]));
            } else {
                float sum = 0.0f, ex[8];
                for (int j = 0; j < k; ++j) { ex[j] = expf(chosen_val[j] - chosen_val[0]); sum += ex[j]; }
                for (int j = 0; j < k; ++j) {
                    ids[int64_t(t) * k + j] = chosen_id[j];
                    gates[int64_t(t) * k + j] = ex[j] / sum;
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Bucketing: one CTA of 1024 threads walks the slots in chunks of 1024.
// ---------------------------------------------------------------------------
constexpr int BK_THREADS = 1024;
constexpr int BK_WARPS = BK_THREADS / 32;
constexpr int BK_MAX_E = 256;

__global__ void __launch_bounds__(BK_THREADS) bucket_kernel(
    const int32_t* __restrict__ ids, int n_slots, int E, int32_t* __restrict__ counts,
    int32_t* __restrict__ offsets, int32_t* __restrict__ perm, int32_t* __restrict__ inv_perm,
    int32_t* __restrict__ zero_words, int n_zero) {
    __shared__ int s_count[BK_MAX_E];
    __shared__ int s_base[BK_MAX_E];
    __shared__ int s_warp[BK_WARPS][BK_MAX_E];   // per-warp counts, then exclusive prefix over warps
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (zero_words != nullptr)
        for (int i = tid; i < n_zero; i += BK_THREADS) zero_words[i] = 0;
    for (int e = tid; e < E; e += BK_THREADS) s_count[e] = 0;
    __syncthreads();
    for (int s = tid; s < n_slots; s += BK_THREADS) atomicAdd(&s_count[ids[s]], 1);
    __syncthreads();
    if (tid == 0) {
        int run = 0;
        for (int e = 0; e < E; ++e) { s_base[e] = run; run += s_count[e]; }
    }
    __syncthreads();
    for (int e = tid; e < E; e += BK_THREADS) {
        counts[e] = s_count[e];
        offsets[e] = s_base[e];
    }
    if (tid == 0) offsets[E] = n_slots;

    for (int s0 = 0; s0 < n_slots; s0 += BK_THREADS) {
        for (int i = tid; i < BK_WARPS * E; i += BK_THREADS) s_warp[i / E][i % E] = 0;
        __syncthreads();
        const int s = s0 + tid;
        const bool valid = s < n_slots;
        const int e = valid ? ids[s] : -1 - lane;    // distinct dummies never match real experts
        const unsigned same = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(same & ((1u << lane) - 1u));
        if (valid && rank == 0) s_warp[warp][e] = __popc(same);
        __syncthreads();
        // exclusive prefix over warps, per expert; chunk total added to the base
        for (int ee = tid; ee < E; ee += BK_THREADS) {
            int run = 0;
            for (int w = 0; w < BK_WARPS; ++w) {
                const int cnt = s_warp[w][ee];
                s_warp[w][ee] = run;
                run += cnt;
            }
            s_count[ee] = run;   // chunk total
        }
        __syncthreads();
        if (valid) {
            const int pos = s_base[e] + s_warp[warp][e] + rank;
            perm[pos] = s;
            if (inv_perm != nullptr) inv_perm[s] = pos;
        }
        __syncthreads();
        for (int ee = tid; ee < E; ee += BK_THREADS) s_base[ee] += s_count[ee];
        __syncthreads();
    }
}

size_t route_smem_bytes(int E) {
    return size_t(RT_TOK + RT_EPASS) * RT_LD * sizeof(bf16) + size_t(RT_TOK) * E * sizeof(float);
}

moe_status launch_route(const bf16* x, int T, int D, const bf16* wr, const float* bias, int E, int k,
                        int32_t* ids, float* gates, int32_t* counts, int32_t* offsets, int32_t* perm,
                        int32_t* inv_perm, bf16* x_frag, int32_t* zero_words, int n_zero,
                        cudaStream_t stream, cudaEvent_t between) {
    const size_t smem = route_smem_bytes(E);
    cudaError_t err = cudaFuncSetAttribute(route_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           int(route_smem_bytes(BK_MAX_E)));
    if (err != cudaSuccess) return MOE_ERR_CUDA;
    route_topk_kernel<<<unsigned(ceil_div(T, RT_TOK)), 128, smem, stream>>>(x, T, D, wr, bias, E, k,
                                                                            ids, gates, x_frag);
    moe_status st = launch_status();
    if (st != MOE_OK) return st;
    if (between) cudaEventRecord(between, stream);
    bucket_kernel<<<1, BK_THREADS, 0, stream>>>(ids, T * k, E, counts, offsets, perm, inv_perm,
                                                zero_words, n_zero);
    return launch_status();
}

}  // namespace moe
