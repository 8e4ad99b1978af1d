// Router, top-k, gate and token bucketing.
//
// "1 卡跑通 Llama 4" (discosf.com), section "混合专家路由": MoE.forward scores
// every token against every expert (router_scores), keeps the top-k experts
// (torch.topk) and later adds the score-weighted expert outputs back into
// their tokens.  "Llama 开源模型系列" (docs.ifdog.com), section "MoE 架构详解":
// the router is a linear layer; Scout keeps 1 of 16 experts, Maverick 8 of 128.
//
// Kernels:
//   router_kernel  16 tokens per CTA; up to 12 warps split the K dimension in
//                  whole groups of 128, each computing 16 x E partial logits
//                  with m16n8k16 tensor-core MMAs (fp32 accumulate) from
//                  fragments loaded straight from global memory.  Partials are
//                  summed in a fixed order (deterministic), the bias added, and
//                  each token's top-k taken by k passes of a warp argmax (ties
//                  -> lower expert index), then the gate.  With an RMSNorm it
//                  normalizes the rows first and writes them out.
//   bucket_kernel  one CTA: per-expert counts, exclusive offsets and the stable
//                  permutation of slots from warp match ranks and a scan over
//                  warps; optionally the weight-streaming FFN's task list.
#include "common.cuh"
#include "ffn_decode.cuh"

namespace moe {

constexpr int RT_TOK = 16;      // tokens per CTA (one m16 tile)
constexpr int RT_MAXW = 12;     // warps splitting K
constexpr size_t RT_SMEM_MAX = 160 * 1024;

// Warps used: the largest divisor of D / 128 that is <= 12 and whose partial
// logits (warps x 16 tokens x E fp32) fit in RT_SMEM_MAX.
inline int router_warps(int D, int E) {
    const int groups = D / kGroup;
    for (int w = RT_MAXW; w > 1; --w)
        if (groups % w == 0 && size_t(w) * RT_TOK * E * sizeof(float) <= RT_SMEM_MAX) return w;
    return 1;
}

// grid (token tiles, ksplit): CTA (i, j) takes tokens 16 i .. 16 i + 15 and
// the j-th of ksplit equal K ranges.  With ksplit > 1 each CTA stores its
// partial logits (summed over its warps) to part_g and the last CTA of a
// tile to arrive (counted in tile_cnt, zeroed beforehand) sums them in
// K-range order -- the same order whichever CTA is last -- and takes the
// top-k.  No CTA waits for another.
// NT: n-tiles of 8 experts per accumulator pass (1, 2 or 4), the smallest
// power of two covering E up to 32 -- few experts keep few registers, so more
// CTAs fit on an SM.
template <int NT>
__global__ void __launch_bounds__(RT_MAXW * 32, NT <= 2 ? 2 : 1) router_kernel(
    const bf16* __restrict__ x, int T, int D, const bf16* __restrict__ wr,
    const float* __restrict__ bias, int E, int k, int32_t* __restrict__ ids,
    float* __restrict__ gates, int ksplit, float* __restrict__ part_g,
    int32_t* __restrict__ tile_cnt, const bf16* __restrict__ gamma, float rms_eps, bf16* __restrict__ xn,
    int32_t* __restrict__ xn_ready) {
    extern __shared__ __align__(16) float part[];     // [nw][RT_TOK][E]
    __shared__ int s_last;
    __shared__ float s_ss[RT_TOK], s_inv[RT_TOK];
    griddep_launch_dependents();
    const int nw = blockDim.x >> 5;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    const int t0 = blockIdx.x * RT_TOK;
    const int groups_per_cta = (D / kGroup) / ksplit;
    const int groups_per_warp = groups_per_cta / nw;
    const int k_begin = (blockIdx.y * groups_per_cta + warp * groups_per_warp) * kGroup;
    const int k_end = k_begin + groups_per_warp * kGroup;
    const bool row_a = t0 + g < T, row_b = t0 + g + 8 < T;
    const bf16* xa_row = x + int64_t(t0 + g) * D;
    const bf16* xb_row = x + int64_t(t0 + g + 8) * D;

    if (gamma != nullptr) {
        // RMSNorm of the tile's rows first ("Llama 开源模型系列", "RMSNorm：为什么
        // 去掉减均值也能工作"): each CTA sums the squares over its own K range
        // (a warp per row, lanes over 8-value chunks, a fixed shuffle tree), the
        // tile's CTAs -- one thread-block cluster -- add the ksplit partial sums
        // in rank (K range) order through distributed shared memory, so every
        // CTA holds the same r = 1 / sqrt(sum / D + eps).  The GEMV below runs on
        // xn = bf16((x * r) * gamma), which the CTA first writes out for the
        // kernels after the router.
        const int k0 = blockIdx.y * groups_per_cta * kGroup, nb = groups_per_cta * kGroup / 8;
        for (int r = warp; r < RT_TOK; r += nw) {
            float ss = 0.0f;
            if (t0 + r < T) {
                const bf16* row = x + int64_t(t0 + r) * D + k0;
                for (int b = lane; b < nb; b += 32) {
                    const uint4 v = ldg_cached(row + 8 * b);
                    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float a = bf16_lo(w[i]), h = bf16_hi(w[i]);
                        ss = fmaf(a, a, ss);
                        ss = fmaf(h, h, ss);
                    }
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
            if (lane == 0) s_ss[r] = ss;
        }
        cluster_sync();
        if (threadIdx.x < RT_TOK) {
            float tot = 0.0f;
            for (int rk = 0; rk < ksplit; ++rk) tot += ld_dsmem_f32(&s_ss[threadIdx.x], rk);
            s_inv[threadIdx.x] = t0 + int(threadIdx.x) < T ? 1.0f / sqrtf(tot / float(D) + rms_eps) : 0.0f;
        }
        cluster_sync();   // every CTA has read the others' sums; s_inv is visible
    }
    // x -> xn = bf16((x * r) * gamma) for 8 values of one row
    auto rms_apply = [&](uint4 v, float r, uint4 gm) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w}, gw[4] = {gm.x, gm.y, gm.z, gm.w};
        uint32_t o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            o[i] = pack_bf16x2((bf16_lo(w[i]) * r) * bf16_lo(gw[i]), (bf16_hi(w[i]) * r) * bf16_hi(gw[i]));
        return make_uint4(o[0], o[1], o[2], o[3]);
    };
    if (gamma != nullptr) {
        // this CTA's part of xn (the tile's rows over its K range) goes out
        // first, and is counted, so kernels that need only xn can start before
        // the GEMV below has finished
        const int k0 = blockIdx.y * groups_per_cta * kGroup, nb = groups_per_cta * kGroup / 8;
        for (int idx = threadIdx.x; idx < RT_TOK * nb; idx += blockDim.x) {
            const int r = idx / nb, kk = k0 + 8 * (idx % nb);
            if (t0 + r >= T) continue;
            const uint4 v = ldg_cached(x + int64_t(t0 + r) * D + kk);
            *reinterpret_cast<uint4*>(xn + int64_t(t0 + r) * D + kk) = rms_apply(v, s_inv[r], ldg_cached(gamma + kk));
        }
        __threadfence();
        __syncthreads();
        if (xn_ready != nullptr && threadIdx.x == 0) atomicAdd(xn_ready, 1);
    }

    for (int e0 = 0; e0 < E; e0 += 8 * NT) {
        float acc[NT][4];
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[n][i] = 0.0f;

        // operands of the next 32-K chunk are loaded while the current one runs
        const int n_tiles = min(NT, (E - e0 + 7) / 8);
        uint4 xa, xb, wv[NT], nxa, nxb, nwv[NT];
        auto load = [&](int kk, uint4& a, uint4& b, uint4 (&w)[NT]) {
            a = row_a ? ldg_cached(xa_row + kk + 8 * c) : make_uint4(0, 0, 0, 0);
            b = row_b ? ldg_cached(xb_row + kk + 8 * c) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                const int e = e0 + n * 8 + g;
                w[n] = (n < n_tiles && e < E) ? ldg_cached(wr + int64_t(e) * D + kk + 8 * c) : make_uint4(0, 0, 0, 0);
            }
        };
        load(k_begin, xa, xb, wv);
        for (int kk = k_begin; kk < k_end; kk += 32) {
            if (kk + 32 < k_end) load(kk + 32, nxa, nxb, nwv);
            if (gamma != nullptr) {   // the same xn values as written out above
                const uint4 gm = ldg_cached(gamma + kk + 8 * c);
                xa = rms_apply(xa, s_inv[g], gm);
                xb = rms_apply(xb, s_inv[g + 8], gm);
            }
            // thread (g, c) holds K values kk + 8c .. kk + 8c + 7 of rows g and g + 8;
            // the two MMAs below use them as K pairs (0,1)(2,3) and (4,5)(6,7)
            // of A, and the expert rows of W_r in the same order as B.
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                if (n >= n_tiles) break;
                mma_bf16_16816(acc[n], xa.x, xb.x, xa.y, xb.y, wv[n].x, wv[n].y);
                mma_bf16_16816(acc[n], xa.z, xb.z, xa.w, xb.w, wv[n].z, wv[n].w);
            }
            xa = nxa;
            xb = nxb;
#pragma unroll
            for (int n = 0; n < NT; ++n) wv[n] = nwv[n];
        }
        // C fragment: rows (tokens) g, g + 8; columns (experts) 2c, 2c + 1 of each n-tile
        float* pw = part + warp * RT_TOK * E;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            const int e = e0 + n * 8 + 2 * c;
            if (e < E) { pw[g * E + e] = acc[n][0]; pw[(g + 8) * E + e] = acc[n][2]; }
            if (e + 1 < E) { pw[g * E + e + 1] = acc[n][1]; pw[(g + 8) * E + e + 1] = acc[n][3]; }
        }
    }
    __syncthreads();

    if (ksplit > 1) {
        // this K range's logits to global memory; the tile's last CTA goes on
        float* mine = part_g + (int64_t(blockIdx.x) * ksplit + blockIdx.y) * RT_TOK * E;
        for (int i = threadIdx.x; i < RT_TOK * E; i += blockDim.x) {
            float a = 0.0f;
            for (int w = 0; w < nw; ++w) a += part[w * RT_TOK * E + i];
            mine[i] = a;
        }
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0) s_last = atomicAdd(&tile_cnt[blockIdx.x], 1) == ksplit - 1;
        __syncthreads();
        if (!s_last) {
            griddep_wait();
            return;
        }
        __threadfence();
        // the tile's logits, summed over the K ranges in order, into part[0,
        // 16 E) (part holds nw x 16 x E >= 16 x E floats): loads are issued
        // eight at a time before they are added, so the sum costs ksplit / 8
        // L2 round trips instead of ksplit dependent ones
        const float* base = part_g + int64_t(blockIdx.x) * ksplit * RT_TOK * E;
        for (int i = threadIdx.x; i < RT_TOK * E; i += blockDim.x) {
            float a = 0.0f;
            for (int j0 = 0; j0 < ksplit; j0 += 8) {
                float v[8];
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    v[j] = j0 + j < ksplit ? __ldcg(base + int64_t(j0 + j) * RT_TOK * E + i) : 0.0f;
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    if (j0 + j < ksplit) a += v[j];
            }
            part[i] = a;
        }
        __syncthreads();
    }
    // logit of token row r, expert e: the sum over warps (one CTA), or the
    // K ranges' sum formed above (split)
    auto logit = [&](int r, int e) {
        if (ksplit > 1) return part[r * E + e];
        float a = 0.0f;
        for (int w = 0; w < nw; ++w) a += part[(w * RT_TOK + r) * E + e];
        return a;
    };

    // top-k per token; lane holds experts lane + 32 i
    for (int r = warp; r < RT_TOK; r += nw) {
        const int t = t0 + r;
        if (t >= T) break;
        float v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = lane + 32 * i;
            float s = -INFINITY;
            if (e < E) {
                s = logit(r, e);
                if (bias) s += bias[e];
            }
            v[i] = s;
        }
        float chosen_val[8];
        int chosen_id[8];
        for (int j = 0; j < k; ++j) {
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
            // remove the winner: a NaN never compares greater or equal
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (lane + 32 * i == bi) v[i] = __int_as_float(0x7fc00000u);
        }
        if (lane == 0) {
            if (k == 1) {
                ids[t] = chosen_id[0];
                gates[t] = 1.0f / (1.0f + expf(-chosen_val[0]));
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
    // reads nothing of the kernel before it (if launched dependent on one),
    // but completes only after it
    griddep_wait();
}

// ---------------------------------------------------------------------------
// Bucketing: one CTA of 1024 threads walks the slots in chunks of 1024.
// ---------------------------------------------------------------------------
constexpr int BK_THREADS = 1024;
constexpr int BK_WARPS = BK_THREADS / 32;
constexpr int BK_MAX_E = 256;

__global__ void __launch_bounds__(BK_THREADS) bucket_kernel(
    const int32_t* __restrict__ ids, int n_slots, int T, int E, int32_t* __restrict__ counts,
    int32_t* __restrict__ offsets, int32_t* __restrict__ perm, int32_t* __restrict__ inv_perm,
    ChunkEntry* __restrict__ chunks, int32_t* __restrict__ n_chunks, int chunk_tokens, int routed_chunk_tokens,
    int32_t* __restrict__ zero_words, int n_zero, int32_t* __restrict__ status) {
    __shared__ int s_count[BK_MAX_E];
    __shared__ int s_base[BK_MAX_E];
    __shared__ int s_warp[BK_WARPS][BK_MAX_E];   // per-warp counts, then exclusive prefix over warps
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    griddep_launch_dependents();
    griddep_wait();   // the router's ids

    if (zero_words != nullptr)
        for (int i = tid; i < n_zero; i += BK_THREADS) zero_words[i] = 0;
    for (int e = tid; e < E; e += BK_THREADS) s_count[e] = 0;
    __syncthreads();
    // ids given by a caller may be out of range: such a slot is counted as
    // expert 0 and the status word says so (the router's are always valid)
    auto expert_of = [&](int s) {
        const int e = ids[s];
        if (unsigned(e) < unsigned(E)) return e;
        if (status) atomicExch(status, DEV_BAD_EXPERT);
        return 0;
    };
    for (int s = tid; s < n_slots; s += BK_THREADS) atomicAdd(&s_count[expert_of(s)], 1);
    __syncthreads();
    if (tid == 0) {
        int run = 0;
        for (int e = 0; e < E; ++e) { s_base[e] = run; run += s_count[e]; }
        if (chunks != nullptr) {
            // task list of the FFN kernels: the shared expert's chunks of
            // <= chunk_tokens tokens, then each routed expert's of
            // <= routed_chunk_tokens
            int n = 0;
            for (int t0 = 0; t0 < T; t0 += chunk_tokens) {
                ChunkEntry ce; ce.expert = -1; ce.start = t0; ce.count = min(chunk_tokens, T - t0); ce.pad = 0;
                chunks[n++] = ce;
            }
            n_chunks[1] = n;
            for (int e = 0; e < E; ++e)
                for (int s = 0; s < s_count[e]; s += routed_chunk_tokens) {
                    ChunkEntry ce; ce.expert = e; ce.start = s_base[e] + s;
                    ce.count = min(routed_chunk_tokens, s_count[e] - s);
                    ce.pad = 0;
                    chunks[n++] = ce;
                }
            n_chunks[0] = n;
        }
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
        const int e = valid ? expert_of(s) : -1 - lane;    // distinct dummies never match real experts
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

// ---------------------------------------------------------------------------
// Bucketing of many slots over several CTAs (the same results as
// bucket_kernel): each CTA takes a block of BK_BLOCK consecutive slots.
//   bucket_hist_kernel   per-block expert counts -> hist[block][E]
//   bucket_scan_kernel   one CTA: counts, offsets, the chunk list, and each
//                        (block, expert)'s first position -> hist
//   bucket_place_kernel  per block: stable positions of its slots (warp match
//                        ranks and a prefix over warps, block by block in slot
//                        order) -> perm, inv_perm
// Three launches chained by programmatic dependent launch; no CTA waits for
// another.
// ---------------------------------------------------------------------------
constexpr int BK_BLOCK = 2 * BK_THREADS;

__device__ __forceinline__ int bucket_expert(const int32_t* ids, int s, int E, int32_t* status) {
    const int e = ids[s];
    if (unsigned(e) < unsigned(E)) return e;
    if (status) atomicExch(status, DEV_BAD_EXPERT);   // given ids out of range count as expert 0
    return 0;
}

__global__ void __launch_bounds__(BK_THREADS) bucket_hist_kernel(const int32_t* __restrict__ ids, int n_slots,
                                                                 int E, int32_t* __restrict__ hist,
                                                                 int32_t* __restrict__ status) {
    __shared__ int s_count[BK_MAX_E];
    griddep_launch_dependents();
    griddep_wait();   // the router's ids
    for (int e = threadIdx.x; e < E; e += BK_THREADS) s_count[e] = 0;
    __syncthreads();
    const int s_end = min(n_slots, (blockIdx.x + 1) * BK_BLOCK);
    for (int s = blockIdx.x * BK_BLOCK + threadIdx.x; s < s_end; s += BK_THREADS)
        atomicAdd(&s_count[bucket_expert(ids, s, E, status)], 1);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += BK_THREADS) hist[blockIdx.x * E + e] = s_count[e];
}

// Inclusive prefix sum over the 32 lanes of a warp.
__device__ __forceinline__ int warp_inclusive_scan(int v, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
    }
    return v;
}

// Exclusive prefix over a[0 .. n) (n <= BK_MAX_E) in shared memory by warp 0;
// returns the total to every lane of warp 0.
__device__ __forceinline__ int warp_exclusive_scan_smem(int* a, int n, int lane) {
    int carry = 0;
    for (int i0 = 0; i0 < n; i0 += 32) {
        const int v = i0 + lane < n ? a[i0 + lane] : 0;
        const int inc = warp_inclusive_scan(v, lane);
        if (i0 + lane < n) a[i0 + lane] = carry + inc - v;
        carry += __shfl_sync(0xffffffffu, inc, 31);
    }
    return carry;
}

__global__ void __launch_bounds__(BK_THREADS) bucket_scan_kernel(
    int32_t* __restrict__ hist, int n_blocks, int n_slots, int T, int E, int32_t* __restrict__ counts,
    int32_t* __restrict__ offsets, ChunkEntry* __restrict__ chunks, int32_t* __restrict__ n_chunks,
    int chunk_tokens, int routed_chunk_tokens) {
    __shared__ int s_count[BK_MAX_E];
    __shared__ int s_base[BK_MAX_E];
    __shared__ int s_cbase[BK_MAX_E];   // first chunk-list entry of each expert
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    griddep_launch_dependents();
    griddep_wait();
    // a warp per expert: lanes over the blocks, a running carry over groups
    // of 32 blocks; each (block, expert) entry becomes that block's first
    // position within the expert (relative; the expert's base is added below)
    for (int e = warp; e < E; e += BK_WARPS) {
        int carry = 0;
        for (int b0 = 0; b0 < n_blocks; b0 += 32) {
            const int b = b0 + lane;
            const int c = b < n_blocks ? hist[b * E + e] : 0;
            const int inc = warp_inclusive_scan(c, lane);
            if (b < n_blocks) hist[b * E + e] = carry + inc - c;
            carry += __shfl_sync(0xffffffffu, inc, 31);
        }
        if (lane == 0) s_count[e] = carry;
    }
    __syncthreads();
    const int n_sh = (T + chunk_tokens - 1) / chunk_tokens;
    if (warp == 0) {
        for (int e = lane; e < E; e += 32) {
            s_base[e] = s_count[e];
            s_cbase[e] = (s_count[e] + routed_chunk_tokens - 1) / routed_chunk_tokens;
        }
        __syncwarp();
        warp_exclusive_scan_smem(s_base, E, lane);
        const int n_routed = warp_exclusive_scan_smem(s_cbase, E, lane);
        if (lane == 0) {
            offsets[E] = n_slots;
            if (chunks != nullptr) {
                n_chunks[1] = n_sh;
                n_chunks[0] = n_sh + n_routed;
            }
        }
    }
    __syncthreads();
    for (int e = tid; e < E; e += BK_THREADS) {
        counts[e] = s_count[e];
        offsets[e] = s_base[e];
    }
    // absolute first positions: add each expert's base
    for (int i = tid; i < n_blocks * E; i += BK_THREADS) hist[i] += s_base[i % E];
    if (chunks != nullptr) {   // the FFN kernels' task list, as bucket_kernel writes it
        for (int c = tid; c < n_sh; c += BK_THREADS) {
            ChunkEntry ce; ce.expert = -1; ce.start = c * chunk_tokens;
            ce.count = min(chunk_tokens, T - c * chunk_tokens); ce.pad = 0;
            chunks[c] = ce;
        }
        // one warp per expert, lanes over its chunks
        for (int e = warp; e < E; e += BK_WARPS) {
            const int cnt = s_count[e];
            for (int j = lane; j * routed_chunk_tokens < cnt; j += 32) {
                ChunkEntry ce; ce.expert = e; ce.start = s_base[e] + j * routed_chunk_tokens;
                ce.count = min(routed_chunk_tokens, cnt - j * routed_chunk_tokens); ce.pad = 0;
                chunks[n_sh + s_cbase[e] + j] = ce;
            }
        }
    }
}

__global__ void __launch_bounds__(BK_THREADS) bucket_place_kernel(const int32_t* __restrict__ ids, int n_slots,
                                                                  int E, const int32_t* __restrict__ hist,
                                                                  int32_t* __restrict__ perm,
                                                                  int32_t* __restrict__ inv_perm) {
    __shared__ int s_count[BK_MAX_E];
    __shared__ int s_base[BK_MAX_E];
    __shared__ int s_warp[BK_WARPS][BK_MAX_E];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    griddep_launch_dependents();
    griddep_wait();   // the bases
    for (int e = tid; e < E; e += BK_THREADS) s_base[e] = hist[blockIdx.x * E + e];
    const int s_begin = blockIdx.x * BK_BLOCK, s_end = min(n_slots, s_begin + BK_BLOCK);
    for (int s0 = s_begin; s0 < s_end; s0 += BK_THREADS) {
        for (int i = tid; i < BK_WARPS * E; i += BK_THREADS) s_warp[i / E][i % E] = 0;
        __syncthreads();
        const int s = s0 + tid;
        const bool valid = s < s_end;
        const int e = valid ? bucket_expert(ids, s, E, nullptr) : -1 - lane;
        const unsigned same = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(same & ((1u << lane) - 1u));
        if (valid && rank == 0) s_warp[warp][e] = __popc(same);
        __syncthreads();
        for (int ee = tid; ee < E; ee += BK_THREADS) {
            int run = 0;
            for (int w = 0; w < BK_WARPS; ++w) {
                const int cnt = s_warp[w][ee];
                s_warp[w][ee] = run;
                run += cnt;
            }
            s_count[ee] = run;
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

int bucket_blocks(int64_t n_slots) { return n_slots >= 2 * BK_BLOCK ? int(ceil_div(n_slots, BK_BLOCK)) : 0; }

size_t router_smem_bytes(int D, int E) { return size_t(router_warps(D, E)) * RT_TOK * E * sizeof(float); }

// K ranges per token tile: with few tiles (a decode batch) the router would
// run on a handful of SMs, so K is split over up to 32 CTAs per tile, each
// with at least two groups of 128.
// With an RMSNorm the split CTAs of a tile form one thread-block cluster, so
// at most 8 (the portable cluster size).
int router_ksplit(int T, int D, bool rms) {
    const int tiles = int(ceil_div(T, RT_TOK)), groups = D / kGroup;
    if (tiles >= 37) return 1;
    for (int ks = rms ? 8 : 32; ks > 1; --ks)
        if (groups % ks == 0 && groups / ks >= 2) return ks;
    return 1;
}

size_t router_partial_floats(int T, int D, int E, bool rms) {
    const int ks = router_ksplit(T, D, rms);
    return ks > 1 ? size_t(ks) * ceil_div(T, RT_TOK) * RT_TOK * E : 0;
}

moe_status launch_route(const bf16* x, int T, int D, const bf16* wr, const float* bias, int E, int k,
                        int32_t* ids, float* gates, int32_t* counts, int32_t* offsets, int32_t* perm,
                        int32_t* inv_perm, const RoutePrep* prep, cudaStream_t stream, cudaEvent_t between,
                        cudaEvent_t ev_scan, cudaEvent_t ev_place) {
    // K split only with scratch for the partial logits (the layer's workspace)
    const bool rms = prep && prep->rms_weight;
    const int ks = (prep && prep->router_part) ? router_ksplit(T, D, rms) : 1;
    const int nw = router_warps(D / ks, E);
    const size_t smem = router_smem_bytes(D / ks, E);
    // n-tiles per pass: the smallest power of two covering E, at most 4 (more
    // experts take several passes over the CTA's K range; 8 n-tiles spilled)
    auto kern = E <= 8 ? router_kernel<1> : E <= 16 ? router_kernel<2> : router_kernel<4>;
    if (allow_max_smem(kern) != MOE_OK) return MOE_ERR_CUDA;
    moe_status st;
    float* part_g = ks > 1 ? prep->router_part : nullptr;
    int32_t* tile_cnt = ks > 1 ? prep->router_tile_cnt : nullptr;
    const dim3 grid(unsigned(ceil_div(T, RT_TOK)), unsigned(ks));
    const bf16* gamma = rms ? prep->rms_weight : nullptr;
    const float eps = rms ? prep->rms_eps : 0.0f;
    bf16* xn = rms ? prep->xn : nullptr;
    int32_t* xn_ready = rms ? prep->xn_ready : nullptr;
    {
        // with an RMSNorm, a tile's ks CTAs form one cluster; the router may
        // overlap the kernel before it when asked (it reads only x, gamma and W_r)
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = grid;
        cfg.blockDim = dim3(nw * 32);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = stream;
        cudaLaunchAttribute attr[2];
        int na = 0;
        if (rms) {
            attr[na].id = cudaLaunchAttributeClusterDimension;
            attr[na].val.clusterDim.x = 1;
            attr[na].val.clusterDim.y = unsigned(ks);
            attr[na].val.clusterDim.z = 1;
            ++na;
        }
        if (prep && prep->router_after_kernel) {
            attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
            attr[na].val.programmaticStreamSerializationAllowed = 1;
            ++na;
        }
        cfg.attrs = attr;
        cfg.numAttrs = na;
        st = cuda_status(cudaLaunchKernelEx(&cfg, kern, x, T, D, wr, bias, E, k, ids, gates, ks, part_g, tile_cnt,
                                            gamma, eps, xn, xn_ready));
    }
    if (st != MOE_OK) return st;
    if (between) cudaEventRecord(between, stream);
    return launch_bucket(ids, T, k, E, counts, offsets, perm, inv_perm, prep, stream, ev_scan, ev_place);
}

moe_status launch_bucket(const int32_t* ids, int T, int k, int E, int32_t* counts, int32_t* offsets, int32_t* perm,
                         int32_t* inv_perm, const RoutePrep* prep, cudaStream_t stream, cudaEvent_t ev_scan,
                         cudaEvent_t ev_place) {
    const int nb = bucket_blocks(int64_t(T) * k);
    if (prep && prep->bucket_hist && nb > 0 && prep->zero_words == nullptr) {
        // many slots: three kernels over ceil(slots / BK_BLOCK) CTAs
        const int n_slots = T * k;
        int32_t* st = prep->status;
        moe_status s = launch_pdl(bucket_hist_kernel, dim3(nb), dim3(BK_THREADS), 0, stream, ids, n_slots, E,
                                  prep->bucket_hist, st);
        if (s != MOE_OK) return s;
        if (ev_scan) cudaEventRecord(ev_scan, stream);
        s = launch_pdl(bucket_scan_kernel, dim3(1), dim3(BK_THREADS), 0, stream, prep->bucket_hist, nb, n_slots, T, E,
                       counts, offsets, prep->chunks, prep->n_chunks, prep->chunk_tokens, prep->routed_chunk_tokens);
        if (s != MOE_OK) return s;
        if (ev_place) cudaEventRecord(ev_place, stream);
        return launch_pdl(bucket_place_kernel, dim3(nb), dim3(BK_THREADS), 0, stream, ids, n_slots, E,
                          (const int32_t*)prep->bucket_hist, perm, inv_perm);
    }
    return launch_pdl(bucket_kernel, dim3(1), dim3(BK_THREADS), 0, stream, ids, T * k, T, E, counts, offsets, perm,
                      inv_perm, prep ? prep->chunks : (ChunkEntry*)nullptr, prep ? prep->n_chunks : (int32_t*)nullptr,
                      prep ? prep->chunk_tokens : 16, prep ? prep->routed_chunk_tokens : 16,
                      prep ? prep->zero_words : (int32_t*)nullptr, prep ? prep->n_zero : 0,
                      prep ? prep->status : (int32_t*)nullptr);
}

}  // namespace moe
