// tcgen05 grouped GEMMs of the MoE layer for many tokens per expert.
//
// The layer ("1 卡跑通 Llama 4" (discosf.com), "混合专家路由"; "Llama 开源模型
// 系列" (docs.ifdog.com), "SwiGLU：门控激活的数学"): each expert runs
// (silu(x Wg^T) * (x Wu^T)) Wd^T on its tokens; routed weights are int4 with
// one fp32 scale per group of 128 K (or the smaller 64 / 32) and zero point 0
// ("Meta Llama Models Llama 4 单卡量化推理与选型指南" (lshu.cn), "量化环节做了
// 什么"), or e4m3 rows; the shared expert is bf16.
//
// One persistent CTA per SM, tiles of 128 output features x 256 tokens:
//   A = weights (M = 128 rows), B = tokens (N = 256 rows), both K-major in
//   shared memory with the 128-byte swizzle, K step 64; D = fp32 in tensor
//   memory (TMEM), two 256-column accumulators so a tile's epilogue overlaps
//   the next tile's MMAs.
// Warp roles (16 warps):
//   warp 0      TMA producer of the token tiles (one thread) and TMEM
//               allocator
//   warp 1      MMA issuer (one thread): tcgen05.mma kind::f16 (bf16) or
//               kind::f8f6f4 (e4m3)
//   warp 2      TMA producer of the weights: int4 codes (for the
//               converters), or bf16 / e4m3 weight tiles, each through a
//               ring of its own that runs ahead of the token ring
//   warps 4-7   epilogue: tcgen05.ld of the accumulator (warp w reads TMEM
//               lanes 32 (w % 4) ..), SwiGLU / gate scaling / combine, stores
//   warps 8-15  int4 modes only: dequantize the stage's codes (w = q * s, s
//               rounded to bf16) into the swizzled A tile; two threads per
//               row, each taking 32 of the stage's 64 K
// Gate/up tiles hold 64 features: A rows alternate 16 gate rows and the same
// 16 up rows, so each epilogue warp finds g (lanes 0..15) and u (lanes 16..31)
// of its 16 features together.  Routed activations are stored with every 8
// consecutive K values in the order x0 x4 x1 x5 x2 x6 x3 x7, the order the
// int4 unpacking produces; the dot products do not depend on the K order.
#include <cuda.h>

#include <cuda_fp8.h>

#include "tc_gemm.cuh"
#include "tcgen05.cuh"

namespace moe {

// Four warpgroups: 0 -- TMA producer (warp 0), MMA issuer (warp 1); 1 --
// epilogue; 2 and 3 -- int4 converters (idle in the bf16 / e4m3 modes).
// Registers: 128 x 64 + 128 x 192 + 256 x 96 <= 512 x 128 (setmaxnreg).
constexpr int TC_THREADS = 512;
constexpr int TC_CTRL_REGS = 64, TC_EPI_REGS = 192, TC_CONV_REGS = 96;
static_assert(128 * TC_CTRL_REGS + 128 * TC_EPI_REGS + 256 * TC_CONV_REGS <= TC_THREADS * 128, "register split");
constexpr int TC_STAGES = 4;
constexpr int TC_B_BYTES = TC_BLOCK_TOKENS * 64 * 2;   // 32 KB
constexpr int TC_A_BYTES = 128 * 64 * 2;               // 16 KB
constexpr int TC_C_BYTES = 128 * 32;                   // int4 codes of the A tile: 4 KB
constexpr int TC_STAGE_BYTES = TC_B_BYTES + TC_A_BYTES;
// The int4 codes have a ring of their own, twice as deep as the stages: they
// are loaded (by warp 2) well ahead, so the converters can fill a stage's A
// tile as soon as its previous MMAs complete, while its token tile is still
// in flight.
constexpr int TC_CSTAGES = 2 * TC_STAGES;
constexpr int TC_TMEM_COLS = 512;
static_assert(TC_STAGE_BYTES % 1024 == 0, "stage alignment");
// bf16 / e4m3 modes: the weight tiles (the routed ones read once from DRAM)
// have a ring of their own, filled by warp 2 up to TC_WSTAGES stages ahead of
// the MMAs, in the space of the stages' weight halves and the (unused) code
// ring; the token tiles keep TC_STAGES slots.  Against one ring of four
// token + weight stages the Maverick-shaped e4m3 GEMMs ran 4 % faster and the
// bf16 ones 2-4 %; three token slots and eight weight slots were slower.
constexpr int TC_WSTAGES = 6;
static_assert(TC_STAGES * TC_B_BYTES + TC_WSTAGES * TC_A_BYTES == TC_STAGES * TC_STAGE_BYTES + TC_CSTAGES * TC_C_BYTES,
              "e4m3 rings");

struct TcSmem {
    uint64_t full[TC_STAGES];      // TMA data of the stage landed (tx counted)
    uint64_t a_ready[TC_STAGES];   // converter warps wrote the A tile
    uint64_t empty[TC_STAGES];     // the stage's MMAs completed
    uint64_t cfull[TC_CSTAGES];    // int4 codes of a code slot landed
    uint64_t cempty[TC_CSTAGES];   // converter warps read the code slot
    uint64_t a_full[TC_WSTAGES];    // bf16 / e4m3: the weight slot landed (tx counted)
    uint64_t a_empty[TC_WSTAGES];   // bf16 / e4m3: the MMAs reading the weight slot completed
    uint64_t acc_full[2];          // accumulator holds a finished tile
    uint64_t acc_empty[2];         // epilogue finished reading the accumulator
    uint32_t tmem_base;
};

// Instruction descriptor: bf16 inputs (kind::f16) or e4m3 inputs (kind::f8f6f4).
__host__ __device__ constexpr uint32_t tc_idesc(int M, int N, bool fp8) { return tc_idesc_fmt(M, N, fp8 ? 0u : 1u); }

__device__ __forceinline__ int frag_pos(int i) { return i < 4 ? 2 * i : 2 * (i - 4) + 1; }

// Tile order: feature blocks in groups of 16; within a group, chunk by chunk.
// A wave of ~148 concurrent tiles then touches ~9 token chunks and 16 weight
// blocks, which stay in L2, instead of every weight block of one chunk.
constexpr int TC_FB_GROUP = 16;
__device__ __forceinline__ void tile_coords(int tile, int n_chunks, int n_fblocks, int& chunk, int& fb) {
    const int gf = min(TC_FB_GROUP, n_fblocks);
    const int n_groups = (n_fblocks + gf - 1) / gf;
    const int g = min(tile / (n_chunks * gf), n_groups - 1);
    const int r = tile - g * n_chunks * gf;
    const int gsize = min(gf, n_fblocks - g * gf);
    chunk = r / gsize;
    fb = g * gf + r % gsize;
}

// N of the MMA for a chunk of `count` tokens: whole multiples of 16 columns.
__device__ __forceinline__ int tile_n(int count) { return min(TC_BLOCK_TOKENS, (count + 15) & ~15); }

// ---------------------------------------------------------------------------
template <int MODE>
__global__ void __launch_bounds__(TC_THREADS, 1) tc_gemm_kernel(
    const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_bs,
    const __grid_constant__ CUtensorMap tm_a0,
    const __grid_constant__ CUtensorMap tm_a1, TcParams p) {
    constexpr bool INT4 = MODE == TC_GATEUP_INT4 || MODE == TC_DOWN_INT4;
    constexpr bool FP8 = MODE == TC_GATEUP_FP8 || MODE == TC_DOWN_FP8;
    constexpr bool GATEUP = MODE == TC_GATEUP_INT4 || MODE == TC_GATEUP_BF16 || MODE == TC_GATEUP_FP8;
    constexpr int KSTEP = FP8 ? 128 : 64;     // K values per 128-byte row of a stage
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* base = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char* cring = base + TC_STAGES * TC_STAGE_BYTES;   // int4 code ring
    TcSmem* sm = reinterpret_cast<TcSmem*>(cring + TC_CSTAGES * TC_C_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < TC_STAGES; ++i) {
            mbar_init(&sm->full[i], 1);
            mbar_init(&sm->a_ready[i], 8);   // the 8 converter warps
            mbar_init(&sm->empty[i], 1);
        }
        for (int i = 0; i < TC_CSTAGES; ++i) { mbar_init(&sm->cfull[i], 1); mbar_init(&sm->cempty[i], 8); }
        for (int i = 0; i < TC_WSTAGES; ++i) { mbar_init(&sm->a_full[i], 1); mbar_init(&sm->a_empty[i], 1); }
        for (int i = 0; i < 2; ++i) { mbar_init(&sm->acc_full[i], 1); mbar_init(&sm->acc_empty[i], 4); }
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&sm->tmem_base, TC_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm->tmem_base;


    const int n_all = p.n_chunks[0], n_sh = p.n_chunks[1];
    const int c_begin = p.routed ? n_sh : 0, c_end = p.routed ? n_all : n_sh;
    const int n_tiles = (c_end - c_begin) * p.n_fblocks;
    const int nk = p.K / KSTEP;
    // token slot pitch, and the e4m3 weight ring after the token slots
    constexpr bool SEPA = !INT4;              // weights through their own ring (warp 2)
    constexpr int B_PITCH = SEPA ? TC_B_BYTES : TC_STAGE_BYTES;
    unsigned char* fring = base + TC_STAGES * TC_B_BYTES;

    if (warp < 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" :: "n"(TC_CTRL_REGS));
    if (warp == 0) {
        // ------------------------- TMA producer of the token tiles -------------------------
        // (int4 codes and the bf16 / e4m3 weights come through their own rings, warp 2)
        if (lane == 0) {
            prefetch_tmap(&tm_b); prefetch_tmap(&tm_bs); prefetch_tmap(&tm_a0); prefetch_tmap(&tm_a1);
            uint32_t it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
                int ci, fb;
                tile_coords(tile, c_end - c_begin, p.n_fblocks, ci, fb);
                const ChunkEntry ce = p.chunks[c_begin + ci];
                // a chunk of a few tokens (an expert's tail) loads a box of only
                // TC_SMALL_TOKENS rows: with the full box it moved as many bytes
                // per stage as a full tile for a sliver of its MMA work
                const bool small = tile_n(ce.count) <= TC_SMALL_TOKENS;
                const CUtensorMap* mb = small ? &tm_bs : &tm_b;
                const uint32_t bbytes = small ? uint32_t(TC_SMALL_TOKENS * 128) : uint32_t(TC_B_BYTES);
                for (int kk = 0; kk < nk; ++kk, ++it) {
                    const uint32_t slot = it % TC_STAGES;
                    if (!mbar_wait(&sm->empty[slot], ((it / TC_STAGES) & 1) ^ 1, p.status)) { ok = false; break; }
                    mbar_arrive_expect_tx(&sm->full[slot], bbytes);
                    tma_load_2d(base + slot * B_PITCH, mb, &sm->full[slot], kk * KSTEP, ce.start);
                }
            }
            // wind down: wait (bounded) for the stages still in flight to land
            for (uint32_t i = 0; i < TC_STAGES && i < it; ++i) {
                const uint32_t j = it - 1 - i;
                mbar_wait(&sm->full[j % TC_STAGES], (j / TC_STAGES) & 1, nullptr);
            }
        }
    } else if (warp == 2 && SEPA) {
        // ------------------------------ bf16 / e4m3 weight producer ------------------------------
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
                int ci, fb;
                tile_coords(tile, c_end - c_begin, p.n_fblocks, ci, fb);
                const ChunkEntry ce = p.chunks[c_begin + ci];
                const int e = ce.expert < 0 ? 0 : ce.expert;
                for (int kk = 0; kk < nk; ++kk, ++it) {
                    const uint32_t as = it % TC_WSTAGES;
                    if (!mbar_wait(&sm->a_empty[as], ((it / TC_WSTAGES) & 1) ^ 1, p.status)) { ok = false; break; }
                    unsigned char* sa = fring + as * TC_A_BYTES;
                    mbar_arrive_expect_tx(&sm->a_full[as], TC_A_BYTES);
                    // 16-row boxes; gate/up: gate rows, up rows, gate rows, ... (same features)
#pragma unroll
                    for (int b = 0; b < 8; ++b) {
                        // the shared expert's matrices hold one expert (no row offset)
                        const int r0 = FP8 ? e * p.n_rows : 0;
                        if (GATEUP)
                            tma_load_2d(sa + b * 2048, (b & 1) ? &tm_a1 : &tm_a0, &sm->a_full[as], kk * KSTEP,
                                        r0 + fb * 64 + (b >> 1) * 16);
                        else
                            tma_load_2d(sa + b * 2048, &tm_a0, &sm->a_full[as], kk * KSTEP,
                                        r0 + fb * 128 + b * 16);
                    }
                }
            }
            // wind down: wait (bounded) for the weight loads still in flight to land
            for (uint32_t i = 0; i < TC_WSTAGES && i < it; ++i) {
                const uint32_t j = it - 1 - i;
                mbar_wait(&sm->a_full[j % TC_WSTAGES], (j / TC_WSTAGES) & 1, nullptr);
            }
        }
    } else if (warp == 2 && INT4) {
        // ------------------------------ int4 code producer ------------------------------
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
                int ci, fb;
                tile_coords(tile, c_end - c_begin, p.n_fblocks, ci, fb);
                const ChunkEntry ce = p.chunks[c_begin + ci];
                const int e = ce.expert < 0 ? 0 : ce.expert;
                const int row = e * p.n_rows + fb * (GATEUP ? 64 : 128);
                for (int kk = 0; kk < nk; ++kk, ++it) {
                    const uint32_t cs = it % TC_CSTAGES;
                    if (!mbar_wait(&sm->cempty[cs], ((it / TC_CSTAGES) & 1) ^ 1, p.status)) { ok = false; break; }
                    unsigned char* sc = cring + cs * TC_C_BYTES;
                    mbar_arrive_expect_tx(&sm->cfull[cs], TC_C_BYTES);
                    if (GATEUP) {   // gate rows, then the same features' up rows
                        tma_load_2d(sc, &tm_a0, &sm->cfull[cs], kk * 32, row);
                        tma_load_2d(sc + 64 * 32, &tm_a1, &sm->cfull[cs], kk * 32, row);
                    } else {
                        tma_load_2d(sc, &tm_a0, &sm->cfull[cs], kk * 32, row);
                        tma_load_2d(sc + 64 * 32, &tm_a0, &sm->cfull[cs], kk * 32, row + 64);
                    }
                }
            }
            // wind down: wait (bounded) for the code loads still in flight to land
            for (uint32_t i = 0; i < TC_CSTAGES && i < it; ++i) {
                const uint32_t j = it - 1 - i;
                mbar_wait(&sm->cfull[j % TC_CSTAGES], (j / TC_CSTAGES) & 1, nullptr);
            }
        }
    } else if (warp == 1) {
        // ------------------------------ MMA issuer ------------------------------
        if (lane == 0) {
            uint32_t it = 0, n = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++n) {
                int ci, fb;
                tile_coords(tile, c_end - c_begin, p.n_fblocks, ci, fb);
                // a partial chunk multiplies only its tokens' columns (rounded up to 16)
                const uint32_t idesc = tc_idesc(128, tile_n(p.chunks[c_begin + ci].count), FP8);
                const uint32_t acc = n & 1;
                if (!mbar_wait(&sm->acc_empty[acc], ((n >> 1) & 1) ^ 1, p.status)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem + acc * 256;
                for (int kk = 0; kk < nk; ++kk, ++it) {
                    const uint32_t slot = it % TC_STAGES;
                    const uint32_t par = (it / TC_STAGES) & 1;
                    const uint32_t as = it % TC_WSTAGES;
                    if (!mbar_wait(&sm->full[slot], par, p.status)) { ok = false; break; }
                    if (INT4 && !mbar_wait(&sm->a_ready[slot], par, p.status)) { ok = false; break; }
                    if (SEPA && !mbar_wait(&sm->a_full[as], (it / TC_WSTAGES) & 1, p.status)) { ok = false; break; }
                    tc_fence_after();
                    const unsigned char* st = base + slot * B_PITCH;
                    const uint64_t bd = sw128_desc(st);
                    const uint64_t ad = sw128_desc(SEPA ? fring + as * TC_A_BYTES : st + TC_B_BYTES);
#pragma unroll
                    for (int k16 = 0; k16 < 4; ++k16)   // +32 bytes (16 bf16 / 32 e4m3 K) per MMA inside the swizzle atom
                        umma<FP8>(d_tmem, ad + 2 * k16, bd + 2 * k16, idesc, (kk | k16) != 0);
                    umma_commit(&sm->empty[slot]);
                    if (SEPA) umma_commit(&sm->a_empty[as]);
                }
                if (ok) umma_commit(&sm->acc_full[acc]);
            }
            // wind down: wait (bounded) for the last MMAs
            if (it > 0) mbar_wait(&sm->empty[(it - 1) % TC_STAGES], ((it - 1) / TC_STAGES) & 1, nullptr);
        }
    }
    } else if (warp < 8) {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" :: "n"(TC_EPI_REGS));
        // ------------------------------ epilogue ------------------------------
        const int ew = warp & 3;                 // TMEM lanes 32 ew .. 32 ew + 31
        uint32_t n = 0;
        for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++n) {
            int ci, fb;
            tile_coords(tile, c_end - c_begin, p.n_fblocks, ci, fb);
            const ChunkEntry ce = p.chunks[c_begin + ci];
            const uint32_t acc = n & 1;
            if (!mbar_wait(&sm->acc_full[acc], (n >> 1) & 1, p.status)) break;
            tc_fence_after();
            const uint32_t taddr = tmem + (uint32_t(32 * ew) << 16) + acc * 256;
            for (int cc = 0; cc < TC_BLOCK_TOKENS / 32; ++cc) {
                if (cc * 32 >= ce.count) break;        // warp-uniform
                uint32_t v[32];
                tmem_ld32(taddr + cc * 32, v);
                const int col0 = cc * 32;
                if (GATEUP) {
                    // lanes 0..15: gate of features f + 0..15; lanes 16..31: up of the same
                    const int f = fb * 64 + ew * 16 + (lane & 15);
                    const int fpos = MODE == TC_GATEUP_INT4 ? (f & ~7) + frag_pos(f & 7) : f;
                    // e4m3: scale of this lane's weight row, and of each column's token row
                    float wrow = 1.0f, tcol = 1.0f;
                    if (FP8) {
                        wrow = (lane < 16 ? p.s0 : p.s1)[int64_t(ce.expert) * p.n_rows + f];
                        tcol = col0 + lane < ce.count ? p.tok_scale[ce.start + col0 + lane] : 0.0f;
                    }
                    // columns in pairs: lanes 0..15 finish the even column (own
                    // gate, partner's up), lanes 16..31 the odd one (partner's
                    // gate, own up) -- one exchange per pair, every lane busy
#pragma unroll
                    for (int jp = 0; jp < 16; ++jp) {
                        float a = __uint_as_float(v[2 * jp]), b = __uint_as_float(v[2 * jp + 1]);
                        if (FP8) {
                            a *= wrow * __shfl_sync(0xffffffffu, tcol, 2 * jp);
                            b *= wrow * __shfl_sync(0xffffffffu, tcol, 2 * jp + 1);
                        }
                        const float recv = __shfl_xor_sync(0xffffffffu, lane < 16 ? b : a, 16);
                        const float g = lane < 16 ? a : recv;
                        const float u = lane < 16 ? recv : b;
                        const int col = col0 + 2 * jp + (lane >> 4);
                        if (col < ce.count)
                            p.h_out[int64_t(ce.start + col) * p.n_rows + fpos] = __float2bfloat16_rn(silu_fast(g) * u);
                    }
                } else if (MODE == TC_DOWN_INT4 || MODE == TC_DOWN_FP8) {
                    const int d = fb * 128 + ew * 32 + lane;
                    const int my_col = col0 + lane;
                    const int my_slot = my_col < ce.count ? p.perm[ce.start + my_col] : 0;
                    float my_gate = my_col < ce.count ? p.gates[my_slot] : 0.0f;
                    float wrow = 1.0f;
                    if (FP8) {   // e4m3: token-row scale folded into the gate, weight-row scale per lane
                        if (my_col < ce.count) my_gate *= p.tok_scale[ce.start + my_col];
                        wrow = p.s0[int64_t(ce.expert) * p.n_rows + d];
                    }
                    if (p.out != nullptr) {
                        // one slot per token: finish the token here,
                        // out[t] = bf16(shared expert + gate * y), t = slot
                        float ys[32];
#pragma unroll
                        for (int j = 0; j < 32; ++j) {   // all loads first, one latency per 32 columns
                            const int slot = __shfl_sync(0xffffffffu, my_slot, j);
                            ys[j] = col0 + j < ce.count ? p.y_r[int64_t(slot) * p.n_rows + d] : 0.0f;
                        }
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const float gt = __shfl_sync(0xffffffffu, my_gate, j) * wrow;
                            const int slot = __shfl_sync(0xffffffffu, my_slot, j);
                            if (col0 + j < ce.count)
                                p.out[int64_t(slot) * p.n_rows + d] = __float2bfloat16_rn(fmaf(__uint_as_float(v[j]), gt, ys[j]));
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            // y is stored by slot (t k + j), so the combine reads it without indirection
                            const float gt = __shfl_sync(0xffffffffu, my_gate, j) * wrow;
                            const int slot = __shfl_sync(0xffffffffu, my_slot, j);
                            if (col0 + j < ce.count) p.y_out[int64_t(slot) * p.n_rows + d] = __uint_as_float(v[j]) * gt;
                        }
                    }
                } else {
                    // shared expert's down projection: fp32 y_s[t] (read by the routed down
                    // projection or the combine)
                    const int d = fb * 128 + ew * 32 + lane;
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int col = col0 + j;
                        if (col < ce.count) p.y_out[int64_t(ce.start + col) * p.n_rows + d] = __uint_as_float(v[j]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm->acc_empty[acc]);
        }
    } else {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" :: "n"(TC_CONV_REGS));
    if (INT4) {
        // ------------------------------ int4 -> bf16 converters ------------------------------
        // thread: A row i, half hh of the stage's 64 K (4 of its 8 code words);
        // a warp reads 16 consecutive code rows, 512 contiguous bytes
        const int i = (threadIdx.x - 256) >> 1, hh = threadIdx.x & 1;
        int code_row, srow_off;
        const float* sbase;
        if (MODE == TC_GATEUP_INT4) {
            const int blk = i >> 4, local = i & 15;
            code_row = (blk & 1) ? 64 + (blk >> 1) * 16 + local : (blk >> 1) * 16 + local;
            srow_off = (blk >> 1) * 16 + local;
            sbase = (blk & 1) ? p.s1 : p.s0;
        } else {
            code_row = i;
            srow_off = i;
            sbase = p.s0;
        }
        // groups of 128, 64 or 32 K: this thread's 32 K of stage kk lie in
        // group (64 kk + 32 hh) >> gsh, a new one every spg stages; a
        // group's scale is loaded two groups ahead
        const int gsh = p.group_shift;
        const int spg = gsh == 7 ? 2 : 1;
        const int ng = p.K >> gsh;
        const __nv_bfloat162 k136 = __floats2bfloat162_rn(136.0f, 136.0f);
        const uint32_t magic = p.bf16_magic;
        uint32_t it = 0;
        for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
            int ci, fb;
            tile_coords(tile, c_end - c_begin, p.n_fblocks, ci, fb);
            const ChunkEntry ce = p.chunks[c_begin + ci];
            const float* srow = sbase + int64_t(ce.expert * p.n_rows + fb * (GATEUP ? 64 : 128) + srow_off) * ng;
            auto scale_of = [&](int kq) { return ldg_f32(srow + ((64 * kq + 32 * hh) >> gsh)); };
            float s_a = scale_of(0), s_b = spg < nk ? scale_of(spg) : 0.0f;
            __nv_bfloat162 s2 = __floats2bfloat162_rn(0.f, 0.f);
            bool ok = true;
            for (int kk = 0; kk < nk; ++kk, ++it) {
                if ((kk & (spg - 1)) == 0) {                  // this thread enters a new group
                    s2 = __floats2bfloat162_rn(s_a, s_a);
                    s_a = s_b;
                    if (kk + 2 * spg < nk) s_b = scale_of(kk + 2 * spg);
                }
                const uint32_t slot = it % TC_STAGES, cs = it % TC_CSTAGES;
                if (!mbar_wait(&sm->cfull[cs], (it / TC_CSTAGES) & 1, p.status)) { ok = false; break; }
                const unsigned char* sc = cring + cs * TC_C_BYTES;
                const uint4 c0 = *reinterpret_cast<const uint4*>(sc + code_row * 32 + hh * 16);
                // the A tile is free once the slot's previous MMAs completed
                if (!mbar_wait(&sm->empty[slot], ((it / TC_STAGES) & 1) ^ 1, p.status)) { ok = false; break; }
                unsigned char* sa = base + slot * TC_STAGE_BYTES + TC_B_BYTES;
                const uint32_t w[4] = {c0.x, c0.y, c0.z, c0.w};
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const int j = 4 * hh + jj;   // 16-byte chunk of the A row (8 K values)
                    // 8 codes k0..k7 -> (k0,k4) (k1,k5) (k2,k6) (k3,k7), each (q * s) in bf16
                    uint32_t o[4];
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        uint32_t t = bf16_lo_nibbles(w[jj] >> (4 * h), magic);   // bf16 136 + q
                        __nv_bfloat162 q = __hsub2(*reinterpret_cast<__nv_bfloat162*>(&t), k136);
                        __nv_bfloat162 r = __hmul2(q, s2);
                        o[h] = *reinterpret_cast<uint32_t*>(&r);
                    }
                    *reinterpret_cast<uint4*>(sa + i * 128 + ((j ^ (i & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
                }
                fence_proxy_async_smem();
                __syncwarp();
                // the code slot is released only after its codes have been used
                // (released right after the load, it was sometimes refilled
                // before the load had read it)
                if (lane == 0) {
                    mbar_arrive(&sm->a_ready[slot]);
                    mbar_arrive(&sm->cempty[cs]);
                }
            }
            if (!ok) break;
        }
    }

    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TC_TMEM_COLS);
    }
}

// x_sorted[p] = x[perm[p] / k], every 8 values reordered x0 x4 x1 x5 x2 x6 x3 x7
__global__ void gather_rows_kernel(const bf16* __restrict__ x, const int32_t* __restrict__ perm, int64_t n,
                                   int k, int D, bf16* __restrict__ out) {
    const int chunks = D / 8;
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n * chunks;
         i += int64_t(gridDim.x) * blockDim.x) {
        const int64_t r = i / chunks;
        const int c = int(i % chunks);
        const uint4 v = *reinterpret_cast<const uint4*>(x + int64_t(perm[r] / k) * D + 8 * c);
        uint4 o;
        o.x = prmt(v.x, v.z, 0x5410); o.y = prmt(v.x, v.z, 0x7632);
        o.z = prmt(v.y, v.w, 0x5410); o.w = prmt(v.y, v.w, 0x7632);
        *reinterpret_cast<uint4*>(out + r * D + 8 * c) = o;
    }
}

// Per-row e4m3 quantization of bf16 x (the same rule as moe_quantize_fp8_rows),
// each token's codes and scale written to the positions of its k slots.
__global__ void __launch_bounds__(256) quantize_fp8_scatter_kernel(const bf16* __restrict__ x, int cols,
                                                                   float scale_ub, const int32_t* __restrict__ inv,
                                                                   int k, uint8_t* __restrict__ q,
                                                                   float* __restrict__ scales) {
    __shared__ float red[8];
    const int64_t t = blockIdx.x;
    const bf16* row = x + t * cols;
    float m = 0.0f;
    for (int c = threadIdx.x * 8; c < cols; c += 256 * 8) {
        const uint4 v = *reinterpret_cast<const uint4*>(row + c);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) m = fmaxf(m, fmaxf(fabsf(bf16_lo(w[i])), fabsf(bf16_hi(w[i]))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    m = red[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) m = fmaxf(m, red[i]);
    const float s = __fdiv_rn(fmaxf(fminf(m, scale_ub), 1e-12f), 448.0f);
    for (int c = threadIdx.x * 8; c < cols; c += 256 * 8) {
        const uint4 v = *reinterpret_cast<const uint4*>(row + c);
        const float f[8] = {__fdiv_rn(bf16_lo(v.x), s), __fdiv_rn(bf16_hi(v.x), s), __fdiv_rn(bf16_lo(v.y), s),
                            __fdiv_rn(bf16_hi(v.y), s), __fdiv_rn(bf16_lo(v.z), s), __fdiv_rn(bf16_hi(v.z), s),
                            __fdiv_rn(bf16_lo(v.w), s), __fdiv_rn(bf16_hi(v.w), s)};
        uint32_t o[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            uint32_t word = 0;
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                __nv_fp8x2_storage_t b = __nv_cvt_float2_to_fp8x2(make_float2(f[4 * h + 2 * i], f[4 * h + 2 * i + 1]),
                                                                  __NV_SATFINITE, __NV_E4M3);
                word |= uint32_t(b) << (16 * i);
            }
            o[h] = word;
        }
        for (int j = 0; j < k; ++j) {
            const int64_t pos = inv[t * k + j];
            *reinterpret_cast<uint2*>(q + pos * cols + c) = make_uint2(o[0], o[1]);
        }
    }
    if (threadIdx.x < k) scales[inv[t * k + threadIdx.x]] = s;
}

moe_status launch_quantize_fp8_scatter(const bf16* x, int64_t rows, int cols, float scale_ub,
                                       const int32_t* inv_perm, int k, uint8_t* q, float* scales,
                                       cudaStream_t stream) {
    if (rows == 0) return MOE_OK;
    quantize_fp8_scatter_kernel<<<unsigned(rows), 256, 0, stream>>>(x, cols, scale_ub, inv_perm, k, q, scales);
    return launch_status();
}

// out[t] = bf16(y_s[t] + sum_j y[t k + j])  (routed outputs stored by slot)
__global__ void combine_slots_kernel(const float* __restrict__ y_s, const float* __restrict__ y, int64_t T, int D,
                                     int k, bf16* __restrict__ out) {
    const int64_t n4 = T * D / 4;
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n4; i += int64_t(gridDim.x) * blockDim.x) {
        const int64_t t = i / (D / 4);
        const int d = int(i % (D / 4)) * 4;
        float4 a = *reinterpret_cast<const float4*>(y_s + t * D + d);
        for (int j = 0; j < k; ++j) {
            const float4 b = *reinterpret_cast<const float4*>(y + (t * k + j) * D + d);
            a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
        }
        uint2 o;
        o.x = pack_bf16x2(a.x, a.y);
        o.y = pack_bf16x2(a.z, a.w);
        *reinterpret_cast<uint2*>(out + t * D + d) = o;
    }
}

moe_status launch_combine_slots(const float* y_s, const float* y, int64_t T, int D, int k, bf16* out,
                                cudaStream_t stream) {
    int64_t blocks = ceil_div(T * D / 4, 256);
    if (blocks > 148 * 16) blocks = 148 * 16;
    combine_slots_kernel<<<unsigned(blocks), 256, 0, stream>>>(y_s, y, T, D, k, out);
    return launch_status();
}

// This file's copy of the wait limit (see c_wait_limit).
moe_status set_wait_limit_tc(uint32_t cycles) {
    return cuda_status(cudaMemcpyToSymbol(c_wait_limit, &cycles, sizeof(cycles)));
}

size_t tc_smem_bytes() {
    return 1024 + size_t(TC_STAGES) * TC_STAGE_BYTES + size_t(TC_CSTAGES) * TC_C_BYTES + sizeof(TcSmem);
}

moe_status launch_tc_gemm(int mode, const TcMaps& maps, const TcParams& prm, cudaStream_t stream) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const size_t smem = tc_smem_bytes();
#define TC_LAUNCH(M)                                                                                     \
    do {                                                                                                 \
        if (allow_max_smem(tc_gemm_kernel<M>) != MOE_OK) return MOE_ERR_CUDA;                         \
        tc_gemm_kernel<M><<<sms, TC_THREADS, smem, stream>>>(maps.b, maps.b_small, maps.a0, maps.a1, prm); \
    } while (0)
    switch (mode) {
        case TC_GATEUP_INT4: TC_LAUNCH(TC_GATEUP_INT4); break;
        case TC_DOWN_INT4: TC_LAUNCH(TC_DOWN_INT4); break;
        case TC_GATEUP_BF16: TC_LAUNCH(TC_GATEUP_BF16); break;
        case TC_GATEUP_FP8: TC_LAUNCH(TC_GATEUP_FP8); break;
        case TC_DOWN_FP8: TC_LAUNCH(TC_DOWN_FP8); break;
        default: TC_LAUNCH(TC_DOWN_BF16); break;
    }
#undef TC_LAUNCH
    return launch_status();
}

moe_status launch_gather_rows(const bf16* x, const int32_t* perm, int64_t n, int k, int D, bf16* out,
                              cudaStream_t stream) {
    if (n == 0) return MOE_OK;
    int64_t blocks = ceil_div(n * (D / 8), 256);
    if (blocks > 148 * 32) blocks = 148 * 32;
    gather_rows_kernel<<<unsigned(blocks), 256, 0, stream>>>(x, perm, n, k, D, out);
    return launch_status();
}

}  // namespace moe
