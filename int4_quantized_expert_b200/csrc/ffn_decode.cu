// Weight-streaming expert FFN for few tokens per expert (decode).
//
// The layer ("1 卡跑通 Llama 4" (discosf.com), "混合专家路由"; "Llama 开源模型
// 系列" (docs.ifdog.com), "SwiGLU：门控激活的数学"):
//   expert_e(x) = (silu(x Wg^T) * (x Wu^T)) Wd^T, and the same with the bf16
//   shared expert, combined as out = bf16(shared(x) + sum_j gate_j expert_j(x)).
// Routed weights are int4 with one fp32 scale per 128 K values and zero point 0
// ("Meta Llama Models Llama 4 单卡量化推理与选型指南" (lshu.cn), "量化环节做了什么").
//
// With a handful of tokens per expert every weight byte is used by only a few
// multiply-adds, so the kernels are bound by HBM bandwidth.  Design:
//   * one persistent CTA per SM; a producer warp takes tasks (32 output rows of
//     one matrix pair x one chunk of <= 16 tokens) from a global counter, shared
//     expert first, and streams the task's weights with 2-D TMA loads
//     (32 rows x 128 bytes, 128-byte swizzle) through a ring of 8 KB stages;
//     the task's int4 scales arrive with one 1-D bulk copy.
//   * 8 consumer warps: 2 row blocks of 16 rows x 4 K phases (stage s goes to
//     phase s % 4).  Each converts int4 codes to exact bf16 integers in
//     registers (no scale multiply per element), runs m16n8k16 tensor-core
//     MMAs against the tokens (fp32 accumulate), and applies the group's scale
//     to the 128-K partial sum.  The 4 K phases are summed through shared
//     memory, then the epilogue applies SwiGLU (gate/up pass) or the gate
//     (down pass).
//   * Tokens are the MMA's N operand (8 per n-tile).  Their rows are read with
//     L1-cached global loads in a layout where every 8 values are stored
//     x0 x4 x1 x5 x2 x6 x3 x7, which is the order the int4 unpacking yields.
#include <cuda.h>

#include "common.cuh"
#include "ffn_decode.cuh"

namespace moe {

constexpr int DC_ROWS = 32;                 // output rows per task
constexpr int DC_KPH = 4;                   // K phases
constexpr int DC_CONSUMERS = 8;             // 2 row blocks x 4 K phases
constexpr int DC_THREADS = (DC_CONSUMERS + 1) * 32;
constexpr int DC_CHUNK = DC_ROWS * 128;     // one matrix tile of a stage: 32 rows x 128 B
constexpr int DC_STAGE = 2 * DC_CHUNK;      // 8 KB
constexpr int DC_NSTAGES = 16;              // ring: 128 KB in flight
constexpr int DC_NT = 2;                    // n-tiles of 8 tokens per task
constexpr int DC_RED_FLOATS = 6 * 32 * DC_NT * 8;   // partial sums of K phases 1..3

struct TaskInfo {
    int32_t kind;       // 0 = shared (bf16), 1 = routed (int4), -1 = done
    int32_t expert;
    int32_t row0;       // first output row (within the expert / shared matrix)
    int32_t start;      // first token row (shared) or sorted slot position (routed)
    int32_t count;      // tokens in this chunk (1..16)
    int32_t n_stages;
    int32_t K;
    int32_t pad;
};

struct DecodeSmem {
    uint64_t full[DC_NSTAGES];
    uint64_t empty[DC_NSTAGES];
    uint64_t sfull[2];
    uint64_t sempty[2];
    uint64_t red_full;    // K phases 1..3 -> phase 0: partial sums written
    uint64_t red_empty;   // phase 0 -> phases 1..3: partial sums consumed
    TaskInfo task[2];
};

__device__ __forceinline__ int sigma8(int g) { return ((g & 1) << 2) | (g >> 1); }

__device__ __forceinline__ uint4 lds128(const unsigned char* p) {
    return *reinterpret_cast<const uint4*>(p);
}

// Address of logical 16-byte chunk j of row r in a 128-byte-swizzled tile.
__device__ __forceinline__ const unsigned char* swz(const unsigned char* tile, int r, int j) {
    return tile + r * 128 + ((j ^ (r & 7)) << 4);
}

// position of element i (0..7) of an 8-block in the x0 x4 x1 x5 x2 x6 x3 x7 layout
__device__ __forceinline__ int frag_pos8(int i) { return i < 4 ? 2 * i : 2 * (i - 4) + 1; }

template <int MODE>   // 0 = gate/up with SwiGLU, 1 = down
__global__ void __launch_bounds__(DC_THREADS, 1) decode_ffn_kernel(
    const __grid_constant__ CUtensorMap tm_r0, const __grid_constant__ CUtensorMap tm_r1,
    const __grid_constant__ CUtensorMap tm_s0, const __grid_constant__ CUtensorMap tm_s1,
    DecodeParams p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // 1024-byte alignment of the ring is required by the 128-byte swizzle
    unsigned char* base = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char* ring = base;
    float* sbuf = reinterpret_cast<float*>(ring + DC_NSTAGES * DC_STAGE);      // 2 scale buffers
    float* red = sbuf + 2 * p.scale_buf_floats;
    DecodeSmem* sm = reinterpret_cast<DecodeSmem*>(red + DC_RED_FLOATS);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < DC_NSTAGES; ++i) { mbar_init(&sm->full[i], 1); mbar_init(&sm->empty[i], 2); }
        for (int i = 0; i < 2; ++i) { mbar_init(&sm->sfull[i], 1); mbar_init(&sm->sempty[i], DC_CONSUMERS); }
        mbar_init(&sm->red_full, (DC_KPH - 1) * 2);
        mbar_init(&sm->red_empty, 2);
        fence_barrier_init();
    }
    __syncthreads();

    const int nbs = p.n_rows_s / DC_ROWS, nbr = p.n_rows_r / DC_ROWS;
    const int n_chunks = *p.n_chunks, n_sh = *p.n_shared_chunks;
    const int n_tasks = n_sh * nbs + (n_chunks - n_sh) * nbr;

    if (warp == DC_CONSUMERS) {
        // ------------------------------ producer ------------------------------
        if (lane == 0) {
            prefetch_tmap(&tm_r0); prefetch_tmap(&tm_r1); prefetch_tmap(&tm_s0); prefetch_tmap(&tm_s1);
            uint32_t it = 0;
            bool ok = true;
            for (uint32_t tn = 0; ok; ++tn) {
                const int t = atomicAdd(p.task_counter, 1);
                const int b = tn & 1;
                if (!mbar_wait(&sm->sempty[b], ((tn >> 1) & 1) ^ 1, p.status)) break;
                TaskInfo ti;
                ti.pad = 0;
                if (t >= n_tasks) {
                    ti.kind = -1;
                    sm->task[b] = ti;
                    mbar_arrive(&sm->sfull[b]);
                    break;
                }
                int ci, blk;
                if (t < n_sh * nbs) { ci = t / nbs; blk = t % nbs; }
                else { const int u = t - n_sh * nbs; ci = n_sh + u / nbr; blk = u % nbr; }
                const ChunkEntry ce = p.chunks[ci];
                ti.kind = ce.expert < 0 ? 0 : 1;
                ti.expert = ce.expert;
                ti.row0 = blk * DC_ROWS;
                ti.start = ce.start;
                ti.count = ce.count;
                ti.K = ti.kind ? p.K_r : p.K_s;
                const int kchunk = ti.kind ? 256 : 64;          // K values per 128-byte tile row
                ti.n_stages = MODE == 0 ? int(ceil_div(ti.K, kchunk)) : int(ceil_div(ti.K, 2 * kchunk));
                sm->task[b] = ti;
                const CUtensorMap* m0 = ti.kind ? &tm_r0 : &tm_s0;
                const CUtensorMap* m1 = ti.kind ? &tm_r1 : &tm_s1;
                const int grow = ti.kind ? ti.expert * p.n_rows_r + ti.row0 : ti.row0;   // global tile row
                if (ti.kind) {
                    const int ng = ti.K / kGroup;
                    const uint32_t bytes = uint32_t(DC_ROWS * ng * 4);
                    float* dst = sbuf + b * p.scale_buf_floats;
                    mbar_arrive_expect_tx(&sm->sfull[b], (MODE == 0 ? 2 : 1) * bytes);
                    bulk_load(dst, p.sc0 + int64_t(grow) * ng, bytes, &sm->sfull[b]);
                    if (MODE == 0) bulk_load(dst + DC_ROWS * ng, p.sc1 + int64_t(grow) * ng, bytes, &sm->sfull[b]);
                } else {
                    mbar_arrive(&sm->sfull[b]);
                }
                const int kbytes = ti.kind ? 128 : 64;   // tile x extent in elements (uint8 codes / bf16)
                for (int s = 0; s < ti.n_stages; ++s, ++it) {
                    const uint32_t slot = it % DC_NSTAGES;
                    if (!mbar_wait(&sm->empty[slot], ((it / DC_NSTAGES) & 1) ^ 1, p.status)) { ok = false; break; }
                    unsigned char* st = ring + slot * DC_STAGE;
                    if (MODE == 0) {
                        mbar_arrive_expect_tx(&sm->full[slot], DC_STAGE);
                        tma_load_2d(st, m0, &sm->full[slot], s * kbytes, grow);
                        tma_load_2d(st + DC_CHUNK, m1, &sm->full[slot], s * kbytes, grow);
                    } else {
                        // two consecutive K tiles of the one matrix; the second only if in range
                        const bool second = (2 * s + 1) * kchunk < ti.K;
                        mbar_arrive_expect_tx(&sm->full[slot], second ? DC_STAGE : DC_CHUNK);
                        tma_load_2d(st, m0, &sm->full[slot], 2 * s * kbytes, grow);
                        if (second) tma_load_2d(st + DC_CHUNK, m0, &sm->full[slot], (2 * s + 1) * kbytes, grow);
                    }
                }
            }
            // wind down: wait (bounded) for every stage still in flight to land
            for (uint32_t i = 0; i < DC_NSTAGES && i < it; ++i) {
                const uint32_t j = it - 1 - i;
                mbar_wait(&sm->full[j % DC_NSTAGES], (j / DC_NSTAGES) & 1, nullptr);
            }
        }
        return;
    }

    // ------------------------------ consumers ------------------------------
    const int rb = warp & 1, q = warp >> 1;
    const int g = lane >> 2, c = lane & 3;
    const int row_a = 16 * rb + sigma8(g), row_b = row_a + 8;
    uint32_t it_base = 0;
    for (uint32_t tn = 0;; ++tn) {
        const int b = tn & 1;
        if (!mbar_wait(&sm->sfull[b], (tn >> 1) & 1, p.status)) break;
        const TaskInfo ti = sm->task[b];
        if (ti.kind < 0) break;
        const float* sc = sbuf + b * p.scale_buf_floats;
        const int ng = ti.K / kGroup;

        // token rows of this chunk for the two n-tiles (column n = g of each)
        const bf16* brow[DC_NT];
#pragma unroll
        for (int nt = 0; nt < DC_NT; ++nt) {
            const int i = nt * 8 + g;
            brow[nt] = nullptr;
            if (i < ti.count) {
                if (ti.kind == 0) brow[nt] = p.b_s + int64_t(ti.start + i) * p.ldb_s;
                else if (MODE == 0) brow[nt] = p.b_r + int64_t(p.perm[ti.start + i] / p.k_top) * p.ldb_r;
                else brow[nt] = p.b_r + int64_t(ti.start + i) * p.ldb_r;
            }
        }
        const int nt_used = ti.count > 8 ? 2 : 1;

        float acc0[DC_NT][4], acc1[DC_NT][4];
#pragma unroll
        for (int nt = 0; nt < DC_NT; ++nt)
#pragma unroll
            for (int r = 0; r < 4; ++r) { acc0[nt][r] = 0.f; acc1[nt][r] = 0.f; }

        bool ok = true;
        for (int s = q; s < ti.n_stages; s += DC_KPH) {
            const uint32_t it = it_base + s;
            const uint32_t slot = it % DC_NSTAGES;
            if (!mbar_wait(&sm->full[slot], (it / DC_NSTAGES) & 1, p.status)) { ok = false; break; }
            const unsigned char* st = ring + slot * DC_STAGE;
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                // MODE 0: tile 0 = gate, tile 1 = up, same K.  MODE 1: two K tiles of one matrix.
                if (MODE == 1 && ch == 1 && (2 * s + 1) * (ti.kind ? 256 : 64) >= ti.K) break;
                if (MODE == 0 && ch == 1) break;   // handled together with tile 0 below
                const unsigned char* t0 = st + ch * DC_CHUNK;
                const unsigned char* t1 = st + DC_CHUNK;
                if (ti.kind == 1) {
                    // ---- int4: 2 groups of 128 K per tile ----
#pragma unroll
                    for (int gi = 0; gi < 2; ++gi) {
                        const int G = (MODE == 0 ? s * 2 : (2 * s + ch) * 2) + gi;
                        if (G >= ng) break;
                        const int j = 4 * gi + c;
                        const uint4 wa = lds128(swz(t0, row_a, j));
                        const uint4 wb = lds128(swz(t0, row_b, j));
                        uint4 va = make_uint4(0, 0, 0, 0), vb = va;
                        if (MODE == 0) { va = lds128(swz(t1, row_a, j)); vb = lds128(swz(t1, row_b, j)); }
                        uint4 xb[DC_NT][4];
#pragma unroll
                        for (int nt = 0; nt < DC_NT; ++nt)
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                xb[nt][i] = (nt < nt_used && brow[nt])
                                                ? ldg_cached(brow[nt] + G * kGroup + 32 * c + 8 * i)
                                                : make_uint4(0, 0, 0, 0);
                        float pg[DC_NT][4], pu[DC_NT][4];
#pragma unroll
                        for (int nt = 0; nt < DC_NT; ++nt)
#pragma unroll
                            for (int r = 0; r < 4; ++r) { pg[nt][r] = 0.f; pu[nt][r] = 0.f; }
                        const uint32_t WA[4] = {wa.x ^ 0x88888888u, wa.y ^ 0x88888888u, wa.z ^ 0x88888888u, wa.w ^ 0x88888888u};
                        const uint32_t WB[4] = {wb.x ^ 0x88888888u, wb.y ^ 0x88888888u, wb.z ^ 0x88888888u, wb.w ^ 0x88888888u};
                        const uint32_t VA[4] = {va.x ^ 0x88888888u, va.y ^ 0x88888888u, va.z ^ 0x88888888u, va.w ^ 0x88888888u};
                        const uint32_t VB[4] = {vb.x ^ 0x88888888u, vb.y ^ 0x88888888u, vb.z ^ 0x88888888u, vb.w ^ 0x88888888u};
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj) {
#pragma unroll
                            for (int h = 0; h < 2; ++h) {
                                uint32_t a0, a1, a2, a3;
                                if (h == 0) {
                                    a0 = int4x2_to_bf16x2<0>(WA[jj]); a2 = int4x2_to_bf16x2<4>(WA[jj]);
                                    a1 = int4x2_to_bf16x2<0>(WB[jj]); a3 = int4x2_to_bf16x2<4>(WB[jj]);
                                } else {
                                    a0 = int4x2_to_bf16x2<8>(WA[jj]); a2 = int4x2_to_bf16x2<12>(WA[jj]);
                                    a1 = int4x2_to_bf16x2<8>(WB[jj]); a3 = int4x2_to_bf16x2<12>(WB[jj]);
                                }
#pragma unroll
                                for (int nt = 0; nt < DC_NT; ++nt) {
                                    if (nt >= nt_used) break;
                                    const uint32_t b0 = h == 0 ? xb[nt][jj].x : xb[nt][jj].z;
                                    const uint32_t b1 = h == 0 ? xb[nt][jj].y : xb[nt][jj].w;
                                    mma_bf16_16816(pg[nt], a0, a1, a2, a3, b0, b1);
                                }
                                if (MODE == 0) {
                                    uint32_t u0, u1, u2, u3;
                                    if (h == 0) {
                                        u0 = int4x2_to_bf16x2<0>(VA[jj]); u2 = int4x2_to_bf16x2<4>(VA[jj]);
                                        u1 = int4x2_to_bf16x2<0>(VB[jj]); u3 = int4x2_to_bf16x2<4>(VB[jj]);
                                    } else {
                                        u0 = int4x2_to_bf16x2<8>(VA[jj]); u2 = int4x2_to_bf16x2<12>(VA[jj]);
                                        u1 = int4x2_to_bf16x2<8>(VB[jj]); u3 = int4x2_to_bf16x2<12>(VB[jj]);
                                    }
#pragma unroll
                                    for (int nt = 0; nt < DC_NT; ++nt) {
                                        if (nt >= nt_used) break;
                                        const uint32_t b0 = h == 0 ? xb[nt][jj].x : xb[nt][jj].z;
                                        const uint32_t b1 = h == 0 ? xb[nt][jj].y : xb[nt][jj].w;
                                        mma_bf16_16816(pu[nt], u0, u1, u2, u3, b0, b1);
                                    }
                                }
                            }
                        }
                        // group scales of rows row_a / row_b
                        const float sga = sc[row_a * ng + G], sgb = sc[row_b * ng + G];
                        float sua = 0.f, sub = 0.f;
                        if (MODE == 0) { sua = sc[(DC_ROWS + row_a) * ng + G]; sub = sc[(DC_ROWS + row_b) * ng + G]; }
#pragma unroll
                        for (int nt = 0; nt < DC_NT; ++nt) {
                            acc0[nt][0] = fmaf(pg[nt][0], sga, acc0[nt][0]);
                            acc0[nt][1] = fmaf(pg[nt][1], sga, acc0[nt][1]);
                            acc0[nt][2] = fmaf(pg[nt][2], sgb, acc0[nt][2]);
                            acc0[nt][3] = fmaf(pg[nt][3], sgb, acc0[nt][3]);
                            if (MODE == 0) {
                                acc1[nt][0] = fmaf(pu[nt][0], sua, acc1[nt][0]);
                                acc1[nt][1] = fmaf(pu[nt][1], sua, acc1[nt][1]);
                                acc1[nt][2] = fmaf(pu[nt][2], sub, acc1[nt][2]);
                                acc1[nt][3] = fmaf(pu[nt][3], sub, acc1[nt][3]);
                            }
                        }
                    }
                } else {
                    // ---- bf16 (shared expert): 64 K per tile; thread c takes 8-blocks c and c + 4 ----
                    const int kt = MODE == 0 ? s * 64 : (2 * s + ch) * 64;
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        const int j = c + 4 * h2;
                        const uint4 wa = lds128(swz(t0, row_a, j));
                        const uint4 wb = lds128(swz(t0, row_b, j));
                        uint4 va = make_uint4(0, 0, 0, 0), vb = va;
                        if (MODE == 0) { va = lds128(swz(t1, row_a, j)); vb = lds128(swz(t1, row_b, j)); }
                        uint4 xb[DC_NT];
#pragma unroll
                        for (int nt = 0; nt < DC_NT; ++nt)
                            xb[nt] = (nt < nt_used && brow[nt]) ? ldg_cached(brow[nt] + kt + 8 * j)
                                                                : make_uint4(0, 0, 0, 0);
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const uint32_t a0 = h == 0 ? prmt(wa.x, wa.z, 0x5410) : prmt(wa.y, wa.w, 0x5410);
                            const uint32_t a2 = h == 0 ? prmt(wa.x, wa.z, 0x7632) : prmt(wa.y, wa.w, 0x7632);
                            const uint32_t a1 = h == 0 ? prmt(wb.x, wb.z, 0x5410) : prmt(wb.y, wb.w, 0x5410);
                            const uint32_t a3 = h == 0 ? prmt(wb.x, wb.z, 0x7632) : prmt(wb.y, wb.w, 0x7632);
#pragma unroll
                            for (int nt = 0; nt < DC_NT; ++nt) {
                                if (nt >= nt_used) break;
                                const uint32_t b0 = h == 0 ? xb[nt].x : xb[nt].z;
                                const uint32_t b1 = h == 0 ? xb[nt].y : xb[nt].w;
                                mma_bf16_16816(acc0[nt], a0, a1, a2, a3, b0, b1);
                            }
                            if (MODE == 0) {
                                const uint32_t u0 = h == 0 ? prmt(va.x, va.z, 0x5410) : prmt(va.y, va.w, 0x5410);
                                const uint32_t u2 = h == 0 ? prmt(va.x, va.z, 0x7632) : prmt(va.y, va.w, 0x7632);
                                const uint32_t u1 = h == 0 ? prmt(vb.x, vb.z, 0x5410) : prmt(vb.y, vb.w, 0x5410);
                                const uint32_t u3 = h == 0 ? prmt(vb.x, vb.z, 0x7632) : prmt(vb.y, vb.w, 0x7632);
#pragma unroll
                                for (int nt = 0; nt < DC_NT; ++nt) {
                                    if (nt >= nt_used) break;
                                    const uint32_t b0 = h == 0 ? xb[nt].x : xb[nt].z;
                                    const uint32_t b1 = h == 0 ? xb[nt].y : xb[nt].w;
                                    mma_bf16_16816(acc1[nt], u0, u1, u2, u3, b0, b1);
                                }
                            }
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm->empty[slot]);
        }
        if (!ok) break;

        // ---- sum the 4 K phases (phases 1..3 hand their partial sums to phase 0) ----
        if (q > 0) {
            if (!mbar_wait(&sm->red_empty, (tn & 1) ^ 1, p.status)) break;
            float* my = red + ((q - 1) * 2 + rb) * 32 * DC_NT * 8 + lane * DC_NT * 8;
#pragma unroll
            for (int nt = 0; nt < DC_NT; ++nt)
#pragma unroll
                for (int r = 0; r < 4; ++r) { my[nt * 8 + r] = acc0[nt][r]; my[nt * 8 + 4 + r] = acc1[nt][r]; }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm->red_full);
        } else {
            if (!mbar_wait(&sm->red_full, tn & 1, p.status)) break;
#pragma unroll
            for (int qq = 1; qq < DC_KPH; ++qq) {
                const float* o = red + ((qq - 1) * 2 + rb) * 32 * DC_NT * 8 + lane * DC_NT * 8;
#pragma unroll
                for (int nt = 0; nt < DC_NT; ++nt)
#pragma unroll
                    for (int r = 0; r < 4; ++r) { acc0[nt][r] += o[nt * 8 + r]; acc1[nt][r] += o[nt * 8 + 4 + r]; }
            }
            // ---- epilogue: C rows (row_a, row_b) x token columns (2c, 2c + 1) of each n-tile ----
#pragma unroll
            for (int nt = 0; nt < DC_NT; ++nt) {
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int col = nt * 8 + 2 * c + (r & 1);
                    if (col >= ti.count) continue;
                    const int n = ti.row0 + (r < 2 ? row_a : row_b);
                    if (MODE == 0) {
                        const float hv = silu_f32(acc0[nt][r]) * acc1[nt][r];
                        const int pos = (n & ~7) + frag_pos8(n & 7);
                        if (ti.kind == 1) p.h_r[int64_t(ti.start + col) * p.n_rows_r + pos] = __float2bfloat16_rn(hv);
                        else p.h_s[int64_t(ti.start + col) * p.n_rows_s + pos] = __float2bfloat16_rn(hv);
                    } else {
                        if (ti.kind == 1) {
                            const int pp = ti.start + col;
                            p.y_r[int64_t(pp) * p.n_rows_r + n] = acc0[nt][r] * p.gates[p.perm[pp]];
                        } else {
                            p.y_s[int64_t(ti.start + col) * p.n_rows_s + n] = acc0[nt][r];
                        }
                    }
                }
            }
        }
        __syncwarp();
        if (q == 0 && lane == 0) mbar_arrive(&sm->red_empty);   // red[] is free again
        if (lane == 0) mbar_arrive(&sm->sempty[b]);
        it_base += ti.n_stages;
    }
}

// out[t] = bf16(y_s[t] + sum_j y_r[inv_perm[t k + j]])
__global__ void combine_kernel(const float* __restrict__ y_s, const float* __restrict__ y_r,
                               const int32_t* __restrict__ inv_perm, int T, int D, int k,
                               bf16* __restrict__ out) {
    const int64_t n4 = int64_t(T) * D / 4;
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n4; i += int64_t(gridDim.x) * blockDim.x) {
        const int64_t t = i / (D / 4);
        const int d = int(i % (D / 4)) * 4;
        float4 a = *reinterpret_cast<const float4*>(y_s + t * D + d);
        for (int j = 0; j < k; ++j) {
            const int64_t pp = inv_perm[t * k + j];
            const float4 b = *reinterpret_cast<const float4*>(y_r + pp * D + d);
            a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
        }
        uint2 o;
        o.x = pack_bf16x2(a.x, a.y);
        o.y = pack_bf16x2(a.z, a.w);
        *reinterpret_cast<uint2*>(out + t * D + d) = o;
    }
}

// One thread: the decode task list (token chunks of <= 16): the shared
// expert's chunks first, then each routed expert's.
__global__ void decode_plan_kernel(const int32_t* __restrict__ counts, const int32_t* __restrict__ offsets,
                                   int T, int E, ChunkEntry* __restrict__ chunks, int32_t* __restrict__ n_chunks,
                                   int32_t* __restrict__ n_shared, int32_t* __restrict__ counters) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    int n = 0;
    for (int t0 = 0; t0 < T; t0 += 16) {
        ChunkEntry ce; ce.expert = -1; ce.start = t0; ce.count = min(16, T - t0); ce.pad = 0;
        chunks[n++] = ce;
    }
    *n_shared = n;
    for (int e = 0; e < E; ++e) {
        for (int s = 0; s < counts[e]; s += 16) {
            ChunkEntry ce; ce.expert = e; ce.start = offsets[e] + s; ce.count = min(16, counts[e] - s); ce.pad = 0;
            chunks[n++] = ce;
        }
    }
    *n_chunks = n;
    counters[0] = 0;
    counters[1] = 0;
}

int decode_max_chunks(int T, int k, int E) { return int(ceil_div(T, 16)) + int(ceil_div(int64_t(T) * k, 16)) + E; }

size_t decode_smem_bytes(int scale_buf_floats) {
    return 1024 + size_t(DC_NSTAGES) * DC_STAGE + 2 * size_t(scale_buf_floats) * 4 + DC_RED_FLOATS * 4 +
           sizeof(DecodeSmem);
}

// ---------------------------------------------------------------------------
// host side: tensor maps and launches
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// 2-D map over a row-major [rows, inner] matrix; box = box_inner x box_rows.
bool make_tmap_2d(CUtensorMap* m, const void* base, bool bf16_elems, uint64_t inner, uint64_t rows,
                  uint32_t box_inner, uint32_t box_rows, bool swizzle128) {
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return false;
    const uint64_t esz = bf16_elems ? 2 : 1;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner * esz};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, bf16_elems ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                    const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

moe_status launch_decode_plan(const int32_t* counts, const int32_t* offsets, int T, int E, void* chunks,
                              int32_t* n_chunks, int32_t* n_shared, int32_t* counters, cudaStream_t stream) {
    decode_plan_kernel<<<1, 32, 0, stream>>>(counts, offsets, T, E, static_cast<ChunkEntry*>(chunks), n_chunks,
                                             n_shared, counters);
    return launch_status();
}

moe_status launch_decode_ffn(int mode, const DecodeMaps& maps, const DecodeParams& prm, cudaStream_t stream) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const size_t smem = decode_smem_bytes(prm.scale_buf_floats);
    cudaError_t e;
    if (mode == 0) {
        e = cudaFuncSetAttribute(decode_ffn_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e != cudaSuccess) return MOE_ERR_CUDA;
        decode_ffn_kernel<0><<<sms, DC_THREADS, smem, stream>>>(maps.r0, maps.r1, maps.s0, maps.s1, prm);
    } else {
        e = cudaFuncSetAttribute(decode_ffn_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e != cudaSuccess) return MOE_ERR_CUDA;
        decode_ffn_kernel<1><<<sms, DC_THREADS, smem, stream>>>(maps.r0, maps.r1, maps.s0, maps.s1, prm);
    }
    return launch_status();
}

moe_status launch_combine(const float* y_s, const float* y_r, const int32_t* inv_perm, int T, int D, int k,
                          bf16* out, cudaStream_t stream) {
    const int64_t n4 = int64_t(T) * D / 4;
    int64_t blocks = ceil_div(n4, 256);
    if (blocks > 148 * 16) blocks = 148 * 16;
    combine_kernel<<<unsigned(blocks), 256, 0, stream>>>(y_s, y_r, inv_perm, T, D, k, out);
    return launch_status();
}

}  // namespace moe
