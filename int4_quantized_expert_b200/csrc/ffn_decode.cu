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
//   * one persistent CTA per SM (512 threads); a producer thread takes tasks
//     (64 output rows of one matrix pair x one chunk of <= 16 tokens x the
//     whole K) from a global counter, shared expert first, and streams each
//     task through a ring of 6 stages.  A stage holds 16 KB of weights (2-D
//     TMA, 64 rows x 128 bytes, 128-byte swizzle), the chunk's token rows for
//     the stage's K range (one 3-D TMA box) and, for int4, the rows' per-group
//     (offset, scale) pairs (one 2-D box).  The benchmark's fp32 weight scales
//     arrive first, one padded 2-D box per matrix.
//   * 12 consumer warps: 4 row blocks of 16 rows x 3 K phases (a stage goes to
//     phase (global stage index) % 3), three per SM sub-partition to hide each
//     one's MMA and load latencies.  Each converts int4 codes to exact fp16
//     integers in registers (no scale multiply per element), runs m16n8k16
//     tensor-core MMAs against the tokens (fp32 accumulate), and applies the
//     group's weight scale (times the token group's power of two) to the
//     128-K partial sum.  At the end of a task every consumer warp hands its
//     partial sums over through shared memory and goes on with the next task.
//   * 3 epilogue warps (the rest of the producer's warpgroup) sum the K
//     phases in a fixed order and apply SwiGLU (gate/up pass) or the gate
//     (down pass), off the consumers' path.
//   * Tokens are the MMA's N operand (8 per n-tile), written by act16_kernel as
//     fp16 rows in the order the int4 unpacking yields, each group of 128
//     scaled by its own power of two.
//   * Every wait is bounded; a timeout sets the status word and the CTA
//     drains its copies in flight and returns.
//   * Launches chain by programmatic dependent launch: each kernel's setup
//     (barriers, tensor-map prefetch, shared-expert tasks) overlaps the tail
//     of the kernel before it.
#include <cuda.h>

#include "common.cuh"
#include "ffn_decode.cuh"

namespace moe {

constexpr int DC_RB = 4;                    // row blocks of 16 rows per task
constexpr int DC_ROWS = 16 * DC_RB;         // output rows per task
constexpr int DC_KPH = 3;                   // K phases
constexpr int DC_CONSUMERS = DC_RB * DC_KPH;   // 12: 3 warps per SM sub-partition
// Four warpgroups: warpgroup 0 holds the producer (warp 0, one thread) and
// gives most of its registers to warpgroups 1 to 3, the 12 consumer warps:
// 128 x 64 + 384 x 144 <= 512 x 128, the registers the block launches with.
constexpr int DC_THREADS = 512;
constexpr int DC_PRODUCER_REGS = 64;
constexpr int DC_CONSUMER_REGS = 144;
static_assert(128 * DC_PRODUCER_REGS + 32 * DC_CONSUMERS * DC_CONSUMER_REGS <= DC_THREADS * 128, "register split");
constexpr int DC_CHUNK = DC_ROWS * 128;     // one matrix tile of a stage: 64 rows x 128 B
constexpr int DC_STAGE = 2 * DC_CHUNK;      // weights of a stage: 16 KB
constexpr int DC_B_OFF = DC_STAGE;          // then the chunk's token rows for the stage's K range
// then the rows' per-group (offset, scale) pairs (8 rows x the stage's groups,
// at most 16) in a 1 KB unit; the token rows take 4 KB (gate/up: 256 K of 8
// routed or 64 K of 16 shared rows) or 8 KB (down: 512 K routed, 128 K
// shared).  With groups of 64 or 32 the stage also carries its weight scales
// (64 rows x the stage's groups, per matrix) in a 4 KB unit.
__host__ __device__ constexpr int dc_c_off(int mode) { return DC_B_OFF + (mode == 0 ? 4096 : 8192); }
__host__ __device__ constexpr int dc_s_off(int mode) { return dc_c_off(mode) + 1024; }
__host__ __device__ constexpr int dc_slot(int mode, int G) {   // a multiple of 1024
    return G == kGroup ? dc_c_off(mode) + 1024 : dc_s_off(mode) + 4096;
}
// K values per stage and groups of G per stage
__host__ __device__ constexpr int dc_kstage(int mode) { return mode == 0 ? 256 : 512; }
// Ring depth: a multiple of the K-phase count.  A stage goes to K phase
// (global stage index) % DC_KPH, so every slot is always consumed by the same
// phase, in order, and no warp ever waits on a slot's next use while its
// current one is still in flight (a parity wait one phase too far ahead
// would return at once).
__host__ __device__ constexpr int dc_nstages(int mode) { return mode == 0 ? 6 : 6; }
constexpr int DC_MAX_STAGES = 6;
static_assert(dc_nstages(0) % DC_KPH == 0 && dc_nstages(1) % DC_KPH == 0, "ring depth vs K phases");
constexpr int DC_NT = 2;                    // n-tiles of 8 tokens per task
constexpr int DC_HELPERS = 3;              // epilogue warps: warps 1..3 (the producer warpgroup)
constexpr int DC_RED_PITCH = DC_NT * 8 + 1; // floats per consumer lane in red[] (odd: no bank conflicts)
constexpr int DC_RED_FLOATS = DC_KPH * DC_RB * 32 * DC_RED_PITCH;   // every consumer warp's partial sums

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
    uint64_t full[DC_MAX_STAGES];
    uint64_t empty[DC_MAX_STAGES];
    uint64_t sfull[2];
    uint64_t sempty[2];
    uint64_t red_full;    // consumers -> epilogue warps: a task's partial sums written
    uint64_t red_empty;   // epilogue warps -> consumers: partial sums consumed
    TaskInfo task[2];
};

__device__ __forceinline__ int sigma8(int g) { return ((g & 1) << 2) | (g >> 1); }

// The first stage of a task (its stages are it_base, it_base + 1, ...) that
// belongs to K phase q: phases take stages by their global index.
__device__ __forceinline__ int first_stage(int q, uint32_t it_base) {
    return int((uint32_t(q) + DC_KPH - it_base % DC_KPH) % DC_KPH);
}

// Row pitch (floats) of a task's scale buffer in shared memory.  When a
// row's K / 128 scales fill whole 16-byte units (ng % 4 == 0), rows are
// copied one by one to a pitch of 4 x an odd number of floats, which puts
// the 8 rows a warp reads at once in distinct banks; otherwise the task's
// rows are one block copy at pitch ng.
__host__ __device__ __forceinline__ bool scale_rows_padded(int ng) { return ng % 4 == 0; }
__host__ __device__ __forceinline__ int scale_row_floats(int ng) {
    return !scale_rows_padded(ng) ? ng : ((ng / 4) % 2 ? ng : ng + 4);
}

// Address of logical 16-byte chunk j of row r in a 128-byte-swizzled tile.
__device__ __forceinline__ const unsigned char* swz(const unsigned char* tile, int r, int j) {
    return tile + r * 128 + ((j ^ (r & 7)) << 4);
}


// The int4 part of a decode task: the warp's stages (those of K phase q) of groups
// of 128 K, one n-tile of 8 tokens.  Returns false if a wait timed out.
//
// Codes enter fp16 MMAs as exact integers: per 32-bit word of 8 codes, one
// shift and four LOP3s give (k0,k4) and (k2,k6) as 1032 + q and (k1,k5),
// (k3,k7) as 1152 + 16 q (f16_lo_nibbles / f16_hi_nibbles, the magic numbers
// held in registers klo, khi).  The token rows (fp16, each group of 128
// scaled by a power of two) store odd positions divided by 16 and every
// 8-block in the order x0 x4 x2 x6 x1 x5 x3 x7, so one accumulator sums q * x
// plus a per-group offset that is added to the group's partial sum.  The
// stage holds the chunk's 8 token rows for its K range and their groups'
// (offset, scale) pairs next to the codes; MMA column g is token row
// sigma8(g).
template <int MODE, int G>
__device__ __forceinline__ bool consume_int4(const TaskInfo& ti, DecodeSmem* sm, const unsigned char* ring,
                                             const float* sc, uint32_t it_base, int q, int lane, int row_a,
                                             int row_b, uint32_t klo, uint32_t khi, float (&acc0)[4],
                                             float (&acc1)[4], int32_t* status) {
    constexpr int GPS = MODE == 0 ? 2 : 4;   // groups per stage
    constexpr int NST = dc_nstages(MODE), SLOT = dc_slot(MODE, G), C_OFF = dc_c_off(MODE);
    const int g = lane >> 2, c = lane & 3;
    const int ng = ti.K / kGroup;
    // byte offsets of this thread's 16-byte code chunks in a swizzled 64 x 128 B
    // tile: chunk 4 gi + c of rows row_a and row_b, for the tile's two groups gi
    uint32_t off_a[2], off_b[2];
#pragma unroll
    for (int gi = 0; gi < 2; ++gi) {
        off_a[gi] = row_a * 128 + (((4 * gi + c) ^ (row_a & 7)) << 4);
        off_b[gi] = row_b * 128 + (((4 * gi + c) ^ (row_b & 7)) << 4);
    }
    const int ldsc = scale_row_floats(ng);   // padded row pitch of the scale buffer
    const float* sga_p = sc + row_a * ldsc;
    const float* sgb_p = sc + row_b * ldsc;
    const float* sua_p = sc + (DC_ROWS + row_a) * ldsc;
    const float* sub_p = sc + (DC_ROWS + row_b) * ldsc;
    // token tile: group gl of the stage in boxes 2 gl, 2 gl + 1 (8 rows x 128 B,
    // 128-byte swizzle); this thread's K chunk 4 c + i of the group is stored
    // at box i >> 1, chunk c + 4 (i & 1) (see act16_kernel)
    const int trow = sigma8(g);
    uint32_t offx[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) offx[i] = (i >> 1) * 1024 + trow * 128 + (((c + 4 * (i & 1)) ^ (trow & 7)) << 4);
    const int tc0 = sigma8(2 * c), tc1 = sigma8(2 * c + 1);   // token rows of C columns 2c, 2c + 1

    // One group of 128 K (group G of the task, gl of the stage).  gl is a
    // compile-time constant at every call, so the register arrays above are
    // indexed statically.
    auto group = [&](const unsigned char* st, const unsigned char* bt, const float* ct, int cg0, int G, int gl) {
        // MODE 0: both groups in tile 0 (gate) and tile 1 (up);
        // MODE 1: groups 0,1 in tile 0 and 2,3 in tile 1 of the one matrix
        const unsigned char* tile = st + (MODE == 0 ? 0 : (gl >> 1) * DC_CHUNK);
        const int gi = gl & 1;
        uint4 xc[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) xc[i] = ld_shared_v4(bt + gl * 2048 + offx[i]);
        const float2 m0 = ld_shared_f32x2(ct + tc0 * 8 + 2 * (cg0 + gl));   // (offset, 2^e) of token row tc0
        const float2 m1 = ld_shared_f32x2(ct + tc1 * 8 + 2 * (cg0 + gl));
        const float cc0 = m0.x, cc1 = m1.x;
        const uint4 wa = ld_shared_v4(tile + off_a[gi]);
        const uint4 wb = ld_shared_v4(tile + off_b[gi]);
        uint4 va = make_uint4(0, 0, 0, 0), vb = va;
        if (MODE == 0) { va = ld_shared_v4(st + DC_CHUNK + off_a[gi]); vb = ld_shared_v4(st + DC_CHUNK + off_b[gi]); }
        const uint32_t WA[4] = {wa.x, wa.y, wa.z, wa.w}, WB[4] = {wb.x, wb.y, wb.z, wb.w};
        const uint32_t VA[4] = {va.x, va.y, va.z, va.w}, VB[4] = {vb.x, vb.y, vb.z, vb.w};
        // one accumulation chain per matrix over the group's 8 MMAs, started
        // at zero; the group offset is added to its sum in fp32
        float pg[4], pu[4];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            const uint32_t wa8 = WA[jj] >> 8, wb8 = WB[jj] >> 8;
            if (jj == 0)
                mma_f16_16816(pg, f16_lo_nibbles(WA[jj], klo), f16_lo_nibbles(WB[jj], klo),
                              f16_lo_nibbles(wa8, klo), f16_lo_nibbles(wb8, klo), xc[jj].x, xc[jj].y,
                              0.0f, 0.0f, 0.0f, 0.0f);
            else
                mma_f16_16816(pg, f16_lo_nibbles(WA[jj], klo), f16_lo_nibbles(WB[jj], klo),
                              f16_lo_nibbles(wa8, klo), f16_lo_nibbles(wb8, klo), xc[jj].x, xc[jj].y);
            if (MODE == 0) {
                const uint32_t va8 = VA[jj] >> 8, vb8 = VB[jj] >> 8;
                if (jj == 0)
                    mma_f16_16816(pu, f16_lo_nibbles(VA[jj], klo), f16_lo_nibbles(VB[jj], klo),
                                  f16_lo_nibbles(va8, klo), f16_lo_nibbles(vb8, klo), xc[jj].x, xc[jj].y,
                                  0.0f, 0.0f, 0.0f, 0.0f);
                else
                    mma_f16_16816(pu, f16_lo_nibbles(VA[jj], klo), f16_lo_nibbles(VB[jj], klo),
                                  f16_lo_nibbles(va8, klo), f16_lo_nibbles(vb8, klo), xc[jj].x, xc[jj].y);
            }
            mma_f16_16816(pg, f16_hi_nibbles(WA[jj], khi), f16_hi_nibbles(WB[jj], khi),
                          f16_hi_nibbles(wa8, khi), f16_hi_nibbles(wb8, khi), xc[jj].z, xc[jj].w);
            if (MODE == 0) {
                const uint32_t va8 = VA[jj] >> 8, vb8 = VB[jj] >> 8;
                mma_f16_16816(pu, f16_hi_nibbles(VA[jj], khi), f16_hi_nibbles(VB[jj], khi),
                              f16_hi_nibbles(va8, khi), f16_hi_nibbles(vb8, khi), xc[jj].z, xc[jj].w);
            }
        }
        // C columns 2c and 2c + 1 (r & 1) are token rows tc0 and tc1; the group's
        // weight scale times the token group's power of two (an exact product)
        const float sga = ld_shared_f32(sga_p + G), sgb = ld_shared_f32(sgb_p + G);
        const float wg[4] = {sga * m0.y, sga * m1.y, sgb * m0.y, sgb * m1.y};
#pragma unroll
        for (int r = 0; r < 4; ++r) acc0[r] = fmaf(pg[r] + ((r & 1) ? cc1 : cc0), wg[r], acc0[r]);
        if (MODE == 0) {
            const float sua = ld_shared_f32(sua_p + G), sub = ld_shared_f32(sub_p + G);
            const float wu[4] = {sua * m0.y, sua * m1.y, sub * m0.y, sub * m1.y};
#pragma unroll
            for (int r = 0; r < 4; ++r) acc1[r] = fmaf(pu[r] + ((r & 1) ? cc1 : cc0), wu[r], acc1[r]);
        }
    };

    bool ok = true;
    for (int s = first_stage(q, it_base); s < ti.n_stages; s += DC_KPH) {
        const uint32_t it = it_base + s;
        const uint32_t slot = it % NST;
        if (!mbar_wait(&sm->full[slot], (it / NST) & 1, status)) { ok = false; break; }
        const unsigned char* st = ring + slot * SLOT;
        const unsigned char* bt = st + DC_B_OFF;
        const float* ct = reinterpret_cast<const float*>(st + C_OFF);
        const int G0 = s * GPS;
        const int cg0 = G0 & 3;   // the offsets tile starts at group G0 rounded down to a multiple of 4
        if (G0 + GPS <= ng) {
            // a full stage: straight-line code, so the groups' loads and
            // unpacking interleave
#pragma unroll
            for (int gl = 0; gl < GPS; ++gl) group(st, bt, ct, cg0, G0 + gl, gl);
        } else {
#pragma unroll
            for (int gl = 0; gl < GPS; ++gl)
                if (G0 + gl < ng) group(st, bt, ct, cg0, G0 + gl, gl);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm->empty[slot]);
    }
    return ok;
}

// The int4 part of a decode task for groups of G = 64 or 32 K ("Meta Llama
// Models Llama 4 单卡量化推理与选型指南", "量化环节做了什么": a smaller
// group_size).  The layout of consume_int4 sums all four 32-K quarters of a
// 128-K block in every MMA, so it cannot apply one scale per 64 or 32 K.
// Here the MMAs go quarter by quarter: thread c takes word c (8 codes) of
// each 32-K quarter of rows row_a and row_b (4-byte loads; the 128-byte
// swizzle puts a warp's 32 words in 32 banks) and the matching token
// 8-block, 8 c .. 8 c + 7 of the quarter (act16 keeps the 8-blocks of such
// groups in their natural order).  A quarter is two MMAs per matrix (low and
// high nibbles); a group chains its G / 32 quarters, adds the group's token
// offset and multiplies by the group's weight scale times the token group's
// power of two.  The stage carries its groups' weight scales and token
// (offset, scale) pairs.
template <int MODE, int G>
__device__ __forceinline__ bool consume_int4_qm(const TaskInfo& ti, DecodeSmem* sm, const unsigned char* ring,
                                                uint32_t it_base, int q, int lane, int row_a, int row_b, uint32_t klo,
                                                uint32_t khi, float (&acc0)[4], float (&acc1)[4], int32_t* status) {
    constexpr int NST = dc_nstages(MODE), SLOT = dc_slot(MODE, G), C_OFF = dc_c_off(MODE), S_OFF = dc_s_off(MODE);
    constexpr int GPS = dc_kstage(MODE) / G;   // groups per stage
    constexpr int QPG = G / 32;                // quarters per group
    const int g = lane >> 2, c = lane & 3;
    const int trow = sigma8(g);
    const int tc0 = sigma8(2 * c), tc1 = sigma8(2 * c + 1);   // token rows of C columns 2c, 2c + 1
    const int ng = ti.K / G;
    bool ok = true;
    for (int s = first_stage(q, it_base); s < ti.n_stages; s += DC_KPH) {
        const uint32_t it = it_base + s;
        const uint32_t slot = it % NST;
        if (!mbar_wait(&sm->full[slot], (it / NST) & 1, status)) { ok = false; break; }
        const unsigned char* st = ring + slot * SLOT;
        const unsigned char* bt = st + DC_B_OFF;
        const float* meta = reinterpret_cast<const float*>(st + C_OFF);   // [8 token rows][GPS][2]
        const float* scl = reinterpret_cast<const float*>(st + S_OFF);    // [matrix][64 rows][GPS]
        const int G0 = s * GPS;
#pragma unroll
        for (int gl = 0; gl < GPS; ++gl) {
            if (G0 + gl >= ng) break;   // the last stage of a task may be partial
            float pg[4], pu[4];
#pragma unroll
            for (int qq = 0; qq < QPG; ++qq) {
                const int Q = gl * QPG + qq;   // quarter of the stage
                const unsigned char* tile = st + (MODE == 0 ? 0 : (Q >> 3) * DC_CHUNK);
                const int ch = Q & 7;
                const uint32_t wa = ld_shared_u32(tile + row_a * 128 + ((ch ^ (row_a & 7)) << 4) + 4 * c);
                const uint32_t wb = ld_shared_u32(tile + row_b * 128 + ((ch ^ (row_b & 7)) << 4) + 4 * c);
                const uint4 xc = ld_shared_v4(bt + (Q >> 1) * 1024 + trow * 128 + ((((Q & 1) * 4 + c) ^ (trow & 7)) << 4));
                const uint32_t wa8 = wa >> 8, wb8 = wb >> 8;
                if (qq == 0)
                    mma_f16_16816(pg, f16_lo_nibbles(wa, klo), f16_lo_nibbles(wb, klo), f16_lo_nibbles(wa8, klo),
                                  f16_lo_nibbles(wb8, klo), xc.x, xc.y, 0.0f, 0.0f, 0.0f, 0.0f);
                else
                    mma_f16_16816(pg, f16_lo_nibbles(wa, klo), f16_lo_nibbles(wb, klo), f16_lo_nibbles(wa8, klo),
                                  f16_lo_nibbles(wb8, klo), xc.x, xc.y);
                mma_f16_16816(pg, f16_hi_nibbles(wa, khi), f16_hi_nibbles(wb, khi), f16_hi_nibbles(wa8, khi),
                              f16_hi_nibbles(wb8, khi), xc.z, xc.w);
                if (MODE == 0) {
                    const unsigned char* up = st + DC_CHUNK;
                    const uint32_t va = ld_shared_u32(up + row_a * 128 + ((ch ^ (row_a & 7)) << 4) + 4 * c);
                    const uint32_t vb = ld_shared_u32(up + row_b * 128 + ((ch ^ (row_b & 7)) << 4) + 4 * c);
                    const uint32_t va8 = va >> 8, vb8 = vb >> 8;
                    if (qq == 0)
                        mma_f16_16816(pu, f16_lo_nibbles(va, klo), f16_lo_nibbles(vb, klo), f16_lo_nibbles(va8, klo),
                                      f16_lo_nibbles(vb8, klo), xc.x, xc.y, 0.0f, 0.0f, 0.0f, 0.0f);
                    else
                        mma_f16_16816(pu, f16_lo_nibbles(va, klo), f16_lo_nibbles(vb, klo), f16_lo_nibbles(va8, klo),
                                      f16_lo_nibbles(vb8, klo), xc.x, xc.y);
                    mma_f16_16816(pu, f16_hi_nibbles(va, khi), f16_hi_nibbles(vb, khi), f16_hi_nibbles(va8, khi),
                                  f16_hi_nibbles(vb8, khi), xc.z, xc.w);
                }
            }
            const float2 m0 = ld_shared_f32x2(meta + (tc0 * GPS + gl) * 2);
            const float2 m1 = ld_shared_f32x2(meta + (tc1 * GPS + gl) * 2);
            const float sga = ld_shared_f32(scl + row_a * GPS + gl), sgb = ld_shared_f32(scl + row_b * GPS + gl);
            const float wg[4] = {sga * m0.y, sga * m1.y, sgb * m0.y, sgb * m1.y};
#pragma unroll
            for (int r = 0; r < 4; ++r) acc0[r] = fmaf(pg[r] + ((r & 1) ? m1.x : m0.x), wg[r], acc0[r]);
            if (MODE == 0) {
                const float* su = scl + DC_ROWS * GPS;
                const float sua = ld_shared_f32(su + row_a * GPS + gl), sub = ld_shared_f32(su + row_b * GPS + gl);
                const float wu[4] = {sua * m0.y, sua * m1.y, sub * m0.y, sub * m1.y};
#pragma unroll
                for (int r = 0; r < 4; ++r) acc1[r] = fmaf(pu[r] + ((r & 1) ? m1.x : m0.x), wu[r], acc1[r]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm->empty[slot]);
    }
    return ok;
}

// One 8-block of a row's fp16 operands (the format act16_kernel describes):
// G / 8 consecutive lanes hold one group of G values; every lane of the warp
// takes part (its shuffles stay inside aligned groups of G / 8 lanes), only
// `valid` lanes store.  b is the 8-block's index in the row.
template <int G>
__device__ __forceinline__ void act16_block(const uint4 v, bool valid, __half* out16_row, float* meta_row, int b) {
    constexpr int LPG = G / 8;   // lanes per group
    const float x[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                        bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(x[i]));
#pragma unroll
    for (int o = LPG / 2; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    int e = 0;
    if (m > 0.0f) {
        e = int((__float_as_uint(m) >> 23) & 0xFF) - 127 - 14;
        e = max(-100, min(e, 113));
    }
    const float down = __uint_as_float(uint32_t(127 - e) << 23);
    const int order[8] = {0, 4, 2, 6, 1, 5, 3, 7};
    __half h[8];
    float ev = 0.0f, od = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        h[i] = __float2half_rn(x[order[i]] * down * (i < 4 ? 1.0f : 0.0625f));
        if (i < 4) ev += __half2float(h[i]); else od += __half2float(h[i]);
    }
    float cs = 1032.0f * ev + 1152.0f * od;
#pragma unroll
    for (int o = LPG / 2; o > 0; o >>= 1) cs += __shfl_xor_sync(0xffffffffu, cs, o);
    if (valid) {
        const int lc = b % LPG;
        int sb = b;   // groups of 64 / 32: 8-blocks in their natural order
        if (G == kGroup) {   // groups of 128: 8-block 4 c + i stored at 8 (i >> 1) + c + 4 (i & 1)
            const int ci = lc >> 2, ii = lc & 3;
            sb = (b & ~15) + 8 * (ii >> 1) + ci + 4 * (ii & 1);
        }
        *reinterpret_cast<uint4*>(out16_row + 8 * sb) = *reinterpret_cast<const uint4*>(h);
        if (lc == 0) *reinterpret_cast<float2*>(meta_row + 2 * (b / LPG)) = make_float2(-cs, __uint_as_float(uint32_t(127 + e) << 23));
    }
}

// The epilogue warps (warps 1..3; `hw` = 0..2): for each task, once the
// consumer warps have handed over their partial sums, sum the K phases and
// finish the task's outputs -- SwiGLU into h (gate/up pass) or the gate-scaled
// y (down pass) -- while the consumers go on with the next task's stages.
// Warp hw takes the task's columns hw, hw + 3, ...: all 64 rows of each, two
// per lane, so consecutive lanes store consecutive rows.
//
// Consumer warp (q, rb) lane (g, c) holds C rows 16 rb + sigma8(g) (r < 2)
// and + 8 (r >= 2) of the task's 64, columns nt * 8 + sigma8(2 c + (r & 1)).
//
// Then, with no wait on another CTA, the last writer finishes what needs
// several tasks' results (an atomic counter says who is last):
//   gate/up pass: a group of 128 rows of h is written by two tasks; the second
//     to finish a token column converts the group into the down pass's fp16
//     operands (act16_block), so no separate conversion pass is needed;
//   down pass: out[t] rows of one 64-row block get one contribution from the
//     shared expert and one per routed slot; the last of them writes
//     out = bf16(y_s + sum_j y_r[slot j]), summed in that fixed order (y_r
//     may also come from the caller, by slot: then the shared expert's
//     contribution is the only one).
template <int MODE, int G>
__device__ __forceinline__ void decode_epilogue(const DecodeParams& p, DecodeSmem* sm, const float* red, int hw,
                                                int lane) {
    uint32_t it_base = 0;
    bool waited = false;
    for (uint32_t tn = 0;; ++tn) {
        const int b = tn & 1;
        if (!mbar_wait(&sm->sfull[b], (tn >> 1) & 1, p.status)) return;
        const TaskInfo ti = sm->task[b];
        if (ti.kind < 0) return;
        if (!waited && (MODE == 1 || ti.kind == 1)) {   // per-slot data comes from the kernels before
            griddep_wait();
            waited = true;
        }
        // column values, lane l holding column l: in the down pass the token the
        // column belongs to and, for a routed column, its slot's gate
        float colgate = 1.0f;
        int coltok = 0, colslot = 0;
        if (MODE == 1 && lane < ti.count) {
            if (ti.kind == 1) {
                colslot = p.perm[ti.start + lane];
                coltok = colslot / p.k_top;
                colgate = p.gates[colslot];
            } else {
                coltok = ti.start + lane;
            }
        }
        if (!mbar_wait(&sm->red_full, tn & 1, p.status)) return;
        for (int col = hw; col < ti.count; col += DC_HELPERS) {
            const float gt = __shfl_sync(0xffffffffu, colgate, col);
            const int yrow = p.y_by_slot ? __shfl_sync(0xffffffffu, colslot, col) : ti.start + col;
            const int nt = col >> 3, cn = col & 7;
            const int jc = ((cn & 3) << 1) | (cn >> 2);             // sigma8(jc) == cn
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int i = half * 32 + lane;                      // row of the task's 64
                const int i16 = i & 15, ih = i16 & 7;
                const int g = ((ih & 3) << 1) | (ih >> 2);          // sigma8(g) == ih
                const int r = (i16 >= 8 ? 2 : 0) + (jc & 1);
                const int ln = g * 4 + (jc >> 1);
                // Phase qq holds the task's stages s with s % DC_KPH == (qq - it_base) % DC_KPH,
                // which depends on the tasks this CTA ran before: the partials are
                // summed in the order of that residue, so every output has the same
                // rounding whichever CTA computed it.
                float v0 = 0.0f, v1 = 0.0f;
#pragma unroll
                for (int rr = 0; rr < DC_KPH; ++rr) {
                    const int qq = int((uint32_t(rr) + it_base) % DC_KPH);
                    const float* o = red + (qq * DC_RB + (i >> 4)) * 32 * DC_RED_PITCH + ln * DC_RED_PITCH + nt * 8;
                    const float a0 = ld_shared_f32(o + r);
                    v0 = rr == 0 ? a0 : v0 + a0;
                    if (MODE == 0) {
                        const float a1 = ld_shared_f32(o + 4 + r);
                        v1 = rr == 0 ? a1 : v1 + a1;
                    }
                }
                const int n = ti.row0 + i;
                if (MODE == 0) {
                    const bf16 hv = __float2bfloat16_rn(silu_f32(v0) * v1);
                    if (ti.kind == 1) p.h_r[int64_t(ti.start + col) * p.n_rows_r + n] = hv;
                    else p.h_s[int64_t(ti.start + col) * p.n_rows_s + n] = hv;
                } else {
                    if (ti.kind == 1) p.y_r[int64_t(yrow) * p.n_rows_r + n] = v0 * gt;
                    else p.y_s[int64_t(ti.start + col) * p.n_rows_s + n] = v0;
                }
            }
        }
        // red[] and the task slot are free again (ti is a copy)
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&sm->red_empty);
            mbar_arrive(&sm->sempty[b]);
        }
        it_base += ti.n_stages;

        // ---- last writers: this warp's stores are made visible first ----
        const int n_mine = ti.count > hw ? (ti.count - hw + DC_HELPERS - 1) / DC_HELPERS : 0;
        const int mycol = hw + DC_HELPERS * lane;                    // lane j < n_mine: this warp's j-th column
        if (MODE == 0 && ti.kind == 1 && G != kGroup) {
            // groups of 64 / 32: the task's 64 rows are whole groups -- convert this
            // warp's columns at once, 4 per pass (8 lanes, the column's 8 8-blocks)
            const int F = p.n_rows_r;
            __threadfence();
            __syncwarp();
            for (int j0 = 0; j0 < n_mine; j0 += 4) {
                const int j = j0 + (lane >> 3);
                const bool valid = j < n_mine;
                const int64_t pos = ti.start + hw + DC_HELPERS * (valid ? j : j0);
                const int bb = (ti.row0 >> 3) + (lane & 7);                 // 8-block of the row
                const uint4 v = valid ? __ldcg(reinterpret_cast<const uint4*>(p.h_r + pos * F + 8 * bb))
                                      : make_uint4(0, 0, 0, 0);
                act16_block<G>(v, valid, p.h16 + pos * F, p.h_meta + pos * act16_meta_pitch(F, G), bb);
            }
        }
        if (MODE == 0 && ti.kind == 1 && G == kGroup) {
            const int F = p.n_rows_r, grp = ti.row0 >> 7;
            __threadfence();
            __syncwarp();
            bool last = false;
            if (lane < n_mine) last = atomicAdd(&p.hcnt[int64_t(ti.start + mycol) * (F >> 7) + grp], 1) == 1;
            uint32_t todo = __ballot_sync(0xffffffffu, last);
            if (todo) __threadfence();
            while (todo) {   // two columns per pass: lanes 0..15 and 16..31, one 8-block each
                const int j0 = __ffs(todo) - 1;
                todo &= todo - 1;
                int j1 = -1;
                if (todo) {
                    j1 = __ffs(todo) - 1;
                    todo &= todo - 1;
                }
                const int j = lane < 16 ? j0 : j1;
                const bool valid = j >= 0;
                const int64_t pos = ti.start + hw + DC_HELPERS * (valid ? j : j0);
                const int bb = grp * 16 + (lane & 15);                  // 8-block of the row
                const uint4 v = valid ? __ldcg(reinterpret_cast<const uint4*>(p.h_r + pos * F + 8 * bb))
                                      : make_uint4(0, 0, 0, 0);
                act16_block<G>(v, valid, p.h16 + pos * F, p.h_meta + pos * act16_meta_pitch(F, G), bb);
            }
        }
        if (MODE == 1 && p.out != nullptr) {
            const int D = p.n_rows_s, blk = ti.row0 >> 6;
            const int tok = __shfl_sync(0xffffffffu, coltok, mycol & 31);
            __threadfence();
            __syncwarp();
            bool last = false;
            if (lane < n_mine) last = atomicAdd(&p.ocnt[int64_t(tok) * (D >> 6) + blk], 1) == p.n_contrib;
            uint32_t todo = __ballot_sync(0xffffffffu, last);
            if (todo) __threadfence();
            while (todo) {
                const int j = __ffs(todo) - 1;
                todo &= todo - 1;
                const int64_t t = __shfl_sync(0xffffffffu, tok, j);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int n = ti.row0 + half * 32 + lane;
                    float a = __ldcg(p.y_s + t * D + n);
                    for (int js = 0; js < p.k_top; ++js) {
                        const int64_t yr = p.inv_perm ? int64_t(__ldcg(p.inv_perm + t * p.k_top + js)) : t * p.k_top + js;
                        a += __ldcg(p.y_r + yr * D + n);
                    }
                    p.out[t * D + n] = __float2bfloat16_rn(a);
                }
            }
        }
    }
}

template <int MODE, int G>   // MODE 0 = gate/up with SwiGLU, 1 = down; G = int4 group size (128, 64, 32)
__global__ void __launch_bounds__(DC_THREADS, 1) decode_ffn_kernel(
    const __grid_constant__ CUtensorMap tm_r0, const __grid_constant__ CUtensorMap tm_r1,
    const __grid_constant__ CUtensorMap tm_s0, const __grid_constant__ CUtensorMap tm_s1,
    const __grid_constant__ CUtensorMap tm_br, const __grid_constant__ CUtensorMap tm_cr,
    const __grid_constant__ CUtensorMap tm_bs, const __grid_constant__ CUtensorMap tm_g0,
    const __grid_constant__ CUtensorMap tm_g1, DecodeParams p) {
    constexpr int NST = dc_nstages(MODE), SLOT = dc_slot(MODE, G), C_OFF = dc_c_off(MODE);
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // 1024-byte alignment of the ring is required by the 128-byte swizzle
    unsigned char* base = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char* ring = base;
    float* sbuf = reinterpret_cast<float*>(ring + NST * SLOT);      // 2 scale buffers
    float* red = sbuf + 2 * p.scale_buf_floats;
    DecodeSmem* sm = reinterpret_cast<DecodeSmem*>(red + DC_RED_FLOATS);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < NST; ++i) { mbar_init(&sm->full[i], 1); mbar_init(&sm->empty[i], DC_RB); }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm->sfull[i], 1);
            mbar_init(&sm->sempty[i], DC_CONSUMERS + DC_HELPERS);
        }
        mbar_init(&sm->red_full, DC_CONSUMERS);
        mbar_init(&sm->red_empty, DC_HELPERS);
        fence_barrier_init();
    }
    griddep_launch_dependents();
    __syncthreads();

    // The shared expert's chunks (16 tokens each) follow from T alone, so its
    // tasks start before the routing step has finished; the routed chunk
    // list is read after the grid dependency wait.
    const int nbs = p.n_rows_s / DC_ROWS, nbr = p.n_rows_r / DC_ROWS;
    const int n_sh = int(ceil_div(p.T, 16));

    if (warp < 4) {
        // ------------------------------ producer ------------------------------
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" :: "n"(DC_PRODUCER_REGS));
        if (warp == 0 && lane == 0) {
            prefetch_tmap(&tm_r0); prefetch_tmap(&tm_r1); prefetch_tmap(&tm_s0); prefetch_tmap(&tm_s1);
            prefetch_tmap(&tm_br); prefetch_tmap(&tm_cr); prefetch_tmap(&tm_bs);
            prefetch_tmap(&tm_g0); prefetch_tmap(&tm_g1);
            uint32_t it = 0;
            bool ok = true, waited = false;
            int n_tasks = n_sh * nbs;   // grows by the routed tasks after the wait
            // With an RMSNorm the shared-expert tasks' token rows are the router's
            // xn: wait (bounded) until every router CTA has written its part.
            if (MODE == 0 && p.xn_ready != nullptr && !wait_counter(p.xn_ready, p.xn_ready_target, p.status))
                ok = false;
            for (uint32_t tn = 0; ok; ++tn) {
                const int t = atomicAdd(p.task_counter, 1);
                // Wait for the kernels before this one before the first load of
                // anything they write: the chunk list (routed tasks) and, in the
                // down pass, every task's input rows.  Only the gate/up pass's
                // shared-expert tasks (rows of the layer input) start before it.
                if (!waited && (MODE == 1 || t >= n_sh * nbs)) {
                    griddep_wait();
                    n_tasks += (*p.n_chunks - n_sh) * nbr;
                    waited = true;
                }
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
                ChunkEntry ce;
                if (t < n_sh * nbs) {
                    ci = t / nbs;
                    blk = t % nbs;
                    ce.expert = -1;
                    ce.start = ci * 16;
                    ce.count = min(16, p.T - ci * 16);
                } else {
                    const int u = t - n_sh * nbs;
                    ci = n_sh + u / nbr;
                    blk = u % nbr;
                    ce = p.chunks[ci];
                }
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
                if (ti.kind && G == kGroup) {
                    // one bulk copy per scale row, rows ldsc floats apart in
                    // shared memory so a warp's 8 rows fall in distinct banks
                    const int ng = ti.K / kGroup, ldsc = scale_row_floats(ng);
                    const uint32_t row_bytes = uint32_t(ng * 4);
                    float* dst = sbuf + b * p.scale_buf_floats;
                    mbar_arrive_expect_tx(&sm->sfull[b], (MODE == 0 ? 2 : 1) * DC_ROWS * uint32_t(ldsc * 4));
                    for (int m = 0; m < (MODE == 0 ? 2 : 1); ++m) {
                        float* d = dst + m * DC_ROWS * ldsc;
                        if (scale_rows_padded(ng))   // one box of ldsc x 64: columns past ng read as zeros
                            tma_load_2d(d, m ? &tm_g1 : &tm_g0, &sm->sfull[b], 0, grow);
                        else                         // 64 rows at pitch ng: a multiple of 16 bytes
                            bulk_load(d, (m ? p.sc1 : p.sc0) + int64_t(grow) * ng, DC_ROWS * row_bytes, &sm->sfull[b]);
                    }
                } else {   // shared expert, or groups of 64 / 32 (their scales come with the stages)
                    mbar_arrive(&sm->sfull[b]);
                }
                const int kbytes = ti.kind ? 128 : 64;   // tile x extent in elements (uint8 codes / bf16)
                // token rows of the chunk (8 routed, 16 shared) for the stage's K range,
                // in boxes of 64 K; routed stages also carry the rows' group (offset, scale) pairs
                const int kstage = (MODE == 0 ? 1 : 2) * kchunk;   // K values per stage
                const int nbox = kstage / 64;
                const uint32_t box_bytes = ti.kind ? 1024u : 2048u;
                // routed stages: the token groups' (offset, scale) pairs (8 rows x 4
                // groups of 128, or x the stage's groups of 64 / 32) and, for groups of
                // 64 / 32, the weight scales of the stage's groups (64 rows per matrix)
                constexpr int GPS = G == kGroup ? 4 : dc_kstage(MODE) / G;
                const uint32_t meta_bytes = 8u * 2u * GPS * 4u;
                const uint32_t scale_bytes = G == kGroup ? 0u : (MODE == 0 ? 2u : 1u) * DC_ROWS * GPS * 4u;
                const uint32_t b_bytes = uint32_t(nbox) * box_bytes + (ti.kind ? meta_bytes + scale_bytes : 0u);
                const CUtensorMap* mb = ti.kind ? &tm_br : &tm_bs;
                for (int s = 0; s < ti.n_stages; ++s, ++it) {
                    const uint32_t slot = it % NST;
                    if (!mbar_wait(&sm->empty[slot], ((it / NST) & 1) ^ 1, p.status)) { ok = false; break; }
                    unsigned char* st = ring + slot * SLOT;
                    if (MODE == 0) {
                        mbar_arrive_expect_tx(&sm->full[slot], DC_STAGE + b_bytes);
                        tma_load_2d(st, m0, &sm->full[slot], s * kbytes, grow);
                        tma_load_2d(st + DC_CHUNK, m1, &sm->full[slot], s * kbytes, grow);
                    } else {
                        // two consecutive K tiles of the one matrix; the second only if in range
                        const bool second = (2 * s + 1) * kchunk < ti.K;
                        mbar_arrive_expect_tx(&sm->full[slot], (second ? DC_STAGE : DC_CHUNK) + b_bytes);
                        tma_load_2d(st, m0, &sm->full[slot], 2 * s * kbytes, grow);
                        if (second) tma_load_2d(st + DC_CHUNK, m0, &sm->full[slot], (2 * s + 1) * kbytes, grow);
                    }
                    // one 3-D box: nbox 64-K chunks x the chunk's rows (chunks beyond K read zeros)
                    tma_load_3d(st + DC_B_OFF, mb, &sm->full[slot], 0, ti.start, s * kstage / 64);
                    if (ti.kind && G == kGroup)   // 4 groups from the stage's first, rounded down to a multiple of 4
                        tma_load_2d(st + C_OFF, &tm_cr, &sm->full[slot], 2 * ((s * kstage / kGroup) & ~3), ti.start);
                    if (ti.kind && G != kGroup) {   // exactly the stage's groups
                        tma_load_2d(st + C_OFF, &tm_cr, &sm->full[slot], 2 * s * GPS, ti.start);
                        unsigned char* sd = st + dc_s_off(MODE);
                        tma_load_2d(sd, &tm_g0, &sm->full[slot], s * GPS, grow);
                        if (MODE == 0) tma_load_2d(sd + DC_ROWS * GPS * 4, &tm_g1, &sm->full[slot], s * GPS, grow);
                    }
                }
            }
            // this grid completes only after the kernels before it
            if (!waited) griddep_wait();
            // wind down: wait (bounded) for every stage still in flight to land
            for (uint32_t i = 0; i < NST && i < it; ++i) {
                const uint32_t j = it - 1 - i;
                mbar_wait(&sm->full[j % NST], (j / NST) & 1, nullptr);
            }
        } else if (warp >= 1 && warp <= DC_HELPERS) {
            decode_epilogue<MODE, G>(p, sm, red, warp - 1, lane);
        }
        return;
    }

    // ------------------------------ consumers ------------------------------
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" :: "n"(DC_CONSUMER_REGS));
    const int ci = warp - 4;
    const int rb = ci % DC_RB, q = ci / DC_RB;   // a stage's DC_RB warps sit on different sub-partitions
    const int g = lane >> 2, c = lane & 3;
    const int row_a = 16 * rb + sigma8(g), row_b = row_a + 8;
    uint32_t it_base = 0;
    bool waited = false;
    for (uint32_t tn = 0;; ++tn) {
        const int b = tn & 1;
        if (!mbar_wait(&sm->sfull[b], (tn >> 1) & 1, p.status)) break;
        const TaskInfo ti = sm->task[b];
        if (ti.kind < 0) break;
        // everything but the shared expert's tokens (the layer input) comes
        // from the kernels before this one
        if (!waited && (MODE == 1 || ti.kind == 1)) {
            griddep_wait();
            waited = true;
        }
        const float* sc = sbuf + b * p.scale_buf_floats;

        const int nt_used = ti.count > 8 ? 2 : 1;

        float acc0[DC_NT][4], acc1[DC_NT][4];
#pragma unroll
        for (int nt = 0; nt < DC_NT; ++nt)
#pragma unroll
            for (int r = 0; r < 4; ++r) { acc0[nt][r] = 0.f; acc1[nt][r] = 0.f; }

        bool ok = true;
        if (ti.kind == 1) {
            // routed chunks hold at most 8 tokens: one n-tile
            if constexpr (G == kGroup)
                ok = consume_int4<MODE, G>(ti, sm, ring, sc, it_base, q, lane, row_a, row_b, p.f16_magic_lo,
                                           p.f16_magic_hi, acc0[0], acc1[0], p.status);
            else
                ok = consume_int4_qm<MODE, G>(ti, sm, ring, it_base, q, lane, row_a, row_b, p.f16_magic_lo,
                                              p.f16_magic_hi, acc0[0], acc1[0], p.status);
        } else {
            // ---------------- bf16 weights (shared expert): 64 K per tile ----------------
            // thread c takes the 8-blocks c and c + 4 of each 64-K tile, of the
            // weight rows and of its token rows nt * 8 + sigma8(g) (in the stage)
            constexpr int UPS = MODE == 0 ? 1 : 2;           // 64-K units per stage
            const int n_units = ti.K / 64;
            const int trow = sigma8(g);
            for (int s = first_stage(q, it_base); s < ti.n_stages; s += DC_KPH) {
                const uint32_t it = it_base + s;
                const uint32_t slot = it % NST;
                if (!mbar_wait(&sm->full[slot], (it / NST) & 1, p.status)) { ok = false; break; }
                const unsigned char* st = ring + slot * SLOT;
#pragma unroll
                for (int ul = 0; ul < UPS; ++ul) {
                    const int U = s * UPS + ul;
                    if (U >= n_units) break;
                    const unsigned char* ta = st + (MODE == 0 ? 0 : ul * DC_CHUNK);
                    const unsigned char* tb = st + DC_B_OFF + ul * 2048;   // 16 token rows x 64 K
                    uint4 xc[DC_NT][2];
#pragma unroll
                    for (int nt = 0; nt < DC_NT; ++nt)
#pragma unroll
                        for (int h2 = 0; h2 < 2; ++h2) xc[nt][h2] = ld_shared_v4(swz(tb, nt * 8 + trow, c + 4 * h2));
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        const int j = c + 4 * h2;
                        const uint4 wa = ld_shared_v4(swz(ta, row_a, j));
                        const uint4 wb = ld_shared_v4(swz(ta, row_b, j));
                        uint4 va = make_uint4(0, 0, 0, 0), vb = va;
                        if (MODE == 0) { va = ld_shared_v4(swz(st + DC_CHUNK, row_a, j)); vb = ld_shared_v4(swz(st + DC_CHUNK, row_b, j)); }
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            // MMA h takes K values 8 j + 4 h .. + 3 of the rows (natural order):
                            // its k-slots 2c, 2c+1 get the first pair, 2c+8, 2c+9 the second
                            const uint32_t a0 = h == 0 ? wa.x : wa.z, a2 = h == 0 ? wa.y : wa.w;
                            const uint32_t a1 = h == 0 ? wb.x : wb.z, a3 = h == 0 ? wb.y : wb.w;
#pragma unroll
                            for (int nt = 0; nt < DC_NT; ++nt) {
                                if (nt >= nt_used) break;
                                const uint32_t b0 = h == 0 ? xc[nt][h2].x : xc[nt][h2].z;
                                const uint32_t b1 = h == 0 ? xc[nt][h2].y : xc[nt][h2].w;
                                mma_bf16_16816(acc0[nt], a0, a1, a2, a3, b0, b1);
                            }
                            if (MODE == 0) {
                                const uint32_t u0 = h == 0 ? va.x : va.z, u2 = h == 0 ? va.y : va.w;
                                const uint32_t u1 = h == 0 ? vb.x : vb.z, u3 = h == 0 ? vb.y : vb.w;
#pragma unroll
                                for (int nt = 0; nt < DC_NT; ++nt) {
                                    if (nt >= nt_used) break;
                                    const uint32_t b0 = h == 0 ? xc[nt][h2].x : xc[nt][h2].z;
                                    const uint32_t b1 = h == 0 ? xc[nt][h2].y : xc[nt][h2].w;
                                    mma_bf16_16816(acc1[nt], u0, u1, u2, u3, b0, b1);
                                }
                            }
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm->empty[slot]);
            }
        }
        if (!ok) break;

        // ---- hand the partial sums to the epilogue warps ----
        if (!mbar_wait(&sm->red_empty, (tn & 1) ^ 1, p.status)) break;
        float* my = red + (q * DC_RB + rb) * 32 * DC_RED_PITCH + lane * DC_RED_PITCH;
#pragma unroll
        for (int nt = 0; nt < DC_NT; ++nt)
#pragma unroll
            for (int r = 0; r < 4; ++r) { my[nt * 8 + r] = acc0[nt][r]; my[nt * 8 + 4 + r] = acc1[nt][r]; }
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&sm->red_full);
            mbar_arrive(&sm->sempty[b]);
        }
        it_base += ti.n_stages;
    }
}

// This file's copy of the wait limit (see c_wait_limit).
moe_status set_wait_limit_decode(uint32_t cycles) {
    return cuda_status(cudaMemcpyToSymbol(c_wait_limit, &cycles, sizeof(cycles)));
}

// shared-expert chunks of 16 tokens, routed ones of 8 (at most one partial chunk per expert)
int decode_max_chunks(int T, int k, int E) { return int(ceil_div(T, 16)) + int(ceil_div(int64_t(T) * k, 8)) + E; }

int decode_task_rows() { return DC_ROWS; }

// scale_row_floats(K / 128) if the task scales load as one padded box, else 0
int decode_scale_pitch(int K) { return scale_rows_padded(K / kGroup) ? scale_row_floats(K / kGroup) : 0; }

// floats of one task's int4 scale buffer: gate and up rows (mode 0) or down
// rows, each row padded to scale_row_floats(K / 128)
int decode_scale_floats(int mode, int K) { return (mode == 0 ? 2 : 1) * DC_ROWS * scale_row_floats(K / kGroup); }

size_t decode_smem_bytes(int mode, int scale_buf_floats, int G) {
    return 1024 + size_t(dc_nstages(mode)) * dc_slot(mode, G) + 2 * size_t(scale_buf_floats) * 4 +
           DC_RED_FLOATS * 4 + sizeof(DecodeSmem);
}

// groups of G per stage of a routed int4 task (4 for groups of 128: the
// (offset, scale) box is 4 groups from the stage's first, rounded down)
int decode_groups_per_stage(int mode, int G) { return G == kGroup ? 4 : dc_kstage(mode) / G; }

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

// 2-D map over a row-major [rows, inner] matrix of 1-, 2- or 4-byte elements;
// box = box_inner x box_rows.
bool make_tmap_2d(CUtensorMap* m, const void* base, int elem_bytes, uint64_t inner, uint64_t rows,
                  uint32_t box_inner, uint32_t box_rows, bool swizzle128) {
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return false;
    const uint64_t esz = uint64_t(elem_bytes);
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner * esz};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    const CUtensorMapDataType dt = elem_bytes == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                   : elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                     : CU_TENSOR_MAP_DATA_TYPE_UINT8;
    CUresult r = fn(m, dt, 2,
                    const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 3-D map over fp16/bf16 token rows [rows, K] seen as (64 K values, row,
// 64-K chunk): a box of box_rows rows x nbox chunks lands as nbox tiles of
// box_rows x 128 bytes, each with the 128-byte swizzle.
bool make_tmap_rows_3d(CUtensorMap* m, const void* base, uint64_t K, uint64_t rows, uint32_t box_rows,
                       uint32_t nbox) {
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {64, rows, K / 64};
    cuuint64_t strides[2] = {K * 2, 128};
    cuuint32_t box[3] = {64, box_rows, nbox};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

moe_status launch_decode_ffn(int mode, int G, const DecodeMaps& maps, const DecodeParams& prm,
                             cudaStream_t stream) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const size_t smem = decode_smem_bytes(mode, prm.scale_buf_floats, G);
    auto kern = mode == 0 ? (G == 32 ? decode_ffn_kernel<0, 32> : G == 64 ? decode_ffn_kernel<0, 64> : decode_ffn_kernel<0, 128>)
                          : (G == 32 ? decode_ffn_kernel<1, 32> : G == 64 ? decode_ffn_kernel<1, 64> : decode_ffn_kernel<1, 128>);
    if (allow_max_smem(kern) != MOE_OK) return MOE_ERR_CUDA;
    return launch_pdl(kern, dim3(sms), dim3(DC_THREADS), smem, stream, maps.r0, maps.r1, maps.s0, maps.s1, maps.br,
                      maps.cr, maps.bs, maps.g0, maps.g1, prm);
}


}  // namespace moe

namespace moe {

// ---------------------------------------------------------------------------
// fp16 operands for the int4 MMAs.
//
// One CTA per output row of a bf16 matrix (the tokens x gathered into
// expert-sorted position order, or the routed experts' hidden h, already by
// position).  Each group of G values (the int4 group size: G / 8 threads, one
// 8-block each) gets its own power of two:
//   scale = 2^-e with e chosen from the group's largest magnitude so that the
//           scaled values stay below 2^15 (fp16 keeps every bf16 value exactly
//           in that range, down to 2^-24 of its largest);
//   out16  every 8-block stored as x0 x4 x2 x6 x1/16 x5/16 x3/16 x7/16 (scaled)
//          -- the K order and the 1/16 factors the int4 unpacking expects --
//          and, for groups of 128 only, inside each group 8-block 4 c + i
//          (c, i = 0..3) stored at 8-block 8 (i >> 1) + c + 4 (i & 1), so that
//          the four threads c of an MMA fragment read distinct shared-memory
//          banks (the quarter-by-quarter MMAs of smaller groups read the
//          8-blocks in their natural order without conflicts);
//   meta   per group, the pair (offset, 2^e): offset = -(1032 * sum of
//          the even-position stored values + 1152 * sum of the odd-position
//          stored values), what the unpacked codes (1032 + q and 1152 + 16 q)
//          add to a dot product, and 2^e, which undoes the scaling on the
//          group's partial sum; rows of act16_meta_pitch(cols, G) floats.
// ---------------------------------------------------------------------------
template <int G>
__global__ void __launch_bounds__(256) act16_kernel(const bf16* __restrict__ in, int cols,
                                                    const int32_t* __restrict__ src_perm, int k,
                                                    __half* __restrict__ out16, float* __restrict__ meta) {
    griddep_launch_dependents();
    griddep_wait();   // the rows (h) or the permutation come from the kernels before
    const int64_t r = blockIdx.x;
    // out row r: input row src_perm[r] / k (tokens into expert-sorted positions), else row r
    const bf16* row = in + (src_perm ? int64_t(src_perm[r] / k) : r) * cols;
    const int nblk = cols / 8;   // a multiple of 16: a group's threads are all valid or all not
    for (int b0 = 0; b0 < nblk; b0 += 256) {
        const int b = b0 + threadIdx.x;
        const bool valid = b < nblk;
        const uint4 v = valid ? *reinterpret_cast<const uint4*>(row + 8 * b) : make_uint4(0, 0, 0, 0);
        act16_block<G>(v, valid, out16 + r * cols, meta + r * act16_meta_pitch(cols, G), b);
    }
}

moe_status launch_act16(const bf16* in, int64_t rows, int cols, int G, const int32_t* src_perm, int k,
                        __half* out16, float* meta, cudaStream_t stream) {
    if (rows == 0) return MOE_OK;
    auto kern = G == 32 ? act16_kernel<32> : G == 64 ? act16_kernel<64> : act16_kernel<128>;
    return launch_pdl(kern, dim3(unsigned(rows)), dim3(256), 0, stream, in, cols, src_perm, k, out16, meta);
}

}  // namespace moe
