// tcgen05 (5th-generation tensor core) grouped GEMMs for many tokens per
// expert: host/device interface.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "ffn_decode.cuh"

namespace moe {

enum TcMode : int32_t {
    TC_GATEUP_INT4 = 0,   // routed gate/up, int4 weights dequantized on chip, SwiGLU -> h (bf16)
    TC_DOWN_INT4 = 1,     // routed down, int4 weights, gate-scaled fp32 y per slot
    TC_GATEUP_BF16 = 2,   // shared gate/up, bf16 weights by TMA, SwiGLU -> h (bf16)
    TC_DOWN_BF16 = 3,     // shared down, bf16 weights -> fp32 y_s [T, D]
    TC_GATEUP_FP8 = 4,    // routed gate/up, e4m3 weights and tokens by TMA, row scales -> h (bf16)
    TC_DOWN_FP8 = 5       // routed down, e4m3 weights and h rows, row scales, gate-scaled fp32 y
};

struct TcParams {
    int32_t K;                 // reduction length
    int32_t n_rows;            // output features of one expert's matrix (F or D)
    int32_t n_fblocks;         // feature blocks per token chunk (64 features for gate/up, 128 otherwise)
    const ChunkEntry* chunks;  // token chunks of <= 256 (shared expert's first)
    const int32_t* n_chunks;   // [0] all chunks, [1] the shared expert's
    int32_t routed;            // 1: chunks [n_shared, n_all); 0: chunks [0, n_shared)
    const float* s0;           // weight scales (gate or down): int4 [E * rows, K / group]; e4m3 [E * rows]
    const float* s1;           // weight scales (up)
    const float* tok_scale;    // e4m3 modes: row scale of each token row of B (by slot position)
    bf16* h_out;               // gate/up output rows [*, n_rows] (row = slot position or token)
    float* y_out;              // down output: routed [slots, n_rows] by slot t * k + j; shared [T, n_rows]
    const float* gates;        // per slot
    const int32_t* perm;       // position -> slot
    bf16* out;                 // routed down with one slot per token: the layer output [T, n_rows]
    const float* y_r;          // ... and the shared expert's y_s it adds
    const int32_t* inv_perm;   // slot -> position
    int32_t k_top;
    int32_t group_shift;       // int4 modes: log2 of the group size (7, 6 or 5: groups of 128, 64, 32)
    uint32_t bf16_magic;       // kBf16Magic, passed at run time so the int4 converters hold it in a register
    int32_t* status;
};

struct TcMaps {
    CUtensorMap b;       // tokens: bf16 [rows, K], box 64 x 256, 128-byte swizzle
    CUtensorMap b_small; // the same tensor, box 64 x TC_SMALL_TOKENS (e4m3: 128 x ...)
    CUtensorMap a0, a1;  // int4 codes uint8 [E * rows, K / 2], box 32 x 64; bf16 weights, box 64 x 16;
                         // or e4m3 weights uint8 [E * rows, K], box 128 x 16
};

constexpr int TC_BLOCK_TOKENS = 256;
// Chunks of at most this many tokens load their token tiles with a box of
// this many rows (the MMAs read only the chunk's rows).
constexpr int TC_SMALL_TOKENS = 64;

size_t tc_smem_bytes();
moe_status launch_tc_gemm(int mode, const TcMaps& maps, const TcParams& prm, cudaStream_t stream);
moe_status launch_quantize_fp8_scatter(const bf16* x, int64_t rows, int cols, float scale_ub,
                                       const int32_t* inv_perm, int k, uint8_t* q, float* scales,
                                       cudaStream_t stream);
moe_status launch_combine_slots(const float* y_s, const float* y, int64_t T, int D, int k, bf16* out,
                                cudaStream_t stream);
moe_status launch_gather_rows(const bf16* x, const int32_t* perm, int64_t n, int k, int D, bf16* out,
                              cudaStream_t stream);

moe_status set_wait_limit_tc(uint32_t cycles);

}  // namespace moe
