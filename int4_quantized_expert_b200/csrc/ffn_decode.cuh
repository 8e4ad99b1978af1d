// Host/device interface of the weight-streaming (decode) expert FFN kernels.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace moe {

// One chunk of <= 16 tokens of one expert (expert -1 = the shared expert).
// For the shared expert `start` is the first token; for a routed expert it is
// the first position in the expert-sorted slot order.
struct ChunkEntry {
    int32_t expert;
    int32_t start;
    int32_t count;
    int32_t pad;
};

struct DecodeParams {
    int32_t n_rows_r;       // output rows of each routed matrix (F for gate/up, D for down)
    int32_t n_rows_s;       // output rows of each shared matrix (F_shared for gate/up, D for down)
    int32_t K_r, K_s;       // reduction lengths (routed, shared)
    int32_t k_top;
    int32_t scale_buf_floats;
    const ChunkEntry* chunks;
    const int32_t* n_chunks;
    const int32_t* n_shared_chunks;
    const int32_t* perm;    // sorted position -> slot (t * k + j)
    const float* gates;     // per slot
    const bf16* b_r;        // B rows, routed: gate/up: tokens (x, fragment order); down: h rows by position
    int32_t ldb_r;
    const bf16* b_s;        // B rows, shared: gate/up: tokens; down: shared h rows
    int32_t ldb_s;
    const float* sc0;       // routed scales: gate/up: gate; down: down   ([E * rows, K / 128])
    const float* sc1;       // routed scales: gate/up: up
    bf16* h_r;              // gate/up outputs (fragment order): routed [T*k, F], shared [T, F_shared]
    bf16* h_s;
    float* y_r;             // down outputs: routed gate * y [T*k, D] (by position), shared [T, D]
    float* y_s;
    int32_t* task_counter;  // zeroed by the plan kernel
    int32_t* status;        // device status word
};

struct DecodeMaps {
    CUtensorMap r0, r1, s0, s1;   // routed tile maps (int4 codes) and shared maps (bf16)
};

bool make_tmap_2d(CUtensorMap* m, const void* base, bool bf16_elems, uint64_t inner, uint64_t rows,
                  uint32_t box_inner, uint32_t box_rows, bool swizzle128);
int decode_max_chunks(int T, int k, int E);
size_t decode_smem_bytes(int scale_buf_floats);
moe_status launch_decode_plan(const int32_t* counts, const int32_t* offsets, int T, int E, void* chunks,
                              int32_t* n_chunks, int32_t* n_shared, int32_t* counters, cudaStream_t stream);
moe_status launch_decode_ffn(int mode, const DecodeMaps& maps, const DecodeParams& prm, cudaStream_t stream);
moe_status launch_combine(const float* y_s, const float* y_r, const int32_t* inv_perm, int T, int D, int k,
                          bf16* out, cudaStream_t stream);

}  // namespace moe
