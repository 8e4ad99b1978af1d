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
    int32_t T;              // tokens (the shared expert's chunks are the 16-token runs of 0..T-1)
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
    const bf16* b_r;        // B rows, routed, by sorted position (fp16 bits; see act16): tokens or h rows
    int32_t ldb_r;
    const bf16* b_s;        // B rows, shared: gate/up: tokens; down: shared h rows
    int32_t ldb_s;
    const float* sc0;       // routed scales: gate/up: gate; down: down   ([E * rows, K / 128])
    const float* sc1;       // routed scales: gate/up: up
    const float* corr_r;    // routed B rows (by position): group offsets negc [rows, K_r / 128] (see act16)
    const float* rscale_r;  // routed B rows (by position): power-of-two scale of each row
    bf16* h_r;              // gate/up outputs: routed [T*k, F] (natural order), shared [T, F_shared] (fragment order)
    bf16* h_s;
    float* y_r;             // down outputs: routed gate * y [T*k, D] (by position), shared [T, D]
    float* y_s;
    const bf16* zero_row;   // zeros, at least max(K_r, K_s) long: B row of a token that does not exist
    const float* zero_corr; // zeros, at least K_r / 128 long
    int32_t* task_counter;  // zeroed by the routing step
    int32_t* status;        // device status word
};

// Extra outputs of the routing step used by the weight-streaming FFN.
struct RoutePrep {
    bf16* x_frag;         // x in bf16 fragment order [T, D] (shared expert)
    ChunkEntry* chunks;   // task list
    int32_t* n_chunks;    // [0] all chunks, [1] the shared expert's
    int32_t chunk_tokens;         // tokens per shared-expert chunk (16 weight streaming, 256 tensor cores)
    int32_t routed_chunk_tokens;  // tokens per routed-expert chunk (8 weight streaming, 256 tensor cores)
    int32_t* zero_words;  // zeroed by the bucketing kernel (or null)
    int32_t n_zero;
    bool router_after_kernel;   // the router may start while the kernel before it runs
};

struct DecodeMaps {
    CUtensorMap r0, r1, s0, s1;   // routed tile maps (int4 codes) and shared maps (bf16)
};

bool make_tmap_2d(CUtensorMap* m, const void* base, bool bf16_elems, uint64_t inner, uint64_t rows,
                  uint32_t box_inner, uint32_t box_rows, bool swizzle128);
int decode_max_chunks(int T, int k, int E);
size_t decode_smem_bytes(int scale_buf_floats);
int decode_task_rows();
int decode_scale_floats(int mode, int K);
moe_status launch_decode_ffn(int mode, const DecodeMaps& maps, const DecodeParams& prm, cudaStream_t stream);
moe_status launch_route(const bf16* x, int T, int D, const bf16* wr, const float* bias, int E, int k,
                        int32_t* ids, float* gates, int32_t* counts, int32_t* offsets, int32_t* perm,
                        int32_t* inv_perm, const RoutePrep* prep, cudaStream_t stream, cudaEvent_t between);
moe_status launch_act16(const bf16* in, int64_t rows, int cols, const int32_t* src_perm, int k, __half* out16,
                        float* negc, float* rscale, cudaStream_t stream);
moe_status launch_combine(const float* y_s, const float* y_r, const int32_t* inv_perm, int T, int D, int k,
                          bf16* out, cudaStream_t stream);

}  // namespace moe
