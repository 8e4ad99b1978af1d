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
    uint32_t f16_magic_lo;  // kF16MagicLo, kF16MagicHi: passed at run time so the int4 unpacking
    uint32_t f16_magic_hi;  // holds them in registers (one LOP3 per two codes)
    const ChunkEntry* chunks;
    const int32_t* n_chunks;
    const int32_t* perm;    // sorted position -> slot (t * k + j)
    const float* gates;     // per slot
    const float* sc0;       // routed scales: gate/up: gate; down: down   ([E * rows, K / 128])
    const float* sc1;       // routed scales: gate/up: up
    bf16* h_r;              // gate/up outputs: routed [T*k, F] by position, shared [T, F_shared]
    bf16* h_s;
    float* y_r;             // down outputs: routed gate * y [T*k, D] by position, shared [T, D]
    float* y_s;
    __half* h16;            // gate/up pass: the down pass's fp16 operands of h [T*k, F] (act16 format)
    float* h_meta;          //   and their per-group (offset, scale) pairs [T*k, act16_meta_pitch(F)]
    int32_t* hcnt;          //   token columns written per (position, group of 128 rows) [T*k, F / 128], zeroed
    bf16* out;              // down pass: the layer output [T, D] (null: none)
    const int32_t* inv_perm;  // slot -> position of y_r's rows (null: y_r is stored by slot)
    int32_t* ocnt;          //   contributions written per (token, block of 64 rows) [T, D / 64], zeroed
    int32_t n_contrib;      //   contributions before the last one (k, or 0 when y_r comes from the caller)
    int32_t y_by_slot;      // down pass: routed y rows stored by slot (t * k + j) instead of by position
    const int32_t* xn_ready;  // gate/up pass with an RMSNorm: the router CTAs that have written the
    int32_t xn_ready_target;  //   normalized x the shared-expert tasks read (they start before the routing ends)
    int32_t* task_counter;  // cleared with the status word
    int32_t* status;        // device status word
};

// Extra outputs of the routing step used by the weight-streaming FFN.
struct RoutePrep {
    ChunkEntry* chunks;   // task list
    int32_t* n_chunks;    // [0] all chunks, [1] the shared expert's
    int32_t chunk_tokens;         // tokens per shared-expert chunk (16 weight streaming, 256 tensor cores)
    int32_t routed_chunk_tokens;  // tokens per routed-expert chunk (8 weight streaming, 256 tensor cores)
    int32_t* zero_words;  // zeroed by the bucketing kernel (or null)
    int32_t n_zero;
    bool router_after_kernel;   // the router may start while the kernel before it runs
    float* router_part;         // router_partial_floats(T, D, E, rms) floats for a K-split router (or null)
    int32_t* router_tile_cnt;   // ceil(T / 16) counters, zero on entry (with router_part)
    const bf16* rms_weight;     // RMSNorm of x in the router (gamma [D]), or null
    float rms_eps;
    bf16* xn;                   // ... and where the router writes it, bf16 [T, D]
    int32_t* xn_ready;          // ... counted by each router CTA once its part of xn is written (or null)
    int32_t* status;            // device status word: out-of-range given expert ids are reported there
    int32_t* bucket_hist;       // bucket_blocks(T * k) * E ints for bucketing many slots over several CTAs (or null)
};

// TMA maps of one weight-streaming launch:
//   r0, r1  routed int4 codes uint8 [E * rows, K / 2] (gate, up; or down), box 128 B x 64 rows, 128-B swizzle
//   s0, s1  shared bf16 weights, box 64 x 64, 128-B swizzle
//   br      routed token rows, fp16 [T * k, K] by position (act16 layout), 3-D box of 8 rows x the
//           stage's 64-K chunks (make_tmap_rows_3d)
//   cr      their per-group (offset, scale) pairs, fp32 [T * k, act16_meta_pitch(K, G)], box
//           2 x decode_groups_per_stage floats x 8 rows
//   bs      shared-expert token rows, bf16 [T, K] (x, or the shared h), 3-D box of 16 rows x chunks
//   g0, g1  routed int4 scales fp32 [E * rows, K / G] (gate, up; or down): groups of 128, box
//           scale_row_floats(K / 128) x 64 (when K / 128 is a multiple of 4) for a task's rows;
//           groups of 64 / 32, box (the stage's groups) x 64 rows, loaded with each stage
struct DecodeMaps {
    CUtensorMap r0, r1, s0, s1, br, cr, bs, g0, g1;
};

// Row pitch (floats) of act16's per-group (offset, scale) pairs: K / G
// groups (G = 128, 64 or 32) rounded up to 4, two floats each, so every row
// starts on 32 bytes.
__host__ __device__ inline int act16_meta_pitch(int cols, int G) { return int(ceil_div(cols / G, 4) * 8); }

bool make_tmap_2d(CUtensorMap* m, const void* base, int elem_bytes, uint64_t inner, uint64_t rows,
                  uint32_t box_inner, uint32_t box_rows, bool swizzle128);
bool make_tmap_rows_3d(CUtensorMap* m, const void* base, uint64_t K, uint64_t rows, uint32_t box_rows,
                       uint32_t nbox);
int decode_scale_pitch(int K);
int decode_max_chunks(int T, int k, int E);
int router_ksplit(int T, int D, bool rms);
size_t router_partial_floats(int T, int D, int E, bool rms);
size_t decode_smem_bytes(int mode, int scale_buf_floats, int G);
int decode_groups_per_stage(int mode, int G);
int decode_task_rows();
int decode_scale_floats(int mode, int K);
moe_status launch_decode_ffn(int mode, int G, const DecodeMaps& maps, const DecodeParams& prm,
                             cudaStream_t stream);
moe_status launch_route(const bf16* x, int T, int D, const bf16* wr, const float* bias, int E, int k,
                        int32_t* ids, float* gates, int32_t* counts, int32_t* offsets, int32_t* perm,
                        int32_t* inv_perm, const RoutePrep* prep, cudaStream_t stream, cudaEvent_t between,
                        cudaEvent_t ev_scan = nullptr, cudaEvent_t ev_place = nullptr);
// The bucketing step alone, from given expert ids [T, k] (counts, offsets,
// the stable permutation and, with `prep`, the FFN's chunk list).
moe_status launch_bucket(const int32_t* ids, int T, int k, int E, int32_t* counts, int32_t* offsets, int32_t* perm,
                         int32_t* inv_perm, const RoutePrep* prep, cudaStream_t stream, cudaEvent_t ev_scan = nullptr,
                         cudaEvent_t ev_place = nullptr);
// CTAs the bucketing of n slots takes (0: one CTA, bucket_kernel)
int bucket_blocks(int64_t n_slots);
moe_status launch_act16(const bf16* in, int64_t rows, int cols, int G, const int32_t* src_perm, int k,
                        __half* out16, float* meta, cudaStream_t stream);

moe_status set_wait_limit_decode(uint32_t cycles);

}  // namespace moe
