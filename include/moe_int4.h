/*
 * moe_int4.h -- C ABI of libmoe_int4: a Llama-4-style mixture-of-experts FFN
 * layer with int4 group-quantized (or FP8 row-quantized) routed experts and a
 * bf16 shared expert, for NVIDIA B200 (sm_100a).
 *
 * Sources of the operations (web pages, cited by title and section):
 *   [P1] "1 卡跑通 Llama 4：从本地部署到多模态推理的完整路径" (discosf.com):
 *        "混合专家路由" (MoE.forward: router scores, torch.topk, scatter_add_
 *        of the score-weighted expert outputs, plus the shared expert) and
 *        "FP8 / Int4 混合量化" (int4_row_quantize).
 *   [P2] "Meta Llama Models Llama 4 单卡量化推理与选型指南" (lshu.cn):
 *        "量化环节做了什么" (bmm_nt: FP8 row-wise weights with per-row
 *        activation quantization, or int4 group-128 weights with zero points
 *        equal to zero; activations stay bf16; a smaller group_size named as
 *        the int4 path's likely next step).
 *   [P4] "Llama" (illegalscreed.cn): introduction (dense and MoE layers
 *        alternate; 16 routed experts, 128 routed + 1 shared).
 *   [P5] "Llama 开源模型系列" (docs.ifdog.com): "MoE 架构详解" (router =
 *        linear layer, top-1 of 16 / top-8 of 128), "SwiGLU：门控激活的数学"
 *        and "RMSNorm：为什么去掉减均值也能工作" (the block's normalization).
 *
 * Conventions for every entry point:
 *   - Pointers named as device pointers must point to device memory of the
 *     current CUDA device; the caller owns all memory.  The library allocates
 *     no device memory, keeps no pointer after a call returns, and never
 *     synchronizes unless the function says so.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  All work is enqueued on it in order.
 *   - The return value reports argument errors (nothing is launched) and
 *     launch errors.  Faults inside kernels surface at the caller's next
 *     synchronization, as with any CUDA call.
 *   - Device pointers must be 16-byte aligned.  Matrices are row-major and
 *     dense (no row padding).  bf16 is IEEE bfloat16 stored in 2 bytes.
 *   - Weights are stored "nt" ([P2] bmm_nt): a projection from K to N
 *     features is a matrix W[N, K] with K contiguous, applied as x * W^T.
 */
#ifndef MOE_INT4_H
#define MOE_INT4_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,          /* null pointer, bad enum, misaligned pointer */
    MOE_ERR_UNSUPPORTED_SHAPE = 2,    /* a size outside the supported range */
    MOE_ERR_WORKSPACE_TOO_SMALL = 3,  /* workspace_bytes < moe_ffn_workspace_size() */
    MOE_ERR_CUDA = 4,                 /* a CUDA runtime call or launch failed */
    MOE_ERR_TIMEOUT = 5               /* a device-side wait gave up (device status word) */
} moe_status;

typedef enum { MOE_DTYPE_BF16 = 0, MOE_DTYPE_FP32 = 1 } moe_dtype;

typedef enum {
    MOE_WEIGHTS_INT4_G128 = 0,  /* int4 codes, two per byte, fp32 scale per group of K
                                   (128 by default; 64 or 32 per moe_layer_desc.group_size) */
    MOE_WEIGHTS_FP8_ROW = 1     /* e4m3 codes, fp32 scale per row */
} moe_weight_format;

typedef enum {
    MOE_PATH_AUTO = 0,     /* chosen from T, k and E */
    MOE_PATH_DECODE = 1,   /* weight-streaming kernels, for few tokens per expert */
    MOE_PATH_PREFILL = 2   /* tcgen05 tensor-core tiles, for many tokens per expert */
} moe_path;

/* Human-readable name of a status code (static string). */
MOE_API const char* moe_status_string(moe_status status);

/* Version of this ABI (bumped on any incompatible change). */
MOE_API int32_t moe_abi_version(void);

/*
 * moe_quantize_int4 -- int4_row_quantize ([P1] "FP8 / Int4 混合量化").
 * For each row of w and each group of `group_size` consecutive columns:
 *   scale = max(max|w|, 1e-6) / 8;  q = clamp(round_half_even(w / scale), -8, 7)
 * with IEEE fp32 division.  Codes are packed two per byte, the even column in
 * the low nibble, as two's-complement nibbles.
 *   w       device, fp32 [rows, cols]
 *   codes   device, uint8 [rows, cols / 2]       (output)
 *   scales  device, fp32 [rows, cols / group_size] (output)
 * Requires group_size 128, 64 or 32 (the smaller groups: [P2]'s next step),
 * cols % 128 == 0, rows >= 0 (0 = no-op).
 */
MOE_API moe_status moe_quantize_int4(const float* w, int64_t rows, int64_t cols, int32_t group_size,
                             uint8_t* codes, float* scales, void* stream);

/*
 * moe_quantize_fp8_rows -- per-row e4m3 quantization ([P2] "量化环节做了什么",
 * quantize_fp8_per_row).  In fp32, for each row r < num_valid_rows:
 *   a = min(max_c |x[r,c]|, scale_ub);  s = max(a, 1e-12) / 448;
 *   q[r,c] = e4m3(x[r,c] / s)   (IEEE division, round to nearest even,
 *                                saturating to +-448)
 * Rows r >= num_valid_rows get q = 0 and s = 0.
 *   x       device, bf16 or fp32 [rows, cols] (x_dtype)
 *   q       device, uint8 [rows, cols]  (e4m3 bit patterns, output)
 *   scales  device, fp32 [rows]         (output)
 *   scale_ub  upper bound on a; +INFINITY for none.  Must be > 0.
 * Requires cols % 8 == 0, 0 <= num_valid_rows <= rows.
 */
MOE_API moe_status moe_quantize_fp8_rows(const void* x, int32_t x_dtype, int64_t rows, int64_t cols,
                                 int64_t num_valid_rows, float scale_ub,
                                 uint8_t* q, float* scales, void* stream);

/*
 * moe_route -- router, top-k, gate and token bucketing ([P1] "混合专家路由";
 * [P5] "MoE 架构详解").
 *   logits[t,e] = sum_d x[t,d] * w_router[e,d] (+ router_bias[e]), fp32 accumulate
 *   topk_ids[t, 0..k-1]: the k largest logits, largest first, equal logits
 *                        ordered by lower expert index
 *   topk_gates[t, j]:    k == 1: sigmoid(logit);  k > 1: softmax over the k
 *                        chosen logits
 *   expert_counts[e]:    number of slots (t, j) with topk_ids[t,j] == e
 *   expert_offsets[e]:   exclusive prefix sum of expert_counts (E + 1 entries)
 *   perm[p]:             slot index s = t*k + j, listed expert by expert, in
 *                        ascending s within each expert
 *   x         device, bf16 [T, D]
 *   w_router  device, bf16 [E, D]
 *   router_bias device, fp32 [E], or NULL for none
 *   outputs   device: int32 [T, k], fp32 [T, k], int32 [E], int32 [E + 1], int32 [T * k]
 * Requires 1 <= T <= 1048576, D a multiple of 128 in [128, 16384],
 * 1 <= k <= min(E, 8), E <= 256.
 */
MOE_API moe_status moe_route(const void* x, int32_t T, int32_t D,
                     const void* w_router, const float* router_bias,
                     int32_t E, int32_t k,
                     int32_t* topk_ids, float* topk_gates, int32_t* expert_counts,
                     int32_t* expert_offsets, int32_t* perm, void* stream);

/*
 * Description of one MoE FFN layer.  All pointers are device pointers.
 *   E routed experts, k experts per token, D model width, F routed hidden
 *   width, F_shared shared-expert hidden width.
 *   INT4_G128: w_gate, w_up uint8 [E, F, D/2]; s_gate, s_up fp32 [E, F, D/G];
 *              w_down uint8 [E, D, F/2]; s_down fp32 [E, D, F/G], G = group_size
 *              (the layout moe_quantize_int4 writes, one expert after another).
 *              G = 128, 64 or 32; groups of 64 and 32 run on the tensor-core
 *              tiles only (AUTO takes PREFILL for them; DECODE is refused with
 *              MOE_ERR_UNSUPPORTED_SHAPE).
 *   FP8_ROW:   w_gate, w_up uint8 [E, F, D]; s_gate, s_up fp32 [E, F];
 *              w_down uint8 [E, D, F]; s_down fp32 [E, D]
 *              (the layout moe_quantize_fp8_rows writes); every expert matmul
 *              quantizes its input rows to e4m3 with bound act_scale_ub.
 *   ws_gate, ws_up bf16 [F_shared, D]; ws_down bf16 [D, F_shared].
 *   path: a moe_path; AUTO picks DECODE when T * k <= 4 * E, else PREFILL.
 *         FP8_ROW layers always run on the tensor-core tiles (PREFILL).
 */
typedef struct moe_layer_desc {
    int32_t E, k, D, F, F_shared;
    int32_t format;        /* moe_weight_format */
    int32_t group_size;    /* INT4_G128: 128, 64 or 32; ignored for FP8_ROW */
    int32_t path;          /* moe_path */
    const void* w_router;      /* bf16 [E, D] */
    const float* router_bias;  /* fp32 [E] or NULL */
    const uint8_t* w_gate; const float* s_gate;
    const uint8_t* w_up;   const float* s_up;
    const uint8_t* w_down; const float* s_down;
    float act_scale_ub;        /* FP8_ROW only; +INFINITY = no bound */
    const void* ws_gate;       /* bf16 [F_shared, D] */
    const void* ws_up;         /* bf16 [F_shared, D] */
    const void* ws_down;       /* bf16 [D, F_shared] */
    /* Optional RMSNorm applied to x before everything else ([P5] "RMSNorm：
     * 为什么去掉减均值也能工作"): x[t,:] -> bf16(x[t,:] / sqrt(mean(x[t,:]^2) +
     * rms_eps) * rms_weight), as moe_rmsnorm computes it.  NULL: none. */
    const void* rms_weight;    /* bf16 [D] (gamma), or NULL */
    float rms_eps;             /* >= 0 (and <= 1); ignored when rms_weight is NULL */
} moe_layer_desc;

/*
 * moe_rmsnorm -- RMSNorm ([P5] "RMSNorm：为什么去掉减均值也能工作"):
 *   out[t, d] = bf16( x[t, d] / sqrt((1/D) sum_i x[t, i]^2 + eps) * gamma[d] )
 * in fp32: the sum of squares in a fixed order, IEEE division and square
 * root, the two products rounded to fp32 and the result to bf16 (nearest
 * even).  The same kernel is the prologue of a layer with rms_weight set.
 *   x      device, bf16 [T, D];  gamma  device, bf16 [D];  out  device, bf16 [T, D]
 * Requires 1 <= T <= 1048576, D a multiple of 128 in [128, 16384],
 * 0 <= eps <= 1.
 */
MOE_API moe_status moe_rmsnorm(const void* x, int32_t T, int32_t D, const void* gamma, float eps, void* out,
                               void* stream);

/*
 * Bytes of device workspace moe_ffn_forward needs for up to T_max tokens
 * (0 if the layer description is invalid).  Includes room for the host
 * staging of moe_ffn_forward_host.  The size depends on `layer->path`: a
 * fixed DECODE or PREFILL path (FP8_ROW layers always take PREFILL) needs
 * only that path's buffers, AUTO the larger of the two, since the path it
 * takes depends on T.
 */
MOE_API size_t moe_ffn_workspace_size(const moe_layer_desc* layer, int32_t T_max);

/*
 * moe_ffn_forward -- the whole layer ([P1] "混合专家路由", MoE.forward):
 *   out[t] = bf16( sum_j gate[t,j] * expert_{ids[t,j]}(x[t]) + shared(x[t]) )
 *   (with layer->rms_weight set, x is first replaced by moe_rmsnorm(x)),
 *   expert_e(x) = (silu(x We_gate^T) * (x We_up^T)) We_down^T  ([P5] SwiGLU),
 *   with int4 (zero point 0) or FP8 row-wise weights ([P2] bmm_nt), fp32
 *   accumulation, and the hidden activation rounded to bf16.
 *   shared(x) is the same SwiGLU with the bf16 shared weights, ungated.
 *   x    device, bf16 [T, D];  out  device, bf16 [T, D] (may not alias x)
 *   workspace  device, >= moe_ffn_workspace_size(layer, T) bytes, 256-byte
 *              aligned; its contents are scratch between calls.
 * Requires 1 <= T; the routing limits of moe_route; D, F and F_shared
 * multiples of 128 in [128, 16384]; format INT4_G128 (FP8_ROW: see below).
 * No host synchronization; no device-to-host copy.
 */
MOE_API moe_status moe_ffn_forward(const moe_layer_desc* layer, const void* x, int32_t T, void* out,
                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * moe_ffn_forward_host -- moe_ffn_forward for host buffers.  Enqueues the
 * copy of x (host, bf16 [T, D]; pinned memory lets it overlap) into the
 * workspace, the layer, and the copy of the result into out (host, bf16
 * [T, D]).  Does not synchronize: `out` is valid after the stream completes.
 */
MOE_API moe_status moe_ffn_forward_host(const moe_layer_desc* layer, const void* x_host, int32_t T,
                                void* out_host, void* workspace, size_t workspace_bytes,
                                void* stream);

/*
 * moe_ffn_forward_timed -- moe_ffn_forward that also records caller-created
 * cudaEvent_t handles (passed as void*) on `stream` for per-kernel timing:
 * events[i] just before the i-th kernel launch of the layer and
 * events[launches] after the last one (n_events >= launches + 1, where
 * launches = moe_ffn_launch_names(...)).  Results are identical to
 * moe_ffn_forward.
 */
MOE_API moe_status moe_ffn_forward_timed(const moe_layer_desc* layer, const void* x, int32_t T, void* out,
                                         void* workspace, size_t workspace_bytes, void* stream,
                                         void* const* events, int32_t n_events);

/*
 * moe_ffn_launch_names -- number of kernel launches moe_ffn_forward makes for
 * this layer and T (0 if the layer is invalid), and their names (static
 * strings) in launch order, written to names[0 .. max_names-1] if non-NULL.
 */
MOE_API int32_t moe_ffn_launch_names(const moe_layer_desc* layer, int32_t T, const char** names,
                                     int32_t max_names);

/*
 * moe_ffn_forward_noalloc -- the layer forward of moe_ffn_forward, for
 * callers that cannot allocate device memory and so cannot pass a workspace:
 * for example a plugin behind a fixed interface that hands over only its
 * input and output buffers, or a runtime that has reserved all device memory
 * for its own pool, where an extra cudaMalloc would fail or would stall the
 * device.  The web pages have no counterpart; this is an interface
 * convenience only.
 *   x    device, bf16 [T, D];  out  device, bf16 [T, D]
 * The library's own scratch is a fixed 8 MiB device array, reserved on every
 * device that loads the library until the process exits.  A call whose
 * scratch need (moe_ffn_workspace_size(layer, T)) exceeds 8 MiB returns
 * MOE_ERR_WORKSPACE_TOO_SMALL and launches nothing; use moe_ffn_forward then.
 * No cudaMalloc, cudaFree or other allocation is made.
 * The first call on each device looks up the array's device address with
 * that device current; make that first call before any stream capture.
 * The address is kept for the life of the process: after cudaDeviceReset
 * on a device, do not call this function on that device again (the array
 * may have moved).
 * All calls on a device share the one array: calls that may overlap on the
 * GPU (different streams, or different host threads) race and corrupt each
 * other's results -- serialize them.  Leftover contents from an earlier call
 * are harmless; what must start at zero is cleared by every call.
 * Argument errors (null or misaligned x / out, unsupported shapes) return
 * before the CUDA runtime is touched.
 */
MOE_API moe_status moe_ffn_forward_noalloc(const moe_layer_desc* layer, const void* x, int32_t T, void* out,
                                           void* stream);

/*
 * moe_ffn_noalloc_device_status -- moe_ffn_device_status for the calls of
 * moe_ffn_forward_noalloc on the current device, whose status word lives in
 * the library's own scratch array: SYNCHRONIZES `stream`, then returns MOE_OK,
 * MOE_ERR_TIMEOUT (a bounded device wait of the last no-alloc call gave up;
 * its output is invalid) or MOE_ERR_CUDA.
 */
MOE_API moe_status moe_ffn_noalloc_device_status(void* stream);

/*
 * Description of a dense SwiGLU FFN layer, the FFN of the dense layers that
 * alternate with the MoE layers ([P4] introduction; [P5] "SwiGLU：门控激活的
 * 数学").  All pointers are device pointers.
 *   w_gate, w_up bf16 [F, D]; w_down bf16 [D, F].
 *   path: a moe_path; AUTO streams the weights (DECODE) for T <= 64 and
 *         uses the tensor-core tiles (PREFILL) above.
 *   rms_weight / rms_eps: as in moe_layer_desc (an RMSNorm of x first; NULL: none).
 */
typedef struct moe_dense_desc {
    int32_t D, F;
    int32_t path;              /* moe_path */
    const void* w_gate;        /* bf16 [F, D] */
    const void* w_up;          /* bf16 [F, D] */
    const void* w_down;        /* bf16 [D, F] */
    const void* rms_weight;    /* bf16 [D], or NULL */
    float rms_eps;
} moe_dense_desc;

/*
 * Bytes of device workspace moe_dense_ffn_forward needs for up to T_max
 * tokens (0 if the description is invalid); with AUTO, the larger of the
 * two paths' needs.
 */
MOE_API size_t moe_dense_ffn_workspace_size(const moe_dense_desc* layer, int32_t T_max);

/*
 * moe_dense_ffn_forward -- out = bf16( (silu(x Wg^T) * (x Wu^T)) Wd^T ) with
 * bf16 weights, fp32 accumulation and the hidden activation rounded to bf16:
 * the MoE layer's shared expert on its own ([P5] "SwiGLU：门控激活的数学").
 *   x    device, bf16 [T, D];  out  device, bf16 [T, D] (may not alias x)
 *   workspace  device, >= moe_dense_ffn_workspace_size(layer, T) bytes,
 *              256-byte aligned; scratch between calls.
 * Requires 1 <= T <= 1048576; D and F multiples of 128 in [128, 16384].
 * No host synchronization.
 */
MOE_API moe_status moe_dense_ffn_forward(const moe_dense_desc* layer, const void* x, int32_t T, void* out,
                                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * Expert parallelism ([P1], the closing section on dependencies: fairscale
 * model-parallel splitting; [P4] introduction: Maverick FP8 on one 8-GPU
 * node).  With the experts spread over P GPUs, a layer is: moe_route on each
 * GPU's own tokens; an all-to-all that sends every slot's row to the GPU
 * holding its expert; moe_expert_ffn_forward there; an all-to-all back; and
 * moe_shared_ffn_combine, which adds the shared expert and sums each token's
 * slots.  The two calls below are those compute steps; the exchanges are the
 * caller's (the Python package's expert-parallel layer uses NCCL).  Rows
 * that arrive from another GPU are in this GPU's memory before either call
 * reads them.
 *
 * moe_expert_ffn_forward -- the routed experts alone, on rows whose expert
 * and gate are given:
 *   y[r] = gates[r] * expert_{expert_ids[r]}(x[r])   (fp32, as in the layer)
 * with `layer`'s routed weights (its router, shared expert and k are not
 * used; expert_ids index its E experts).
 *   x  device, bf16 [n, D] (already normalized if the layer has an RMSNorm)
 *   expert_ids  device, int32 [n], 0 <= id < E;  gates  device, fp32 [n]
 *   y  device, fp32 [n, D] (output)
 *   workspace  device, >= moe_expert_ffn_workspace_size(layer, n) bytes,
 *              256-byte aligned.
 * An id out of range is counted as expert 0 and reported by
 * moe_ffn_device_status(workspace) as MOE_ERR_INVALID_ARG.
 */
MOE_API size_t moe_expert_ffn_workspace_size(const moe_layer_desc* layer, int32_t n_max);
MOE_API moe_status moe_expert_ffn_forward(const moe_layer_desc* layer, const void* x, int32_t n,
                                          const int32_t* expert_ids, const float* gates, float* y,
                                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * moe_shared_ffn_combine -- the rest of the layer for T tokens whose k slots'
 * routed outputs are given:
 *   out[t] = bf16( shared(x[t]) + sum_{j < k} y_slots[t, j] )
 * summed in that order, as moe_ffn_forward does (with layer->rms_weight set,
 * x is first replaced by moe_rmsnorm(x)).
 *   x  device, bf16 [T, D];  y_slots  device, fp32 [T, k, D];  out  device, bf16 [T, D]
 *   workspace  device, >= moe_shared_ffn_workspace_size(layer, T) bytes, 256-byte aligned.
 */
MOE_API size_t moe_shared_ffn_workspace_size(const moe_layer_desc* layer, int32_t T_max);
MOE_API moe_status moe_shared_ffn_combine(const moe_layer_desc* layer, const void* x, int32_t T,
                                          const float* y_slots, void* out, void* workspace,
                                          size_t workspace_bytes, void* stream);

/*
 * moe_ffn_device_status -- SYNCHRONIZES `stream`, then reads the device
 * status word that the kernels of the last call on this workspace
 * (moe_ffn_forward, moe_dense_ffn_forward, moe_expert_ffn_forward,
 * moe_shared_ffn_combine) set.  Returns MOE_OK, MOE_ERR_TIMEOUT (a bounded
 * device wait gave up; the outputs of that call are invalid),
 * MOE_ERR_INVALID_ARG (moe_expert_ffn_forward was given an expert id out of
 * range) or MOE_ERR_CUDA.  The word is cleared at the start of every call.
 */
MOE_API moe_status moe_ffn_device_status(const void* workspace, void* stream);

/*
 * moe_set_wait_limit -- the limit, in SM clock cycles, of every bounded
 * device wait that reports to a status word (the kernels' waits on their
 * pipeline barriers), for the current device.  cycles <= 0 restores the
 * default of 2e9 cycles (about one second).  A lowered limit makes waits give
 * up as soon as they miss their first try, so the next layer call ends with
 * MOE_ERR_TIMEOUT in its status word: it exists to test that path.  Waits
 * that let a kernel's own copies in flight land before it exits keep the
 * default.  Synchronous; call it while no kernel of this library is running.
 * The pages have no counterpart.
 */
MOE_API moe_status moe_set_wait_limit(int64_t cycles);

#ifdef __cplusplus
}
#endif

#endif /* MOE_INT4_H */
