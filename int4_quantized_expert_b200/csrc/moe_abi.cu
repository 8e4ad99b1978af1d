// extern "C" entry points of libmoe_int4: argument checks, workspace layout,
// and the stream-ordered launch sequence of each operation.
#include <math.h>
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "ffn_decode.cuh"
#include "tc_gemm.cuh"
#include "norm.cuh"

namespace moe {
moe_status launch_quantize_int4(const float* w, int64_t rows, int64_t cols, int group_size, uint8_t* codes,
                                float* scales, cudaStream_t stream);
moe_status launch_quantize_fp8_rows(const void* x, int32_t x_dtype, int64_t rows, int64_t cols,
                                    int64_t num_valid, float scale_ub, uint8_t* q, float* scales,
                                    cudaStream_t stream);
}  // namespace moe

using namespace moe;

namespace {

constexpr int kMaxT = 1 << 20;
constexpr int kMaxDim = 16384;
constexpr size_t kMaxDecodeSmem = 227 * 1024;

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

bool valid_dim(int32_t v) { return v >= 128 && v <= kMaxDim && v % 128 == 0; }

moe_status check_route_shape(int32_t T, int32_t D, int32_t E, int32_t k) {
    if (T < 1 || T > kMaxT) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!valid_dim(D)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (E < 1 || E > 256 || k < 1 || k > E || k > 8) return MOE_ERR_UNSUPPORTED_SHAPE;
    return MOE_OK;
}

// Workspace regions, each 256-byte aligned.  The regions up to `common_end`
// are shared by both paths; the rest is laid out per path from there, and a
// workspace must be large enough for either.
struct WsLayout {
    size_t status, rt_cnt, dec_cnt, zeros_end, counters, rt_part, ids, gates, counts, offsets, perm, inv_perm, chunks, nchunks;
    size_t bk_hist;   // per-block expert counts of the multi-CTA bucketing
    size_t xn;   // RMSNorm of x (layers with rms_weight)
    size_t common_end;
    // weight-streaming path
    size_t x16, x_meta, h_r, h16, h_meta, h_s, y_r, y_s;
    // tensor-core path (row counts padded to whole 256-token tiles)
    size_t x_sorted, h_sorted, h_s_pad, y_pos, y_shared;
    size_t xq, xq_scale, hq, hq_scale;   // e4m3 activations of FP8_ROW layers
    // host staging of moe_ffn_forward_host
    size_t x_in, out;
    size_t total;
};

inline bool int4_group_ok(int g) { return g == 128 || g == 64 || g == 32; }

enum { PATH_SEL_DECODE = 1, PATH_SEL_PREFILL = 2 };

WsLayout ws_layout(const moe_layer_desc& L, int64_t T, int path) {
    WsLayout w;
    memset(&w, 0, sizeof(w));
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off += (bytes + 255) & ~size_t(255);
        return o;
    };
    const int64_t S = T * L.k;
    const int64_t S_pad = ceil_div(S, TC_BLOCK_TOKENS) * TC_BLOCK_TOKENS;
    const int64_t T_pad = ceil_div(T, TC_BLOCK_TOKENS) * TC_BLOCK_TOKENS;
    w.status = take(64);
    w.counters = take(64);   // task counters of the weight-streaming kernels
    const bool rms = L.rms_weight != nullptr;
    const bool rt_split = router_ksplit(int(T), L.D, rms) > 1;
    w.rt_cnt = take(rt_split ? size_t(ceil_div(T, 16)) * 4 : 0);   // router tile counters
    // weight-streaming path: the epilogues' last-writer counters, per (position,
    // group of 128 rows of h) and per (token, block of 64 output rows)
    w.dec_cnt = take(path == PATH_SEL_DECODE ? size_t(S * (L.F / 128) + T * (L.D / 64)) * 4 : 0);
    w.zeros_end = off;   // [status, zeros_end) is cleared at the start of every call
    w.rt_part = take(router_partial_floats(int(T), L.D, L.E, rms) * 4);
    w.ids = take(S * 4);
    w.gates = take(S * 4);
    w.counts = take(size_t(L.E) * 4);
    w.offsets = take(size_t(L.E + 1) * 4);
    w.perm = take(S * 4);
    w.inv_perm = take(S * 4);
    w.bk_hist = take(size_t(bucket_blocks(S)) * L.E * 4);
    w.chunks = take(size_t(decode_max_chunks(int(T), L.k, L.E)) * sizeof(ChunkEntry));
    w.nchunks = take(16);
    w.xn = take(L.rms_weight ? size_t(T) * L.D * 2 : 0);
    w.common_end = off;
    if (path == PATH_SEL_DECODE) {
        w.x16 = take(S * L.D * 2);                 // tokens by expert-sorted position
        w.x_meta = take(S * act16_meta_pitch(L.D, L.group_size) * 4);
        w.h_r = take(S * L.F * 2);
        w.h16 = take(S * L.F * 2);
        w.h_meta = take(S * act16_meta_pitch(L.F, L.group_size) * 4);
        w.h_s = take(T * L.F_shared * 2);
        w.y_r = take(S * L.D * 4);
        w.y_s = take(T * L.D * 4);
    } else {
        if (L.format == MOE_WEIGHTS_FP8_ROW) {
            w.xq = take(S_pad * L.D);
            w.xq_scale = take(S * 4);
            w.hq = take(S_pad * L.F);
            w.hq_scale = take(S * 4);
        } else {
            w.x_sorted = take(S_pad * L.D * 2);
        }
        w.h_sorted = take(S_pad * L.F * 2);
        w.h_s_pad = take(T_pad * L.F_shared * 2);
        w.y_pos = take(S * L.D * 4);
        w.y_shared = take(T * L.D * 4);
    }
    w.x_in = take(T * L.D * 2);
    w.out = take(T * L.D * 2);
    w.total = off;
    return w;
}

bool decode_fits(const moe_layer_desc& L);

// Workspace for every call with this descriptor and at most T tokens: the
// fixed path's layout, or the larger of the two when the path depends on T.
size_t ws_bytes(const moe_layer_desc& L, int64_t T) {
    const size_t a = ws_layout(L, T, PATH_SEL_DECODE).total;
    const size_t b = ws_layout(L, T, PATH_SEL_PREFILL).total;
    if (L.format == MOE_WEIGHTS_FP8_ROW || L.path == MOE_PATH_PREFILL) return b;
    if (L.path == MOE_PATH_AUTO && !decode_fits(L)) return b;   // AUTO never takes the decode path
    if (L.path == MOE_PATH_DECODE) return a;
    return a > b ? a : b;
}

// Whether the weight-streaming kernels take this layer.  Groups of 128 keep
// a task's scales in shared memory (it must fit); groups of 64 / 32 load
// each stage's scales with it, as a TMA box of the stage's groups (at least
// as many as a row has) whose rows (K / G scales) must be whole 16-byte units.
bool decode_fits(const moe_layer_desc& L) {
    const int G = L.group_size;
    if (L.format == MOE_WEIGHTS_INT4_G128 && G != 128)
        return (L.D / G) % 4 == 0 && (L.F / G) % 4 == 0 && L.D / G >= decode_groups_per_stage(0, G) &&
               L.F / G >= decode_groups_per_stage(1, G) && decode_smem_bytes(0, 0, G) <= kMaxDecodeSmem &&
               decode_smem_bytes(1, 0, G) <= kMaxDecodeSmem;
    return decode_smem_bytes(0, decode_scale_floats(0, L.D), 128) <= kMaxDecodeSmem &&
           decode_smem_bytes(1, decode_scale_floats(1, L.F), 128) <= kMaxDecodeSmem;
}

int choose_path(const moe_layer_desc& L, int64_t T) {
    if (L.format == MOE_WEIGHTS_FP8_ROW) return PATH_SEL_PREFILL;   // e4m3 layers run on tensor-core tiles
    if (L.path == MOE_PATH_DECODE) return PATH_SEL_DECODE;
    if (L.path == MOE_PATH_PREFILL) return PATH_SEL_PREFILL;
    return T * L.k <= 4 * int64_t(L.E) && decode_fits(L) ? PATH_SEL_DECODE : PATH_SEL_PREFILL;
}

moe_status check_layer(const moe_layer_desc* L) {
    if (!L) return MOE_ERR_INVALID_ARG;
    if (L->E < 1 || L->E > 256 || L->k < 1 || L->k > L->E || L->k > 8) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!valid_dim(L->D) || !valid_dim(L->F) || !valid_dim(L->F_shared)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (L->format != MOE_WEIGHTS_INT4_G128 && L->format != MOE_WEIGHTS_FP8_ROW) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (L->format == MOE_WEIGHTS_INT4_G128 && !int4_group_ok(L->group_size)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (L->format == MOE_WEIGHTS_FP8_ROW && !(L->act_scale_ub > 0.0f)) return MOE_ERR_INVALID_ARG;
    if (L->path < MOE_PATH_AUTO || L->path > MOE_PATH_PREFILL) return MOE_ERR_INVALID_ARG;
    const void* ptrs[] = {L->w_router, L->w_gate, L->s_gate, L->w_up, L->s_up, L->w_down, L->s_down,
                          L->ws_gate, L->ws_up, L->ws_down};
    for (const void* p : ptrs)
        if (!p || !aligned16(p)) return MOE_ERR_INVALID_ARG;
    if (L->router_bias && !aligned16(L->router_bias)) return MOE_ERR_INVALID_ARG;
    if (L->rms_weight && (!aligned16(L->rms_weight) || !(L->rms_eps >= 0.0f) || L->rms_eps > 1.0f))
        return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

// Optional per-launch timing: event i is recorded before the i-th kernel of
// the layer, the last one after the final kernel.
struct Marks {
    void* const* ev = nullptr;
    int32_t n = 0;
    int32_t i = 0;
    void mark(cudaStream_t st) {
        if (ev && i < n) cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), st);
        ++i;
    }
    // the event j places after the current one (or null)
    cudaEvent_t event(int j) const { return (ev && i + j < n) ? static_cast<cudaEvent_t>(ev[i + j]) : nullptr; }
};

const char* const kDecodeLaunches[] = {"router", "bucket", "act16_x", "decode_gate_up", "decode_down"};
constexpr int32_t kDecodeLaunchCount = 5;

template <typename T>
T* at(void* base, size_t off) {
    return reinterpret_cast<T*>(static_cast<unsigned char*>(base) + off);
}

// A launch's tensor maps depend only on the layer description, the workspace,
// the input pointer, T and the path; a call with the same ones reuses them.
struct MapCacheKey {
    moe_layer_desc L;
    const void* ws;
    const void* x;
    int64_t T;
    int path;
    bool valid;
};

MapCacheKey make_key(const moe_layer_desc& L, const void* ws, const void* x, int64_t T, int path) {
    MapCacheKey k;
    memset(&k, 0, sizeof(k));
    memcpy(&k.L, &L, sizeof(L));
    k.ws = ws;
    k.x = x;
    k.T = T;
    k.path = path;
    k.valid = true;
    return k;
}

bool same_key(const MapCacheKey& a, const MapCacheKey& b) {
    return a.valid && b.valid && memcmp(&a.L, &b.L, sizeof(a.L)) == 0 && a.ws == b.ws && a.x == b.x &&
           a.T == b.T && a.path == b.path;
}

// With an RMSNorm the router normalizes x itself and writes xn to the
// workspace for the kernels after it; counters[2] counts its CTAs once done.
void set_rms(RoutePrep& prep, const moe_layer_desc& L, void* ws, const WsLayout& W) {
    if (!L.rms_weight) return;
    prep.rms_weight = static_cast<const bf16*>(L.rms_weight);
    prep.rms_eps = L.rms_eps;
    prep.xn = at<bf16>(ws, W.xn);
    prep.xn_ready = at<int32_t>(ws, W.counters) + 2;
}

// Rows whose expert and gate the caller gives (the routed experts alone: the
// compute step of an expert-parallel layer).  The router and the shared
// expert are skipped and each row's gate-scaled output goes to y by row.
struct PreRouted {
    const int32_t* ids;   // [T] expert of each row
    const float* gates;   // [T]
    float* y;             // [T, D] fp32
};

moe_status ffn_decode_path(const moe_layer_desc& L, const bf16* x, const bf16* xin, int T, bf16* out, void* ws,
                           const WsLayout& W, cudaStream_t st, Marks& mk, const PreRouted* pr = nullptr) {
    int32_t* status = at<int32_t>(ws, W.status);
    int32_t* counters = at<int32_t>(ws, W.counters);
    int32_t* perm = at<int32_t>(ws, W.perm);
    int32_t* inv = at<int32_t>(ws, W.inv_perm);
    float* gates = at<float>(ws, W.gates);
    bf16* h_r = at<bf16>(ws, W.h_r);
    bf16* h_s = at<bf16>(ws, W.h_s);
    float* y_r = at<float>(ws, W.y_r);
    float* y_s = at<float>(ws, W.y_s);
    ChunkEntry* chunks = at<ChunkEntry>(ws, W.chunks);
    int32_t* nch = at<int32_t>(ws, W.nchunks);
    const int64_t S = int64_t(T) * L.k;

    // Launch order: router, bucket, act16_x, gate/up, act16_h, down, combine;
    // every launch after the first may start while the one before it runs
    // (programmatic dependent launch) and waits before reading its outputs.
    RoutePrep prep;
    memset(&prep, 0, sizeof(prep));
    if (router_ksplit(T, L.D, L.rms_weight != nullptr) > 1) {   // K-split router (few token tiles)
        prep.router_part = at<float>(ws, W.rt_part);
        prep.router_tile_cnt = at<int32_t>(ws, W.rt_cnt);
    }
    prep.chunks = chunks;
    prep.n_chunks = nch;
    prep.zero_words = nullptr;      // the task counters are cleared with the status word
    prep.n_zero = 0;
    prep.chunk_tokens = 16;
    prep.routed_chunk_tokens = 8;   // one 8-column n-tile per routed chunk
    prep.bucket_hist = at<int32_t>(ws, W.bk_hist);
    prep.router_after_kernel = false;
    set_rms(prep, L, ws, W);
    moe_status s;
    if (pr) {   // the rows' experts are given: bucketing only
        prep.status = at<int32_t>(ws, W.status);
        s = launch_bucket(pr->ids, T, 1, L.E, at<int32_t>(ws, W.counts), at<int32_t>(ws, W.offsets), perm, inv,
                          &prep, st);
        gates = const_cast<float*>(pr->gates);
    } else {
        mk.mark(st);
        const bool multi = bucket_blocks(int64_t(T) * L.k) > 0;
        s = launch_route(x, T, L.D, static_cast<const bf16*>(L.w_router), L.router_bias, L.E, L.k,
                         at<int32_t>(ws, W.ids), gates, at<int32_t>(ws, W.counts), at<int32_t>(ws, W.offsets), perm,
                         inv, &prep, st, mk.event(0), multi ? mk.event(1) : nullptr, multi ? mk.event(2) : nullptr);
        mk.i += multi ? 3 : 1;
    }
    if (s != MOE_OK) return s;
    mk.mark(st);
    s = launch_act16(xin, S, L.D, L.group_size, perm, L.k, at<__half>(ws, W.x16), at<float>(ws, W.x_meta), st);
    if (s != MOE_OK) return s;

    // tensor maps: built once per (layer, workspace, input, T) and thread
    static thread_local MapCacheKey dkey;
    static thread_local DecodeMaps dm1, dm2;
    const MapCacheKey key = make_key(L, ws, x, T, PATH_SEL_DECODE);
    if (!same_key(key, dkey)) {
        dkey.valid = false;
        auto build = [&](DecodeMaps& m1, DecodeMaps& m2) -> bool {
        const uint64_t E = uint64_t(L.E);
        const uint32_t rows = uint32_t(decode_task_rows());
        const int G = L.group_size;
        // weights; token rows (8 per routed chunk, 16 per shared chunk) and group offsets
        bool ok = make_tmap_2d(&m1.r0, L.w_gate, 1, L.D / 2, E * L.F, 128, rows, true) &&
                  make_tmap_2d(&m1.r1, L.w_up, 1, L.D / 2, E * L.F, 128, rows, true) &&
                  make_tmap_2d(&m1.s0, L.ws_gate, 2, L.D, L.F_shared, 64, rows, true) &&
                  make_tmap_2d(&m1.s1, L.ws_up, 2, L.D, L.F_shared, 64, rows, true) &&
                  make_tmap_rows_3d(&m1.br, at<__half>(ws, W.x16), L.D, S, 8, 4) &&
                  make_tmap_2d(&m1.cr, at<float>(ws, W.x_meta), 4, act16_meta_pitch(L.D, G), S,
                               2 * decode_groups_per_stage(0, G), 8, false) &&
                  make_tmap_rows_3d(&m1.bs, xin, L.D, T, 16, 1) &&
                  make_tmap_2d(&m2.r0, L.w_down, 1, L.F / 2, E * L.D, 128, rows, true) &&
                  make_tmap_2d(&m2.s0, L.ws_down, 2, L.F_shared, L.D, 64, rows, true) &&
                  make_tmap_rows_3d(&m2.br, at<__half>(ws, W.h16), L.F, S, 8, 8) &&
                  make_tmap_2d(&m2.cr, at<float>(ws, W.h_meta), 4, act16_meta_pitch(L.F, G), S,
                               2 * decode_groups_per_stage(1, G), 8, false) &&
                  make_tmap_rows_3d(&m2.bs, h_s, L.F_shared, T, 16, 2);
        if (G == 128) {
            // the task scales: one box per matrix when their rows are whole 16-byte units
            const int pd = decode_scale_pitch(L.D), pf = decode_scale_pitch(L.F);
            if (pd) ok = ok && make_tmap_2d(&m1.g0, L.s_gate, 4, L.D / kGroup, E * L.F, pd, rows, false) &&
                         make_tmap_2d(&m1.g1, L.s_up, 4, L.D / kGroup, E * L.F, pd, rows, false);
            else m1.g0 = m1.g1 = m1.r0;   // unused: the scales come by bulk copy
            if (pf) ok = ok && make_tmap_2d(&m2.g0, L.s_down, 4, L.F / kGroup, E * L.D, pf, rows, false);
            else m2.g0 = m2.r0;
        } else {
            // groups of 64 / 32: each stage's scales, (the stage's groups) x 64 rows
            const uint32_t g0 = uint32_t(decode_groups_per_stage(0, G)), g1 = uint32_t(decode_groups_per_stage(1, G));
            ok = ok && make_tmap_2d(&m1.g0, L.s_gate, 4, L.D / G, E * L.F, g0, rows, false) &&
                 make_tmap_2d(&m1.g1, L.s_up, 4, L.D / G, E * L.F, g0, rows, false) &&
                 make_tmap_2d(&m2.g0, L.s_down, 4, L.F / G, E * L.D, g1, rows, false);
        }
        if (!ok) return false;
        m2.r1 = m2.r0;
        m2.s1 = m2.s0;
        m2.g1 = m2.g0;
            return true;
        };
        if (!build(dm1, dm2)) return MOE_ERR_CUDA;
        dkey = key;
    }
    const DecodeMaps& m1 = dm1;
    const DecodeMaps& m2 = dm2;

    DecodeParams p;
    memset(&p, 0, sizeof(p));
    p.T = T;
    p.n_rows_r = L.F;
    p.n_rows_s = L.F_shared;
    p.K_r = L.D;
    p.K_s = L.D;
    p.k_top = L.k;
    p.scale_buf_floats = L.group_size == 128 ? decode_scale_floats(0, L.D) : 0;
    p.f16_magic_lo = kF16MagicLo;
    p.f16_magic_hi = kF16MagicHi;
    p.chunks = chunks;
    p.n_chunks = nch;
    p.perm = perm;
    p.gates = gates;
    p.sc0 = L.s_gate;
    p.sc1 = L.s_up;
    p.h_r = h_r;
    p.h_s = h_s;
    p.h16 = at<__half>(ws, W.h16);      // the gate/up epilogue also writes h's fp16 operands
    p.h_meta = at<float>(ws, W.h_meta);
    p.hcnt = at<int32_t>(ws, W.dec_cnt);
    if (L.rms_weight) {   // the shared-expert tasks read the router's xn: wait for all its CTAs
        p.xn_ready = counters + 2;
        p.xn_ready_target = int32_t(ceil_div(T, 16)) * router_ksplit(T, L.D, true);
    }
    p.task_counter = counters;
    p.status = status;
    if (pr) p.n_rows_s = 0;   // no shared-expert tasks
    mk.mark(st);
    s = launch_decode_ffn(0, L.group_size, m1, p, st);
    if (s != MOE_OK) return s;

    p.n_rows_r = L.D;
    p.n_rows_s = L.D;
    p.K_r = L.F;
    p.K_s = L.F_shared;
    p.scale_buf_floats = L.group_size == 128 ? decode_scale_floats(1, L.F) : 0;
    p.sc0 = L.s_down;
    p.sc1 = nullptr;
    p.y_r = y_r;
    p.y_s = y_s;
    p.out = out;                        // the down epilogue finishes each token
    p.inv_perm = inv;
    p.n_contrib = L.k;
    p.ocnt = at<int32_t>(ws, W.dec_cnt) + S * (L.F / 128);
    p.task_counter = counters + 1;
    if (pr) {   // gate-scaled y of each row, by row; no shared expert, no combine
        p.n_rows_s = 0;
        p.y_r = pr->y;
        p.y_by_slot = 1;
        p.out = nullptr;
    }
    mk.mark(st);
    s = launch_decode_ffn(1, L.group_size, m2, p, st);
    mk.mark(st);
    return s;
}

// Kernel launches of the tensor-core path, in order (the combine only when a
// token has more than one routed slot).
int prefill_launches(const moe_layer_desc& L, int64_t T, const char** names, int max_names) {
    const bool fp8 = L.format == MOE_WEIGHTS_FP8_ROW;
    const char* list[11];
    int n = 0;
    list[n++] = "router";
    list[n++] = "bucket";
    if (bucket_blocks(T * L.k) > 0) {   // the bucketing's three kernels
        list[n++] = "bucket_scan";
        list[n++] = "bucket_place";
    }
    list[n++] = fp8 ? "quantize_x" : "gather";
    list[n++] = "tc_shared_gate_up";
    list[n++] = "tc_shared_down";
    list[n++] = "tc_gate_up";
    if (fp8) list[n++] = "quantize_h";
    list[n++] = "tc_down";
    if (L.k > 1) list[n++] = "combine";
    for (int i = 0; i < n && i < max_names && names; ++i) names[i] = list[i];
    return n;
}

// The kernels one forward launches, in order (an RMSNorm runs inside the router).
int32_t layer_launch_names(const moe_layer_desc& L, int64_t T, const char** names, int32_t max_names) {
    if (choose_path(L, T) != PATH_SEL_DECODE) return prefill_launches(L, T, names, max_names);
    for (int32_t i = 0; i < kDecodeLaunchCount && i < max_names && names; ++i) names[i] = kDecodeLaunches[i];
    return kDecodeLaunchCount;
}

moe_status ffn_prefill_path(const moe_layer_desc& L, const bf16* x, const bf16* xin, int T, bf16* out, void* ws,
                            const WsLayout& W, cudaStream_t st, Marks& mk, const PreRouted* pr = nullptr) {
    int32_t* status = at<int32_t>(ws, W.status);
    int32_t* perm = at<int32_t>(ws, W.perm);
    int32_t* inv = at<int32_t>(ws, W.inv_perm);
    float* gates = at<float>(ws, W.gates);
    ChunkEntry* chunks = at<ChunkEntry>(ws, W.chunks);
    int32_t* nch = at<int32_t>(ws, W.nchunks);
    const int64_t S = int64_t(T) * L.k;
    const uint64_t S_pad = uint64_t(ceil_div(S, TC_BLOCK_TOKENS) * TC_BLOCK_TOKENS);
    const uint64_t T_pad = uint64_t(ceil_div(T, TC_BLOCK_TOKENS) * TC_BLOCK_TOKENS);
    bf16* x_sorted = at<bf16>(ws, W.x_sorted);
    bf16* h_sorted = at<bf16>(ws, W.h_sorted);
    bf16* h_s = at<bf16>(ws, W.h_s_pad);
    float* y_pos = at<float>(ws, W.y_pos);

    RoutePrep prep;
    memset(&prep, 0, sizeof(prep));   // unsplit router: the tensor-core path has many token tiles
    prep.chunks = chunks;
    prep.n_chunks = nch;
    prep.chunk_tokens = TC_BLOCK_TOKENS;
    prep.routed_chunk_tokens = TC_BLOCK_TOKENS;
    prep.bucket_hist = at<int32_t>(ws, W.bk_hist);
    set_rms(prep, L, ws, W);
    moe_status s;
    if (pr) {   // the rows' experts are given: bucketing only
        prep.status = at<int32_t>(ws, W.status);
        s = launch_bucket(pr->ids, T, 1, L.E, at<int32_t>(ws, W.counts), at<int32_t>(ws, W.offsets), perm, inv,
                          &prep, st);
        gates = const_cast<float*>(pr->gates);
    } else {
        mk.mark(st);
        const bool multi = bucket_blocks(int64_t(T) * L.k) > 0;
        s = launch_route(x, T, L.D, static_cast<const bf16*>(L.w_router), L.router_bias, L.E, L.k,
                         at<int32_t>(ws, W.ids), gates, at<int32_t>(ws, W.counts), at<int32_t>(ws, W.offsets), perm,
                         inv, &prep, st, mk.event(0), multi ? mk.event(1) : nullptr, multi ? mk.event(2) : nullptr);
        mk.i += multi ? 3 : 1;
    }
    if (s != MOE_OK) return s;
    mk.mark(st);
    const bool fp8 = L.format == MOE_WEIGHTS_FP8_ROW;
    if (fp8)   // e4m3 rows of x, written to each token's slot positions
        s = launch_quantize_fp8_scatter(xin, T, L.D, L.act_scale_ub, inv, L.k, at<uint8_t>(ws, W.xq),
                                        at<float>(ws, W.xq_scale), st);
    else
        s = launch_gather_rows(xin, perm, S, L.k, L.D, x_sorted, st);
    if (s != MOE_OK) return s;

    static thread_local MapCacheKey pkey;
    static thread_local TcMaps pm[4];
    const MapCacheKey key = make_key(L, ws, x, T, PATH_SEL_PREFILL);
    if (!same_key(key, pkey)) {
        pkey.valid = false;
        auto build = [&](TcMaps& m_gu, TcMaps& m_dn, TcMaps& m_sgu, TcMaps& m_sdn) -> bool {
        const uint64_t E = uint64_t(L.E);
        bool ok;
        if (fp8)
            ok = make_tmap_2d(&m_gu.b, at<uint8_t>(ws, W.xq), 1, L.D, S_pad, 128, TC_BLOCK_TOKENS, true) &&
                 make_tmap_2d(&m_gu.b_small, at<uint8_t>(ws, W.xq), 1, L.D, S_pad, 128, TC_SMALL_TOKENS, true) &&
                 make_tmap_2d(&m_gu.a0, L.w_gate, 1, L.D, E * L.F, 128, 16, true) &&
                 make_tmap_2d(&m_gu.a1, L.w_up, 1, L.D, E * L.F, 128, 16, true) &&
                 make_tmap_2d(&m_dn.b, at<uint8_t>(ws, W.hq), 1, L.F, S_pad, 128, TC_BLOCK_TOKENS, true) &&
                 make_tmap_2d(&m_dn.b_small, at<uint8_t>(ws, W.hq), 1, L.F, S_pad, 128, TC_SMALL_TOKENS, true) &&
                 make_tmap_2d(&m_dn.a0, L.w_down, 1, L.F, E * L.D, 128, 16, true);
        else
            ok = make_tmap_2d(&m_gu.b, x_sorted, 2, L.D, S_pad, 64, TC_BLOCK_TOKENS, true) &&
                 make_tmap_2d(&m_gu.b_small, x_sorted, 2, L.D, S_pad, 64, TC_SMALL_TOKENS, true) &&
                 make_tmap_2d(&m_gu.a0, L.w_gate, 1, L.D / 2, E * L.F, 32, 64, false) &&
                 make_tmap_2d(&m_gu.a1, L.w_up, 1, L.D / 2, E * L.F, 32, 64, false) &&
                 make_tmap_2d(&m_dn.b, h_sorted, 2, L.F, S_pad, 64, TC_BLOCK_TOKENS, true) &&
                 make_tmap_2d(&m_dn.b_small, h_sorted, 2, L.F, S_pad, 64, TC_SMALL_TOKENS, true) &&
                 make_tmap_2d(&m_dn.a0, L.w_down, 1, L.F / 2, E * L.D, 32, 64, false);
        // the shared expert's token tiles come straight from x: a 256-row box that
        // runs past row T - 1 reads zeros there
        ok = ok && make_tmap_2d(&m_sgu.b, xin, 2, L.D, uint64_t(T), 64, TC_BLOCK_TOKENS, true) &&
                 make_tmap_2d(&m_sgu.b_small, xin, 2, L.D, uint64_t(T), 64, TC_SMALL_TOKENS, true) &&
                  make_tmap_2d(&m_sgu.a0, L.ws_gate, 2, L.D, L.F_shared, 64, 16, true) &&
                  make_tmap_2d(&m_sgu.a1, L.ws_up, 2, L.D, L.F_shared, 64, 16, true) &&
                  make_tmap_2d(&m_sdn.b, h_s, 2, L.F_shared, T_pad, 64, TC_BLOCK_TOKENS, true) &&
                 make_tmap_2d(&m_sdn.b_small, h_s, 2, L.F_shared, T_pad, 64, TC_SMALL_TOKENS, true) &&
                  make_tmap_2d(&m_sdn.a0, L.ws_down, 2, L.F_shared, L.D, 64, 16, true);
        if (!ok) return false;
        m_dn.a1 = m_dn.a0;
        m_sdn.a1 = m_sdn.a0;
            return true;
        };
        if (!build(pm[0], pm[1], pm[2], pm[3])) return MOE_ERR_CUDA;
        pkey = key;
    }
    TcMaps& m_gu = pm[0];
    TcMaps& m_dn = pm[1];
    TcMaps& m_sgu = pm[2];
    TcMaps& m_sdn = pm[3];

    TcParams p;
    memset(&p, 0, sizeof(p));
    p.chunks = chunks;
    p.n_chunks = nch;
    p.gates = gates;
    p.perm = perm;
    p.inv_perm = inv;
    p.k_top = L.k;
    p.group_shift = L.group_size == 32 ? 5 : L.group_size == 64 ? 6 : 7;   // int4: log2 of the group
    p.bf16_magic = kBf16Magic;
    p.status = status;
    float* y_shared = at<float>(ws, W.y_shared);

    if (!pr) {   // (rows with given experts: no shared expert)
        // shared gate/up -> h_s (bf16, natural order, by token)
        p.K = L.D; p.n_rows = L.F_shared; p.n_fblocks = L.F_shared / 64; p.routed = 0;
        p.h_out = h_s;
        mk.mark(st);
        s = launch_tc_gemm(TC_GATEUP_BF16, m_sgu, p, st);
        if (s != MOE_OK) return s;
        // shared down -> y_s (fp32, by token)
        p.K = L.F_shared; p.n_rows = L.D; p.n_fblocks = L.D / 128;
        p.h_out = nullptr; p.y_out = y_shared;
        mk.mark(st);
        s = launch_tc_gemm(TC_DOWN_BF16, m_sdn, p, st);
        if (s != MOE_OK) return s;
    }
    // routed gate/up -> h (bf16 by slot position; int4: fragment order, e4m3: natural order)
    p.K = L.D; p.n_rows = L.F; p.n_fblocks = L.F / 64; p.routed = 1;
    p.s0 = L.s_gate; p.s1 = L.s_up; p.h_out = h_sorted; p.y_out = nullptr;
    p.tok_scale = fp8 ? at<float>(ws, W.xq_scale) : nullptr;
    mk.mark(st);
    s = launch_tc_gemm(fp8 ? TC_GATEUP_FP8 : TC_GATEUP_INT4, m_gu, p, st);
    if (s != MOE_OK) return s;
    if (fp8) {   // e4m3 rows of h (every expert matmul quantizes its input rows)
        mk.mark(st);
        s = launch_quantize_fp8_rows(h_sorted, MOE_DTYPE_BF16, S, L.F, S, L.act_scale_ub, at<uint8_t>(ws, W.hq),
                                     at<float>(ws, W.hq_scale), st);
        if (s != MOE_OK) return s;
    }
    // routed down: with one slot per token it finishes the layer (shared + gate * y);
    // otherwise gate * y by slot, summed per token by the combine
    p.K = L.F; p.n_rows = L.D; p.n_fblocks = L.D / 128;
    p.s0 = L.s_down; p.s1 = nullptr; p.h_out = nullptr;
    p.tok_scale = fp8 ? at<float>(ws, W.hq_scale) : nullptr;
    if (pr) { p.out = nullptr; p.y_r = nullptr; p.y_out = pr->y; }   // gate * y by row
    else if (L.k == 1) { p.out = out; p.y_r = y_shared; p.y_out = nullptr; }
    else { p.out = nullptr; p.y_r = nullptr; p.y_out = y_pos; }
    mk.mark(st);
    s = launch_tc_gemm(fp8 ? TC_DOWN_FP8 : TC_DOWN_INT4, m_dn, p, st);
    if (s != MOE_OK) return s;
    if (pr) return MOE_OK;
    if (L.k > 1) {
        mk.mark(st);
        s = launch_combine_slots(y_shared, y_pos, T, L.D, L.k, out, st);
    }
    mk.mark(st);
    return s;
}

moe_status ffn_forward_impl(const moe_layer_desc* layer, const void* x, int32_t T, void* out, void* workspace,
                            size_t workspace_bytes, cudaStream_t st, Marks mk = Marks()) {
    moe_status s = check_layer(layer);
    if (s != MOE_OK) return s;
    s = check_route_shape(T, layer->D, layer->E, layer->k);
    if (s != MOE_OK) return s;
    if (!x || !out || !workspace || !aligned16(x) || !aligned16(out) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return MOE_ERR_INVALID_ARG;
    const int path = choose_path(*layer, T);
    const WsLayout W = ws_layout(*layer, T, path);
    if (workspace_bytes < W.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    if (path == PATH_SEL_DECODE && !decode_fits(*layer)) return MOE_ERR_UNSUPPORTED_SHAPE;
    // the device status word and the zero rows read in place of missing tokens
    if (cudaMemsetAsync(at<int32_t>(workspace, W.status), 0, W.zeros_end - W.status, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    // With the block's RMSNorm the router normalizes x on the way and writes
    // xn; every kernel after it reads xn.
    const bf16* xr = static_cast<const bf16*>(x);
    const bf16* xin = layer->rms_weight ? at<bf16>(workspace, W.xn) : xr;
    if (path == PATH_SEL_DECODE)
        return ffn_decode_path(*layer, xr, xin, T, static_cast<bf16*>(out), workspace, W, st, mk);
    return ffn_prefill_path(*layer, xr, xin, T, static_cast<bf16*>(out), workspace, W, st, mk);
}

}  // namespace

extern "C" {

const char* moe_status_string(moe_status status) {
    switch (status) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
        case MOE_ERR_CUDA: return "CUDA error";
        case MOE_ERR_TIMEOUT: return "device wait timed out";
    }
    return "unknown status";
}

int32_t moe_abi_version(void) { return 2; }

moe_status moe_quantize_int4(const float* w, int64_t rows, int64_t cols, int32_t group_size, uint8_t* codes,
                             float* scales, void* stream) {
    if (!int4_group_ok(group_size)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (rows < 0 || cols <= 0 || cols % 128 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (rows == 0) return MOE_OK;
    if (!w || !codes || !scales || !aligned16(w) || !aligned16(codes) || !aligned16(scales))
        return MOE_ERR_INVALID_ARG;
    return launch_quantize_int4(w, rows, cols, group_size, codes, scales, as_stream(stream));
}

moe_status moe_quantize_fp8_rows(const void* x, int32_t x_dtype, int64_t rows, int64_t cols,
                                 int64_t num_valid_rows, float scale_ub, uint8_t* q, float* scales,
                                 void* stream) {
    if (x_dtype != MOE_DTYPE_BF16 && x_dtype != MOE_DTYPE_FP32) return MOE_ERR_INVALID_ARG;
    if (rows < 0 || cols <= 0 || cols % 8 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (num_valid_rows < 0 || num_valid_rows > rows) return MOE_ERR_INVALID_ARG;
    if (!(scale_ub > 0.0f)) return MOE_ERR_INVALID_ARG;   // also rejects NaN
    if (rows == 0) return MOE_OK;
    if (!x || !q || !scales || !aligned16(x) || !aligned16(q) || !aligned16(scales)) return MOE_ERR_INVALID_ARG;
    return launch_quantize_fp8_rows(x, x_dtype, rows, cols, num_valid_rows, scale_ub, q, scales,
                                    as_stream(stream));
}

moe_status moe_route(const void* x, int32_t T, int32_t D, const void* w_router, const float* router_bias,
                     int32_t E, int32_t k, int32_t* topk_ids, float* topk_gates, int32_t* expert_counts,
                     int32_t* expert_offsets, int32_t* perm, void* stream) {
    moe_status s = check_route_shape(T, D, E, k);
    if (s != MOE_OK) return s;
    const void* ptrs[] = {x, w_router, topk_ids, topk_gates, expert_counts, expert_offsets, perm};
    for (const void* p : ptrs)
        if (!p || !aligned16(p)) return MOE_ERR_INVALID_ARG;
    if (router_bias && !aligned16(router_bias)) return MOE_ERR_INVALID_ARG;
    return launch_route(static_cast<const bf16*>(x), T, D, static_cast<const bf16*>(w_router), router_bias, E, k,
                        topk_ids, topk_gates, expert_counts, expert_offsets, perm, nullptr, nullptr,
                        as_stream(stream), nullptr);
}

size_t moe_ffn_workspace_size(const moe_layer_desc* layer, int32_t T_max) {
    if (check_layer(layer) != MOE_OK || T_max < 1 || T_max > kMaxT) return 0;
    return ws_bytes(*layer, T_max);
}

moe_status moe_ffn_forward(const moe_layer_desc* layer, const void* x, int32_t T, void* out, void* workspace,
                           size_t workspace_bytes, void* stream) {
    return ffn_forward_impl(layer, x, T, out, workspace, workspace_bytes, as_stream(stream));
}

moe_status moe_ffn_forward_host(const moe_layer_desc* layer, const void* x_host, int32_t T, void* out_host,
                                void* workspace, size_t workspace_bytes, void* stream) {
    moe_status s = check_layer(layer);
    if (s != MOE_OK) return s;
    s = check_route_shape(T, layer->D, layer->E, layer->k);
    if (s != MOE_OK) return s;
    if (!x_host || !out_host || !workspace) return MOE_ERR_INVALID_ARG;
    const WsLayout W = ws_layout(*layer, T, choose_path(*layer, T));
    if (workspace_bytes < W.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t st = as_stream(stream);
    const size_t bytes = size_t(T) * layer->D * 2;
    void* xd = at<void>(workspace, W.x_in);
    void* od = at<void>(workspace, W.out);
    if (cudaMemcpyAsync(xd, x_host, bytes, cudaMemcpyHostToDevice, st) != cudaSuccess) return MOE_ERR_CUDA;
    s = ffn_forward_impl(layer, xd, T, od, workspace, workspace_bytes, st);
    if (s != MOE_OK) return s;
    if (cudaMemcpyAsync(out_host, od, bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
}

moe_status moe_ffn_forward_timed(const moe_layer_desc* layer, const void* x, int32_t T, void* out,
                                 void* workspace, size_t workspace_bytes, void* stream, void* const* events,
                                 int32_t n_events) {
    if (!layer) return MOE_ERR_INVALID_ARG;
    const int32_t need = layer_launch_names(*layer, T, nullptr, 0);
    if (!events || n_events < need + 1) return MOE_ERR_INVALID_ARG;
    for (int32_t i = 0; i < n_events; ++i)
        if (!events[i]) return MOE_ERR_INVALID_ARG;
    Marks mk;
    mk.ev = events;
    mk.n = n_events;
    return ffn_forward_impl(layer, x, T, out, workspace, workspace_bytes, as_stream(stream), mk);
}

int32_t moe_ffn_launch_names(const moe_layer_desc* layer, int32_t T, const char** names, int32_t max_names) {
    if (check_layer(layer) != MOE_OK || T < 1) return 0;
    return layer_launch_names(*layer, T, names, max_names);
}

moe_status moe_rmsnorm(const void* x, int32_t T, int32_t D, const void* gamma, float eps, void* out,
                       void* stream) {
    if (T < 1 || T > kMaxT || !valid_dim(D)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!x || !gamma || !out || !aligned16(x) || !aligned16(gamma) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
    if (!(eps >= 0.0f) || eps > 1.0f) return MOE_ERR_INVALID_ARG;
    return launch_rmsnorm(static_cast<const bf16*>(x), T, D, static_cast<const bf16*>(gamma), eps,
                          static_cast<bf16*>(out), as_stream(stream));
}

moe_status moe_ffn_device_status(const void* workspace, void* stream) {
    if (!workspace) return MOE_ERR_INVALID_ARG;
    int32_t v = 0;
    cudaStream_t st = as_stream(stream);
    if (cudaMemcpyAsync(&v, workspace, 4, cudaMemcpyDeviceToHost, st) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
    return v == DEV_OK ? MOE_OK : v == DEV_BAD_EXPERT ? MOE_ERR_INVALID_ARG : MOE_ERR_TIMEOUT;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Layer forward without caller-provided scratch.
//
// The scratch lives in one file-scope device array of kNoAllocScratchBytes.
// Every device that loads this library reserves it for the life of the
// process, so it is kept small: it covers the layer's intermediate buffers for
// decode-sized batches only.  Host code cannot use the array's name as a
// device address (it names a host-side shadow), so the first call on each
// device asks the runtime for the real address, with that device current,
// and remembers it.  Calls share the array and it keeps whatever the previous
// call left; the layer path already clears what must start at zero (the
// device status word and the task counters) on every call.  The status word
// sits at the array's start, where moe_ffn_noalloc_device_status reads it.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;   // 8 MiB
constexpr int kNoAllocMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mutex;
void* g_noalloc_addr[kNoAllocMaxDevices] = {};

moe_status noalloc_scratch_address(void** addr) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (g_noalloc_addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
        g_noalloc_addr[dev] = p;
    }
    *addr = g_noalloc_addr[dev];
    return MOE_OK;
}

}  // namespace

extern "C" moe_status moe_ffn_forward_noalloc(const moe_layer_desc* layer, const void* x, int32_t T, void* out,
                                              void* stream) {
    moe_status s = check_layer(layer);
    if (s != MOE_OK) return s;
    s = check_route_shape(T, layer->D, layer->E, layer->k);
    if (s != MOE_OK) return s;
    // argument errors first: nothing below touches the CUDA runtime until they pass
    if (!x || !out || !aligned16(x) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
    if (ws_layout(*layer, T, choose_path(*layer, T)).total > kNoAllocScratchBytes) return MOE_ERR_WORKSPACE_TOO_SMALL;
    void* scratch = nullptr;
    s = noalloc_scratch_address(&scratch);
    if (s != MOE_OK) return s;
    return ffn_forward_impl(layer, x, T, out, scratch, kNoAllocScratchBytes, as_stream(stream));
}

extern "C" moe_status moe_ffn_noalloc_device_status(void* stream) {
    void* scratch = nullptr;
    moe_status s = noalloc_scratch_address(&scratch);
    if (s != MOE_OK) return s;
    return moe_ffn_device_status(scratch, stream);
}

extern "C" moe_status moe_set_wait_limit(int64_t cycles) {
    // the default, or the caller's limit (at most the default)
    const uint32_t c = cycles > 0 && cycles < int64_t(kWaitCycles) ? uint32_t(cycles) : kWaitCycles;
    moe_status s = set_wait_limit_decode(c);
    if (s != MOE_OK) return s;
    return set_wait_limit_tc(c);
}

// ---------------------------------------------------------------------------
// Dense SwiGLU FFN layer: the FFN of the dense layers that alternate with the
// MoE layers ("Llama" (illegalscreed.cn), introduction: dense and MoE layers
// alternate; "Llama 开源模型系列" (docs.ifdog.com), "SwiGLU：门控激活的数学"):
//   out = bf16( (silu(x Wg^T) * (x Wu^T)) Wd^T ), bf16 weights, the hidden
// activation rounded to bf16 -- the MoE layer's shared expert without the
// routed experts.  It runs the shared-expert kernels of either path:
//   weight streaming: [rmsnorm,] dense_prep, decode gate/up, decode down (its epilogue writes out)
//   tensor cores:     [rmsnorm,] dense_prep, copy to whole tiles, gate/up, down, combine
// dense_prep writes the token chunk list the kernels take their tasks from.
// ---------------------------------------------------------------------------
namespace {

constexpr int32_t kDenseDecodeMaxT = 64;   // AUTO streams the weights up to this many tokens

struct DenseWs {
    size_t status, counters, ocnt, zeros_end, chunks, nchunks, xn;
    size_t h, y;          // hidden [T(_pad), F] bf16, fp32 result [T, D]
    size_t total;
};

int dense_path(const moe_dense_desc& L, int64_t T) {
    if (L.path == MOE_PATH_DECODE) return PATH_SEL_DECODE;
    if (L.path == MOE_PATH_PREFILL) return PATH_SEL_PREFILL;
    return T <= kDenseDecodeMaxT ? PATH_SEL_DECODE : PATH_SEL_PREFILL;
}

DenseWs dense_layout(const moe_dense_desc& L, int64_t T, int path) {
    DenseWs w;
    memset(&w, 0, sizeof(w));
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off += (bytes + 255) & ~size_t(255);
        return o;
    };
    const int64_t T_pad = ceil_div(T, TC_BLOCK_TOKENS) * TC_BLOCK_TOKENS;
    const int64_t rows = path == PATH_SEL_DECODE ? T : T_pad;
    w.status = take(64);
    w.counters = take(64);
    w.ocnt = take(path == PATH_SEL_DECODE ? size_t(T) * (L.D / 64) * 4 : 0);   // contributions per output block
    w.zeros_end = off;
    w.chunks = take(size_t(ceil_div(T, 16)) * sizeof(ChunkEntry));
    w.nchunks = take(16);
    w.xn = take(L.rms_weight ? size_t(T) * L.D * 2 : 0);
    w.h = take(size_t(rows) * L.F * 2);
    w.y = take(size_t(T) * L.D * 4);
    w.total = off;
    return w;
}

moe_status check_dense(const moe_dense_desc* L) {
    if (!L) return MOE_ERR_INVALID_ARG;
    if (!valid_dim(L->D) || !valid_dim(L->F)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (L->path < MOE_PATH_AUTO || L->path > MOE_PATH_PREFILL) return MOE_ERR_INVALID_ARG;
    const void* ptrs[] = {L->w_gate, L->w_up, L->w_down};
    for (const void* p : ptrs)
        if (!p || !aligned16(p)) return MOE_ERR_INVALID_ARG;
    if (L->rms_weight && (!aligned16(L->rms_weight) || !(L->rms_eps >= 0.0f) || L->rms_eps > 1.0f))
        return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

// The chunk list of the shared-expert tasks: chunks of `ct` tokens; both
// counts of the list header = the number of chunks (no routed chunks).
__global__ void dense_prep_kernel(ChunkEntry* chunks, int32_t* n_chunks, int T, int ct) {
    const int n = (T + ct - 1) / ct;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        ChunkEntry ce;
        ce.expert = -1;
        ce.start = i * ct;
        ce.count = min(ct, T - i * ct);
        ce.pad = 0;
        chunks[i] = ce;
    }
    if (threadIdx.x == 0) { n_chunks[0] = n; n_chunks[1] = n; }
}

struct DenseKey {
    moe_dense_desc L;
    const void* ws;
    const void* x;
    int64_t T;
    int path;
    bool valid;
};

DenseKey dense_key(const moe_dense_desc& L, const void* ws, const void* x, int64_t T, int path) {
    DenseKey k;
    memset(&k, 0, sizeof(k));
    memcpy(&k.L, &L, sizeof(L));
    k.ws = ws;
    k.x = x;
    k.T = T;
    k.path = path;
    k.valid = true;
    return k;
}

bool same_dense_key(const DenseKey& a, const DenseKey& b) {
    return a.valid && b.valid && memcmp(&a.L, &b.L, sizeof(a.L)) == 0 && a.ws == b.ws && a.x == b.x &&
           a.T == b.T && a.path == b.path;
}

// y_add (fp32 [T, k_add, D], or null): outputs of each token's k_add routed
// slots, added in slot order (the shared-expert half of an expert-parallel
// MoE layer): out = bf16(ffn(x) + sum_j y_add[t, j]).
moe_status dense_forward_impl(const moe_dense_desc* layer, const void* x, int32_t T, void* out, void* ws,
                              size_t ws_bytes, cudaStream_t st, const float* y_add = nullptr, int k_add = 0) {
    moe_status s = check_dense(layer);
    if (s != MOE_OK) return s;
    const moe_dense_desc& L = *layer;
    if (T < 1 || T > kMaxT) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!x || !out || !ws || !aligned16(x) || !aligned16(out) || (reinterpret_cast<uintptr_t>(ws) & 255u))
        return MOE_ERR_INVALID_ARG;
    const int path = dense_path(L, T);
    const DenseWs W = dense_layout(L, T, path);
    if (ws_bytes < W.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    if (cudaMemsetAsync(at<int32_t>(ws, W.status), 0, W.zeros_end - W.status, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    const bf16* xin = static_cast<const bf16*>(x);
    if (L.rms_weight) {
        s = launch_rmsnorm(xin, T, L.D, static_cast<const bf16*>(L.rms_weight), L.rms_eps, at<bf16>(ws, W.xn), st);
        if (s != MOE_OK) return s;
        xin = at<bf16>(ws, W.xn);
    }
    ChunkEntry* chunks = at<ChunkEntry>(ws, W.chunks);
    int32_t* nch = at<int32_t>(ws, W.nchunks);
    int32_t* status = at<int32_t>(ws, W.status);
    bf16* h = at<bf16>(ws, W.h);
    float* y = at<float>(ws, W.y);
    dense_prep_kernel<<<1, 256, 0, st>>>(chunks, nch, T, path == PATH_SEL_DECODE ? 16 : TC_BLOCK_TOKENS);
    s = launch_status();
    if (s != MOE_OK) return s;

    if (path == PATH_SEL_DECODE) {
        static thread_local DenseKey key_d;
        static thread_local DecodeMaps m1, m2;
        const DenseKey key = dense_key(L, ws, xin, T, path);
        if (!same_dense_key(key, key_d)) {
            key_d.valid = false;
            const uint32_t rows = uint32_t(decode_task_rows());
            bool ok = make_tmap_2d(&m1.s0, L.w_gate, 2, L.D, L.F, 64, rows, true) &&
                      make_tmap_2d(&m1.s1, L.w_up, 2, L.D, L.F, 64, rows, true) &&
                      make_tmap_rows_3d(&m1.bs, xin, L.D, T, 16, 1) &&
                      make_tmap_2d(&m2.s0, L.w_down, 2, L.F, L.D, 64, rows, true) &&
                      make_tmap_rows_3d(&m2.bs, h, L.F, T, 16, 2);
            if (!ok) return MOE_ERR_CUDA;
            // no routed tasks: the routed maps are never used; valid copies fill them
            m1.r0 = m1.r1 = m1.g0 = m1.g1 = m1.s0;
            m1.br = m1.cr = m1.bs;
            m2.s1 = m2.r0 = m2.r1 = m2.g0 = m2.g1 = m2.s0;
            m2.br = m2.cr = m2.bs;
            key_d = key;
        }
        DecodeParams p;
        memset(&p, 0, sizeof(p));
        p.T = T;
        p.n_rows_r = decode_task_rows();   // routed rows: unused (no routed chunks)
        p.n_rows_s = L.F;
        p.K_r = L.D;
        p.K_s = L.D;
        p.k_top = y_add ? k_add : 0;   // routed outputs by slot, if any, are given: the shared
        p.n_contrib = 0;                 // expert's contribution is each output's only one
        p.y_r = const_cast<float*>(y_add);
        p.scale_buf_floats = 0;
        p.f16_magic_lo = kF16MagicLo;
        p.f16_magic_hi = kF16MagicHi;
        p.chunks = chunks;
        p.n_chunks = nch;
        p.h_s = h;
        p.task_counter = at<int32_t>(ws, W.counters);
        p.status = status;
        s = launch_decode_ffn(0, 128, m1, p, st);
        if (s != MOE_OK) return s;
        p.n_rows_s = L.D;
        p.K_r = L.F;
        p.K_s = L.F;
        p.y_s = y;
        p.out = static_cast<bf16*>(out);
        p.ocnt = at<int32_t>(ws, W.ocnt);
        p.task_counter = at<int32_t>(ws, W.counters) + 1;
        return launch_decode_ffn(1, 128, m2, p, st);
    }

    const uint64_t T_pad = uint64_t(ceil_div(T, TC_BLOCK_TOKENS) * TC_BLOCK_TOKENS);
    static thread_local DenseKey key_p;
    static thread_local TcMaps mg, md;
    const DenseKey key = dense_key(L, ws, xin, T, path);
    if (!same_dense_key(key, key_p)) {
        key_p.valid = false;
        bool ok = make_tmap_2d(&mg.b, xin, 2, L.D, uint64_t(T), 64, TC_BLOCK_TOKENS, true) &&
                 make_tmap_2d(&mg.b_small, xin, 2, L.D, uint64_t(T), 64, TC_SMALL_TOKENS, true) &&
                  make_tmap_2d(&mg.a0, L.w_gate, 2, L.D, L.F, 64, 16, true) &&
                  make_tmap_2d(&mg.a1, L.w_up, 2, L.D, L.F, 64, 16, true) &&
                  make_tmap_2d(&md.b, h, 2, L.F, T_pad, 64, TC_BLOCK_TOKENS, true) &&
                 make_tmap_2d(&md.b_small, h, 2, L.F, T_pad, 64, TC_SMALL_TOKENS, true) &&
                  make_tmap_2d(&md.a0, L.w_down, 2, L.F, L.D, 64, 16, true);
        if (!ok) return MOE_ERR_CUDA;
        md.a1 = md.a0;
        key_p = key;
    }
    TcParams p;
    memset(&p, 0, sizeof(p));
    p.chunks = chunks;
    p.n_chunks = nch;
    p.k_top = 1;
    p.group_shift = 7;
    p.bf16_magic = kBf16Magic;
    p.status = status;
    p.K = L.D; p.n_rows = L.F; p.n_fblocks = L.F / 64; p.routed = 0;
    p.h_out = h;
    s = launch_tc_gemm(TC_GATEUP_BF16, mg, p, st);
    if (s != MOE_OK) return s;
    p.K = L.F; p.n_rows = L.D; p.n_fblocks = L.D / 128;
    p.h_out = nullptr; p.y_out = y;
    s = launch_tc_gemm(TC_DOWN_BF16, md, p, st);
    if (s != MOE_OK) return s;
    return launch_combine_slots(y, y_add, T, L.D, y_add ? k_add : 0, static_cast<bf16*>(out), st);
}

}  // namespace

extern "C" size_t moe_dense_ffn_workspace_size(const moe_dense_desc* layer, int32_t T_max) {
    if (check_dense(layer) != MOE_OK || T_max < 1 || T_max > kMaxT) return 0;
    if (layer->path != MOE_PATH_AUTO) return dense_layout(*layer, T_max, dense_path(*layer, T_max)).total;
    const size_t a = dense_layout(*layer, T_max, PATH_SEL_DECODE).total;
    const size_t b = dense_layout(*layer, T_max, PATH_SEL_PREFILL).total;
    return a > b ? a : b;
}

extern "C" moe_status moe_dense_ffn_forward(const moe_dense_desc* layer, const void* x, int32_t T, void* out,
                                            void* workspace, size_t workspace_bytes, void* stream) {
    return dense_forward_impl(layer, x, T, out, workspace, workspace_bytes, as_stream(stream));
}

// ---- expert parallelism: the routed experts on given rows; the shared
// expert plus the combine of given routed outputs ----
namespace {
moe_layer_desc one_slot_layer(const moe_layer_desc& L) {
    moe_layer_desc L1 = L;   // rows with one expert each, no RMSNorm (the rows arrive normalized)
    L1.k = 1;
    L1.rms_weight = nullptr;
    return L1;
}

moe_dense_desc shared_as_dense(const moe_layer_desc& L) {
    moe_dense_desc d;
    memset(&d, 0, sizeof(d));
    d.D = L.D;
    d.F = L.F_shared;
    d.path = L.path;
    d.w_gate = L.ws_gate;
    d.w_up = L.ws_up;
    d.w_down = L.ws_down;
    d.rms_weight = L.rms_weight;
    d.rms_eps = L.rms_eps;
    return d;
}
}  // namespace

extern "C" size_t moe_expert_ffn_workspace_size(const moe_layer_desc* layer, int32_t n_max) {
    if (check_layer(layer) != MOE_OK || n_max < 1 || n_max > kMaxT) return 0;
    return ws_bytes(one_slot_layer(*layer), n_max);
}

extern "C" moe_status moe_expert_ffn_forward(const moe_layer_desc* layer, const void* x, int32_t n,
                                             const int32_t* expert_ids, const float* gates, float* y,
                                             void* workspace, size_t workspace_bytes, void* stream) {
    moe_status s = check_layer(layer);
    if (s != MOE_OK) return s;
    const moe_layer_desc L = one_slot_layer(*layer);
    s = check_route_shape(n, L.D, L.E, 1);
    if (s != MOE_OK) return s;
    const void* ptrs[] = {x, expert_ids, gates, y, workspace};
    for (const void* ptr : ptrs)
        if (!ptr || !aligned16(ptr)) return MOE_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return MOE_ERR_INVALID_ARG;
    const int path = choose_path(L, n);
    const WsLayout W = ws_layout(L, n, path);
    if (workspace_bytes < W.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    if (path == PATH_SEL_DECODE && !decode_fits(L)) return MOE_ERR_UNSUPPORTED_SHAPE;
    cudaStream_t st = as_stream(stream);
    if (cudaMemsetAsync(at<int32_t>(workspace, W.status), 0, W.zeros_end - W.status, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    PreRouted pr{expert_ids, gates, y};
    Marks mk;
    const bf16* xr = static_cast<const bf16*>(x);
    if (path == PATH_SEL_DECODE) return ffn_decode_path(L, xr, xr, n, nullptr, workspace, W, st, mk, &pr);
    return ffn_prefill_path(L, xr, xr, n, nullptr, workspace, W, st, mk, &pr);
}

extern "C" size_t moe_shared_ffn_workspace_size(const moe_layer_desc* layer, int32_t T_max) {
    if (check_layer(layer) != MOE_OK) return 0;
    const moe_dense_desc d = shared_as_dense(*layer);
    return moe_dense_ffn_workspace_size(&d, T_max);
}

extern "C" moe_status moe_shared_ffn_combine(const moe_layer_desc* layer, const void* x, int32_t T,
                                             const float* y_slots, void* out, void* workspace,
                                             size_t workspace_bytes, void* stream) {
    moe_status s = check_layer(layer);
    if (s != MOE_OK) return s;
    if (!y_slots || !aligned16(y_slots)) return MOE_ERR_INVALID_ARG;
    const moe_dense_desc d = shared_as_dense(*layer);
    return dense_forward_impl(&d, x, T, out, workspace, workspace_bytes, as_stream(stream), y_slots, layer->k);
}

