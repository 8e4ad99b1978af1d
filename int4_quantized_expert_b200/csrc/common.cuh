// Shared device helpers for libmoe_int4 (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <mutex>
#include <set>
#include <utility>

#include "moe_int4.h"

namespace moe {

typedef __nv_bfloat16 bf16;

// Device status word values (written into the workspace's first int32).
enum : int32_t { DEV_OK = 0, DEV_TIMEOUT = 1, DEV_BAD_EXPERT = 2 };

constexpr int kGroup = 128;   // int4 group size along K

__host__ __device__ inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

inline moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

inline moe_status launch_status() { return cuda_status(cudaGetLastError()); }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---------------------------------------------------------------------------
// Programmatic dependent launch.  A kernel launched with launch_pdl may start
// while the kernel before it in the stream is still running: it runs code
// that reads none of that kernel's outputs, then calls griddep_wait(), which
// returns once the preceding kernel has completed and its writes are visible.
// Every kernel of a chain calls griddep_wait() before it completes, so each
// completion implies the completion of everything before it.  Kernels call
// griddep_launch_dependents() as they start, letting the next kernel launch.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Allow a kernel the device's largest dynamic shared memory, once per device.
template <typename... KArgs>
inline moe_status allow_max_smem(void (*kernel)(KArgs...)) {
    static std::mutex mu;
    static std::set<std::pair<const void*, int>> done;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(mu);
    const auto key = std::make_pair(reinterpret_cast<const void*>(kernel), dev);
    if (done.count(key)) return MOE_OK;
    int optin = 0;
    cudaFuncAttributes fa;
    if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
        cudaFuncGetAttributes(&fa, kernel) != cudaSuccess ||
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             optin - int(fa.sharedSizeBytes)) != cudaSuccess)   // static shared memory counts too
        return MOE_ERR_CUDA;
    done.insert(key);
    return MOE_OK;
}

template <typename... KArgs, typename... Args>
inline moe_status launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                             Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cuda_status(cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...));
}

// ---------------------------------------------------------------------------
// Read-only global loads that do not allocate in L1 (weights are streamed once)
// ---------------------------------------------------------------------------
// (Not volatile: they read memory no thread of the kernel writes, so the
// compiler may schedule them freely.)
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// Read-only global load that may be cached in L1 (small operands reused by many warps)
__device__ __forceinline__ uint4 ldg_cached(const void* p) {
    uint4 v;
    asm("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ float ldg_f32(const float* p) {
    float v;
    asm("ld.global.nc.f32 %0, [%1];" : "=f"(v) : "l"(p));
    return v;
}

// ---------------------------------------------------------------------------
// bf16x2 helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);   // .x = lo (low half)
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// Two int4 codes -> exact bf16x2 values q in [-8, 7].
// `w` holds 8 two's-complement nibbles n0..n7 (n0 in bits 0..3).  For a shift
// s in {0, 4, 8, 12}, the nibbles at bit positions s and s + 16 are moved into
// the low mantissa bits of two bf16 numbers with exponent 2^7 (0x4300 = 128.0,
// mantissa step 1), after flipping each nibble's sign bit (q + 8 in 0..15):
// the pair then holds 128 + q + 8, and subtracting 136 gives q exactly.
template <int SHIFT>
__device__ __forceinline__ uint32_t int4x2_to_bf16x2(uint32_t w_xor88) {
    uint32_t t = ((w_xor88 >> SHIFT) & 0x000F000Fu) | 0x43004300u;
    __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&t);
    const __nv_bfloat162 bias = __floats2bfloat162_rn(136.0f, 136.0f);
    v = __hsub2(v, bias);
    return *reinterpret_cast<uint32_t*>(&v);
}

// ---------------------------------------------------------------------------
// Warp-level tensor-core MMA: m16n8k16, bf16 inputs, fp32 accumulate.
// A fragment (16x16, row major): a0 = (r, k..k+1), a1 = (r+8, k..k+1),
//   a2 = (r, k+8..k+9), a3 = (r+8, k+8..k+9), r = lane/4, k = 2*(lane%4).
// B fragment (16x8): b0 = (k..k+1, n), b1 = (k+8..k+9, n), n = lane/4.
// C fragment (16x8): c0,c1 = (r, 2*(lane%4) + {0,1}), c2,c3 = (r+8, ...).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma_bf16_16816(float c[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The same shape with fp16 inputs: d = a * b + c (c separate from d).
__device__ __forceinline__ void mma_f16_16816(float d[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1, float c0, float c1, float c2, float c3) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%11,%12,%13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(c0), "f"(c1), "f"(c2), "f"(c3));
}

__device__ __forceinline__ void mma_f16_16816(float d[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
    mma_f16_16816(d, a0, a1, a2, a3, b0, b1, d[0], d[1], d[2], d[3]);
}

// int4 codes -> exact fp16 integers, two per instruction.  0x6400 is 1024.0
// in fp16, whose mantissa step is 1; a nibble placed in mantissa bits 0..3
// with its top bit flipped (two's-complement q -> q + 8) reads 1032 + q, and
// one in bits 4..7 reads 1024 + 16 (q + 8) = 1152 + 16 q.  Each is one LOP3
// (w & mask) ^ magic with the mask as the immediate and the magic in a
// register: kF16MagicLo / kF16MagicHi, which the caller passes in as a run-
// time value.  Written with both as compile-time constants the expression
// takes two ALU instructions, since one LOP3 holds one immediate.
// The same for bf16 (mantissa step 1 at 128.0 = 0x4300): nibbles in bits
// 0..3 of each half read 136 + q.
constexpr uint32_t kBf16Magic = 0x43084308u;
__device__ __forceinline__ uint32_t bf16_lo_nibbles(uint32_t w, uint32_t magic) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0x6a;" : "=r"(d) : "r"(w), "n"(0x000F000F), "r"(magic));
    return d;
}
constexpr uint32_t kF16MagicLo = 0x64086408u;
constexpr uint32_t kF16MagicHi = 0x64806480u;
__device__ __forceinline__ uint32_t f16_lo_nibbles(uint32_t w, uint32_t magic_lo) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0x6a;" : "=r"(d) : "r"(w), "n"(0x000F000F), "r"(magic_lo));   // (a & b) ^ c
    return d;
}
__device__ __forceinline__ uint32_t f16_hi_nibbles(uint32_t w, uint32_t magic_hi) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0x6a;" : "=r"(d) : "r"(w), "n"(0x00F000F0), "r"(magic_hi));
    return d;
}

__device__ __forceinline__ float silu_f32(float z) { return z / (1.0f + expf(-z)); }

// silu with the hardware exponential and division (a few ulps of fp32; used
// where the result is rounded to bf16 at once).  For z below about -88 the
// denominator overflows and the result is 0, as silu's is to fp32 precision.
__device__ __forceinline__ float silu_fast(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

}  // namespace moe

// ---------------------------------------------------------------------------
// mbarrier / TMA / bulk-copy helpers (sm_90+ PTX, used on sm_100a).
// Every wait is bounded: after ~kWaitCycles SM cycles it records DEV_TIMEOUT
// in the device status word and returns false; callers then wind down.
// ---------------------------------------------------------------------------
namespace moe {

constexpr uint32_t kWaitCycles = 2000000000u;   // about one second at 1.9 GHz

// The limit of the waits that report to a status word, in SM cycles.  It is
// kWaitCycles unless a test lowers it (moe_set_wait_limit) to make waits run
// out on purpose; waits that drain a CTA's own copies in flight (no status
// word) always keep kWaitCycles.  Each translation unit that waits on
// mbarriers has its own copy, set by set_wait_limit_<unit>().
static __constant__ uint32_t c_wait_limit = kWaitCycles;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Shared-memory accesses written as ld.shared / st.shared.  Given generic
// pointers into dynamic shared memory the compiler may emit generic loads,
// which take the slower L1TEX path (measured on the weight-streaming
// kernel's operand loads: 3-4 % of its time).  Volatile, so they keep their
// order with the mbarrier operations around them.
__device__ __forceinline__ uint4 ld_shared_v4(const void* p) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(smem_u32(p)));
    return v;
}
__device__ __forceinline__ uint32_t ld_shared_u32(const void* p) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)));
    return v;
}
__device__ __forceinline__ float ld_shared_f32(const float* p) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(smem_u32(p)));
    return v;
}
__device__ __forceinline__ float2 ld_shared_f32x2(const float* p) {
    float2 v;
    asm volatile("ld.shared.v2.f32 {%0,%1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(smem_u32(p)));
    return v;
}
__device__ __forceinline__ void st_shared_v4(void* p, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" :: "r"(smem_u32(p)), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}"
                 :: "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}"
                 :: "r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}

__device__ __forceinline__ int32_t ld_volatile(const int32_t* p) {
    return *reinterpret_cast<const volatile int32_t*>(p);
}

// try_wait with a suspend-time hint: a thread whose phase is not complete
// sleeps until it completes (or about hint_ns pass), so a waiter wakes as
// soon as its data lands and issues nothing meanwhile.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns) : "memory");
    return ok != 0;
}

// Thread-block cluster barrier (every thread of every CTA of the cluster).
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// A float in the shared memory of CTA `rank` of this cluster, at the address
// `p` has in this CTA.
__device__ __forceinline__ float ld_dsmem_f32(const float* p, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(p)), "r"(rank));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    return v;
}

// Bounded wait until a global counter written by other CTAs (atomicAdd after
// a __threadfence) reaches `target`; acquire semantics.  Followed by a proxy
// fence, so TMA (async-proxy) reads issued after it see what the counted
// writers stored.
__device__ __forceinline__ bool wait_counter(const int32_t* cnt, int32_t target, int32_t* status) {
    const uint32_t t0 = uint32_t(clock64());
    for (;;) {
        int32_t v;
        asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(cnt) : "memory");
        if (v >= target) break;
        if (uint32_t(clock64()) - t0 > c_wait_limit) {
            atomicExch(status, DEV_TIMEOUT);
            return false;
        }
        __nanosleep(256);
    }
    asm volatile("fence.proxy.async.global;" ::: "memory");
    return true;
}

// Non-blocking test of a phase (try_wait may suspend the thread for a while).
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}

// Bounded wait for the phase with the given parity to complete.  The
// device status word (another wait of this launch timed out) and the clock
// are checked only every 64 sleeps, so a wait that misses its first try costs
// no global-memory round trip.  With a lowered limit (tests) the waiter only
// polls, without ever suspending, so the limit decides when it gives up.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int32_t* status) {
    if (status != nullptr && c_wait_limit != kWaitCycles) {
        const uint32_t t0 = uint32_t(clock64());
        for (;;) {
            if (mbar_test_wait(bar, parity)) return true;
            if (uint32_t(clock64()) - t0 > c_wait_limit) {
                atomicExch(status, DEV_TIMEOUT);
                return false;
            }
        }
    }
    if (mbar_try_wait(bar, parity)) return true;
    const uint32_t t0 = uint32_t(clock64());   // 32-bit differences: the limit is below 2^32 cycles
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait_sleep(bar, parity, 10000u)) return true;
        if ((i & 63u) == 0) {
            if (status && ld_volatile(status) != DEV_OK) return false;
            if (uint32_t(clock64()) - t0 > kWaitCycles) {
                if (status) atomicExch(status, DEV_TIMEOUT);
                return false;
            }
        }
    }
}

// 2-D tiled TMA load global -> shared, completion counted on `bar` (bytes).
__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, uint64_t* bar, int32_t x,
                                            int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];"
        :: "r"(smem_u32(dst)), "l"(tmap), "r"(smem_u32(bar)), "r"(x), "r"(y) : "memory");
}

// 3-D tiled TMA load global -> shared, completion counted on `bar` (bytes).
__device__ __forceinline__ void tma_load_3d(void* dst, const void* tmap, uint64_t* bar, int32_t x, int32_t y,
                                            int32_t z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];"
        :: "r"(smem_u32(dst)), "l"(tmap), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z) : "memory");
}

// 1-D bulk copy global -> shared (16-byte aligned addresses, size % 16 == 0).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        :: "r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const void* tmap) {
    asm volatile("prefetch.tensormap [%0];" :: "l"(tmap) : "memory");
}

// Named barrier over a subset of the CTA's warps.
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t threads) {
    asm volatile("bar.sync %0, %1;" :: "r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ bool elect_one() {
    uint32_t pred = 0;
    asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(pred));
    return pred != 0;
}

}  // namespace moe
