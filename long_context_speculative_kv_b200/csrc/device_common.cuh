// device_common.cuh -- sm_100a device helpers for libwmtp: bounded mbarrier waits, TMA tile
// loads, ldmatrix / mma.sync fragments, bf16 packing and the device status word.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace wmtp {

// ---------------------------------------------------------------------------------------------
// Device status word: bit flags, read and cleared by wmtp_device_status().
enum : unsigned int {
    kStatusDeviceIndex = 1u,   // a page id outside [0, num_pages): the tile was skipped
    kStatusTimeout = 2u,       // a bounded wait gave up: the kernel returned early
};

// Defined once: the whole library is one translation unit (capi.cu includes every kernel).
__device__ unsigned int g_status = 0;

__device__ __forceinline__ void flag_status(unsigned int bit) { atomicOr(&g_status, bit); }

// ---------------------------------------------------------------------------------------------
// Time source for bounded waits (nanoseconds).
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Every spin-wait in this library gives up after this long, flags kStatusTimeout and lets the
// kernel return.  Healthy waits last microseconds.
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s

// Build-time timestamp trace for measurement (off unless WMTP_TRACE is defined): named points of
// CTA (0, 0) record the global timer; read with wmtp_trace_read.
// WMTP_TRACE_TILE(role, t) records tile t - kTraceT0 (of the first 32 tiles from kTraceT0) of one
// role in slot 64 + 32 role + (t - kTraceT0).
#ifdef WMTP_TRACE
constexpr int kTraceSlots = 64 + 32 * 12;
#ifndef WMTP_TRACE_T0
#define WMTP_TRACE_T0 0
#endif
constexpr int kTraceT0 = WMTP_TRACE_T0;
__device__ unsigned long long g_trace[kTraceSlots];
#define WMTP_TRACE_AT(i)                                                            \
    do {                                                                            \
        if (blockIdx.x == 0 && blockIdx.y == 0 && (i) < kTraceSlots) g_trace[(i)] = global_ns(); \
    } while (0)
#define WMTP_TRACE_TILE(role, t)                                                    \
    do {                                                                            \
        const int tt_ = (int)(t) - kTraceT0;                                        \
        if (tt_ >= 0 && tt_ < 32) WMTP_TRACE_AT(64 + 32 * (role) + tt_);             \
    } while (0)
// the latest time any CTA passed this point (slot i)
#define WMTP_TRACE_MAX(i) atomicMax(&g_trace[(i)], (unsigned long long)global_ns())
#else
#define WMTP_TRACE_MAX(i) \
    do {                  \
    } while (0)
#define WMTP_TRACE_AT(i) \
    do {                 \
    } while (0)
#define WMTP_TRACE_TILE(role, t) \
    do {                         \
    } while (0)
#endif

// ---------------------------------------------------------------------------------------------
// mbarrier (shared::cta).
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}"
                 ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}"
                 ::"r"(smem_addr(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(smem_addr(bar)), "r"(parity) : "memory");
    return ok != 0;
}

// Waits for the phase of `parity` to complete.  Returns false (and flags kStatusTimeout) after
// kWaitLimitNs: the caller must then stop using the pipeline.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    uint32_t spins = 0;
    while (!mbar_try_wait(bar, parity)) {
        if ((++spins & 255u) == 0u && global_ns() - t0 > kWaitLimitNs) {
            flag_status(kStatusTimeout);
            return false;
        }
    }
    return true;
}

// ---------------------------------------------------------------------------------------------
// TMA: 3-D tiled load of one box into shared memory, completing on an mbarrier (no multicast).
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y, int z, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4}], [%5], %6;"
        ::"r"(smem_addr(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z),
          "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

// L2 prefetch of one 3-D box (no shared memory, no completion to wait for): warms L2 only.
__device__ __forceinline__ void tma_prefetch_3d(const CUtensorMap* map, int x, int y, int z) {
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z)
                 : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// L2 policy for data read exactly once per call (the KV stream).
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// ---------------------------------------------------------------------------------------------
// Programmatic dependent launch.  Every kernel of the library lets the next kernel on the stream
// launch early (its CTAs then block in pdl_wait) and waits for its own predecessor to finish,
// with memory visible, before it touches global memory that kernel may write.  The attention
// kernels trigger only after their own wait, so the LSE merge that follows one may read the
// request lengths (final by then, and not written by the attention kernel) before its wait.
// Without the launch attribute both are no-ops.
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ---------------------------------------------------------------------------------------------
// Thread-block clusters: the hardware cluster barrier (every thread of every CTA of the cluster
// arrives; release / acquire order shared-memory writes before it with reads after it) and
// loads from another CTA's shared memory (distributed shared memory; no TMA, no multicast).
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Address of the same shared-memory offset in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t map_shared_rank(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

// (Reads of partials the cluster barrier has published: no ordering constraints of their own, so
// the compiler may batch them.)
__device__ __forceinline__ float ld_dsmem_f32(uint32_t addr) {
    float v;
    asm("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ float4 ld_dsmem_v4(uint32_t addr) {
    float4 v;
    asm("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
        : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
    return v;
}

// ---------------------------------------------------------------------------------------------
// ldmatrix / mma.sync (bf16 in, fp32 accumulate).
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                              uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

// D(16x8) += A(16x16, row) * B(16x8, col)
__device__ __forceinline__ void mma_bf16_16816(float* d, const uint32_t* a, uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// ---------------------------------------------------------------------------------------------
// fp16 MMA and fp8 (E4M3) widening, for the fp8-KV path: every E4M3 value and every bf16 query
// of normal magnitude is exact in fp16, so the products see the stored numbers unrounded.
__device__ __forceinline__ void mma_f16_16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Four E4M3 codes (a 32-bit word, lowest byte first) -> two fp16x2 words: lo = codes 0, 1 and
// hi = codes 2, 3 (the lower code in the lower half), with one cvt per pair.
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t codes, uint32_t& lo, uint32_t& hi) {
    asm("{\n\t.reg .b16 c01, c23;\n\t"
        "mov.b32 {c01, c23}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, c01;\n\t"
        "cvt.rn.f16x2.e4m3x2 %1, c23;\n\t}"
        : "=r"(lo), "=r"(hi) : "r"(codes));
}

// Two fp32 values -> two E4M3 codes (round to nearest even, saturating at +-448): `lo` in the
// lower byte, `hi` in the upper.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
    uint16_t d;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
    return (uint32_t)d;
}

// bf16x2 -> fp16x2 through fp32 (exact for values fp16 represents).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w) {
    return pack_f16x2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// Transposes the 8x8 16-bit matrix a warp holds in the ldmatrix fragment layout.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t a) {
    uint32_t d;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
    return d;
}

__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

}  // namespace wmtp
