// capi.cu -- the C ABI of libwmtp.so (declared in include/wmtp.h): host-side argument checks,
// TMA tensor-map encoding, workspace layout and kernel launches.  One translation unit holds all
// device code, so the device status word needs no relocatable device code.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdlib>
#include <cstdio>
#include <cstring>
#include <utility>
#include <atomic>
#include <mutex>

#include "wmtp.h"
#include "wmtp_loop.h"
#include "attn_kernels.cuh"
#include "attn_tc_kernels.cuh"
#include "ring_accept_kernels.cuh"
#include "loop_kernels.cuh"
#include "synth_kernels.cuh"

namespace wmtp {

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    int sm_count = 0;
    int major = 0;
    bool ok = false;
};

std::mutex g_mu;
std::atomic<unsigned long long> g_launches{0};

// Checks the launch just issued and counts it.
int launched() {
    if (cudaGetLastError() != cudaSuccess) return WMTP_ERR_CUDA;
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return WMTP_OK;
}
DeviceInfo g_dev[kMaxDevices];
bool g_dev_done[kMaxDevices] = {};
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int current_device(int* dev) {
    if (cudaGetDevice(dev) != cudaSuccess) return WMTP_ERR_CUDA;
    if (*dev < 0 || *dev >= kMaxDevices) return WMTP_ERR_CUDA;
    return WMTP_OK;
}

int device_info(DeviceInfo* out) {
    int dev;
    int rc = current_device(&dev);
    if (rc != WMTP_OK) return rc;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_dev_done[dev]) {
        DeviceInfo d;
        if (cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
            return WMTP_ERR_CUDA;
        d.ok = (d.major == 10);
        g_dev[dev] = d;
        g_dev_done[dev] = true;
    }
    *out = g_dev[dev];
    return out->ok ? WMTP_OK : WMTP_ERR_UNSUPPORTED;
}

int encoder(PFN_cuTensorMapEncodeTiled_v12000* fn) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_encode == nullptr) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || p == nullptr)
            return WMTP_ERR_CUDA;
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    *fn = g_encode;
    return WMTP_OK;
}

// A [n_blocks][rows][128] bf16 tensor viewed as 3-D (dim, row, block), read in 64x64 boxes with
// the 128-byte swizzle.  Rows past `rows` and blocks past `n_blocks` read as zero.  fp8: the
// same with 1-byte elements, read in 128x64 boxes (one 128-byte row per key).
int encode_rows_map(CUtensorMap* map, const void* base, long long rows, long long n_blocks,
                    bool fp8 = false) {
    PFN_cuTensorMapEncodeTiled_v12000 enc;
    int rc = encoder(&enc);
    if (rc != WMTP_OK) return rc;
    const cuuint64_t esz = fp8 ? 1 : 2;
    cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)rows, (cuuint64_t)n_blocks};
    cuuint64_t strides[2] = {(cuuint64_t)kD * esz, (cuuint64_t)rows * kD * esz};
    cuuint32_t box[3] = {fp8 ? 128u : 64u, (cuuint32_t)kTileKeys, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                     const_cast<void*>(base), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? WMTP_OK : WMTP_ERR_CUDA;
}

// Q of a call, [B, n_q, Hq, 128] bf16, viewed per kv head as 4-D (dim, g, h, b * n_q + i) and
// read in boxes of (64 dims, G heads, 1 kv head, n_q queries): one box lands as the unit's rows
// i * G + g, 128 bytes each, 128-byte swizzled (the tcgen05 A-operand layout).
int encode_q_map(CUtensorMap* map, const void* q, int B, int n_q, int Hq, int Hkv) {
    PFN_cuTensorMapEncodeTiled_v12000 enc;
    int rc = encoder(&enc);
    if (rc != WMTP_OK) return rc;
    const int G = Hq / Hkv;
    cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)G, (cuuint64_t)Hkv, (cuuint64_t)B * n_q};
    cuuint64_t strides[3] = {(cuuint64_t)kD * 2, (cuuint64_t)G * kD * 2, (cuuint64_t)Hq * kD * 2};
    cuuint32_t box[4] = {64, (cuuint32_t)G, 1, (cuuint32_t)n_q};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(q), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? WMTP_OK : WMTP_ERR_CUDA;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Stream-K plan: a CTA takes at least this many tiles (fewer, fuller CTAs measured slower for
// the small windowed calls, and more only lengthens the tail).
constexpr int kMinTilesPerCta = 2;

struct Shape {
    int B, n_q, Hq, Hkv, G, rows_total, rows_blk, n_rb, units;
};

int check_shape(int B, int n_q, int Hq, int Hkv, int D, Shape* s) {
    if (B < 1 || n_q < 1 || Hq < 1 || Hkv < 1) return WMTP_ERR_ARG;
    if (D != WMTP_HEAD_DIM) return WMTP_ERR_SHAPE;
    if (Hq % Hkv != 0 || Hq / Hkv > WMTP_MAX_GROUP || n_q > WMTP_MAX_QUERIES || B > kMaxBatch)
        return WMTP_ERR_SHAPE;
    s->B = B; s->n_q = n_q; s->Hq = Hq; s->Hkv = Hkv; s->G = Hq / Hkv;
    s->rows_total = n_q * s->G;
    s->rows_blk = s->rows_total < kRowsPerBlock ? s->rows_total : kRowsPerBlock;
    s->n_rb = (s->rows_total + kRowsPerBlock - 1) / kRowsPerBlock;
    s->units = B * Hkv * s->n_rb;
    return WMTP_OK;
}

// Workspace: a 256-byte control block (word 0: the fused append's ticket, zero between calls),
// then [slots][rows_blk][128] fp32 partial outputs, then [slots][rows_blk] fp32 partial LSEs
// (slot = CTA + unit; rows_blk = rows per unit).
constexpr size_t kWsControl = 256;
size_t ws_o_bytes(long long slots, int rows_blk) { return (size_t)slots * rows_blk * kD * sizeof(float); }
size_t ws_total_bytes(long long slots, int rows_blk) {
    size_t a = (ws_o_bytes(slots, rows_blk) + 255) & ~size_t(255);
    return kWsControl + a + (size_t)slots * rows_blk * sizeof(float);
}

// ---------------------------------------------------------------------------------------------
// Launch helpers.  Every kernel goes out with programmatic stream serialization (PDL): it lets
// its successor launch early and waits for its predecessor before touching global memory (see
// pdl_wait in device_common.cuh).
template <typename... KArgs, typename... Args>
int launch(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
           Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...) != cudaSuccess) {
        (void)cudaGetLastError();
        return WMTP_ERR_CUDA;
    }
    return launched();
}

// The same with a cluster of `cs` CTAs along x.
template <typename... KArgs, typename... Args>
int launch_cluster(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                   int cs, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)cs;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...) != cudaSuccess) {
        (void)cudaGetLastError();
        return WMTP_ERR_CUDA;
    }
    return launched();
}

// Sets a kernel's dynamic shared-memory limit once per device (under the library mutex, so
// concurrent first calls from several host threads do not race on the flags).
template <typename K>
int set_smem_once(K kern, int bytes, bool (&done)[kMaxDevices]) {
    int dev;
    if (current_device(&dev) != WMTP_OK) return WMTP_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!done[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
            return WMTP_ERR_CUDA;
        done[dev] = true;
    }
    return WMTP_OK;
}

// ---------------------------------------------------------------------------------------------
// Kernel selection: one table, by the rows of a unit (rows_blk = min(64, n_q * G)) and the KV
// element type.  Measured at 1M keys on B200 (fraction of the measured HBM copy peak):
//   bf16  rows <= 16      mma.sync (1 m-tile, 4 key groups, 4 stages, 1 CTA/SM)      1.02-1.03
//         rows 17..32     mma.sync (2, 2, 2 stages, 2 CTAs/SM)                       0.98
//         rows 33..64     tcgen05 / TMEM (K pair slots 3, V ring 3, S buffers 2)     0.96
//         > 64 rows       mma.sync (4, 1, 2 stages, 2 CTAs/SM) per 64-row block
//   fp8   rows <= 16      mma.sync, Q in shared memory (1, 4, 2 stages, 3 CTAs/SM)   0.82
//         rows 17..64     tcgen05: QK^T on the E4M3 key codes, V widened by converter warps
//         > 64 rows       mma.sync (4, 1, 4 stages, 2 CTAs/SM) per 64-row block
// The 1-CTA mma.sync layouts above 16 rows were latency-bound (one consumer warp per SM
// sub-partition); two independent CTA pipelines per SM fixed that.  The tcgen05 kernel needs
// the whole unit in one 64-row block (its Q arrives as one TMA box of n_q x G rows).
// Build-time option for measurement sweeps: the smallest unit (in rows) the tcgen05 kernel takes
// (bf16: 33, where the mma.sync layouts fall behind; fp8: 17, the tcgen05 kernel's QK^T on the
// key codes beats the register-widening layout from 17 rows, 318 vs 338 us at 1M keys, 32 rows).
#ifndef WMTP_TC_MIN_ROWS
#define WMTP_TC_MIN_ROWS 33
#endif
#ifndef WMTP_TC8_MIN_ROWS
#define WMTP_TC8_MIN_ROWS 17
#endif
// fp8 tcgen05 rings (build-time for sweeps): K pair slots (16 KiB of codes each) and V slots
// (16 KiB fp16 each, an even number).  A V slot stays busy from its TMA issue through the
// landing, the widening and PV (~2.9 us at 1M keys), so the V ring needs ~6 slots to keep a tile
// every ~0.5 us.
#ifndef WMTP_TC8_NK
#define WMTP_TC8_NK 3
#endif
#ifndef WMTP_TC8_NV
#define WMTP_TC8_NV 6
#endif
enum class Kern { kSplit16, kSplit32, kSplit64, kTc, kSplit16Fp8, kSplit32Fp8, kSplit64Fp8, kTcFp8 };

Kern select_kernel(const Shape& s, bool kv8) {
    const bool tc = s.rows_total <= kRowsPerBlock && s.rows_blk >= (kv8 ? WMTP_TC8_MIN_ROWS : WMTP_TC_MIN_ROWS);
    if (tc) return kv8 ? Kern::kTcFp8 : Kern::kTc;
    if (s.rows_blk <= 16) return kv8 ? Kern::kSplit16Fp8 : Kern::kSplit16;
    if (s.rows_blk <= 32) return kv8 ? Kern::kSplit32Fp8 : Kern::kSplit32;
    return kv8 ? Kern::kSplit64Fp8 : Kern::kSplit64;
}

// Build-time option for measurement sweeps: 32-row units on one CTA per SM with four stages
// (half the split partials per unit) instead of two CTAs with two stages.
#ifndef WMTP_SPLIT32_ONE_CTA
#define WMTP_SPLIT32_ONE_CTA 0
#endif

// Stages of the two-CTA layout of units of 17-32 rows (build-time for sweeps).  Its key groups
// merge through the held stage of a unit's last tile, which leaves room for three 32 KiB stages in
// two CTAs per SM (1M-key verify at 32 rows 313 -> 307 us; the ring layout of <= 16 rows gained
// nothing from a third stage: 15.9 vs 15.9 us for the 64 MiB window call).
#ifndef WMTP_SPLIT32_NSTAGE
#define WMTP_SPLIT32_NSTAGE 3
#endif

// CTAs per SM of each kernel (the grid is sm_count times this).  Units of at most 16 rows read
// from the ring run two CTAs of two stages per SM: a large window is mostly L2-resident, and the
// 8-row consumer (~0.7 us a tile) rather than HBM then sets the pace, so two pipelines per SM
// help (64 MiB window call 19.6 -> 15.4 us); from the paged cache one CTA of four stages per SM
// already streams at the HBM rate.
int ctas_per_sm(Kern k, bool ring = false) {
    switch (k) {
        case Kern::kSplit16: return ring ? 2 : 1;
        case Kern::kSplit32: return WMTP_SPLIT32_ONE_CTA ? 1 : 2;
        case Kern::kSplit16Fp8: return 3;
        case Kern::kTc: case Kern::kTcFp8: return 1;
        default: return 2;
    }
}
constexpr int kMaxCtasPerSm = 3;

// LSE-merge grid: (units, rows per block, C head-dim chunks), with the smallest C whose one round
// of loads (8 C x kMergeBatch partials) covers a unit's expected partials (~P / units + 1).
dim3 merge_grid(const Shape& s, int P) {
    const long long per_unit = (long long)P / (s.units > 0 ? s.units : 1) + 1;
    const int C = per_unit <= 8 * kMergeBatch ? 1 : (per_unit <= 16 * kMergeBatch ? 2 : 4);
    return dim3((unsigned)s.units, (unsigned)s.rows_blk, (unsigned)C);
}

template <int SRC, int NMT, int NKG, int NSTAGE, int MINB, bool KV8 = false, bool QS = false,
          bool MS = false>
int launch_attn_t(const CUtensorMap& km, const CUtensorMap& vm, const AttnArgs& a, int sm_count,
                  const Shape& s, cudaStream_t st) {
    using Lay = SmemLayout<NMT, NKG, NSTAGE, KV8, QS, MS>;
    auto kern = attn_split_kernel<SRC, NMT, NKG, NSTAGE, MINB, KV8, QS, false, MS>;
    static bool attr_set[kMaxDevices] = {};
    int rc = set_smem_once(kern, Lay::kAlloc, attr_set);
    if (rc != WMTP_OK) return rc;
    const int grid = sm_count * MINB;
    rc = launch(kern, dim3(grid), dim3((NMT * NKG + 1) * 32), Lay::kAlloc, st, km, vm, a);
    if (rc != WMTP_OK) return rc;
    return launch(lse_merge_kernel<SRC>, merge_grid(s, grid), dim3(kMergeThreads), 0, st, a, grid);
}

template <int SRC, int NK, int NV, int NSB, bool KV8 = false>
int launch_attn_tc_t(const CUtensorMap& km, const CUtensorMap& vm, const void* q, const AttnArgs& a,
                     int sm_count, const Shape& s, cudaStream_t st) {
    using Lay = TcLayout<NK, NV, NSB, KV8>;
    auto kern = attn_tc_kernel<SRC, NK, NV, NSB, KV8>;
    static bool attr_set[kMaxDevices] = {};
    int rc = set_smem_once(kern, Lay::kAlloc, attr_set);
    if (rc != WMTP_OK) return rc;
    CUtensorMap qm;
    rc = encode_q_map(&qm, q, s.B, s.n_q, s.Hq, s.Hkv);
    if (rc != WMTP_OK) return rc;
    const int grid = sm_count;
    rc = launch(kern, dim3(grid), dim3(tc_threads<KV8>()), Lay::kAlloc, st, km, vm, qm, a);
    if (rc != WMTP_OK) return rc;
    return launch(lse_merge_kernel<SRC>, merge_grid(s, grid), dim3(kMergeThreads), 0, st, a, grid);
}

template <int SRC>
int launch_attn(const CUtensorMap& km, const CUtensorMap& vm, const AttnArgs& a, int sm_count,
                const Shape& s, cudaStream_t st, bool kv8 = false) {
    switch (select_kernel(s, kv8)) {
        case Kern::kSplit16:
            if (SRC == kSrcRing) return launch_attn_t<SRC, 1, 4, 2, 2>(km, vm, a, sm_count, s, st);
            return launch_attn_t<SRC, 1, 4, 4, 1>(km, vm, a, sm_count, s, st);
        case Kern::kSplit32:
#if WMTP_SPLIT32_ONE_CTA
            return launch_attn_t<SRC, 2, 2, 4, 1>(km, vm, a, sm_count, s, st);
#else
            return launch_attn_t<SRC, 2, 2, WMTP_SPLIT32_NSTAGE, 2, false, false, true>(km, vm, a, sm_count, s, st);
#endif
        case Kern::kSplit64: return launch_attn_t<SRC, 4, 1, 2, 2>(km, vm, a, sm_count, s, st);
        case Kern::kTc: return launch_attn_tc_t<SRC, 3, 3, 2>(km, vm, a.q, a, sm_count, s, st);
        case Kern::kSplit16Fp8: return launch_attn_t<SRC, 1, 4, 2, 3, true, true>(km, vm, a, sm_count, s, st);
        case Kern::kSplit32Fp8: return launch_attn_t<SRC, 2, 2, 4, 2, true>(km, vm, a, sm_count, s, st);
        case Kern::kSplit64Fp8: return launch_attn_t<SRC, 4, 1, 4, 2, true>(km, vm, a, sm_count, s, st);
        case Kern::kTcFp8:
            return launch_attn_tc_t<SRC, WMTP_TC8_NK, WMTP_TC8_NV, 2, true>(km, vm, a.q, a, sm_count, s, st);
    }
    return WMTP_ERR_ARG;
}

// ---------------------------------------------------------------------------------------------
// The windowed draft call: the cluster window kernel, one unit per cluster.  The cluster size is
// the largest of 16, 8, 4, 2 that leaves every CTA at least two tiles of the longest possible
// window and lets all units' clusters be resident at once (the occupancy query counts the
// clusters the GPU can hold with this kernel's shared memory); else 1 (one CTA per unit, no
// merge).  Queried once per device, kernel and size.
template <typename K>
int cluster_capacity(K kern, int smem, int threads, int cs, int (&cache)[kMaxDevices][5],
                     bool (&init)[kMaxDevices][5]) {
    int dev;
    if (current_device(&dev) != WMTP_OK) return 0;
    const int k = cs == 16 ? 4 : cs == 8 ? 3 : cs == 4 ? 2 : cs == 2 ? 1 : 0;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!init[dev][k]) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(cs, 1, 1);
        cfg.blockDim = dim3(threads);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)cs;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
            (void)cudaGetLastError();
            n = 0;
        }
        cache[dev][k] = n;
        init[dev][k] = true;
    }
    return cache[dev][k];
}

// Build-time options for measurement sweeps: the largest cluster size, and the stage count /
// CTAs per SM of the cluster layout for units of at most 16 rows.  Two stages and two CTAs per SM
// (94 KB of shared memory each) rather than four stages and one CTA: the smaller CTAs let eight
// 16-CTA clusters be resident at once (at 160 KB per CTA only clusters of 8 fit; 8 units of a
// 64 MiB window: 27.7 -> 20.2 us, a call that now takes the stream-K path, 15.5 us).
#ifndef WMTP_CL_MAX
#define WMTP_CL_MAX 16
#endif
static_assert(WMTP_CL_MAX <= kClusterMax, "the cluster merge handles at most kClusterMax ranks");
#ifndef WMTP_CL16_NSTAGE
#define WMTP_CL16_NSTAGE 2
#endif
#ifndef WMTP_CL16_MINB
#define WMTP_CL16_MINB 2
#endif

template <int NMT, int NKG, int NSTAGE, int MINB, bool KV8 = false, bool QS = false>
int launch_window_cluster_t(const CUtensorMap& km, const CUtensorMap& vm, const AttnArgs& a,
                            const Shape& s, int max_tiles, cudaStream_t st) {
    using Lay = SmemLayout<NMT, NKG, NSTAGE, KV8, QS>;
    auto kern = attn_split_kernel<kSrcRing, NMT, NKG, NSTAGE, MINB, KV8, QS, true>;
    constexpr int kThreads = (NMT * NKG + 1) * 32;
    static bool attr_set[kMaxDevices] = {};
    static int cap[kMaxDevices][5];
    static bool cap_init[kMaxDevices][5] = {};
    {
        int dev;
        if (current_device(&dev) != WMTP_OK) return WMTP_ERR_CUDA;
        std::lock_guard<std::mutex> lk(g_mu);
        if (!attr_set[dev]) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::kAlloc) != cudaSuccess ||
                cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
                return WMTP_ERR_CUDA;
            attr_set[dev] = true;
        }
    }
    int cs = 1;
    for (int c = WMTP_CL_MAX; c >= 2; c >>= 1) {
        if (2 * c > max_tiles) continue;
        const int n = cluster_capacity(kern, Lay::kAlloc, kThreads, c, cap, cap_init);
        if (n > 0 && s.units <= n) { cs = c; break; }
    }
#ifdef WMTP_CL_REPORT
    std::fprintf(stderr, "[wmtp] window cluster: units %d, size %d, %d threads, %d bytes shared\n",
                 s.units, cs, kThreads, Lay::kAlloc);
#endif
    return launch_cluster(kern, dim3(cs, s.units), dim3(kThreads), Lay::kAlloc, st, cs, km, vm, a);
}

int launch_window_cluster(const CUtensorMap& km, const CUtensorMap& vm, const AttnArgs& a,
                          const Shape& s, int max_tiles, cudaStream_t st, bool kv8) {
    // the mma.sync layouts of the stream-K kernel, by the unit's rows (the windowed units are
    // short, so the tcgen05 kernel's deeper pipeline does not pay here)
    if (s.rows_blk <= 16)
        return kv8 ? launch_window_cluster_t<1, 4, 2, 3, true, true>(km, vm, a, s, max_tiles, st)
                   : launch_window_cluster_t<1, 4, WMTP_CL16_NSTAGE, WMTP_CL16_MINB>(km, vm, a, s, max_tiles, st);
    if (s.rows_blk <= 32)
        return kv8 ? launch_window_cluster_t<2, 2, 4, 2, true>(km, vm, a, s, max_tiles, st)
                   : launch_window_cluster_t<2, 2, 2, 2>(km, vm, a, s, max_tiles, st);
    return kv8 ? launch_window_cluster_t<4, 1, 4, 2, true>(km, vm, a, s, max_tiles, st)
               : launch_window_cluster_t<4, 1, 2, 2>(km, vm, a, s, max_tiles, st);
}

// Common front half of the three attention calls.
int prepare(const Shape& s, const void* q, const void* out, const float* lse, void* ws,
            size_t ws_bytes, float sm_scale, DeviceInfo* dev, AttnArgs* a, bool kv8 = false,
            float k_scale = 1.f, float v_scale = 1.f, bool ring = false) {
    if (q == nullptr || out == nullptr || ws == nullptr) return WMTP_ERR_ARG;
    if (!(sm_scale > 0.f) || !std::isfinite(sm_scale)) return WMTP_ERR_ARG;
    if (!(k_scale > 0.f) || !std::isfinite(k_scale) || !(v_scale > 0.f) || !std::isfinite(v_scale))
        return WMTP_ERR_ARG;
    if (!std::isfinite(sm_scale * k_scale * 1.4426950408889634f)) return WMTP_ERR_ARG;
    if (!aligned(q, 16) || !aligned(out, 16) || (lse && !aligned(lse, 4)) || !aligned(ws, 256))
        return WMTP_ERR_ALIGN;
    int rc = device_info(dev);
    if (rc != WMTP_OK) return rc;
    const int grid = dev->sm_count * ctas_per_sm(select_kernel(s, kv8), ring);
    if (grid > kMaxParts) return WMTP_ERR_SHAPE;           // the merge's per-row weight table
    const long long slots = (long long)grid + s.units;
    if (ws_bytes < ws_total_bytes(slots, s.rows_blk)) return WMTP_ERR_WORKSPACE;
    std::memset(a, 0, sizeof(*a));
    a->q = reinterpret_cast<const __nv_bfloat16*>(q);
    a->out = reinterpret_cast<__nv_bfloat16*>(const_cast<void*>(out));
    a->lse = const_cast<float*>(lse);
    uint8_t* wsb = reinterpret_cast<uint8_t*>(ws);
    a->ticket = reinterpret_cast<unsigned int*>(wsb);
    a->ws_o = reinterpret_cast<float*>(wsb + kWsControl);
    a->ws_lse = reinterpret_cast<float*>(wsb + kWsControl +
                                         ((ws_o_bytes(slots, s.rows_blk) + 255) & ~size_t(255)));
    a->B = s.B; a->n_q = s.n_q; a->Hq = s.Hq; a->Hkv = s.Hkv; a->G = s.G; a->n_rb = s.n_rb;
    a->rows_total = s.rows_total;
    a->rows_blk = s.rows_blk;
    a->scale_log2 = sm_scale * k_scale * 1.4426950408889634f;
    a->v_scale = v_scale;
    a->min_tiles_per_cta = kMinTilesPerCta;
    return WMTP_OK;
}

int paged_call(const wmtp_bf16* q, const void* k_pool, const void* v_pool,
               const int32_t* page_table, const int32_t* kv_len, const int32_t* tree_parent,
               int B, int n_q, int Hq, int Hkv, int D, int page_size, int max_pages, int num_pages,
               float sm_scale, wmtp_bf16* out, float* lse, void* ws, size_t ws_bytes,
               cudaStream_t st, bool kv8 = false, float k_scale = 1.f, float v_scale = 1.f) {
    Shape s;
    int rc = check_shape(B, n_q, Hq, Hkv, D, &s);
    if (rc != WMTP_OK) return rc;
    if (page_size != WMTP_PAGE_SIZE) return WMTP_ERR_SHAPE;
    if (k_pool == nullptr || v_pool == nullptr || page_table == nullptr || kv_len == nullptr)
        return WMTP_ERR_ARG;
    if (max_pages < 1 || num_pages < 1) return WMTP_ERR_ARG;
    if ((long long)num_pages * Hkv > 0x7fffffffll) return WMTP_ERR_SHAPE;
    if (!aligned(k_pool, 16) || !aligned(v_pool, 16) || !aligned(page_table, 4) ||
        !aligned(kv_len, 4) || (tree_parent && !aligned(tree_parent, 4)))
        return WMTP_ERR_ALIGN;
    DeviceInfo dev;
    AttnArgs a;
    rc = prepare(s, q, out, lse, ws, ws_bytes, sm_scale, &dev, &a, kv8, k_scale, v_scale);
    if (rc != WMTP_OK) return rc;
    a.tree_parent = tree_parent;
    a.page_table = page_table;
    a.kv_len = kv_len;
    a.max_pages = max_pages;
    a.num_pages = num_pages;
    CUtensorMap km, vm;
    if ((rc = encode_rows_map(&km, k_pool, WMTP_PAGE_SIZE, (long long)num_pages * Hkv, kv8)) != WMTP_OK) return rc;
    if ((rc = encode_rows_map(&vm, v_pool, WMTP_PAGE_SIZE, (long long)num_pages * Hkv, kv8)) != WMTP_OK) return rc;
    return launch_attn<kSrcPaged>(km, vm, a, dev.sm_count, s, st, kv8);
}

}  // namespace
}  // namespace wmtp

// ---------------------------------------------------------------------------------------------
// Scratch for draft_attn_window_noalloc: split partials of callers that cannot allocate device
// memory.  Host code must not use this name as a device address (on the host it is only a
// stand-in); the address comes from cudaGetSymbolAddress, once per device.
static __device__ __align__(256) unsigned char wmtp_noalloc_scratch[WMTP_NOALLOC_SCRATCH_BYTES];

namespace wmtp {
namespace {

void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up on first use).
int noalloc_scratch(void** out) {
    int dev;
    if (current_device(&dev) != WMTP_OK) return WMTP_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, wmtp_noalloc_scratch) != cudaSuccess || p == nullptr)
            return WMTP_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return WMTP_OK;
}

}  // namespace
}  // namespace wmtp

using namespace wmtp;

// The failure path of every bounded wait, on purpose: lane 0 waits on an mbarrier that nothing
// arrives on, gives up after limit_ns, flags the timeout status and returns (no trap, no fault).
__global__ void selftest_wait_timeout_kernel(uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
        const uint64_t t0 = global_ns();
        uint32_t spins = 0;
        while (!mbar_try_wait(&bar, 0u)) {
            if ((++spins & 255u) == 0u && global_ns() - t0 > limit_ns) {
                flag_status(kStatusTimeout);
                break;
            }
        }
    }
    __syncwarp();
}

extern "C" {

const char* wmtp_status_string(int status) {
    switch (status) {
        case WMTP_OK: return "ok";
        case WMTP_ERR_ARG: return "invalid argument";
        case WMTP_ERR_SHAPE: return "unsupported shape";
        case WMTP_ERR_ALIGN: return "misaligned pointer";
        case WMTP_ERR_WORKSPACE: return "workspace too small";
        case WMTP_ERR_CUDA: return "CUDA error";
        case WMTP_ERR_DEVICE_INDEX: return "device-side index out of range";
        case WMTP_ERR_UNSUPPORTED: return "unsupported device (needs sm_100)";
        case WMTP_ERR_TIMEOUT: return "device-side wait timed out";
        case WMTP_ERR_SCRATCH_LIMIT: return "shape exceeds the built-in scratch of the no-alloc call";
        default: return "unknown status";
    }
}

size_t wmtp_workspace_bytes(int B, int n_q, int Hq, int Hkv, int D) {
    Shape s;
    if (check_shape(B, n_q, Hq, Hkv, D, &s) != WMTP_OK) return 0;
    DeviceInfo dev;
    if (device_info(&dev) != WMTP_OK) return 0;
    return ws_total_bytes((long long)dev.sm_count * kMaxCtasPerSm + s.units, s.rows_blk);
}

}  // extern "C"

namespace wmtp {
namespace {

// Ring append of rows of CH 16-byte pieces (bf16: 16, fp8: 8).
template <int CH>
int ring_append_call(void* ring_k, void* ring_v, int64_t* ring_len, const void* k_new,
                     const void* v_new, int B, int n_new, int Hkv, int D, int n_sink, int capacity,
                     wmtp_stream_t stream) {
    if (ring_k == nullptr || ring_v == nullptr || ring_len == nullptr) return WMTP_ERR_ARG;
    if (B < 1 || n_new < 0 || Hkv < 1 || n_sink < 0 || capacity <= n_sink) return WMTP_ERR_ARG;
    if (D != WMTP_HEAD_DIM) return WMTP_ERR_SHAPE;
    if (B > 65535) return WMTP_ERR_SHAPE;                      // grid.y
    if (n_new == 0) return WMTP_OK;
    if (k_new == nullptr || v_new == nullptr) return WMTP_ERR_ARG;
    if (!aligned(ring_k, 16) || !aligned(ring_v, 16) || !aligned(k_new, 16) || !aligned(v_new, 16) ||
        !aligned(ring_len, 8))
        return WMTP_ERR_ALIGN;
    DeviceInfo dev;
    int rc = device_info(&dev);
    if (rc != WMTP_OK) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // upper bound on surviving rows per request: the sink plus the ring's other slots
    const long long surv = (long long)(n_new < capacity ? n_new : capacity);
    const long long work = surv * Hkv * CH;
    long long chunks = (work + 256 * 4 - 1) / (256 * 4);     // ~4 pieces per thread
    const long long max_chunks = (long long)dev.sm_count * 8;
    if (chunks > max_chunks) chunks = max_chunks;
    if (chunks < 1) chunks = 1;
    const int single = (chunks == 1);
    rc = launch(ring_append_kernel<CH>, dim3((unsigned)chunks, B), dim3(256), 0, st,
                reinterpret_cast<uint4*>(ring_k), reinterpret_cast<uint4*>(ring_v),
                reinterpret_cast<long long*>(ring_len), reinterpret_cast<const uint4*>(k_new),
                reinterpret_cast<const uint4*>(v_new), n_new, Hkv, n_sink, capacity, single);
    if (rc != WMTP_OK || single) return rc;
    return launch(ring_len_add_kernel, dim3((B + 255) / 256), dim3(256), 0, st,
                  reinterpret_cast<long long*>(ring_len), B, n_new);
}

// The windowed draft call, optionally with the ring append of the call's new rows fused in
// (n_new > 0: positions [ring_len[b], ring_len[b] + n_new) get the rows of k_new / v_new and
// ring_len advances, as ring_kv_append would).  stream_k: the stream-K kernel with workspace
// partials and the LSE merge kernel instead of the cluster kernel (the no-alloc entry point).
// Windowed calls of few units whose key sets hold at least this many tiles per SM in all (units x
// the longest key set's tiles / SMs) take the stream-K path.
constexpr int kWindowStreamKTilesPerSm = 7;

int window_call(const wmtp_bf16* q, void* ring_k, void* ring_v, int64_t* ring_len,
                const void* k_new, const void* v_new, int n_new,
                int B, int n_q, int Hq, int Hkv, int D, int n_sink, int window, int capacity,
                float sm_scale, wmtp_bf16* out, float* lse, void* ws, size_t ws_bytes,
                wmtp_stream_t stream, bool kv8, float k_scale, float v_scale, bool stream_k = false) {
    Shape s;
    int rc = check_shape(B, n_q, Hq, Hkv, D, &s);
    if (rc != WMTP_OK) return rc;
    if (ring_k == nullptr || ring_v == nullptr || ring_len == nullptr) return WMTP_ERR_ARG;
    if (n_sink < 0 || window < 0 || capacity <= n_sink || window > capacity - n_sink) return WMTP_ERR_ARG;
    if ((long long)B * Hkv > 0x7fffffffll) return WMTP_ERR_SHAPE;
    if (!aligned(ring_k, 16) || !aligned(ring_v, 16) || !aligned(ring_len, 8)) return WMTP_ERR_ALIGN;
    if (n_new < 0) return WMTP_ERR_ARG;
    if (n_new > 0) {
        if (k_new == nullptr || v_new == nullptr) return WMTP_ERR_ARG;
        if (!aligned(k_new, 16) || !aligned(v_new, 16)) return WMTP_ERR_ALIGN;
    }
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    DeviceInfo dev;
    AttnArgs a;
    rc = prepare(s, q, out, lse, ws, ws_bytes, sm_scale, &dev, &a, kv8, k_scale, v_scale, true);
    if (rc != WMTP_OK) return rc;
    // tiles of the longest key set: the sink's, the window's, one more where the window wraps
    const int max_tiles = (n_sink + kTileKeys - 1) / kTileKeys + (window + kTileKeys - 1) / kTileKeys + 1;
    // the cluster kernel (one launch) unless its clusters of at most 16 CTAs leave SMs idle (few
    // units) while the call holds many tiles (a long window): then the stream-K kernel over every
    // SM plus the LSE merge (64 MiB NoPE call, 8 units: 20.1 -> 15.5 us; 8 requests x 8 MiB,
    // 32 units: the cluster kernel, 14.3 vs 17.8 us; 8 MiB, 4 units: cluster, 9.7 vs 12.1 us)
    const bool use_sk = stream_k || s.units > 65535 ||
                        ((long long)s.units * WMTP_CL_MAX < dev.sm_count &&
                         (long long)s.units * max_tiles >= (long long)kWindowStreamKTilesPerSm * dev.sm_count);
    // the fused append covers new rows that all fall in the call's key set (n_new <= window);
    // otherwise the append runs as its own kernel first
    const bool fused = n_new > 0 && n_new <= window && !use_sk;
    if (n_new > 0 && !fused) {
        rc = kv8 ? ring_append_call<8>(ring_k, ring_v, ring_len, k_new, v_new, B, n_new, Hkv, D, n_sink,
                                       capacity, stream)
                 : ring_append_call<16>(ring_k, ring_v, ring_len, k_new, v_new, B, n_new, Hkv, D, n_sink,
                                        capacity, stream);
        if (rc != WMTP_OK) return rc;
    }
    a.ring_len = reinterpret_cast<const long long*>(ring_len);
    a.ring_len_w = reinterpret_cast<long long*>(ring_len);
    a.n_sink = n_sink;
    a.window = window;
    a.capacity = capacity;
    if (fused) {
        a.k_new = reinterpret_cast<const uint4*>(k_new);
        a.v_new = reinterpret_cast<const uint4*>(v_new);
        a.ring_kw = reinterpret_cast<uint4*>(ring_k);
        a.ring_vw = reinterpret_cast<uint4*>(ring_v);
        a.n_new = n_new;
    }
    CUtensorMap km, vm;
    if ((rc = encode_rows_map(&km, ring_k, capacity, (long long)B * Hkv, kv8)) != WMTP_OK) return rc;
    if ((rc = encode_rows_map(&vm, ring_v, capacity, (long long)B * Hkv, kv8)) != WMTP_OK) return rc;
    if (use_sk) return launch_attn<kSrcRing>(km, vm, a, dev.sm_count, s, st, kv8);
    return launch_window_cluster(km, vm, a, s, max_tiles, st, kv8);
}

}  // namespace
}  // namespace wmtp

extern "C" {

int ring_kv_append(wmtp_bf16* ring_k, wmtp_bf16* ring_v, int64_t* ring_len, const wmtp_bf16* k_new,
                   const wmtp_bf16* v_new, int B, int n_new, int Hkv, int D, int n_sink, int capacity,
                   wmtp_stream_t stream) {
    return wmtp::ring_append_call<16>(ring_k, ring_v, ring_len, k_new, v_new, B, n_new, Hkv, D, n_sink,
                                      capacity, stream);
}

int ring_kv_append_fp8(uint8_t* ring_k, uint8_t* ring_v, int64_t* ring_len, const uint8_t* k_new,
                       const uint8_t* v_new, int B, int n_new, int Hkv, int D, int n_sink, int capacity,
                       wmtp_stream_t stream) {
    return wmtp::ring_append_call<8>(ring_k, ring_v, ring_len, k_new, v_new, B, n_new, Hkv, D, n_sink,
                                     capacity, stream);
}

int draft_attn_window(const wmtp_bf16* q, const wmtp_bf16* ring_k, const wmtp_bf16* ring_v,
                      const int64_t* ring_len, int B, int n_q, int Hq, int Hkv, int D, int n_sink,
                      int window, int capacity, float sm_scale, wmtp_bf16* out, float* lse, void* ws,
                      size_t ws_bytes, wmtp_stream_t stream) {
    return window_call(q, const_cast<wmtp_bf16*>(ring_k), const_cast<wmtp_bf16*>(ring_v),
                       const_cast<int64_t*>(ring_len), nullptr, nullptr, 0, B, n_q, Hq, Hkv, D, n_sink,
                       window, capacity, sm_scale, out, lse, ws, ws_bytes, stream, false, 1.f, 1.f);
}

int draft_attn_window_append(const wmtp_bf16* q, wmtp_bf16* ring_k, wmtp_bf16* ring_v, int64_t* ring_len,
                             const wmtp_bf16* k_new, const wmtp_bf16* v_new, int n_new, int B, int n_q,
                             int Hq, int Hkv, int D, int n_sink, int window, int capacity, float sm_scale,
                             wmtp_bf16* out, float* lse, void* ws, size_t ws_bytes, wmtp_stream_t stream) {
    return window_call(q, ring_k, ring_v, ring_len, k_new, v_new, n_new, B, n_q, Hq, Hkv, D, n_sink,
                       window, capacity, sm_scale, out, lse, ws, ws_bytes, stream, false, 1.f, 1.f);
}

int draft_attn_window_append_fp8(const wmtp_bf16* q, uint8_t* ring_k, uint8_t* ring_v, int64_t* ring_len,
                                 const uint8_t* k_new, const uint8_t* v_new, int n_new, int B, int n_q,
                                 int Hq, int Hkv, int D, int n_sink, int window, int capacity,
                                 float sm_scale, float k_scale, float v_scale, wmtp_bf16* out, float* lse,
                                 void* ws, size_t ws_bytes, wmtp_stream_t stream) {
    return window_call(q, ring_k, ring_v, ring_len, k_new, v_new, n_new, B, n_q, Hq, Hkv, D, n_sink,
                       window, capacity, sm_scale, out, lse, ws, ws_bytes, stream, true, k_scale, v_scale);
}

int draft_attn_window_fp8(const wmtp_bf16* q, const uint8_t* ring_k, const uint8_t* ring_v,
                          const int64_t* ring_len, int B, int n_q, int Hq, int Hkv, int D, int n_sink,
                          int window, int capacity, float sm_scale, float k_scale, float v_scale,
                          wmtp_bf16* out, float* lse, void* ws, size_t ws_bytes, wmtp_stream_t stream) {
    return window_call(q, const_cast<uint8_t*>(ring_k), const_cast<uint8_t*>(ring_v),
                       const_cast<int64_t*>(ring_len), nullptr, nullptr, 0, B, n_q, Hq, Hkv, D, n_sink,
                       window, capacity, sm_scale, out, lse, ws, ws_bytes, stream, true, k_scale, v_scale);
}

int draft_attn_full_fp8(const wmtp_bf16* q, const uint8_t* k_pool, const uint8_t* v_pool,
                        const int32_t* page_table, const int32_t* kv_len, int B, int n_q, int Hq, int Hkv,
                        int D, int page_size, int max_pages, int num_pages, float sm_scale, float k_scale,
                        float v_scale, wmtp_bf16* out, float* lse, void* ws, size_t ws_bytes,
                        wmtp_stream_t stream) {
    return paged_call(q, k_pool, v_pool, page_table, kv_len, nullptr, B, n_q, Hq, Hkv, D, page_size,
                      max_pages, num_pages, sm_scale, out, lse, ws, ws_bytes,
                      reinterpret_cast<cudaStream_t>(stream), true, k_scale, v_scale);
}

int verify_attn_fp8(const wmtp_bf16* q, const uint8_t* k_pool, const uint8_t* v_pool,
                    const int32_t* page_table, const int32_t* kv_len, const int32_t* tree_parent, int B,
                    int n_q, int Hq, int Hkv, int D, int page_size, int max_pages, int num_pages,
                    float sm_scale, float k_scale, float v_scale, wmtp_bf16* out, float* lse, void* ws,
                    size_t ws_bytes, wmtp_stream_t stream) {
    return paged_call(q, k_pool, v_pool, page_table, kv_len, tree_parent, B, n_q, Hq, Hkv, D, page_size,
                      max_pages, num_pages, sm_scale, out, lse, ws, ws_bytes,
                      reinterpret_cast<cudaStream_t>(stream), true, k_scale, v_scale);
}

int draft_attn_full(const wmtp_bf16* q, const wmtp_bf16* k_pool, const wmtp_bf16* v_pool,
                    const int32_t* page_table, const int32_t* kv_len, int B, int n_q, int Hq, int Hkv,
                    int D, int page_size, int max_pages, int num_pages, float sm_scale, wmtp_bf16* out,
                    float* lse, void* ws, size_t ws_bytes, wmtp_stream_t stream) {
    return paged_call(q, k_pool, v_pool, page_table, kv_len, nullptr, B, n_q, Hq, Hkv, D, page_size,
                      max_pages, num_pages, sm_scale, out, lse, ws, ws_bytes,
                      reinterpret_cast<cudaStream_t>(stream));
}

int verify_attn(const wmtp_bf16* q, const wmtp_bf16* k_pool, const wmtp_bf16* v_pool,
                const int32_t* page_table, const int32_t* kv_len, const int32_t* tree_parent, int B,
                int n_q, int Hq, int Hkv, int D, int page_size, int max_pages, int num_pages,
                float sm_scale, wmtp_bf16* out, float* lse, void* ws, size_t ws_bytes,
                wmtp_stream_t stream) {
    return paged_call(q, k_pool, v_pool, page_table, kv_len, tree_parent, B, n_q, Hq, Hkv, D,
                      page_size, max_pages, num_pages, sm_scale, out, lse, ws, ws_bytes,
                      reinterpret_cast<cudaStream_t>(stream));
}

int accept_greedy(const float* logits, const int32_t* tokens, const int32_t* tree_parent, int B,
                  int n_q, int V, int32_t* accepted, int32_t* n_accepted, wmtp_stream_t stream) {
    if (logits == nullptr || tokens == nullptr || accepted == nullptr || n_accepted == nullptr)
        return WMTP_ERR_ARG;
    if (B < 1 || n_q < 1 || V < 1 || n_q > WMTP_MAX_QUERIES) return WMTP_ERR_ARG;
    if (!aligned(logits, 4) || !aligned(tokens, 4) || !aligned(accepted, 4) || !aligned(n_accepted, 4) ||
        (tree_parent && !aligned(tree_parent, 4)))
        return WMTP_ERR_ALIGN;
    DeviceInfo dev;
    int rc = device_info(&dev);
    if (rc != WMTP_OK) return rc;
    return launch(accept_greedy_kernel, dim3(B), dim3(256), 0, reinterpret_cast<cudaStream_t>(stream),
                  logits, tokens, tree_parent, n_q, V, accepted, n_accepted);
}

int accept_stochastic(const float* p, const float* q, const int32_t* tokens, const uint32_t* u_accept,
                      const uint32_t* u_sample, int B, int n_q, int V, int32_t* accepted,
                      int32_t* n_accepted, wmtp_stream_t stream) {
    if (p == nullptr || tokens == nullptr || u_sample == nullptr || accepted == nullptr ||
        n_accepted == nullptr)
        return WMTP_ERR_ARG;
    if (B < 1 || n_q < 1 || n_q > WMTP_MAX_QUERIES || V < 1 || V >= (1 << 24)) return WMTP_ERR_ARG;
    if (n_q > 1 && (q == nullptr || u_accept == nullptr)) return WMTP_ERR_ARG;
    if (!aligned(p, 4) || !aligned(tokens, 4) || !aligned(u_sample, 4) || !aligned(accepted, 4) ||
        !aligned(n_accepted, 4) || (q && !aligned(q, 4)) || (u_accept && !aligned(u_accept, 4)))
        return WMTP_ERR_ALIGN;
    DeviceInfo dev;
    int rc = device_info(&dev);
    if (rc != WMTP_OK) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (V <= 4096)
        return launch(accept_stochastic_kernel<256>, dim3(B), dim3(256), 0, st, p, q, tokens,
                      u_accept, u_sample, n_q, V, accepted, n_accepted);
    return launch(accept_stochastic_kernel<1024>, dim3(B), dim3(1024), 0, st, p, q, tokens, u_accept,
                  u_sample, n_q, V, accepted, n_accepted);
}

int draft_attn_window_noalloc(const wmtp_bf16* q, const wmtp_bf16* ring_k, const wmtp_bf16* ring_v,
                              const int64_t* ring_len, int B, int n_q, int Hq, int Hkv, int D,
                              int n_sink, int window, int capacity, float sm_scale, wmtp_bf16* out,
                              float* lse, wmtp_stream_t stream) {
    // the device check comes first, so an unsupported GPU reports WMTP_ERR_UNSUPPORTED as every
    // other call does, before the scratch lookup
    DeviceInfo dev;
    int rc = device_info(&dev);
    if (rc != WMTP_OK) return rc;
    void* scratch = nullptr;
    rc = noalloc_scratch(&scratch);
    if (rc != WMTP_OK) return rc;
    rc = window_call(q, const_cast<wmtp_bf16*>(ring_k), const_cast<wmtp_bf16*>(ring_v),
                     const_cast<int64_t*>(ring_len), nullptr, nullptr, 0, B, n_q, Hq, Hkv, D, n_sink, window,
                     capacity, sm_scale, out, lse, scratch, WMTP_NOALLOC_SCRATCH_BYTES, stream, false, 1.f,
                     1.f, /*stream_k=*/true);
    return rc == WMTP_ERR_WORKSPACE ? WMTP_ERR_SCRATCH_LIMIT : rc;
}

int ring_kv_append_at(wmtp_bf16* ring_k, wmtp_bf16* ring_v, int64_t* ring_len, const wmtp_bf16* k_new,
                      const wmtp_bf16* v_new, const int64_t* pos, const int32_t* n_new, int B, int n_max,
                      int Hkv, int D, int n_sink, int capacity, wmtp_stream_t stream) {
    if (ring_k == nullptr || ring_v == nullptr || ring_len == nullptr || k_new == nullptr ||
        v_new == nullptr || pos == nullptr || n_new == nullptr)
        return WMTP_ERR_ARG;
    if (reinterpret_cast<const void*>(pos) == reinterpret_cast<const void*>(ring_len)) return WMTP_ERR_ARG;
    if (B < 1 || n_max < 1 || Hkv < 1 || n_sink < 0 || capacity <= n_sink) return WMTP_ERR_ARG;
    if (D != WMTP_HEAD_DIM) return WMTP_ERR_SHAPE;
    if (B > 65535) return WMTP_ERR_SHAPE;
    if (!aligned(ring_k, 16) || !aligned(ring_v, 16) || !aligned(k_new, 16) || !aligned(v_new, 16) ||
        !aligned(ring_len, 8) || !aligned(pos, 8) || !aligned(n_new, 4))
        return WMTP_ERR_ALIGN;
    DeviceInfo dev;
    int rc = device_info(&dev);
    if (rc != WMTP_OK) return rc;
    const long long surv = (long long)(n_max < capacity ? n_max : capacity);
    long long chunks = (surv * Hkv * 16 + 256 * 4 - 1) / (256 * 4);
    const long long max_chunks = (long long)dev.sm_count * 8;
    if (chunks > max_chunks) chunks = max_chunks;
    if (chunks < 1) chunks = 1;
    return launch(ring_append_at_kernel, dim3((unsigned)chunks, B), dim3(256), 0,
                  reinterpret_cast<cudaStream_t>(stream), reinterpret_cast<uint4*>(ring_k),
                  reinterpret_cast<uint4*>(ring_v), reinterpret_cast<long long*>(ring_len),
                  reinterpret_cast<const uint4*>(k_new), reinterpret_cast<const uint4*>(v_new),
                  reinterpret_cast<const long long*>(pos), reinterpret_cast<const int*>(n_new), n_max,
                  Hkv, n_sink, capacity);
}

int spec_commit(const int32_t* accepted, const int32_t* n_accepted, int B, int n_q, int32_t* history,
                int64_t max_tokens, int64_t* n_tokens, int64_t* append_pos, int32_t* n_append,
                int32_t* verify_len, int n_q_verify, int32_t* draft_len, int n_draft,
                wmtp_stream_t stream) {
    if (accepted == nullptr || n_accepted == nullptr || history == nullptr || n_tokens == nullptr ||
        append_pos == nullptr || n_append == nullptr)
        return WMTP_ERR_ARG;
    if (B < 1 || n_q < 1 || n_q > WMTP_MAX_QUERIES || max_tokens < 1 || n_draft < 0 || n_q_verify < 0)
        return WMTP_ERR_ARG;
    if (max_tokens + (int64_t)n_q_verify + (int64_t)n_draft >= ((int64_t)1 << 31)) return WMTP_ERR_ARG;
    if (!aligned(accepted, 4) || !aligned(n_accepted, 4) || !aligned(history, 4) ||
        !aligned(n_tokens, 8) || !aligned(append_pos, 8) || !aligned(n_append, 4) ||
        (verify_len && !aligned(verify_len, 4)) || (draft_len && !aligned(draft_len, 4)))
        return WMTP_ERR_ALIGN;
    DeviceInfo dev;
    int rc = device_info(&dev);
    if (rc != WMTP_OK) return rc;
    return launch(spec_commit_kernel, dim3((B + 127) / 128), dim3(128), 0,
                  reinterpret_cast<cudaStream_t>(stream), accepted, n_accepted, B, n_q, history,
                  (long long)max_tokens, reinterpret_cast<long long*>(n_tokens),
                  reinterpret_cast<long long*>(append_pos), n_append, verify_len, n_q_verify,
                  draft_len, n_draft);
}

int wmtp_synth_draft_tokens(const int32_t* history, const int64_t* n_tokens, int B, int64_t max_tokens,
                            int gamma, int V, uint64_t target_seed, uint64_t draft_seed, uint32_t agree24,
                            int32_t* tokens, wmtp_stream_t stream) {
    if (history == nullptr || n_tokens == nullptr || tokens == nullptr) return WMTP_ERR_ARG;
    if (B < 1 || V < 2 || gamma < 0 || gamma + 1 > WMTP_MAX_QUERIES || max_tokens < 1 ||
        agree24 > (1u << 24))
        return WMTP_ERR_ARG;
    if (!aligned(history, 4) || !aligned(n_tokens, 8) || !aligned(tokens, 4)) return WMTP_ERR_ALIGN;
    DeviceInfo dev;
    int rc = device_info(&dev);
    if (rc != WMTP_OK) return rc;
    return launch(synth::draft_tokens_kernel, dim3(B), dim3(256), 0, reinterpret_cast<cudaStream_t>(stream),
                  history, reinterpret_cast<const long long*>(n_tokens), (long long)max_tokens, gamma, V,
                  (unsigned long long)target_seed, (unsigned long long)draft_seed, (unsigned int)agree24,
                  tokens);
}

int wmtp_synth_target_logits(const int32_t* history, const int64_t* n_tokens, int B, int64_t max_tokens,
                             const int32_t* tokens, const int32_t* tree_parent, int n_q, int V,
                             uint64_t target_seed, float* logits, wmtp_stream_t stream) {
    if (history == nullptr || n_tokens == nullptr || tokens == nullptr || logits == nullptr)
        return WMTP_ERR_ARG;
    if (B < 1 || B > 65535 || V < 2 || n_q < 1 || n_q > WMTP_MAX_QUERIES || max_tokens < 1)
        return WMTP_ERR_ARG;
    if (!aligned(history, 4) || !aligned(n_tokens, 8) || !aligned(tokens, 4) || !aligned(logits, 4) ||
        (tree_parent && !aligned(tree_parent, 4)))
        return WMTP_ERR_ALIGN;
    DeviceInfo dev;
    int rc = device_info(&dev);
    if (rc != WMTP_OK) return rc;
    return launch(synth::target_logits_kernel, dim3(n_q, B), dim3(256), 0,
                  reinterpret_cast<cudaStream_t>(stream), history,
                  reinterpret_cast<const long long*>(n_tokens), (long long)max_tokens, tokens, tree_parent,
                  n_q, V, (unsigned long long)target_seed, logits);
}

uint64_t wmtp_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

#ifdef WMTP_TRACE
// Measurement builds only: copies the timestamp trace of CTA (0, 0) of the last traced launch.
WMTP_API int wmtp_trace_read(unsigned long long* host, int n) {
    if (host == nullptr || n < 1 || n > kTraceSlots) return WMTP_ERR_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess) return WMTP_ERR_CUDA;
    return cudaMemcpyFromSymbol(host, g_trace, sizeof(unsigned long long) * n) == cudaSuccess ? WMTP_OK
                                                                                            : WMTP_ERR_CUDA;
}
#endif

int wmtp_selftest_wait_timeout(uint64_t limit_ns, wmtp_stream_t stream) {
    if (limit_ns < 1000000ull || limit_ns > kWaitLimitNs) return WMTP_ERR_ARG;
    return launch(selftest_wait_timeout_kernel, dim3(1), dim3(32), 0,
                  reinterpret_cast<cudaStream_t>(stream), limit_ns);
}

int wmtp_device_status(wmtp_stream_t stream) {
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return WMTP_ERR_CUDA;
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_status, sizeof v) != cudaSuccess) return WMTP_ERR_CUDA;
    if (v != 0 && cudaMemcpyToSymbol(g_status, &zero, sizeof zero) != cudaSuccess) return WMTP_ERR_CUDA;
    if (v & kStatusDeviceIndex) return WMTP_ERR_DEVICE_INDEX;
    if (v & kStatusTimeout) return WMTP_ERR_TIMEOUT;
    return WMTP_OK;
}

}  // extern "C"
