// attn_tc_kernels.cuh -- split-KV attention on the 5th-generation tensor cores (tcgen05) for
// units of up to 64 query rows: the multi-query verify of the Windowed-MTP decode step (Pith
// verdict on arXiv 2607.21535, pith_extraction.key_machinery: the target verifies gamma + 1
// positions, or a tree, with full attention), where QK^T and PV are dense [rows x 128] x
// [128 x 64] contractions per key tile.
//
// Same work split, tile walk, masks, partial format and merge as attn_split_kernel; only the
// math engine differs.  Tiles go in pairs (CTA-local tiles 2q, 2q + 1).  Roles (384 threads, one
// CTA per SM; 512 with fp8 KV):
//   warp 0        K producer: each pair's K tiles into one pair slot of an NK-deep ring (laid
//                 out so the 128 keys of a 64-dim half are consecutive rows), and each unit's Q
//                 rows (one box of n_q x G rows per 64-dim half) into a Q double buffer;
//   warp 6        V producer: each tile's V into an NV-deep ring.  K is released as soon as
//                 QK^T has read it and V after PV;
//   warp 1        owns the tensor memory; lane 0 issues S = Q K^T for a pair into a 128-column
//                 S buffer: one M = 64, N = 128, K = 16 MMA per k-step when both tiles belong to
//                 the same unit, else two N = 64 sequences; fp32 in TMEM.  It forwards the tiles'
//                 descriptions to the softmax warps through the S barrier;
//   warp 7        lane 0 issues O += P V (M = 64, N = 128 dims, K = 64 keys; O stays in TMEM)
//                 into the tile's group's O once the softmax group has written P(t).  Two issuers
//                 keep the tensor core's queue fed while the other waits;
//   warps 2..5, 8..11   softmax, two groups of four warps taking alternate tiles (group g the
//                 CTA's tiles it with it % 2 == g, i.e. column half g of each S buffer), each with
//                 its own running maxima and sums and its own O accumulator in TMEM; one warp per
//                 sub-partition could not keep up with the tile rate.  The M = 64 accumulator
//                 keeps row r in TMEM lane 32 (r / 16) + r % 16, so warp w sees rows
//                 16 (w % 4) .. + 15; with the 16x32bx2 load both half-warps read those rows,
//                 lanes 0-15 keys 0-31 and lanes 16-31 keys 32-63 (and O dims 0-63 / 64-127).
//                 Each thread masks, exponentiates against the row's running maximum and writes
//                 its half of the P row (128-byte swizzled) for the PV MMA.  The maximum is only
//                 moved when a row's maximum grows by more than 2^8 (log2 units), and only then
//                 is that O row rescaled in TMEM, so the common tile touches no O at all.  After
//                 each tile a group publishes its rows' maxima and sums; the group holding a
//                 unit's last tile combines both groups' (O, max, sum) like two split-KV partials
//                 and writes the result, and a group starts a new unit only after that
//                 combination (its O is then free);
//   warps 12..15  (fp8 KV only) converters, two pairs taking alternate tiles: each E4M3 V tile
//                 lands in the upper half of its fp16 slot and is widened in place (PV then runs
//                 on fp16 operands, P too), and the pair that takes a unit's first tile splits the
//                 unit's bf16 Q rows into two E4M3 terms.  K is not converted at all: QK^T runs as
//                 kind::f8f6f4 on the E4M3 key codes as TMA lands them, against Q = 2^-k (hi + lo)
//                 with hi = e4m3(2^k q), lo = e4m3(2^k q - hi) and one power of two 2^k per row
//                 (bf16's 8 significant bits fit in two 4-bit E4M3 significands), and the row's
//                 2^-k goes into its softmax scale.
// Tensor memory: NSB S pair buffers of 128 columns, then O of group 0 and O of group 1 (128
// columns each).  Every wait is bounded; on a timeout all roles stop, each MMA issuer waits
// (bounded) for its own MMAs, all meet at the final barrier and warp 1 frees the tensor memory.
#pragma once

#include "attn_kernels.cuh"
#include "tcgen05.cuh"

namespace wmtp {

// 384 threads; with fp8 KV four more warps (12..15) widen the fp8 tiles into fp16 operands.
template <bool KV8>
constexpr int tc_threads() { return KV8 ? 512 : 384; }
constexpr float kRescaleThreshold = 8.f;   // log2 units

// Tiles go in pairs (CTA-local tiles 2q and 2q + 1): pair q's K tiles share one K slot and one
// S buffer of 128 columns, so a pair of the same unit needs one N = 128 QK^T instead of two
// N = 64 ones (the tensor core's cost per tile drops from ~656 to ~512 cycles).

template <int NSB>
struct TcCols {
    static constexpr uint32_t kO = NSB * 128;                    // O of group g: [kO + 128 g, + 128)
    static constexpr uint32_t kAlloc = 512;
    static_assert(NSB * 128 + 256 <= 512, "tensor memory holds NSB S pair buffers and two O");
};

// K ring: NK pair slots of 32 KiB laid out [tile 0, dims 0-63][tile 1, dims 0-63][tile 0, dims
// 64-127][tile 1, dims 64-127], so 128 keys of one 64-dim half are 128 consecutive 128-byte rows
// (the K-major operand of an N = 128 MMA).
// fp8 KV: the producers land each E4M3 tile (one 128-byte x 64-key box) in the upper 64-dim half
// of its fp16 slot, and the converter warps widen it in place (see widen_rows).
// fp8 KV: a K pair slot holds the two tiles' E4M3 codes, [tile 0: 64 keys x 128 bytes][tile 1],
// again 128 consecutive 128-byte rows; the Q buffer holds the unit's hi and lo E4M3 terms,
// [64 rows x 128 bytes] each, in place of the bf16 rows the TMA brought.
template <int NK, int NV, int NSB, bool KV8 = false>
struct TcLayout {
    static constexpr int kPBufs = 4;                             // P buffers (one tile each)
    static constexpr int kStage8 = KV8 ? 1 : 0;                  // (fp8: V landing barriers)
    static constexpr int kTileHalf = kHalfBytes;                 // 64 rows x 128 bytes
    static constexpr int kKSlotBytes = KV8 ? 2 * kTileBytes8 : 2 * kTileBytes;
    static constexpr int kKOff = 0;                              // NK x pair slot
    static constexpr int kVOff = kKOff + NK * kKSlotBytes;       // NV x [64 keys][128]
    static constexpr int kQOff = kVOff + NV * kTileBytes;        // 2 x [64 rows][128]
    static constexpr int kQBytes = kTileBytes;
    static constexpr int kPOff = kQOff + 2 * kQBytes;            // kPBufs x [64 rows][64 keys]
    static constexpr int kPBytes = kHalfBytes;
    static constexpr int kBarOff = kPOff + kPBufs * kPBytes;
    // kfull[NK] kempty[NK] vfull[NV] vempty[NV] q_full[2] q_free[2] s_full[NSB] s_free[NSB]
    // p_full[P] p_free[P] mma_done[2] merge_done; fp8: v8full[NV] (codes landed), q_conv[2]
    static constexpr int kNumBars = 2 * NK + 2 * NV + 4 + 2 * NSB + 2 * kPBufs + 3 + kStage8 * NV + 2;
    static constexpr int kPubOff = kBarOff + kNumBars * 8;        // per group: max[64], sum[64]
    static constexpr int kPubUnitOff = kPubOff + 2 * 2 * 64 * 4;  // per group: its last tile's unit
    // fp8: softmax scale of each row of the last 8 units (the unit's scale times its row's 2^-k),
    // a ring indexed by the unit ordinal, and the V tiles' descriptions for the converters
    static constexpr int kQScaleOff = kPubUnitOff + 16;
    static constexpr int kQScaleRing = 8;
    static constexpr int kVMetaOff = kQScaleOff + kStage8 * kQScaleRing * 64 * 4;
    static constexpr int kKMetaOff = kVMetaOff + kStage8 * NV * (int)sizeof(TileMeta);
    static constexpr int kSMetaOff = kKMetaOff + 2 * NK * (int)sizeof(TileMeta);
    static constexpr int kPMetaOff = kSMetaOff + 2 * NSB * (int)sizeof(TileMeta);
    static constexpr int kPlanOff = kPMetaOff + kPBufs * (int)sizeof(TileMeta);
    static constexpr int kPlanBytes = 2 * kMaxBatch * 4;
    static constexpr int kTmemOff = kPlanOff + kPlanBytes;
    static constexpr int kTotal = kTmemOff + 16;
    static constexpr int kAlloc = kTotal + 1024;
};

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int x, int y, int z, int w) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];"
        ::"r"(smem_addr(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w),
          "r"(smem_addr(bar))
        : "memory");
}

// Widens one fp8 tile in place.  The E4M3 codes (a 128-byte x 64-key TMA box, 128-byte swizzle)
// sit where the fp16 tile's upper half (dims 64-127) goes; `lo` is the fp16 lower half.  Thread
// r (0 .. 63) owns key row r: it reads its whole code row, then writes dims 0-63 into `lo` and
// dims 64-127 over the code row it has just read (no other row is touched, so no thread can
// overwrite codes another still needs).  Rows at or past `nvalid` become zeros.
__device__ __forceinline__ void widen_rows(uint32_t codes_hi, uint32_t lo, int nvalid, int r) {
    uint32_t w[32];
    if (r < nvalid) {
#pragma unroll
        for (int c = 0; c < 8; ++c)
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(w[4 * c]), "=r"(w[4 * c + 1]), "=r"(w[4 * c + 2]), "=r"(w[4 * c + 3])
                         : "r"(codes_hi + (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4))));
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        // codes 16 c .. 16 c + 15 -> fp16 dims 16 c .. 16 c + 15: half c / 4, chunks 2 (c % 4), + 1
        uint32_t h[8];
        if (r < nvalid) {
            e4m3x4_to_f16x2x2(w[4 * c], h[0], h[1]);
            e4m3x4_to_f16x2x2(w[4 * c + 1], h[2], h[3]);
            e4m3x4_to_f16x2x2(w[4 * c + 2], h[4], h[5]);
            e4m3x4_to_f16x2x2(w[4 * c + 3], h[6], h[7]);
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) h[j] = 0u;
        }
        const uint32_t hb = ((c >> 2) ? codes_hi : lo) + (uint32_t)(r * 128);
        const int c0 = 2 * (c & 3);
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};"
                     :: "r"(hb + (uint32_t)((c0 ^ (r & 7)) << 4)), "r"(h[0]), "r"(h[1]), "r"(h[2]), "r"(h[3])
                     : "memory");
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};"
                     :: "r"(hb + (uint32_t)(((c0 + 1) ^ (r & 7)) << 4)), "r"(h[4]), "r"(h[5]), "r"(h[6]), "r"(h[7])
                     : "memory");
    }
}

template <int SRC, int NK, int NV, int NSB, bool KV8 = false>
__global__ void __launch_bounds__(tc_threads<KV8>(), 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
               const __grid_constant__ CUtensorMap qmap, const AttnArgs a) {
    using L = TcLayout<NK, NV, NSB, KV8>;
    constexpr int kPB = L::kPBufs;
    constexpr int kS8 = L::kStage8;
    using TCOL = TcCols<NSB>;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base for the 128-byte swizzle, by pointer arithmetic on the shared array
    // (an integer round trip would make every access through it a generic one)
    uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
    uint64_t* kfull = bars;
    uint64_t* kempty = kfull + NK;
    uint64_t* vfull = kempty + NK;
    uint64_t* vempty = vfull + NV;
    uint64_t* q_full = vempty + NV;
    uint64_t* q_free = q_full + 2;
    uint64_t* s_full = q_free + 2;
    uint64_t* s_free = s_full + NSB;
    uint64_t* p_full = s_free + NSB;
    uint64_t* p_free = p_full + kPB;
    uint64_t* mma_done = p_free + kPB;
    uint64_t* merge_done = mma_done + 2;
    uint64_t* v8full = merge_done + 1;                  // fp8: [NV] codes of a V tile landed
    uint64_t* q_conv = v8full + kS8 * NV;               // fp8: the unit's Q split into E4M3 terms
    float* qscale = reinterpret_cast<float*>(smem + L::kQScaleOff);     // fp8: [8 units][64 rows]
    TileMeta* vmeta = reinterpret_cast<TileMeta*>(smem + L::kVMetaOff); // fp8: [NV]
    float* pub = reinterpret_cast<float*>(smem + L::kPubOff);           // [group][max | sum][row]
    volatile int* pub_unit = reinterpret_cast<volatile int*>(smem + L::kPubUnitOff);
    TileMeta* kmeta = reinterpret_cast<TileMeta*>(smem + L::kKMetaOff);
    TileMeta* smeta = reinterpret_cast<TileMeta*>(smem + L::kSMetaOff);
    TileMeta* pmeta = reinterpret_cast<TileMeta*>(smem + L::kPMetaOff);
    int* plan_tiles = reinterpret_cast<int*>(smem + L::kPlanOff);
    int* plan_len = plan_tiles + kMaxBatch;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemOff);
    __shared__ long long s_range[2];

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    uint64_t pol = 0;                          // the producers' L2 policy for the KV stream
    if ((warp == 0 || warp == 6) && lane == 0) pol = l2_evict_first_policy();
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&kmap);
        prefetch_tensormap(&vmap);
        prefetch_tensormap(&qmap);
        if (SRC == kSrcPaged) prefetch_first_tiles(a, &kmap, &vmap, KV8, 4);
    }
    pdl_wait();
    pdl_launch_dependents();   // after the wait, as attn_split_kernel (the LSE merge plans early)

    // ---- plan (as attn_split_kernel) -----------------------------------------------------
    if (warp == 0) {
        for (int b = lane; b < a.B; b += 32) {
            const int Lb = request_len<SRC>(a, b);
            plan_len[b] = Lb;
            plan_tiles[b] = request_tiles<SRC>(a, Lb);
        }
        __syncwarp();
        if (lane == 0) {
            long long T = 0;
            for (int b = 0; b < a.B; ++b) T += (long long)plan_tiles[b] * a.Hkv * a.n_rb;
            const int peff = plan_ctas(T, gridDim.x, a.min_tiles_per_cta);
            const long long c = blockIdx.x;
            s_range[0] = c < peff ? cta_begin(c, T, peff) : 0;
            s_range[1] = c < peff ? cta_begin(c + 1, T, peff) : 0;
            // K pair slot: one arrival per tile (the producer's); V slot: the producer's (bf16) or
            // both warps of the converter pair that widened it (fp8)
            for (int k = 0; k < NK; ++k) { mbar_init(&kfull[k], 2); mbar_init(&kempty[k], 1); }
            for (int k = 0; k < NV; ++k) { mbar_init(&vfull[k], KV8 ? 2 : 1); mbar_init(&vempty[k], 1); }
            if (KV8) {
                for (int k = 0; k < NV; ++k) mbar_init(&v8full[k], 1);
                mbar_init(&q_conv[0], 2);
                mbar_init(&q_conv[1], 2);
            }
            for (int k = 0; k < 2; ++k) { mbar_init(&q_full[k], 1); mbar_init(&q_free[k], 1); }
            for (int k = 0; k < NSB; ++k) {
                mbar_init(&s_full[k], 2);      // tensor-core completion + the forwarded descriptions
                mbar_init(&s_free[k], 8);      // both groups' warps have read their tile's scores
            }
            for (int k = 0; k < kPB; ++k) {
                mbar_init(&p_full[k], 4);
                mbar_init(&p_free[k], 1);
            }
            mbar_init(&mma_done[0], 1);
            mbar_init(&mma_done[1], 1);
            mbar_init(merge_done, 4);
            pub_unit[0] = -1;
            pub_unit[1] = -1;
            fence_barrier_init();
        }
    }
    __syncthreads();
    const long long t_begin = s_range[0], t_end = s_range[1];
    if (t_begin >= t_end) return;
    const uint32_t n = (uint32_t)(t_end - t_begin);

    // ---- tensor memory (whole warp 1) ------------------------------------------------------
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, TCOL::kAlloc);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0 || warp == 6) {
        // =========================== producers ===============================================
        if (lane == 0) {
            const bool is_k = (warp == 0);
            TileWalker<SRC> walk;
            walk.init(a, plan_tiles);
            uint32_t uidx = 0, it = 0;
            int ord = 0;
            const uint32_t q_bytes = (uint32_t)a.rows_total * 256u;
            bool alive = true;
            for (long long t = t_begin; t < t_end; ++t, ++it) {
                TileMeta m;
                int ty = 0, tz = 0;
                walk.describe(a, plan_tiles, plan_len, t, t_begin, t_end, m, ty, tz);
                m.ord = ord;
                if (m.flags & kLast) ++ord;
                if (is_k) {
                    if (m.flags & kFirst) {
                        const uint32_t qb = uidx & 1u;
                        if (!mbar_wait_bounded(&q_free[qb], ((uidx >> 1) & 1u) ^ 1u)) { alive = false; break; }
                        uint8_t* qdst = smem + L::kQOff + qb * L::kQBytes;
                        mbar_arrive_expect_tx(&q_full[qb], q_bytes);
                        tma_load_4d(qdst, &qmap, &q_full[qb], 0, 0, m.h, m.b * a.n_q);
                        tma_load_4d(qdst + kHalfBytes, &qmap, &q_full[qb], 64, 0, m.h, m.b * a.n_q);
                        ++uidx;
                    }
                    const uint32_t pq = it >> 1, sub = it & 1u, ks = pq % NK;
                    if (sub == 0u && !mbar_wait_bounded(&kempty[ks], ((pq / NK) & 1u) ^ 1u)) { alive = false; break; }
                    kmeta[2 * ks + sub] = m;
                    WMTP_TRACE_TILE(0, it);
                    if (KV8) {
                        // fp8: the codes land as they are (QK^T reads E4M3 keys)
                        uint8_t* dst8 = smem + L::kKOff + ks * L::kKSlotBytes + sub * kTileBytes8;
                        if (m.nvalid > 0) {
                            mbar_arrive_expect_tx(&kfull[ks], kTileBytes8);
                            tma_load_3d(dst8, &kmap, &kfull[ks], 0, ty, tz, pol);
                        } else {
                            mbar_arrive(&kfull[ks]);
                        }
                        if (sub == 0u && t + 1 == t_end) mbar_arrive(&kfull[ks]);   // pair without tile 1
                        continue;
                    }
                    uint8_t* dst = smem + L::kKOff + ks * L::kKSlotBytes + sub * kHalfBytes;
                    if (m.nvalid > 0) {
                        mbar_arrive_expect_tx(&kfull[ks], kTileBytes);
                        tma_load_3d(dst, &kmap, &kfull[ks], 0, ty, tz, pol);
                        tma_load_3d(dst + kTileBytes, &kmap, &kfull[ks], 64, ty, tz, pol);
                    } else {
                        mbar_arrive(&kfull[ks]);
                    }
                    if (sub == 0u && t + 1 == t_end) mbar_arrive(&kfull[ks]);   // pair without tile 1
                } else if (KV8) {
                    const uint32_t vs = it % NV;
                    if (!mbar_wait_bounded(&vempty[vs], ((it / NV) & 1u) ^ 1u)) { alive = false; break; }
                    vmeta[vs] = m;
                    WMTP_TRACE_TILE(1, it);
                    if (m.nvalid > 0) {
                        mbar_arrive_expect_tx(&v8full[vs], kTileBytes8);
                        tma_load_3d(smem + L::kVOff + vs * kTileBytes + kHalfBytes, &vmap, &v8full[vs], 0, ty, tz, pol);
                    } else {
                        mbar_arrive(&v8full[vs]);
                    }
                } else {
                    const uint32_t vs = it % NV;
                    if (!mbar_wait_bounded(&vempty[vs], ((it / NV) & 1u) ^ 1u)) { alive = false; break; }
                    uint8_t* dst = smem + L::kVOff + vs * kTileBytes;
                    if (m.nvalid > 0) {
                        mbar_arrive_expect_tx(&vfull[vs], kTileBytes);
                        tma_load_3d(dst, &vmap, &vfull[vs], 0, ty, tz, pol);
                        tma_load_3d(dst + kHalfBytes, &vmap, &vfull[vs], 64, ty, tz, pol);
                    } else {
                        mbar_arrive(&vfull[vs]);
                    }
                }
            }
            // drain: every issued stage released (no copy still landing at exit)
            const uint32_t depth = is_k ? NK : NV;
            const uint32_t used = is_k ? (it + 1) / 2 : it;          // K: pair slots
            uint64_t* empty = is_k ? kempty : vempty;
            for (uint32_t k = (used > depth ? used - depth : 0); k < used && alive; ++k)
                if (!mbar_wait_bounded(&empty[k % depth], (k / depth) & 1u)) break;
        }
    } else if (warp == 1) {
        // =========================== S issuer (QK^T) =========================================
        if (lane == 0) {
            constexpr uint32_t kIdescS64 = KV8 ? tc::idesc_e4m3_f32(64, 64, false, false)
                                               : tc::idesc_bf16_f32(64, 64, false, false);
            constexpr uint32_t kIdescS128 = KV8 ? tc::idesc_e4m3_f32(64, 128, false, false)
                                                : tc::idesc_bf16_f32(64, 128, false, false);
            uint64_t* q_ready = KV8 ? q_conv : q_full;   // fp8: Q split into E4M3 terms first
            // descriptors of the ring bases; a k-step or buffer offset is added as (bytes >> 4)
            const uint64_t dK = tc::smem_desc(smem_addr(smem + L::kKOff), 16, 1024);
            const uint64_t dQ = tc::smem_desc(smem_addr(smem + L::kQOff), 16, 1024);
            uint32_t uidx = 0;
            const uint32_t npairs = (n + 1) / 2;
            bool ok = true;
            for (uint32_t pq = 0; pq < npairs && ok; ++pq) {
                const uint32_t ks = pq % NK, sb = pq % NSB;
                if (!mbar_wait_bounded(&kfull[ks], (pq / NK) & 1u)) break;
                WMTP_TRACE_TILE(7, 2 * pq);
                const bool has1 = 2 * pq + 1 < n;
                TileMeta mt[2];
                uint32_t qb[2] = {0u, 0u};
                for (uint32_t sub = 0; sub < (has1 ? 2u : 1u); ++sub) {
                    mt[sub] = kmeta[2 * ks + sub];
                    if (mt[sub].flags & kFirst) {
                        if (!mbar_wait_bounded(&q_ready[uidx & 1u], (uidx >> 1) & 1u)) { ok = false; break; }
                        ++uidx;
                    }
                    qb[sub] = (uidx - 1u) & 1u;
                }
                if (!ok) break;
                if (!mbar_wait_bounded(&s_free[sb], ((pq / NSB) & 1u) ^ 1u)) break;
                WMTP_TRACE_TILE(6, 2 * pq);
                smeta[2 * sb] = mt[0];
                if (has1) smeta[2 * sb + 1] = mt[1];
                tc::fence_after_sync();
                const uint32_t kslot = ks * (uint32_t)L::kKSlotBytes;
                const bool paired = has1 && mt[0].nvalid > 0 && mt[1].nvalid > 0 && mt[0].unit == mt[1].unit;
                if (KV8) {
                    // E4M3: k-step j covers dims 32 j .. 32 j + 31 (32 bytes of every row); the hi
                    // and lo terms of Q accumulate into the same scores
                    if (paired) {
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const uint32_t qoff = qb[0] * (uint32_t)L::kQBytes + (uint32_t)((j >> 2) * kHalfBytes + (j & 3) * 32);
                            const uint32_t koff = kslot + (uint32_t)((j & 3) * 32);
                            tc::mma_f8_ss(tmem + sb * 128u, dQ + (qoff >> 4), dK + (koff >> 4), kIdescS128, j > 0);
                        }
                    } else {
                        for (uint32_t sub = 0; sub < (has1 ? 2u : 1u); ++sub) {
                            if (mt[sub].nvalid <= 0) continue;
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                const uint32_t qoff = qb[sub] * (uint32_t)L::kQBytes +
                                                      (uint32_t)((j >> 2) * kHalfBytes + (j & 3) * 32);
                                const uint32_t koff = kslot + sub * (uint32_t)kTileBytes8 + (uint32_t)((j & 3) * 32);
                                tc::mma_f8_ss(tmem + sb * 128u + 64u * sub, dQ + (qoff >> 4), dK + (koff >> 4),
                                              kIdescS64, j > 0);
                            }
                        }
                    }
                } else if (paired) {
                    // one N = 128 MMA per k-step: keys of both tiles are consecutive rows
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint32_t qoff = qb[0] * (uint32_t)L::kQBytes + (uint32_t)((j >> 2) * kHalfBytes + (j & 3) * 32);
                        const uint32_t koff = kslot + (uint32_t)((j >> 2) * kTileBytes + (j & 3) * 32);
                        tc::mma_f16_ss(tmem + sb * 128u, dQ + (qoff >> 4), dK + (koff >> 4), kIdescS128, j > 0);
                    }
                } else {
                    for (uint32_t sub = 0; sub < (has1 ? 2u : 1u); ++sub) {
                        if (mt[sub].nvalid <= 0) continue;
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const uint32_t qoff = qb[sub] * (uint32_t)L::kQBytes +
                                                  (uint32_t)((j >> 2) * kHalfBytes + (j & 3) * 32);
                            const uint32_t koff = kslot + sub * (uint32_t)kHalfBytes +
                                                  (uint32_t)((j >> 2) * kTileBytes + (j & 3) * 32);
                            tc::mma_f16_ss(tmem + sb * 128u + 64u * sub, dQ + (qoff >> 4), dK + (koff >> 4),
                                           kIdescS64, j > 0);
                        }
                    }
                }
                tc::commit(&kempty[ks]);
                tc::commit(&s_full[sb]);
                mbar_arrive(&s_full[sb]);
                WMTP_TRACE_TILE(3, 2 * pq);
                if (mt[0].flags & kLast) tc::commit(&q_free[qb[0]]);
                if (has1 && (mt[1].flags & kLast)) tc::commit(&q_free[qb[1]]);
            }
            // every MMA of this thread complete before the tensor memory is freed
            tc::commit(&mma_done[0]);
            mbar_wait_bounded(&mma_done[0], 0);
        }
    } else if (warp == 7) {
        // =========================== PV issuer ===============================================
        if (lane == 0) {
            constexpr uint32_t kIdescO = KV8 ? tc::idesc_f16_f32(64, 128, false, true)
                                             : tc::idesc_bf16_f32(64, 128, false, true);
            const uint64_t dP = tc::smem_desc(smem_addr(smem + L::kPOff), 16, 1024);
            const uint64_t dV = tc::smem_desc(smem_addr(smem + L::kVOff), 8192, 1024);
            uint32_t o_init[2] = {0u, 0u};
            int o_unit[2] = {-1, -1};
            for (uint32_t t = 0; t < n; ++t) {
                const uint32_t sb = t % kPB, vs = t % NV, g = t & 1u;
                // the softmax group of tile t has written P(t) (and read its description) by now
                if (!mbar_wait_bounded(&p_full[sb], (t / kPB) & 1u)) break;
                const TileMeta m = pmeta[sb];
                if (!mbar_wait_bounded(&vfull[vs], (t / NV) & 1u)) break;
                tc::fence_after_sync();
                if (m.unit != o_unit[g]) { o_unit[g] = m.unit; o_init[g] = 0u; }
                if (m.nvalid > 0) {
                    const uint32_t poff = sb * (uint32_t)L::kPBytes;
                    const uint32_t voff = vs * (uint32_t)kTileBytes;
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        tc::mma_f16_ss(tmem + TCOL::kO + 128u * g, dP + ((poff + 32u * j) >> 4),
                                       dV + ((voff + 2048u * j) >> 4), kIdescO, (o_init[g] | (uint32_t)j) != 0u);
                    o_init[g] = 1u;
                }
                tc::commit(&p_free[sb]);
                tc::commit(&vempty[vs]);
                WMTP_TRACE_TILE(5, t);
            }
            tc::commit(&mma_done[1]);
            mbar_wait_bounded(&mma_done[1], 0);
        }
    } else if (KV8 && warp >= 12) {
        // =========================== converters (fp8 KV) =====================================
        // Pair 0 (warps 12-13) takes the even tiles, pair 1 (warps 14-15) the odd ones; NV is
        // even, so each V slot belongs to one pair and its phases are waited on in order.  Thread
        // r of a pair owns key row r of its V tiles (widened to fp16 in place).  Pair 0 also
        // splits every unit's bf16 Q rows into the E4M3 hi / lo terms, strictly in unit order
        // (before its tile t it converts every unit up to tile t's), so its waits on the Q
        // buffers' phases are in order too: unit u + 2's Q cannot land before unit u is
        // converted (its buffer is freed only after unit u's last QK^T).
        static_assert(!KV8 || NV % 2 == 0, "each V slot belongs to one converter pair");
        const uint32_t pair = (uint32_t)(warp - 12) >> 1;
        const int r = threadIdx.x - 384 - 64 * (int)pair;            // 0 .. 63
        // Splits unit u's Q row r in place (the unit's rows form one row block of <= 64 rows).
        auto convert_q = [&](uint32_t u) -> bool {
            const uint32_t qb = u & 1u;
            if (!mbar_wait_bounded(&q_full[qb], (u >> 1) & 1u)) return false;
            const uint32_t row = smem_addr(smem + L::kQOff + qb * L::kQBytes) + (uint32_t)(r * 128);
            const bool live = r < a.rows_total;
            // chunk c of the bf16 boxes (box c / 8): dims 8 c .. 8 c + 7 of the row
            auto bchunk = [&](int c) -> uint32_t {
                return row + (uint32_t)((c >> 3) * kHalfBytes) + (uint32_t)(((c & 7) ^ (r & 7)) << 4);
            };
            float amax = 0.f;
            if (live) {
#pragma unroll 4
                for (int c = 0; c < 16; ++c) {
                    uint32_t w4[4];
                    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(w4[0]), "=r"(w4[1]), "=r"(w4[2]), "=r"(w4[3]) : "r"(bchunk(c)) : "memory");
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w4[k] << 16)),
                                                 fabsf(__uint_as_float(w4[k] & 0xffff0000u))));
                }
            }
            // 2^k q < 2^8 for the row's largest |q| (E4M3 reaches 448); the row's scores come out
            // 2^k too large, so its softmax scale carries 2^-k
            int e = 0;
            if (amax > 0.f) (void)frexpf(amax, &e);
            const int k2 = 8 - e;
            const float up = ldexpf(1.f, k2);
            qscale[(u % L::kQScaleRing) * 64 + r] = ldexpf(a.scale_log2, -k2);
            // output chunk c holds the codes of dims 16 c .. 16 c + 15 (lowest dim in the lowest
            // byte): hi in chunk c of box 0's space, lo in chunk c of box 1's space.  Writing hi
            // chunk c clobbers bf16 dims 8 c .. of box 0, which output chunks <= c have read
            // already; the lo chunks would clobber box 1 dims still unread, so they are held in
            // registers and written last.
            uint32_t lo[8][4];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint32_t w8[8];
                if (live) {
                    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(w8[0]), "=r"(w8[1]), "=r"(w8[2]), "=r"(w8[3]) : "r"(bchunk(2 * c)) : "memory");
                    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(w8[4]), "=r"(w8[5]), "=r"(w8[6]), "=r"(w8[7]) : "r"(bchunk(2 * c + 1)) : "memory");
                } else {
#pragma unroll
                    for (int k = 0; k < 8; ++k) w8[k] = 0u;
                }
                uint32_t hi4[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t wa = w8[2 * k], wb = w8[2 * k + 1];
                    const float x0 = __uint_as_float(wa << 16) * up;
                    const float x1 = __uint_as_float(wa & 0xffff0000u) * up;
                    const float x2 = __uint_as_float(wb << 16) * up;
                    const float x3 = __uint_as_float(wb & 0xffff0000u) * up;
                    hi4[k] = f32x2_to_e4m3x2(x0, x1) | (f32x2_to_e4m3x2(x2, x3) << 16);
                    uint32_t h01, h23;
                    e4m3x4_to_f16x2x2(hi4[k], h01, h23);
                    const float2 v01 = __half22float2(*reinterpret_cast<const __half2*>(&h01));
                    const float2 v23 = __half22float2(*reinterpret_cast<const __half2*>(&h23));
                    lo[c][k] = f32x2_to_e4m3x2(x0 - v01.x, x1 - v01.y) |
                               (f32x2_to_e4m3x2(x2 - v23.x, x3 - v23.y) << 16);
                }
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};"
                             :: "r"(row + (uint32_t)((c ^ (r & 7)) << 4)), "r"(hi4[0]), "r"(hi4[1]),
                                "r"(hi4[2]), "r"(hi4[3]) : "memory");
            }
#pragma unroll
            for (int c = 0; c < 8; ++c)
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};"
                             :: "r"(row + (uint32_t)kHalfBytes + (uint32_t)((c ^ (r & 7)) << 4)),
                                "r"(lo[c][0]), "r"(lo[c][1]), "r"(lo[c][2]), "r"(lo[c][3]) : "memory");
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(&q_conv[qb]);
            return true;
        };
        uint32_t next_u = 0;                                         // pair 0: next unit to split
        bool qok = true;
        TileMeta last{};
        for (uint32_t t = pair; t < n; t += 2) {
            const uint32_t vs = t % NV;
            if (!mbar_wait_bounded(&v8full[vs], (t / NV) & 1u)) break;
            const TileMeta m = vmeta[vs];
            last = m;
            if (pair == 0u) {
                while (qok && next_u <= (uint32_t)m.ord) qok = convert_q(next_u++);
                if (!qok) break;
            }
            // rows past the valid keys come out as zeros (codes there may be anything)
            const uint32_t base = smem_addr(smem + L::kVOff + vs * kTileBytes);
            widen_rows(base + kHalfBytes, base, kTileKeys, r);
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(&vfull[vs]);
            if (lane == 0 && (warp & 1) == 0) WMTP_TRACE_TILE(2, t);
        }
        // pair 0's last tile (n - 2) ended its unit: tile n - 1 starts one more unit
        if (pair == 0u && qok && n >= 2 && (n & 1u) == 0u && (last.flags & kLast) &&
            next_u == (uint32_t)last.ord + 1u)
            (void)convert_q(next_u);
    } else {
        // =========================== softmax warps (two groups) ==============================
        const uint32_t grp = warp >= 8 ? 1u : 0u;
        const int gwarp0 = grp ? 8 : 2;                  // the group's first warp
        const int gtid = threadIdx.x - 32 * gwarp0;      // 0 .. 127 within the group
        const int sp = warp & 3;
        const int half = lane >> 4;
        const int row = 16 * sp + (lane & 15);
        const uint32_t lane_base = (uint32_t)(32 * sp) << 16;
        const uint32_t o_own = TCOL::kO + 128u * grp, o_oth = TCOL::kO + 128u * (grp ^ 1u);
        float* pub_m_own = pub + (2 * grp) * 64;
        float* pub_l_own = pub + (2 * grp + 1) * 64;
        const float* pub_m_oth = pub + (2 * (grp ^ 1u)) * 64;
        const float* pub_l_oth = pub + (2 * (grp ^ 1u) + 1) * 64;
        float m_used = -INFINITY, l_part = 0.f;
        float rs = a.scale_log2;                         // this row's score scale (log2 units)
        unsigned long long vis = 0ull;
        bool row_ok = false;
        int Lpre = 0, my_unit = -1;
        bool alive = true;
        for (uint32_t it = grp; it < n && alive; it += 2) {
            const uint32_t sq = (it >> 1) % NSB;             // S pair buffer
            const uint32_t scol = sq * 128u + 64u * grp;     // this tile's 64 score columns
            const uint32_t sb = it % kPB;                    // P buffer
            if (!mbar_wait_bounded(&s_full[sq], ((it >> 1) / NSB) & 1u)) { alive = false; break; }
            if (lane == 0 && warp == gwarp0) WMTP_TRACE_TILE(8, it);
            tc::fence_after_sync();
            const TileMeta m = smeta[2 * sq + grp];
            if (m.unit != my_unit) {
                // first tile of a unit for this group: the previous unit's combination (which
                // reads this group's O) must be done before this group's O is overwritten
                if (m.ord >= 1 && !mbar_wait_bounded(merge_done, (uint32_t)(m.ord - 1) & 1u)) {
                    alive = false;
                    break;
                }
                my_unit = m.unit;
                Lpre = m.L_tot - a.n_q;
                const int R = m.rb * kRowsPerBlock + row;
                row_ok = R < a.rows_total;
                vis = row_ok ? step_visibility(a, m.b, R / a.G) : 0ull;
                m_used = -INFINITY;
                l_part = 0.f;
                // fp8: the row's Q carries 2^k (written before the unit's first QK^T was issued,
                // so before these scores completed)
                if (KV8) rs = qscale[((uint32_t)m.ord % L::kQScaleRing) * 64 + row];
            }
            // ---- this thread's 32 scores from tensor memory ---------------------------------
            __syncwarp();
            uint32_t sr[32];
            tc::ld_16x32bx2_x16<32>(tmem + lane_base + scol, sr);
            tc::ld_16x32bx2_x16<32>(tmem + lane_base + scol + 16u, sr + 16);
            tc::wait_ld();
            if (lane == 0 && warp == gwarp0) WMTP_TRACE_TILE(9, it);
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_free[sq]);
            // ---- key mask of this row: valid rows of the tile, prefix keys, visible step keys --
            uint32_t mk = 0u;
            if (row_ok && m.nvalid > 0) {
                if (m.nvalid == kTileKeys && m.pos0 + kTileKeys <= Lpre) {
                    mk = ~0u;
                } else {
                    const int d = Lpre - m.pos0;           // keys [0, d) of the tile are prefix
                    const unsigned long long valid =
                        m.nvalid >= 64 ? ~0ull : ((1ull << m.nvalid) - 1ull);
                    const unsigned long long pre =
                        d >= 64 ? ~0ull : (d <= 0 ? 0ull : ((1ull << d) - 1ull));
                    const unsigned long long step =
                        d >= 64 ? 0ull : (d >= 0 ? (vis << d) : (-d >= 64 ? 0ull : (vis >> (-d))));
                    mk = (uint32_t)(((pre | step) & valid) >> (32 * half));
                }
            }
            // ---- maximum over the row (both half-warps), running maximum -------------------
            float x[32];
            if (mk == ~0u) {
#pragma unroll
                for (int j = 0; j < 32; ++j) x[j] = __uint_as_float(sr[j]);
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) x[j] = ((mk >> j) & 1u) ? __uint_as_float(sr[j]) : -INFINITY;
            }
            float mx8[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) mx8[j] = fmaxf(fmaxf(x[j], x[j + 8]), fmaxf(x[j + 16], x[j + 24]));
            float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16)) * rs;
            float alpha = 1.f;
            bool rescale = false;
            if (mx > m_used + kRescaleThreshold || (m_used == -INFINITY && mx != -INFINITY)) {
                if (m_used != -INFINITY) {
                    alpha = fast_exp2(m_used - mx);
                    rescale = true;
                }
                m_used = mx;
                l_part *= alpha;
            }
            const float m_sub = (m_used == -INFINITY) ? 0.f : m_used;
            uint32_t pk[16];
            float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float p0 = fast_exp2(fmaf(x[2 * j], rs, -m_sub));
                const float p1 = fast_exp2(fmaf(x[2 * j + 1], rs, -m_sub));
                // fp16 (fp8 KV) or bf16 weights for PV; the row sum over the fp32 weights (the
                // rounded weights would cost two unpacks a pair; the sums differ by at most 2^-9
                // of a weight, within the tolerance)
                pk[j] = KV8 ? pack_f16x2(p0, p1) : pack_bf16x2(p0, p1);
                ls[j & 3] += p0 + p1;
            }
            l_part += (ls[0] + ls[1]) + (ls[2] + ls[3]);
            if (lane == 0 && warp == gwarp0) WMTP_TRACE_TILE(10, it);
            // ---- P to shared memory (its buffer is free once PV of tile it - NSB is done) -----
            if (it >= (uint32_t)kPB && !mbar_wait_bounded(&p_free[sb], ((it / kPB) & 1u) ^ 1u)) {
                alive = false;
                break;
            }
            {
                uint8_t* prow = smem + L::kPOff + sb * L::kPBytes + row * 128;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int chunk = 4 * half + c;
                    *reinterpret_cast<uint4*>(prow + ((chunk ^ (row & 7)) << 4)) =
                        make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
                }
            }
            if (lane == 0 && warp == gwarp0) WMTP_TRACE_TILE(11, it);
            // V rows past the valid keys may hold anything (NaN tails): zero them before PV
            if (m.nvalid > 0 && m.nvalid < kTileKeys) {
                const uint32_t vs = it % NV;
                if (!mbar_wait_bounded(&vfull[vs], (it / NV) & 1u)) { alive = false; break; }
                uint8_t* vt = smem + L::kVOff + vs * kTileBytes;
                const int nrow = kTileKeys - m.nvalid;
                for (int idx = gtid; idx < nrow * 16; idx += 128) {
                    const int r = m.nvalid + idx / 16, c16 = idx % 16;
                    *reinterpret_cast<uint4*>(vt + (c16 >> 3) * kHalfBytes + r * 128 + (c16 & 7) * 16) =
                        make_uint4(0u, 0u, 0u, 0u);
                }
            }
            // ---- rare: move this warp's O rows to the new maximum (after this group's
            //      previous PV, tile it - 2, is done) --------------------------------------------
            if (__any_sync(0xffffffffu, rescale)) {
                if (it >= 2u) {
                    const uint32_t pb = (it - 2u) % kPB;
                    if (!mbar_wait_bounded(&p_free[pb], ((it - 2u) / kPB) & 1u)) { alive = false; break; }
                }
                tc::fence_after_sync();
                const float f = rescale ? alpha : 1.f;
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t o[16];
                    __syncwarp();
                    tc::ld_16x32bx2_x16<64>(tmem + lane_base + o_own + 16u * c, o);
                    tc::wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * f);
                    tc::st_16x32bx2_x16<64>(tmem + lane_base + o_own + 16u * c, o);
                }
                tc::wait_st();
            }
            // ---- publish this group's row state for the unit-end combination -----------------
            const float l_row = l_part + __shfl_xor_sync(0xffffffffu, l_part, 16);
            if (half == 0) {
                pub_m_own[row] = m_used;
                pub_l_own[row] = l_row;
            }
            if (warp == gwarp0 && lane == 0) {
                pmeta[sb] = m;                           // the PV issuer's copy of the description
                pub_unit[grp] = m.unit;
            }
            fence_proxy_async();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[sb]);
            if (lane == 0 && warp == gwarp0) WMTP_TRACE_TILE(4, it);
            // ---- unit end: combine both groups' (O, max, sum), write the rows ----------------
            if (m.flags & kLast) {
                if (!mbar_wait_bounded(&p_free[sb], (it / kPB) & 1u)) { alive = false; break; }
                // the other group's last tile of this unit, if any, is tile it - 1: its P (and so
                // its published state) is complete once its p_full phase has, and its PV before
                // ours
                bool other = false;
                float m_o = -INFINITY, l_o = 0.f;
                if (it >= 1u) {
                    const uint32_t pb = (it - 1u) % kPB;
                    if (!mbar_wait_bounded(&p_full[pb], ((it - 1u) / kPB) & 1u)) { alive = false; break; }
                    if (pub_unit[grp ^ 1u] == m.unit) {
                        other = true;
                        m_o = pub_m_oth[row];
                        l_o = pub_l_oth[row];
                    }
                }
                tc::fence_after_sync();
                const float M = fmaxf(m_used, m_o);
                const float w_own = (m_used == -INFINITY) ? 0.f : fast_exp2(m_used - M);
                const float w_oth = (!other || m_o == -INFINITY) ? 0.f : fast_exp2(m_o - M);
                const float l_sum = l_row * w_own + l_o * w_oth;
                const float inv = l_sum > 0.f ? a.v_scale / l_sum : 0.f;
                const float lse2 = l_sum > 0.f ? M + __log2f(l_sum) : -INFINITY;
                const bool use_own = w_own > 0.f, use_oth = w_oth > 0.f;
                const int R = m.rb * kRowsPerBlock + row;
                const int i = R / a.G, g = R - (R / a.G) * a.G;
                const size_t orow = ((size_t)m.b * a.n_q + i) * a.Hq + (size_t)m.h * a.G + g;
                const int slot = (int)blockIdx.x + m.unit;
#pragma unroll 1
                for (int c = 0; c < 4; ++c) {
                    uint32_t o[16], o2[16];
                    __syncwarp();
                    tc::ld_16x32bx2_x16<64>(tmem + lane_base + o_own + 16u * c, o);
                    tc::ld_16x32bx2_x16<64>(tmem + lane_base + o_oth + 16u * c, o2);
                    tc::wait_ld();
                    if (row_ok) {
                        const int d0 = 64 * half + 16 * c;
                        float v[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            float acc = use_own ? __uint_as_float(o[j]) * w_own : 0.f;
                            if (use_oth) acc += __uint_as_float(o2[j]) * w_oth;
                            v[j] = acc * inv;
                        }
                        if (m.flags & kWhole) {
                            uint4* op = reinterpret_cast<uint4*>(a.out + orow * kD + d0);
                            op[0] = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                               pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
                            op[1] = make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]),
                                               pack_bf16x2(v[12], v[13]), pack_bf16x2(v[14], v[15]));
                        } else {
                            float4* wo = reinterpret_cast<float4*>(
                                a.ws_o + ((size_t)slot * a.rows_blk + row) * kD + d0);
                            wo[0] = make_float4(v[0], v[1], v[2], v[3]);
                            wo[1] = make_float4(v[4], v[5], v[6], v[7]);
                            wo[2] = make_float4(v[8], v[9], v[10], v[11]);
                            wo[3] = make_float4(v[12], v[13], v[14], v[15]);
                        }
                    }
                }
                if (row_ok && half == 0) {
                    if (m.flags & kWhole) {
                        if (a.lse != nullptr) a.lse[orow] = lse2 * kLn2;
                    } else {
                        a.ws_lse[(size_t)slot * a.rows_blk + row] = lse2;
                    }
                }
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(merge_done);
            }
        }
    }

    // ---- all roles done (or stopped): free the tensor memory --------------------------------
    __syncwarp();
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, TCOL::kAlloc);
    }
}

}  // namespace wmtp
