// attn_tct_kernels.cuh -- split-KV attention for units of at most 32 query rows on the 5th-
// generation tensor cores, with the contraction transposed so every MMA is full height:
//
//   S^T[key][row]  = K Q^T    (M = 128 keys of a pair of tiles, N = 32 rows, K = 128 dims)
//   O^T[dim][row] += V^T P^T  (M = 128 head dims, N = 32 rows, K = the step's keys)
//
// The decode and verify shapes of the Windowed-MTP step (Pith verdict on arXiv 2607.21535,
// pith_extraction.key_machinery: gamma + 1 verify positions, G = 8 query heads per kv head) give
// 8..32 rows per kv head; an M = 64 or 128 tile over rows would leave half of it or more empty.
//
// Work split, tile walk, masks, partial format and merge are those of attn_split_kernel.  Tiles
// go in pairs (CTA-local tiles 2q, 2q + 1) sharing one 32 KiB K pair slot whose 128 keys are 128
// consecutive 128-byte rows per 64-dim half: the K-major A operand of M = 128.  A pair of one
// unit is one step; otherwise each tile is a step of its own (the other half's lanes masked).
//
// Roles (384 threads; 640 with fp8 KV):
//   warp 0        K producer (pair slots) and each unit's Q rows (a 4-D TMA box per 64-dim half
//                 that lands as the unit's rows, the N = 32 K-major B operand);
//   warp 1        S issuer: 8 MMAs M128 N32 K16 per step into one of NSB S buffers (32 columns);
//   warp 2        V producer (one slot per tile);
//   warp 3        PV issuer: 4 MMAs M128 N32 K16 per tile with V^T read MN-major from the V slot
//                 and P^T K-major from the step's P buffer, into the unit's O^T buffer (two
//                 buffers alternate between units);
//   warps 4..11   softmax, two warps per scheduler: warp 4 + 4 hh + q owns TMEM lanes 32 q .. + 31
//                 (key t of the step for S^T, head dim t for O^T) and rows 16 hh .. + 15.  Each
//                 step a thread reads its 16 scores, masks, and tests them against the rows'
//                 running maxima (shared, in shared memory).  Only when some score exceeds its
//                 row's maximum by more than 2^8 (log2 units; always on a unit's first step) do the
//                 warps agree, through a bounded rendezvous, on new maxima (a reduce over the lanes
//                 and a combine over the lane quarters), rescale their per-lane row sums and their
//                 O^T columns.  Then P = 2^(x - m) (<= 2^8) goes to the P buffer as P^T.  At a
//                 unit's end the row sums are reduced the same way and each thread writes head dim
//                 t of its 16 rows (partials when the unit is split);
//   warps 12..19  (fp8 KV only) converters: the E4M3 codes land in the upper half of each fp16
//                 slot and are widened in place, each tile of a pair by its own two warps (four
//                 for K, four for V); the unit's Q is widened bf16 -> fp16 in place.
// Every wait is bounded; the softmax warps meet only through mbarriers with bounded waits, so a
// warp that gives up cannot leave the others blocked.  On a timeout all roles stop, the issuers
// wait (bounded) for their own MMAs, all meet at the final barrier and warp 1 frees the tensor
// memory.
#pragma once

#include "attn_tc_kernels.cuh"

namespace wmtp {

template <bool KV8>
constexpr int tct_threads() { return KV8 ? 640 : 384; }

constexpr int kTctRows = 32;                     // N of both MMAs: rows per unit, padded

template <int NK, int NV, int NSB>
struct TctCols {
    static constexpr uint32_t kO = NSB * kTctRows;               // O^T of unit parity u: kO + 32 u
    static constexpr uint32_t kAlloc = (NSB * kTctRows + 2 * kTctRows) <= 128 ? 128u : 256u;
    static_assert(NSB * kTctRows + 2 * kTctRows <= 256, "S buffers and two O^T fit 256 columns");
};

// One step: one or both tiles of a pair, of one unit.
struct StepMeta {
    TileMeta tm[2];
    int inc;          // bit s: tile 2q + s belongs to this step
    int it0;          // CTA-local index of tile 2q
};

template <int NK, int NV, int NSB, bool KV8>
struct TctLayout {
    static constexpr int kPBufs = 4;
    static constexpr int kKSlotBytes = 2 * kTileBytes;           // pair slot, 32 KiB
    static constexpr int kKOff = 0;
    static constexpr int kVOff = kKOff + NK * kKSlotBytes;       // NV x [64 keys][128] (two halves)
    static constexpr int kQOff = kVOff + NV * kTileBytes;        // 2 x [half][32 rows][128 B]
    static constexpr int kQHalf = kTctRows * 128;                // 4 KiB: one 64-dim half
    static constexpr int kQBytes = 2 * kQHalf;
    static constexpr int kPOff = kQOff + 2 * kQBytes;            // kPBufs x [sub][32 rows][128 B]
    static constexpr int kPBytes = 2 * kTctRows * 128;
    static constexpr int kBarOff = kPOff + kPBufs * kPBytes;
    // kfull[NK] kempty[NK] vfull[NV] vempty[NV] q_full[2] q_free[2] s_full[NSB] s_free[NSB]
    // p_full[P] p_free[P] o_free[2] sm_sync mma_done[2]; fp8: k8full[2 NK] v8full[NV] q_conv[2]
    static constexpr int kNumBars = 2 * NK + 2 * NV + 4 + 2 * NSB + 2 * kPBufs + 2 + 1 + 2 +
                                    (KV8 ? 2 * NK + NV + 2 : 0);
    static constexpr int kMOff = (kBarOff + kNumBars * 8 + 15) / 16 * 16;   // running row maxima [32]
    static constexpr int kAlphaOff = kMOff + kTctRows * 4;        // row rescale factors [32]
    static constexpr int kRedOff = kAlphaOff + kTctRows * 4;      // per-warp row values [4][32]
    static constexpr int kFlagOff = kRedOff + 4 * kTctRows * 4;   // per-warp flags [2][8]
    static constexpr int kVisOff = kFlagOff + 64;                 // row visibility masks [32]
    static constexpr int kKMetaOff = kVisOff + kTctRows * 8;
    static constexpr int kSMetaOff = kKMetaOff + 2 * NK * (int)sizeof(TileMeta);
    static constexpr int kPMetaOff = kSMetaOff + NSB * (int)sizeof(StepMeta);
    static constexpr int kPlanOff = kPMetaOff + kPBufs * (int)sizeof(StepMeta);
    static constexpr int kTmemOff = kPlanOff + 2 * kMaxBatch * 4;
    static constexpr int kTotal = kTmemOff + 16;
    static constexpr int kAlloc = kTotal + 1024;
    static_assert(kBarOff % 8 == 0 && kMOff % 16 == 0 && kAlphaOff % 16 == 0 && kVisOff % 8 == 0,
                  "alignment");
};

// Warp transpose-reduce of 32 values per lane (value n of every lane belongs to row n): after it,
// lane n holds row n's reduction over the warp.  16 + 8 + 4 + 2 + 1 shuffles.
template <bool MAX>
__device__ __forceinline__ float warp_rows_reduce(float (&v)[32], int lane) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < off; ++i) {
            const float send = upper ? v[i] : v[i + off];
            const float keep = upper ? v[i + off] : v[i];
            const float got = __shfl_xor_sync(0xffffffffu, send, off);
            v[i] = MAX ? fmaxf(keep, got) : keep + got;
        }
    }
    return v[0];
}

template <int SRC, int NK, int NV, int NSB, bool KV8 = false>
__global__ void __launch_bounds__(tct_threads<KV8>(), 1)
attn_tct_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                const __grid_constant__ CUtensorMap qmap, const AttnArgs a) {
    using L = TctLayout<NK, NV, NSB, KV8>;
    using TCOL = TctCols<NK, NV, NSB>;
    constexpr int kPB = L::kPBufs;
    extern __shared__ uint8_t smem_raw[];
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
    uint64_t* o_free = p_free + kPB;
    uint64_t* sm_sync = o_free + 2;
    uint64_t* mma_done = sm_sync + 1;
    uint64_t* k8full = mma_done + 2;                     // fp8: [2 NK]
    uint64_t* v8full = k8full + (KV8 ? 2 * NK : 0);      // fp8: [NV]
    uint64_t* q_conv = v8full + (KV8 ? NV : 0);          // fp8: [2]
    float* m_s = reinterpret_cast<float*>(smem + L::kMOff);
    float* alpha_s = reinterpret_cast<float*>(smem + L::kAlphaOff);
    float* red_s = reinterpret_cast<float*>(smem + L::kRedOff);
    int* flag_s = reinterpret_cast<int*>(smem + L::kFlagOff);
    unsigned long long* vis_s = reinterpret_cast<unsigned long long*>(smem + L::kVisOff);
    TileMeta* kmeta = reinterpret_cast<TileMeta*>(smem + L::kKMetaOff);
    StepMeta* smeta = reinterpret_cast<StepMeta*>(smem + L::kSMetaOff);
    StepMeta* pmeta = reinterpret_cast<StepMeta*>(smem + L::kPMetaOff);
    int* plan_tiles = reinterpret_cast<int*>(smem + L::kPlanOff);
    int* plan_len = plan_tiles + kMaxBatch;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemOff);
    __shared__ long long s_range[2];

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    pdl_launch_dependents();
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&kmap);
        prefetch_tensormap(&vmap);
        prefetch_tensormap(&qmap);
    }
    pdl_wait();

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
            for (int k = 0; k < NK; ++k) { mbar_init(&kfull[k], KV8 ? 4 : 2); mbar_init(&kempty[k], 1); }
            for (int k = 0; k < NV; ++k) { mbar_init(&vfull[k], KV8 ? 2 : 1); mbar_init(&vempty[k], 1); }
            if (KV8) {
                for (int k = 0; k < 2 * NK; ++k) mbar_init(&k8full[k], 1);
                for (int k = 0; k < NV; ++k) mbar_init(&v8full[k], 1);
                mbar_init(&q_conv[0], 2);
                mbar_init(&q_conv[1], 2);
            }
            for (int k = 0; k < 2; ++k) { mbar_init(&q_full[k], 1); mbar_init(&q_free[k], 1); }
            for (int k = 0; k < NSB; ++k) { mbar_init(&s_full[k], 2); mbar_init(&s_free[k], 8); }
            for (int k = 0; k < kPB; ++k) { mbar_init(&p_full[k], 8); mbar_init(&p_free[k], 1); }
            mbar_init(&o_free[0], 8);
            mbar_init(&o_free[1], 8);
            mbar_init(sm_sync, 8);
            mbar_init(&mma_done[0], 1);
            mbar_init(&mma_done[1], 1);
            fence_barrier_init();
        }
    }
    __syncthreads();
    const long long t_begin = s_range[0], t_end = s_range[1];
    if (t_begin >= t_end) return;
    const uint32_t n = (uint32_t)(t_end - t_begin);
    const uint32_t npairs = (n + 1) / 2;

    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, TCOL::kAlloc);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0 || warp == 2) {
        // =========================== producers ===============================================
        if (lane == 0) {
            const bool is_k = (warp == 0);
            const uint64_t pol = l2_evict_first_policy();
            TileWalker<SRC> walk;
            walk.init(a, plan_tiles);
            uint32_t uidx = 0, it = 0;
            const uint32_t q_bytes = (uint32_t)a.rows_total * 256u;
            bool alive = true;
            for (long long t = t_begin; t < t_end; ++t, ++it) {
                TileMeta m;
                int ty = 0, tz = 0;
                walk.describe(a, plan_tiles, plan_len, t, t_begin, t_end, m, ty, tz);
                m.ord = (int)uidx - ((m.flags & kFirst) ? 0 : 1);   // the tile's unit index in the CTA
                if (is_k) {
                    if (m.flags & kFirst) {
                        const uint32_t qb = uidx & 1u;
                        if (!mbar_wait_bounded(&q_free[qb], ((uidx >> 1) & 1u) ^ 1u)) { alive = false; break; }
                        uint8_t* qdst = smem + L::kQOff + qb * L::kQBytes;
                        mbar_arrive_expect_tx(&q_full[qb], q_bytes);
                        tma_load_4d(qdst, &qmap, &q_full[qb], 0, 0, m.h, m.b * a.n_q);
                        tma_load_4d(qdst + L::kQHalf, &qmap, &q_full[qb], 64, 0, m.h, m.b * a.n_q);
                        ++uidx;
                    }
                    const uint32_t pq = it >> 1, sub = it & 1u, ks = pq % NK;
                    if (sub == 0u && !mbar_wait_bounded(&kempty[ks], ((pq / NK) & 1u) ^ 1u)) { alive = false; break; }
                    kmeta[2 * ks + sub] = m;
                    if (KV8) {
                        uint64_t* lb = &k8full[2 * ks + sub];
                        if (m.nvalid > 0) {
                            mbar_arrive_expect_tx(lb, kTileBytes8);
                            tma_load_3d(smem + L::kKOff + ks * L::kKSlotBytes + kTileBytes + sub * kHalfBytes,
                                        &kmap, lb, 0, ty, tz, pol);
                        } else {
                            mbar_arrive(lb);
                        }
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
                } else {
                    const uint32_t vs = it % NV;
                    if (!mbar_wait_bounded(&vempty[vs], ((it / NV) & 1u) ^ 1u)) { alive = false; break; }
                    uint8_t* dst = smem + L::kVOff + vs * kTileBytes;
                    if (KV8) {
                        if (m.nvalid > 0) {
                            mbar_arrive_expect_tx(&v8full[vs], kTileBytes8);
                            tma_load_3d(dst + kHalfBytes, &vmap, &v8full[vs], 0, ty, tz, pol);
                        } else {
                            mbar_arrive(&v8full[vs]);
                        }
                    } else if (m.nvalid > 0) {
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
            const uint32_t used = is_k ? (it + 1) / 2 : it;
            uint64_t* empty = is_k ? kempty : vempty;
            for (uint32_t k = (used > depth ? used - depth : 0); k < used && alive; ++k)
                if (!mbar_wait_bounded(&empty[k % depth], (k / depth) & 1u)) break;
        }
    } else if (warp == 1) {
        // =========================== S issuer: S^T = K Q^T ===================================
        if (lane == 0) {
            constexpr uint32_t kIdescS = KV8 ? tc::idesc_f16_f32(128, kTctRows, false, false)
                                             : tc::idesc_bf16_f32(128, kTctRows, false, false);
            uint64_t* q_ready = KV8 ? q_conv : q_full;
            const uint64_t dK = tc::smem_desc(smem_addr(smem + L::kKOff), 16, 1024);
            const uint64_t dQ = tc::smem_desc(smem_addr(smem + L::kQOff), 16, 1024);
            uint32_t uidx = 0, step = 0;
            bool ok = true;
            for (uint32_t pq = 0; pq < npairs && ok; ++pq) {
                const uint32_t ks = pq % NK;
                if (!mbar_wait_bounded(&kfull[ks], (pq / NK) & 1u)) break;
                const bool has1 = 2 * pq + 1 < n;
                TileMeta mt[2];
                mt[0] = kmeta[2 * ks];
                if (has1) mt[1] = kmeta[2 * ks + 1];
                const bool paired = has1 && mt[0].unit == mt[1].unit;
                const int nsteps = paired ? 1 : (has1 ? 2 : 1);
                for (int si = 0; si < nsteps && ok; ++si, ++step) {
                    StepMeta sm;
                    sm.tm[0] = mt[0];
                    sm.tm[1] = has1 ? mt[1] : mt[0];
                    sm.inc = paired ? 3 : (si == 0 ? 1 : 2);
                    sm.it0 = (int)(2 * pq);
                    const int f_flags = (sm.inc & 1) ? mt[0].flags : mt[1].flags;
                    const int l_flags = (sm.inc & 2) ? mt[1].flags : mt[0].flags;
                    if (f_flags & kFirst) {
                        if (!mbar_wait_bounded(&q_ready[uidx & 1u], (uidx >> 1) & 1u)) { ok = false; break; }
                        ++uidx;
                    }
                    const uint32_t qb = (uidx - 1u) & 1u;
                    const uint32_t sb = step % NSB;
                    if (!mbar_wait_bounded(&s_free[sb], ((step / NSB) & 1u) ^ 1u)) { ok = false; break; }
                    smeta[sb] = sm;
                    tc::fence_after_sync();
                    const uint32_t kslot = ks * (uint32_t)L::kKSlotBytes;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint32_t qoff = qb * (uint32_t)L::kQBytes + (uint32_t)((j >> 2) * L::kQHalf + (j & 3) * 32);
                        const uint32_t koff = kslot + (uint32_t)((j >> 2) * kTileBytes + (j & 3) * 32);
                        tc::mma_f16_ss(tmem + sb * (uint32_t)kTctRows, dK + (koff >> 4), dQ + (qoff >> 4), kIdescS, j > 0);
                    }
                    tc::commit(&s_full[sb]);
                    mbar_arrive(&s_full[sb]);
                    if (l_flags & kLast) tc::commit(&q_free[qb]);
                }
                tc::commit(&kempty[ks]);
            }
            tc::commit(&mma_done[0]);
            mbar_wait_bounded(&mma_done[0], 0);
        }
    } else if (warp == 3) {
        // =========================== PV issuer: O^T += V^T P^T ===============================
        if (lane == 0) {
            constexpr uint32_t kIdescO = KV8 ? tc::idesc_f16_f32(128, kTctRows, true, false)
                                             : tc::idesc_bf16_f32(128, kTctRows, true, false);
            const uint64_t dP = tc::smem_desc(smem_addr(smem + L::kPOff), 16, 1024);
            const uint64_t dV = tc::smem_desc(smem_addr(smem + L::kVOff), 8192, 1024);
            uint32_t step = 0, units = 0, o_init = 0;
            int cur_unit = -1;
            bool ok = true;
            for (uint32_t pq = 0; pq < npairs && ok; ++pq) {
                // the steps of pair q, as the S issuer forms them (read from the P metadata)
                int done_inc = 0;
                const int want_inc = (2 * pq + 1 < n) ? 3 : 1;
                while (done_inc != want_inc) {
                    const uint32_t pb = step % kPB;
                    if (!mbar_wait_bounded(&p_full[pb], (step / kPB) & 1u)) { ok = false; break; }
                    const StepMeta sm = pmeta[pb];
                    const int f_unit = (sm.inc & 1) ? sm.tm[0].unit : sm.tm[1].unit;
                    if (f_unit != cur_unit) {
                        // a new unit: its O^T buffer is free once the unit two back was read out
                        cur_unit = f_unit;
                        const uint32_t ob = units & 1u;
                        if (!mbar_wait_bounded(&o_free[ob], ((units >> 1) & 1u) ^ 1u)) { ok = false; break; }
                        ++units;
                        o_init = 0;
                    }
                    const uint32_t ob = (units - 1u) & 1u;
#pragma unroll
                    for (int sub = 0; sub < 2; ++sub) {
                        if (!((sm.inc >> sub) & 1)) continue;
                        const uint32_t tix = (uint32_t)sm.it0 + (uint32_t)sub;
                        const uint32_t vs = tix % NV;
                        if (!mbar_wait_bounded(&vfull[vs], (tix / NV) & 1u)) { ok = false; break; }
                    }
                    if (!ok) break;
                    tc::fence_after_sync();
#pragma unroll
                    for (int sub = 0; sub < 2; ++sub) {
                        if (!((sm.inc >> sub) & 1) || sm.tm[sub].nvalid <= 0) continue;
                        const uint32_t vs = ((uint32_t)sm.it0 + (uint32_t)sub) % NV;
                        const uint32_t poff = pb * (uint32_t)L::kPBytes + (uint32_t)sub * (kTctRows * 128u);
                        const uint32_t voff = vs * (uint32_t)kTileBytes;
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            tc::mma_f16_ss(tmem + TCOL::kO + (uint32_t)kTctRows * ob, dV + ((voff + 2048u * j) >> 4),
                                           dP + ((poff + 32u * j) >> 4), kIdescO, (o_init | (uint32_t)j) != 0u);
                        o_init = 1u;
                    }
                    tc::commit(&p_free[pb]);
                    for (int sub = 0; sub < 2; ++sub)
                        if ((sm.inc >> sub) & 1) tc::commit(&vempty[((uint32_t)sm.it0 + (uint32_t)sub) % NV]);
                    done_inc |= sm.inc;
                    ++step;
                }
            }
            tc::commit(&mma_done[1]);
            mbar_wait_bounded(&mma_done[1], 0);
        }
    } else if (KV8 && warp >= 12) {
        // =========================== converters (fp8 KV) =====================================
        // warps 12-15 widen K (warps 12-13 the pair's tile 0, 14-15 its tile 1, and the unit's Q
        // where that tile starts a unit), warps 16-19 V (16-17 even tiles, 18-19 odd tiles);
        // thread r owns key row r of its tile.
        const bool conv_k = warp < 16;
        const uint32_t mysub = (uint32_t)(((warp - (conv_k ? 12 : 16)) >> 1) & 1);
        const int r = (int)threadIdx.x - 32 * (conv_k ? 12 : 16) - 64 * (int)mysub;   // 0 .. 63
        for (uint32_t t = mysub; t < n; t += 2) {
            if (conv_k) {
                const uint32_t pq = t >> 1, ks = pq % NK;
                if (!mbar_wait_bounded(&k8full[2 * ks + mysub], (pq / NK) & 1u)) break;
                const TileMeta m = kmeta[2 * ks + mysub];
                if (m.flags & kFirst) {
                    const uint32_t uq = (uint32_t)m.ord;            // this unit's index in the CTA
                    const uint32_t qb = uq & 1u;
                    if (!mbar_wait_bounded(&q_full[qb], (uq >> 1) & 1u)) break;
                    const uint32_t qa = smem_addr(smem + L::kQOff + qb * L::kQBytes);
                    for (int i = r; i < L::kQBytes / 16; i += 64) {
                        uint32_t v0, v1, v2, v3;
                        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                     : "=r"(v0), "=r"(v1), "=r"(v2), "=r"(v3) : "r"(qa + 16u * i));
                        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};"
                                     :: "r"(qa + 16u * i), "r"(bf16x2_to_f16x2(v0)), "r"(bf16x2_to_f16x2(v1)),
                                        "r"(bf16x2_to_f16x2(v2)), "r"(bf16x2_to_f16x2(v3))
                                     : "memory");
                    }
                    fence_proxy_async();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&q_conv[qb]);
                }
                if (m.nvalid > 0) {
                    const uint32_t base = smem_addr(smem + L::kKOff + ks * L::kKSlotBytes + mysub * kHalfBytes);
                    widen_rows(base + kTileBytes, base, m.nvalid, r);
                }
                fence_proxy_async();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&kfull[ks]);
                    if (mysub == 0u && t + 1 == n) mbar_arrive(&kfull[ks]);   // pair without tile 1
                }
            } else {
                const uint32_t vs = t % NV;
                if (!mbar_wait_bounded(&v8full[vs], (t / NV) & 1u)) break;
                const uint32_t base = smem_addr(smem + L::kVOff + vs * kTileBytes);
                widen_rows(base + kHalfBytes, base, kTileKeys, r);
                fence_proxy_async();
                __syncwarp();
                if (lane == 0) mbar_arrive(&vfull[vs]);
            }
        }
    } else if (warp >= 4 && warp < 12) {
        // =========================== softmax / epilogue warps ================================
        // warp 4 + 4 hh + q: TMEM lanes 32 q .. + 31 (key t of a step, head dim t of O^T) and the
        // 16 rows 16 hh .. + 15; two warps per scheduler
        const int q = warp & 3, hh = (warp - 4) >> 2;
        const int t = 32 * q + lane;
        const int row0 = 16 * hh;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const int nrows = a.rows_total;                  // <= 32 (one row block per unit)
        constexpr int RH = kTctRows / 2;
        float l_part[RH];
#pragma unroll
        for (int i = 0; i < RH; ++i) l_part[i] = 0.f;
        uint32_t sync_phase = 0, units = 0;
        int cur_unit = -1, Lpre = 0;
        bool alive = true;
        auto sm_rendezvous = [&]() -> bool {
            __syncwarp();
            if (lane == 0) mbar_arrive(sm_sync);
            const bool r_ok = mbar_wait_bounded(sm_sync, sync_phase);
            sync_phase ^= 1u;
            return r_ok;
        };
        // 16 values per lane, value i of row row0 + i: lane L ends with row row0 + (L & 15)
        // reduced over all 32 lanes (reduce-scatter over 16 lanes, then across the halves)
        auto rows16_reduce = [&](float (&v)[RH], bool is_max) -> float {
#pragma unroll
            for (int off = 8; off >= 1; off >>= 1) {
                const bool upper = (lane & off) != 0;
#pragma unroll
                for (int i = 0; i < off; ++i) {
                    const float send = upper ? v[i] : v[i + off];
                    const float keep = upper ? v[i + off] : v[i];
                    const float got = __shfl_xor_sync(0xffffffffu, send, off);
                    v[i] = is_max ? fmaxf(keep, got) : keep + got;
                }
            }
            const float o16 = __shfl_xor_sync(0xffffffffu, v[0], 16);
            return is_max ? fmaxf(v[0], o16) : v[0] + o16;
        };
        uint32_t step = 0;
        for (uint32_t pq = 0; pq < npairs && alive; ++pq) {
            int done_inc = 0;
            const int want_inc = (2 * pq + 1 < n) ? 3 : 1;
            while (done_inc != want_inc && alive) {
                const uint32_t sb = step % NSB, pb = step % kPB;
                if (!mbar_wait_bounded(&s_full[sb], (step / NSB) & 1u)) { alive = false; break; }
                tc::fence_after_sync();
                const StepMeta sm = smeta[sb];
                // scalar fields only (constant indices), so nothing of the step lives in local memory
                const bool inc0 = (sm.inc & 1) != 0, inc1 = (sm.inc & 2) != 0;
                const int f_unit = inc0 ? sm.tm[0].unit : sm.tm[1].unit;
                const int f_flags = inc0 ? sm.tm[0].flags : sm.tm[1].flags;
                const int f_Ltot = inc0 ? sm.tm[0].L_tot : sm.tm[1].L_tot;
                const int f_rb = inc0 ? sm.tm[0].rb : sm.tm[1].rb;
                const int f_b = inc0 ? sm.tm[0].b : sm.tm[1].b;
                const int l_flags = inc1 ? sm.tm[1].flags : sm.tm[0].flags;
                const int l_unit = inc1 ? sm.tm[1].unit : sm.tm[0].unit;
                const int l_rb = inc1 ? sm.tm[1].rb : sm.tm[0].rb;
                const int l_b = inc1 ? sm.tm[1].b : sm.tm[0].b;
                const int l_h = inc1 ? sm.tm[1].h : sm.tm[0].h;
                // ---- scores of key t for this warp's 16 rows --------------------------------
                uint32_t sr[RH];
                __syncwarp();
                tc::ld_32x32b_x16(tmem + lane_base + sb * (uint32_t)kTctRows + (uint32_t)row0, sr);
                tc::wait_ld();
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s_free[sb]);
                if (f_unit != cur_unit) {
                    // ---- a new unit: every warp is done with the previous unit's row state ---
                    if (!sm_rendezvous()) { alive = false; break; }
                    cur_unit = f_unit;
                    Lpre = f_Ltot - a.n_q;
                    if (warp == 4) {
                        const int R = f_rb * kRowsPerBlock + lane;
                        m_s[lane] = -INFINITY;
                        vis_s[lane] = step_visibility(a, f_b, R < a.rows_total ? R / a.G : 0);
                    }
#pragma unroll
                    for (int i = 0; i < RH; ++i) l_part[i] = 0.f;
                    if (!sm_rendezvous()) { alive = false; break; }
                }
                // ---- mask: the step's tiles, valid keys, rows, in-step visibility ------------
                const int sub = t >> 6, kk = t & 63;
                const int k_nvalid = sub ? sm.tm[1].nvalid : sm.tm[0].nvalid;
                const int k_pos0 = sub ? sm.tm[1].pos0 : sm.tm[0].pos0;
                const bool key_ok = (sub ? inc1 : inc0) && kk < k_nvalid;
                const int off = k_pos0 + kk - Lpre;              // >= 0: a key of this call's rows
                float x[RH];
                if (key_ok && off < 0) {
#pragma unroll
                    for (int i = 0; i < RH; ++i)
                        x[i] = row0 + i < nrows ? __uint_as_float(sr[i]) * a.scale_log2 : -INFINITY;
                } else {
#pragma unroll
                    for (int i = 0; i < RH; ++i) {
                        const bool ok = key_ok && row0 + i < nrows && off < 64 &&
                                        ((vis_s[row0 + i] >> (off & 63)) & 1ull);
                        x[i] = ok ? __uint_as_float(sr[i]) * a.scale_log2 : -INFINITY;
                    }
                }
                // ---- lazy maxima: the common step moves none ----------------------------------
                const float4* m4 = reinterpret_cast<const float4*>(m_s + row0);
                bool grow = false;
#pragma unroll
                for (int i = 0; i < RH / 4; ++i) {
                    const float4 v = m4[i];
                    grow |= (x[4 * i] > v.x + kRescaleThreshold) | (x[4 * i + 1] > v.y + kRescaleThreshold) |
                            (x[4 * i + 2] > v.z + kRescaleThreshold) | (x[4 * i + 3] > v.w + kRescaleThreshold);
                }
                grow = __any_sync(0xffffffffu, grow);
                // flags double-buffered by step parity: a warp can be at most one rendezvous ahead
                int* fl = flag_s + 8 * (step & 1u);
                if (lane == 0) fl[warp - 4] = grow ? 1 : 0;
                if (!sm_rendezvous()) { alive = false; break; }
                const bool any_grow = ((fl[0] | fl[1] | fl[2] | fl[3]) | (fl[4] | fl[5] | fl[6] | fl[7])) != 0;
                if (any_grow) {
                    // ---- new maxima: reduce over the lanes, combine the four lane quarters --------
                    float v[RH];
#pragma unroll
                    for (int i = 0; i < RH; ++i) v[i] = x[i];
                    const float rm = rows16_reduce(v, true);
                    if (lane < 16) red_s[q * kTctRows + row0 + lane] = rm;
                    if (!sm_rendezvous()) { alive = false; break; }
                    if (warp == 4) {
                        const float mo = m_s[lane];
                        float mn = mo;
#pragma unroll
                        for (int w = 0; w < 4; ++w) mn = fmaxf(mn, red_s[w * kTctRows + lane]);
                        alpha_s[lane] = (mo == -INFINITY || mn == -INFINITY) ? (mo == -INFINITY ? 0.f : 1.f)
                                                                             : fast_exp2(mo - mn);
                        m_s[lane] = mn;
                    }
                    if (!sm_rendezvous()) { alive = false; break; }
                    const float4* a4 = reinterpret_cast<const float4*>(alpha_s + row0);
#pragma unroll
                    for (int i = 0; i < RH / 4; ++i) {
                        const float4 av = a4[i];
                        l_part[4 * i] *= av.x; l_part[4 * i + 1] *= av.y;
                        l_part[4 * i + 2] *= av.z; l_part[4 * i + 3] *= av.w;
                    }
                    // O^T lane t, this warp's 16 columns, once the unit's previous PV is done
                    if (!(f_flags & kFirst) && step >= 1u) {
                        const uint32_t pp = (step - 1u) % kPB;
                        if (!mbar_wait_bounded(&p_free[pp], ((step - 1u) / kPB) & 1u)) { alive = false; break; }
                        tc::fence_after_sync();
                        const uint32_t ocol = TCOL::kO + (uint32_t)kTctRows * (units & 1u) + (uint32_t)row0;
                        uint32_t o[16];
                        __syncwarp();
                        tc::ld_32x32b_x16(tmem + lane_base + ocol, o);
                        tc::wait_ld();
#pragma unroll
                        for (int j = 0; j < 16; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha_s[row0 + j]);
                        tc::st_32x32b_x16(tmem + lane_base + ocol, o);
                        tc::wait_st();
                    }
                }
                // ---- P^T to the step's P buffer (free once the PV of step - kPB is done) -------
                if (step >= (uint32_t)kPB && !mbar_wait_bounded(&p_free[pb], ((step / kPB) & 1u) ^ 1u)) {
                    alive = false;
                    break;
                }
                {
                    // plain shared stores (no asm barrier between rows), so the compiler can overlap
                    // the rows' exponentials and stores
                    float mrow[RH];
#pragma unroll
                    for (int i = 0; i < RH / 4; ++i) {
                        const float4 v4 = m4[i];
                        mrow[4 * i] = v4.x; mrow[4 * i + 1] = v4.y; mrow[4 * i + 2] = v4.z; mrow[4 * i + 3] = v4.w;
                    }
                    uint16_t* prow = reinterpret_cast<uint16_t*>(smem + L::kPOff + pb * L::kPBytes +
                                                                 sub * (kTctRows * 128));
                    const int colb = kk * 2;
#pragma unroll
                    for (int i = 0; i < RH; ++i) {
                        const int rr = row0 + i;
                        const float m_use = (mrow[i] == -INFINITY) ? 0.f : mrow[i];
                        const float p = fast_exp2(x[i] - m_use);
                        uint16_t h;
                        float pr;
                        if (KV8) {
                            const __half hp = __float2half_rn(p);
                            h = __half_as_ushort(hp);
                            pr = __half2float(hp);
                        } else {
                            const __nv_bfloat16 bp = __float2bfloat16_rn(p);
                            h = __bfloat16_as_ushort(bp);
                            pr = __bfloat162float(bp);
                        }
                        l_part[i] += pr;
                        prow[(rr * 128 + ((((colb >> 4) ^ (rr & 7)) << 4) | (colb & 15))) >> 1] = h;
                    }
                }
                // V rows past the valid keys may hold anything (NaN tails): zero them before PV
#pragma unroll
                for (int s2 = 0; s2 < 2; ++s2) {
                    const TileMeta& tv = sm.tm[s2];
                    if (!((sm.inc >> s2) & 1) || tv.nvalid <= 0 || tv.nvalid >= kTileKeys) continue;
                    const uint32_t tix = (uint32_t)sm.it0 + (uint32_t)s2;
                    const uint32_t vs = tix % NV;
                    if (!mbar_wait_bounded(&vfull[vs], (tix / NV) & 1u)) { alive = false; break; }
                    uint8_t* vt = smem + L::kVOff + vs * kTileBytes;
                    const int nrow = kTileKeys - tv.nvalid;
                    for (int idx = t + 128 * hh; idx < nrow * 16; idx += 256) {
                        const int rv = tv.nvalid + idx / 16, c16 = idx % 16;
                        *reinterpret_cast<uint4*>(vt + (c16 >> 3) * kHalfBytes + rv * 128 + (c16 & 7) * 16) =
                            make_uint4(0u, 0u, 0u, 0u);
                    }
                }
                if (!alive) break;
                if (warp == 4 && lane == 0) pmeta[pb] = sm;
                fence_proxy_async();
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[pb]);
                // ---- unit end: row sums, O^T readout, the rows or the partials ---------------
                if (l_flags & kLast) {
                    if (!mbar_wait_bounded(&p_free[pb], (step / kPB) & 1u)) { alive = false; break; }
                    tc::fence_after_sync();
                    float v[RH];
#pragma unroll
                    for (int i = 0; i < RH; ++i) v[i] = l_part[i];
                    const float rs = rows16_reduce(v, false);
                    if (lane < 16) red_s[q * kTctRows + row0 + lane] = rs;
                    if (!sm_rendezvous()) { alive = false; break; }
                    const uint32_t ocol = TCOL::kO + (uint32_t)kTctRows * (units & 1u) + (uint32_t)row0;
                    const int slot = (int)blockIdx.x + l_unit;
                    uint32_t o[16];
                    __syncwarp();
                    tc::ld_32x32b_x16(tmem + lane_base + ocol, o);
                    tc::wait_ld();
#pragma unroll
                    for (int j = 0; j < RH; ++j) {
                        const int i = row0 + j;
                        if (i >= nrows) continue;
                        const float l = (red_s[i] + red_s[kTctRows + i]) + (red_s[2 * kTctRows + i] + red_s[3 * kTctRows + i]);
                        const float val = l > 0.f ? __uint_as_float(o[j]) * (a.v_scale / l) : 0.f;
                        const int R = l_rb * kRowsPerBlock + i;
                        if (l_flags & kWhole) {
                            const int qi = R / a.G, g = R - (R / a.G) * a.G;
                            const size_t orow = ((size_t)l_b * a.n_q + qi) * a.Hq + (size_t)l_h * a.G + g;
                            a.out[orow * kD + t] = __float2bfloat16_rn(val);
                        } else {
                            a.ws_o[((size_t)slot * a.rows_blk + i) * kD + t] = val;
                        }
                    }
                    if (q == 0 && lane < 16 && row0 + lane < nrows) {
                        const int i = row0 + lane;
                        const float l = (red_s[i] + red_s[kTctRows + i]) + (red_s[2 * kTctRows + i] + red_s[3 * kTctRows + i]);
                        const float lse2 = l > 0.f ? m_s[i] + __log2f(l) : -INFINITY;
                        const int R = l_rb * kRowsPerBlock + i;
                        if (l_flags & kWhole) {
                            if (a.lse != nullptr) {
                                const int qi = R / a.G, g = R - (R / a.G) * a.G;
                                a.lse[((size_t)l_b * a.n_q + qi) * a.Hq + (size_t)l_h * a.G + g] = lse2 * kLn2;
                            }
                        } else {
                            a.ws_lse[(size_t)slot * a.rows_blk + i] = lse2;
                        }
                    }
                    tc::fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&o_free[units & 1u]);
                    ++units;
                }
                done_inc |= sm.inc;
                ++step;
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
