// attn_kernels.cuh -- split-KV decode/verify attention for sm_100a.
//
// One kernel template serves the three attention calls of the Windowed-MTP decode step
// (Windowed-MTP, arXiv 2607.21535; Pith verdict, pith_extraction.key_machinery):
//   * draft_attn_window: keys = the attention sink plus the recent window, read from the ring as
//     at most three contiguous slot ranges (never a dense mask);
//   * draft_attn_full:   keys = the whole paged KV cache (the native draft it replaces);
//   * verify_attn:       keys = the paged prefix plus the step's nodes (chain-causal or tree).
//
// Work decomposition.  A "unit" is (request b, kv head h, row block rb); its rows are the
// n_q * G query rows (query i, packed GQA head g: row = i * G + g) of that kv head, 64 per row
// block.  Its keys are cut into tiles of 64 keys (one page, or a piece of one ring range).  The
// tiles of all units form one flat sequence of T tiles; CTA c of the P_eff working CTAs takes the
// tiles [floor(c T / P_eff), floor((c+1) T / P_eff)), so every CTA streams the same number of
// bytes whatever the lengths and ring wrap (stream-K).  A unit entirely inside one CTA is
// finished there; otherwise each CTA writes an (o, lse) partial to workspace slot c + u and
// lse_merge_kernel combines them (slots are unique: c' > c implies u' >= u).
//
// Inside a CTA: one producer warp streams K/V tiles with TMA (two 64x64 bf16 boxes per tensor,
// 128-byte swizzle) through an NSTAGE ring of mbarrier-guarded stages; NMT x NKG consumer warps
// each own one 16-row m-tile and 64/NKG keys of every tile and run QK^T and PV on the tensor
// cores (mma.sync m16n8k16 bf16, fp32 accumulate) with an online base-2 softmax.
#pragma once

#include "device_common.cuh"

namespace wmtp {

constexpr int kD = 128;
constexpr int kTileKeys = 64;
constexpr int kRowsPerBlock = 64;
constexpr int kHalfBytes = kTileKeys * 64 * 2;      // one 64x64 bf16 box: 8 KiB
constexpr int kTileBytes = 2 * kHalfBytes;          // K or V tile: 16 KiB
constexpr int kStageBytes = 2 * kTileBytes;         // K + V: 32 KiB
constexpr int kTileBytes8 = kTileKeys * kD;         // fp8 K or V tile: one 128x64 byte box, 8 KiB
constexpr int kStageBytes8 = 2 * kTileBytes8;       // fp8 K + V: 16 KiB
constexpr int kMaxBatch = 256;
constexpr int kClusterMax = 16;                   // largest window cluster (non-portable size)
constexpr float kLn2 = 0.693147180559945309f;

enum SourceKind : int { kSrcPaged = 0, kSrcRing = 1 };

struct AttnArgs {
    const __nv_bfloat16* q;      // [B, n_q, Hq, D]
    __nv_bfloat16* out;          // [B, n_q, Hq, D]
    float* lse;                  // [B, n_q, Hq] or null
    float* ws_o;                 // [slots][rows_blk][D]   normalised partial outputs
    float* ws_lse;               // [slots][rows_blk]      base-2 partial log-sum-exp
    int B, n_q, Hq, Hkv, G, n_rb;
    int rows_total;              // n_q * G
    int rows_blk;                // rows per unit (min(64, rows_total)): the workspace slot height
    float scale_log2;            // sm_scale * log2(e) (fp8 KV: times the key scale)
    float v_scale;               // output multiplier (fp8 KV: the value scale; else 1)
    const int* tree_parent;      // [B, n_q] or null (chain / causal)
    // paged source
    const int* page_table;       // [B, max_pages]
    const int* kv_len;           // [B]
    int max_pages, num_pages;
    // ring source
    const long long* ring_len;   // [B]
    int n_sink, window, capacity;
    // plan
    int min_tiles_per_cta;
    // fused ring append (cluster window kernel only): positions [L_old, L_old + n_new) of each
    // request, rows of k_new / v_new [B, n_new, Hkv, D], are written to their ring slots (and
    // into the shared-memory tiles that hold them); the last CTA to have read ring_len advances
    // it by n_new.  n_new = 0: no append.
    const uint4* k_new;
    const uint4* v_new;
    uint4* ring_kw;              // ring K/V base (the same arrays the tensor maps read)
    uint4* ring_vw;
    long long* ring_len_w;       // ring_len, written once per call by the last CTA
    unsigned int* ticket;        // workspace word, zero between calls
    int n_new;
};

// Per-stage tile description, written by the producer before the stage's barrier completes.
struct TileMeta {
    int b, h, rb, unit;
    int pos0;       // logical position of the tile's row 0
    int nvalid;     // rows [0, nvalid) are keys of this unit; 0 = skipped tile
    int L_tot;      // request length (keys) including this call's n_q positions
    int flags;      // kFirst | kLast | kWhole
    int ord;        // units this CTA finished before this tile's unit (tcgen05 kernel only)
    int slot0;      // ring slot of row 0 (ring source)
};
enum : int { kFirst = 1, kLast = 2, kWhole = 4 };

// ---------------------------------------------------------------------------------------------
// Key ranges of a request.
// Ring: sink slots [0, ns) hold positions [0, ns); the recent window positions [r0, L) sit in
// ring slots starting at slot(r0) and wrap at most once (slot(p) = n_sink + (p - n_sink) mod
// (C - n_sink)).  Paged: one range of L keys.
struct Ranges {
    int n;               // number of ranges (<= 3)
    int slot0[3], pos0[3], len[3];
};

__device__ __forceinline__ Ranges ring_ranges(long long L_ll, int s, int W, int C) {
    Ranges r;
    r.n = 0;
    const int L = (int)L_ll;
    const int ns = L < s ? L : s;
    if (ns > 0) { r.slot0[r.n] = 0; r.pos0[r.n] = 0; r.len[r.n] = ns; ++r.n; }
    if (L > s) {
        const int r0 = (L - W) > s ? (L - W) : s;
        const int n = L - r0;
        const int a = s + (r0 - s) % (C - s);
        const int first = n < (C - a) ? n : (C - a);
        r.slot0[r.n] = a; r.pos0[r.n] = r0; r.len[r.n] = first; ++r.n;
        if (n - first > 0) { r.slot0[r.n] = s; r.pos0[r.n] = r0 + first; r.len[r.n] = n - first; ++r.n; }
    }
    return r;
}

template <int SRC>
__device__ __forceinline__ int request_len(const AttnArgs& a, int b) {
    long long L = (SRC == kSrcPaged) ? (long long)a.kv_len[b] : a.ring_len[b];
    if (L < 0) L = 0;
    if (L > 0x7fffffffll) L = 0x7fffffffll;
    return (int)L;
}

template <int SRC>
__device__ __forceinline__ int request_tiles(const AttnArgs& a, int L) {
    if (SRC == kSrcPaged) return (L + kTileKeys - 1) / kTileKeys;
    Ranges r = ring_ranges(L, a.n_sink, a.window, a.capacity);
    int t = 0;
    for (int k = 0; k < r.n; ++k) t += (r.len[k] + kTileKeys - 1) / kTileKeys;
    return t;
}

__device__ __forceinline__ long long cta_begin(long long c, long long T, long long P) {
    return c * T / P;
}

__device__ __forceinline__ int plan_ctas(long long T, int P_launch, int min_tiles) {
    long long want = (T + min_tiles - 1) / min_tiles;
    if (want < 1) want = 1;
    return (int)(want < P_launch ? want : P_launch);
}

// CTA whose tile range contains tile t (largest c with begin(c) <= t).
__device__ __forceinline__ int cta_of_tile(long long t, long long T, int P) {
    long long c = ((t + 1) * P + T - 1) / T - 1;
    return (int)c;
}

// ---------------------------------------------------------------------------------------------
// Walks a CTA's flat tile range in order and describes each tile: its unit, key positions,
// valid rows, first/last/whole flags, and the TMA row/block coordinates of its K/V boxes.
template <int SRC>
struct TileWalker {
    int b = 0;
    long long b_start = 0, per_b = 0;
    // position of the last described tile, for the O(1) step to the next one (producers walk
    // their ranges in order; a division-free step keeps the producer loop short)
    long long cur_t = -1;
    int nt_b = 0, unit_in_b = 0, tile = 0;
    // page id of the next tile, loaded one step ahead so its latency hides behind this step
    int pf_b = -1, pf_tile = -1, pf_page = -1;

    __device__ __forceinline__ void init(const AttnArgs& a, const int* plan_tiles) {
        b = 0;
        b_start = 0;
        per_b = (long long)plan_tiles[0] * a.Hkv * a.n_rb;
        cur_t = -1;
    }

    __device__ __forceinline__ void describe(const AttnArgs& a, const int* plan_tiles,
                                             const int* plan_len, long long t, long long t_begin,
                                             long long t_end, TileMeta& m, int& ty, int& tz) {
        const int units_b = a.Hkv * a.n_rb;
        if (cur_t >= 0 && t == cur_t + 1) {
            if (++tile == nt_b) {
                tile = 0;
                if (++unit_in_b == units_b) {
                    unit_in_b = 0;
                    b_start += per_b;
                    do {
                        ++b;
                        per_b = (long long)plan_tiles[b] * units_b;
                    } while (per_b == 0);              // t < total tiles: some later request has tiles
                    nt_b = plan_tiles[b];
                }
            }
        } else {
            while (t >= b_start + per_b) {
                b_start += per_b;
                ++b;
                per_b = (long long)plan_tiles[b] * units_b;
            }
            nt_b = plan_tiles[b];
            const long long off = t - b_start;
            unit_in_b = (int)(off / nt_b);
            tile = (int)(off - (long long)unit_in_b * nt_b);
        }
        cur_t = t;
        const int h = unit_in_b / a.n_rb;
        const int rb = unit_in_b - h * a.n_rb;
        const long long u_start = b_start + (long long)unit_in_b * nt_b;
        m.b = b; m.h = h; m.rb = rb;
        m.unit = (b * a.Hkv + h) * a.n_rb + rb;
        m.L_tot = plan_len[b];
        m.flags = ((t == t_begin || tile == 0) ? kFirst : 0) |
                  ((t == t_end - 1 || tile == nt_b - 1) ? kLast : 0) |
                  ((u_start >= t_begin && u_start + nt_b <= t_end) ? kWhole : 0);
        if (SRC == kSrcPaged) {
            int page;
            if (pf_b == b && pf_tile == tile) {
                page = pf_page;
            } else {
                page = tile < a.max_pages ? a.page_table[(size_t)b * a.max_pages + tile] : -1;
            }
            // next tile of this request: the following tile of this unit, or tile 0 of the next
            // unit (the same pages, another kv head or row block)
            const int nxt = (tile + 1 < nt_b) ? tile + 1 : 0;
            pf_b = b;
            pf_tile = nxt;
            pf_page = nxt < a.max_pages ? a.page_table[(size_t)b * a.max_pages + nxt] : -1;
            m.pos0 = tile * kTileKeys;
            const int rem = m.L_tot - m.pos0;
            m.nvalid = rem < kTileKeys ? rem : kTileKeys;
            if (page < 0 || page >= a.num_pages) {
                flag_status(kStatusDeviceIndex);
                m.nvalid = 0;
            }
            ty = 0;
            tz = page * a.Hkv + h;
        } else {
            Ranges r = ring_ranges(m.L_tot, a.n_sink, a.window, a.capacity);
            int tl = tile, k = 0;
            for (; k < r.n; ++k) {
                const int ntk = (r.len[k] + kTileKeys - 1) / kTileKeys;
                if (tl < ntk) break;
                tl -= ntk;
            }
            if (k >= r.n) k = r.n - 1;   // unreachable: tile < request_tiles
            const int rem = r.len[k] - tl * kTileKeys;
            m.pos0 = r.pos0[k] + tl * kTileKeys;
            m.nvalid = rem < kTileKeys ? rem : kTileKeys;
            ty = r.slot0[k] + tl * kTileKeys;
            tz = b * a.Hkv + h;
            m.slot0 = ty;
        }
    }
};

// Before the PDL wait (paged source, one thread): this CTA's first n tiles, planned from the
// lengths and page table as they read at that moment, are prefetched into L2, so that their DRAM
// latency overlaps the predecessor's tail.  The predecessor may still be writing those inputs; a
// stale read only warms the wrong lines (nothing is loaded into shared memory or used), and every
// read stays inside the table and every prefetch inside a valid page.  Requests beyond 16 skip it.
__device__ __forceinline__ void prefetch_first_tiles(const AttnArgs& a, const CUtensorMap* kmap,
                                                     const CUtensorMap* vmap, bool kv8, int n) {
    if (a.B > 16) return;
    const int units_b = a.Hkv * a.n_rb;
    long long T = 0;
    for (int b = 0; b < a.B; ++b) {
        const int L = a.kv_len[b];
        T += (long long)((L > 0 ? L : 0) + kTileKeys - 1) / kTileKeys * units_b;
    }
    const int peff = plan_ctas(T, gridDim.x, a.min_tiles_per_cta);
    const long long c = blockIdx.x;
    if (c >= peff) return;
    long long t = cta_begin(c, T, peff);
    const long long t1 = cta_begin(c + 1, T, peff);
    for (int k = 0; k < n && t < t1; ++k, ++t) {
        long long b_start = 0;
        int b = 0, nt = 0;
        for (; b < a.B; ++b) {
            const int L = a.kv_len[b];
            nt = ((L > 0 ? L : 0) + kTileKeys - 1) / kTileKeys;
            if (t < b_start + (long long)nt * units_b) break;
            b_start += (long long)nt * units_b;
        }
        if (b >= a.B || nt == 0) return;
        const int unit_in_b = (int)((t - b_start) / nt);
        const int tile = (int)((t - b_start) - (long long)unit_in_b * nt);
        if (tile >= a.max_pages) return;
        const int page = a.page_table[(size_t)b * a.max_pages + tile];
        if (page < 0 || page >= a.num_pages) return;
        const int tz = page * a.Hkv + unit_in_b / a.n_rb;
        tma_prefetch_3d(kmap, 0, 0, tz);
        tma_prefetch_3d(vmap, 0, 0, tz);
        if (!kv8) {
            tma_prefetch_3d(kmap, 64, 0, tz);
            tma_prefetch_3d(vmap, 64, 0, tz);
        }
    }
}

// The unit of flat tile t (b, h, rb, unit and L_tot only; no page-table read), so that the
// consumers can start their first unit (its Q loads) while the first tile is still in flight.
__device__ __forceinline__ void unit_of_tile(const AttnArgs& a, const int* plan_tiles,
                                             const int* plan_len, long long t, TileMeta& m) {
    const int units_b = a.Hkv * a.n_rb;
    int b = 0;
    long long b_start = 0, per_b = (long long)plan_tiles[0] * units_b;
    while (t >= b_start + per_b) {
        b_start += per_b;
        ++b;
        per_b = (long long)plan_tiles[b] * units_b;
    }
    const int unit_in_b = (int)((t - b_start) / plan_tiles[b]);
    m.b = b;
    m.h = unit_in_b / a.n_rb;
    m.rb = unit_in_b - m.h * a.n_rb;
    m.unit = (b * a.Hkv + m.h) * a.n_rb + m.rb;
    m.L_tot = plan_len[b];
}

// ---------------------------------------------------------------------------------------------
// Cluster window mode: one unit per cluster of CL_size CTAs (grid (CL_size, units)), CTA r of
// the cluster takes the unit's tiles [floor(r nt / CL_size), floor((r + 1) nt / CL_size)).  The
// ring's tiles of one unit: its at most three slot ranges cut into 64-key tiles.
struct RingUnitWalker {
    Ranges r;
    int b, h, rb, unit, L_tot;

    __device__ __forceinline__ void describe(const AttnArgs& a, int tile, int t_begin, int t_end,
                                             TileMeta& m, int& ty, int& tz) const {
        int tl = tile, k = 0;
        for (; k < r.n; ++k) {
            const int ntk = (r.len[k] + kTileKeys - 1) / kTileKeys;
            if (tl < ntk) break;
            tl -= ntk;
        }
        if (k >= r.n) k = r.n - 1;   // unreachable: tile < tiles of the unit
        const int rem = r.len[k] - tl * kTileKeys;
        m.b = b; m.h = h; m.rb = rb; m.unit = unit;
        m.L_tot = L_tot;
        m.pos0 = r.pos0[k] + tl * kTileKeys;
        m.nvalid = rem < kTileKeys ? rem : kTileKeys;
        m.flags = (tile == t_begin ? kFirst : 0) | (tile == t_end - 1 ? kLast : 0);
        m.ord = 0;
        ty = r.slot0[k] + tl * kTileKeys;
        tz = b * a.Hkv + h;
        m.slot0 = ty;
    }
};

// Visibility bitmask of the step's in-call keys for query i: bit j set when the key at
// position L_tot - n_q + j is visible (chain: j <= i; tree: j on i's root path).
__device__ __forceinline__ unsigned long long step_visibility(const AttnArgs& a, int b, int i) {
    if (a.tree_parent != nullptr) {
        unsigned long long msk = 0ull;
        int cur = i;
        for (int k = 0; k < 64 && cur >= 0 && cur < a.n_q; ++k) {
            msk |= 1ull << cur;
            const int nxt = a.tree_parent[(size_t)b * a.n_q + cur];
            cur = (nxt < cur) ? nxt : -1;
        }
        return msk;
    }
    return (i >= 63) ? ~0ull : ((1ull << (i + 1)) - 1ull);
}

// ---------------------------------------------------------------------------------------------
// Shared-memory layout (dynamic; stage buffers 1024-byte aligned for the 128-byte swizzle).
// QS (fp8 KV only): the unit's Q rows are kept in shared memory as fp16, in a space the unit-end
// key-group merge reuses one m-tile at a time.
// MS: the key-group merge at a unit's end goes through the stage of the unit's last tile (held
// until the merge is done) instead of a space of its own, which leaves room for a third stage in
// two CTAs per SM.
template <int NMT, int NKG, int NSTAGE, bool KV8 = false, bool QS = false, bool MS = false>
struct SmemLayout {
    static constexpr int kStagesBytes = NSTAGE * (KV8 ? kStageBytes8 : kStageBytes);
    static constexpr int kMergeStride = kD + 4;                      // floats per merge row
    static constexpr int kMergeMT = QS ? 1 : NMT;                    // m-tiles merged at once
    static constexpr int kMergeFloats = (NKG - 1) * kMergeMT * 16 * kMergeStride;
    static constexpr int kMergeMLFloats = (NKG - 1) * kMergeMT * 16 * 2;
    static_assert(!MS || (!QS && (kMergeFloats + kMergeMLFloats) * 4 <= (KV8 ? kStageBytes8 : kStageBytes)),
                  "the merge rows fit one stage");
    // fp16 Q row: 128 dims + 32 bytes of padding, so the 8-byte fragment reads of four rows in a
    // half-warp start 8 banks apart
    static constexpr int kQStride = 2 * kD + 32;
    static constexpr int kQBytes = QS ? NMT * 16 * kQStride : 0;
    static constexpr int kMergeOff = kStagesBytes;
    static constexpr int kQOff = kMergeOff;                          // QS: aliases the merge rows
    static constexpr int kMergeBytes = MS ? kQBytes : ((kQBytes > kMergeFloats * 4) ? kQBytes : kMergeFloats * 4);
    static constexpr int kMergeMLOff = kMergeOff + kMergeBytes;
    static constexpr int kBarOff = kMergeMLOff + (MS ? 0 : kMergeMLFloats * 4);
    static constexpr int kMetaOff = kBarOff + (2 * NSTAGE + 1) * 8;
    static constexpr int kPlanOff = kMetaOff + NSTAGE * (int)sizeof(TileMeta);
    static constexpr int kPlanBytes = 2 * kMaxBatch * 4;            // tiles per request, length
    static constexpr int kTotal = kPlanOff + kPlanBytes;
    static constexpr int kAlloc = kTotal + 1024;                     // slack for base alignment
    // cluster window mode: the CTA's (o, lse) partial of its unit lives in the stage space once
    // the pipeline has drained: [NMT * 16 rows][128] fp32 normalised outputs, then the rows'
    // base-2 LSEs
    static constexpr int kPartOff = 0;
    static constexpr int kPartLseOff = NMT * 16 * kD * 4;
    static_assert(kPartLseOff + NMT * 16 * 4 <= kStagesBytes, "partial fits the stage space");
};

// Swizzled shared address of 16-byte chunk `chunk` (0..15) of key row `row` in a K/V tile
// stored as two 64x64 boxes with the TMA 128-byte swizzle (chunk' = chunk ^ (row & 7)).
__device__ __forceinline__ uint32_t tile_chunk_addr(uint32_t base, int row, int chunk) {
    return base + (uint32_t)((chunk >> 3) * kHalfBytes + row * 128 + (((chunk & 7) ^ (row & 7)) << 4));
}

// Same for an fp8 tile: one 128-byte row per key, 16-byte chunks 0..7 swizzled the same way.
__device__ __forceinline__ uint32_t tile8_chunk_addr(uint32_t base, int row, int chunk) {
    return base + (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// ---------------------------------------------------------------------------------------------
// Cluster window mode, end of the kernel: merges the cluster's per-CTA partials of its unit
// through distributed shared memory.  Every thread of the CTA calls it exactly once.  CTA `me`
// takes the unit's rows me, me + size, ...; one warp per row: lane k reads rank k's LSE (ranks
// without tiles hold no partial), then lane l sums head dims 4 l .. 4 l + 3 over the ranks with
// one 16-byte remote load per rank.  The second cluster barrier keeps every CTA's shared memory
// alive until its siblings have read it.
template <int NMT, int NKG, int NSTAGE, bool KV8, bool QS>
__device__ __forceinline__ void cluster_merge_rows(const AttnArgs& a, uint8_t* smem,
                                                   const RingUnitWalker& wk, int nt, int warp,
                                                   int lane) {
    using L = SmemLayout<NMT, NKG, NSTAGE, KV8, QS>;
    constexpr int kWarps = NMT * NKG + 1;
    cluster_sync_all();
    if (warp == 0 && lane == 0) WMTP_TRACE_AT(29);
    const int cs = (int)gridDim.x, me = (int)blockIdx.x;
    const int rows_u = min(kRowsPerBlock, a.rows_total - wk.rb * kRowsPerBlock);
    const uint32_t part = smem_addr(smem + L::kPartOff);
    const uint32_t plse = smem_addr(smem + L::kPartLseOff);
    const bool has = lane < cs && (long long)(lane + 1) * nt / cs > (long long)lane * nt / cs;
    const uint32_t has_mask = __ballot_sync(0xffffffffu, has);     // ranks holding a partial
    for (int rr = me + warp * cs; rr < rows_u; rr += kWarps * cs) {
        // one round of remote loads: rank `lane`'s LSE and this lane's four head dims of every
        // rank's partial are all in flight at once (a dependent round per step would cost one
        // distributed-shared-memory round trip each)
        float x = -INFINITY;
        if (has) x = ld_dsmem_f32(map_shared_rank(plse + 4u * rr, lane));
        const uint32_t po = part + 4u * (uint32_t)(rr * kD + 4 * lane);
        float4 v[kClusterMax];
#pragma unroll
        for (int k = 0; k < kClusterMax; ++k)
            v[k] = ((has_mask >> k) & 1u) ? ld_dsmem_v4(map_shared_rank(po, (uint32_t)k))
                                          : make_float4(0.f, 0.f, 0.f, 0.f);
        float mx = x;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const float w = (has && mx != -INFINITY) ? exp2f(x - mx) : 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        float wsum = 0.f;
#pragma unroll
        for (int k = 0; k < kClusterMax; ++k) {
            const float wk = __shfl_sync(0xffffffffu, w, k);
            if (wk > 0.f) {
                acc.x += wk * v[k].x; acc.y += wk * v[k].y; acc.z += wk * v[k].z; acc.w += wk * v[k].w;
                wsum += wk;
            }
        }
        const int R = wk.rb * kRowsPerBlock + rr;
        const int i = R / a.G, g = R - (R / a.G) * a.G;
        const size_t orow = ((size_t)wk.b * a.n_q + i) * a.Hq + (size_t)wk.h * a.G + g;
        const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
        uint2 pk;
        pk.x = pack_bf16x2(acc.x * inv, acc.y * inv);
        pk.y = pack_bf16x2(acc.z * inv, acc.w * inv);
        *reinterpret_cast<uint2*>(a.out + orow * kD + 4 * lane) = pk;
        if (a.lse != nullptr && lane == 0) a.lse[orow] = wsum > 0.f ? (mx + log2f(wsum)) * kLn2 : -INFINITY;
    }
    if (warp == 0 && lane == 0) WMTP_TRACE_AT(30);
    __syncwarp();
    cluster_sync_all();
}

// ---------------------------------------------------------------------------------------------
// KV8 = true: K and V are fp8 (E4M3) codes, one 128-byte row per key and head, scaled by the
// key and value scales (the key scale folded into scale_log2).  The tiles stream at half the
// bytes; consumers widen them to fp16 in registers (exact) and run fp16 MMAs, with Q widened to
// fp16 as well.  QK^T: ldmatrix on the fp8 tile hands each thread four consecutive dims of one
// key, so the MMA's k index is permuted consistently in Q (loaded in the same order) and K.
// PV: the widened V fragments are transposed in registers (movmatrix), which permutes the
// output's head dims in a fixed way that the final store undoes.
//
// QS = true (fp8 only) keeps the unit's Q in shared memory as fp16 instead of in registers: each
// A fragment is read per k-step, the kernel fits in 128 registers, and three CTAs share an SM
// (the fp8 kernel is bound by per-warp dependency chains, so more warps per SM is what helps).
//
// CL = true (ring source only): the cluster window kernel.  Grid (cluster size, units), one unit
// per cluster; each CTA streams its share of the unit's tiles, keeps its (o, lse) partial in
// shared memory, and the cluster merges the partials through distributed shared memory (CTA r
// merges rows r, r + size, ...), so the call is one launch with no workspace partials.  With
// a.n_new > 0 the call also appends the request's new draft rows: the consumer warps that own a
// new row's key slot copy it from k_new / v_new into the tile (after the TMA landed) and into
// the ring, and the last CTA to have read ring_len advances it.
// Fused append: every CTA counts in once it has read ring_len; the last one to count in advances
// ring_len by n_new for every request and clears the ticket for the next call.
__device__ __forceinline__ void fused_append_ticket(const AttnArgs& a) {
    __threadfence();
    const unsigned int total = gridDim.x * gridDim.y;
    if (atomicAdd(a.ticket, 1u) == total - 1u) {
        __threadfence();
        for (int b = 0; b < a.B; ++b) a.ring_len_w[b] = a.ring_len_w[b] + a.n_new;
        *a.ticket = 0u;
        __threadfence();
    }
}

template <int SRC, int NMT, int NKG, int NSTAGE, int MINB, bool KV8 = false, bool QS = false,
          bool CL = false, bool MS = false>
__global__ void __launch_bounds__((NMT * NKG + 1) * 32, MINB)
attn_split_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                  const AttnArgs a) {
    static_assert(!(MS && CL), "the cluster kernel keeps its merge space");
    using L = SmemLayout<NMT, NKG, NSTAGE, KV8, QS, MS>;
    static_assert(!QS || KV8, "shared-memory Q is an fp8-KV layout");
    static_assert(!CL || SRC == kSrcRing, "the cluster kernel reads the ring");
    constexpr int kStage = KV8 ? kStageBytes8 : kStageBytes;
    constexpr int NWC = NMT * NKG;            // consumer warps
    constexpr int KPW = kTileKeys / NKG;      // keys per consumer warp per tile
    constexpr int NT = KPW / 8;               // S n-tiles per warp
    static_assert(KPW % 16 == 0, "keys per warp must be a multiple of 16");

    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base for the 128-byte swizzle, by pointer arithmetic on the shared array
    // (an integer round trip would make every access through it a generic one)
    uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    float* merge_o = reinterpret_cast<float*>(smem + L::kMergeOff);
    float* merge_ml = reinterpret_cast<float*>(smem + L::kMergeMLOff);
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
    uint64_t* empty_bar = full_bar + NSTAGE;
    uint64_t* sync_bar = full_bar + 2 * NSTAGE;   // consumer-warp rendezvous at unit ends
    TileMeta* meta = reinterpret_cast<TileMeta*>(smem + L::kMetaOff);
    int* plan_tiles = reinterpret_cast<int*>(smem + L::kPlanOff);
    int* plan_len = plan_tiles + kMaxBatch;
    __shared__ long long s_range[2];          // this CTA's [t_begin, t_end)
    __shared__ int s_peff;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) WMTP_TRACE_AT(0);
    uint64_t pol = 0;                          // the producer's L2 policy for the KV stream
    if (warp == NWC && lane == 0) {
        prefetch_tensormap(&kmap);
        prefetch_tensormap(&vmap);
        pol = l2_evict_first_policy();
        if (!CL && SRC == kSrcPaged) prefetch_first_tiles(a, &kmap, &vmap, KV8, NSTAGE);
    }
    // the successor may launch once this kernel's predecessor is done (so it may read, before
    // its own wait, inputs this kernel does not write: the LSE merge reads the lengths early)
    pdl_wait();
    pdl_launch_dependents();
    if (threadIdx.x == 0) WMTP_TRACE_AT(1);

    __shared__ RingUnitWalker s_walk;          // cluster mode: this CTA's unit
    // ---- plan: lengths -> tiles per request -> this CTA's tile range ------------------------
    if (CL) {
        if (warp == NWC && lane == 0) {
            const int u = blockIdx.y;
            RingUnitWalker wk;
            wk.rb = u % a.n_rb;
            wk.h = (u / a.n_rb) % a.Hkv;
            wk.b = u / (a.n_rb * a.Hkv);
            wk.unit = u;
            const long long L_old = a.ring_len[wk.b];
            long long Lt = L_old + a.n_new;
            if (Lt < 0) Lt = 0;
            if (Lt > 0x7fffffffll) Lt = 0x7fffffffll;
            wk.L_tot = (int)Lt;
            wk.r = ring_ranges(wk.L_tot, a.n_sink, a.window, a.capacity);
            int nt = 0;
            for (int k = 0; k < wk.r.n; ++k) nt += (wk.r.len[k] + kTileKeys - 1) / kTileKeys;
            const long long cs = gridDim.x, c = blockIdx.x;
            s_walk = wk;
            s_range[0] = c * nt / cs;
            s_range[1] = (c + 1) * nt / cs;
            s_peff = nt;
            // a CTA with tiles counts in after its first TMA is issued (off the critical path)
            if (a.n_new > 0 && s_range[0] >= s_range[1]) fused_append_ticket(a);
            for (int s = 0; s < NSTAGE; ++s) {
                mbar_init(&full_bar[s], 1);
                mbar_init(&empty_bar[s], NWC);
            }
            mbar_init(sync_bar, NWC);
            fence_barrier_init();
        }
    } else if (warp == NWC) {
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
            s_peff = peff;
            s_range[0] = c < peff ? cta_begin(c, T, peff) : 0;
            s_range[1] = c < peff ? cta_begin(c + 1, T, peff) : 0;
            for (int s = 0; s < NSTAGE; ++s) {
                mbar_init(&full_bar[s], 1);
                mbar_init(&empty_bar[s], NWC);
            }
            mbar_init(sync_bar, NWC);
            fence_barrier_init();
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) WMTP_TRACE_AT(2);
    const long long t_begin = s_range[0], t_end = s_range[1];
    if (!CL && t_begin >= t_end) return;

    if (warp == NWC) {
        // =========================== producer warp =========================================
        if (lane == 0 && t_begin < t_end) {
            if (threadIdx.x == 32 * NWC) WMTP_TRACE_AT(42);
            TileWalker<SRC> walk;
            if (!CL) walk.init(a, plan_tiles);
            uint32_t it = 0;
            for (long long t = t_begin; t < t_end; ++t, ++it) {
                TileMeta m;
                int ty = 0, tz = 0;
                if (it == 0) WMTP_TRACE_AT(40);
                if (CL)
                    s_walk.describe(a, (int)t, (int)t_begin, (int)t_end, m, ty, tz);
                else
                    walk.describe(a, plan_tiles, plan_len, t, t_begin, t_end, m, ty, tz);
                if (it == 0) WMTP_TRACE_AT(41);
                const int stage = (int)(it % NSTAGE);
                const uint32_t phase = (it / NSTAGE) & 1u;
                if (!mbar_wait_bounded(&empty_bar[stage], phase ^ 1u)) break;
                meta[stage] = m;
                uint8_t* st = smem + (size_t)stage * kStage;
                if (m.nvalid > 0 && KV8) {
                    mbar_arrive_expect_tx(&full_bar[stage], kStageBytes8);
                    tma_load_3d(st, &kmap, &full_bar[stage], 0, ty, tz, pol);
                    tma_load_3d(st + kTileBytes8, &vmap, &full_bar[stage], 0, ty, tz, pol);
                } else if (m.nvalid > 0) {
                    mbar_arrive_expect_tx(&full_bar[stage], kStageBytes);
                    tma_load_3d(st, &kmap, &full_bar[stage], 0, ty, tz, pol);
                    tma_load_3d(st + kHalfBytes, &kmap, &full_bar[stage], 64, ty, tz, pol);
                    tma_load_3d(st + kTileBytes, &vmap, &full_bar[stage], 0, ty, tz, pol);
                    tma_load_3d(st + kTileBytes + kHalfBytes, &vmap, &full_bar[stage], 64, ty, tz, pol);
                } else {
                    mbar_arrive(&full_bar[stage]);
                }
                WMTP_TRACE_TILE(0, it);
                if (CL && it == 0 && a.n_new > 0) fused_append_ticket(a);
            }
            // Drain: wait (bounded) until the consumers released every stage, so no TMA copy is
            // in flight into this CTA's shared memory when it exits.
            const uint32_t issued = it;
            for (uint32_t k = (issued > NSTAGE ? issued - NSTAGE : 0); k < issued; ++k) {
                if (!mbar_wait_bounded(&empty_bar[k % NSTAGE], (k / NSTAGE) & 1u)) break;
            }
        }
        if (CL) {
            __syncwarp();
            cluster_merge_rows<NMT, NKG, NSTAGE, KV8, QS>(a, smem, s_walk, s_peff, warp, lane);
        }
        return;
    }

    // ============================= consumer warps ==========================================
    const int mt = warp % NMT;        // m-tile (16 rows)
    const int kg = warp / NMT;        // key group
    const int gid = lane >> 2, tig = lane & 3;
    const int key0 = kg * KPW;

    uint32_t qa[8][4];                // Q A-fragments, 8 k-steps of 16 dims
    float o[16][4];                   // O accumulator: 16 n-tiles of 8 dims
    float m_r[2], l_r[2];             // running max (log2 domain) and sum, rows gid / gid+8
    unsigned long long vis[2];        // in-step visibility bitmask per row
    int row_ok[2];
    int Lpre = 0;

    // head dim of accumulator pair (o[n][0], o[n][1]): 8 n + 2 tig; with fp8 KV the transposed
    // V fragments put n-tile 2 j + h at dims 16 j + 4 tig + 2 h
    auto out_dim = [](int n, int tg) -> int {
        return KV8 ? 16 * (n >> 1) + 4 * tg + 2 * (n & 1) : 8 * n + 2 * tg;
    };
    // per-lane ldmatrix row/chunk offsets
    const int k_row_l = (lane & 7) + ((lane >> 4) << 3);   // K: matrices (n0,k0) (n0,k8) (n8,k0) (n8,k8)
    const int k_chk_l = (lane >> 3) & 1;
    const int v_row_l = (lane & 7) + (((lane >> 3) & 1) << 3);   // V^T: (k0,d0) (k8,d0) (k0,d8) (k8,d8)
    const int v_chk_l = lane >> 4;

    uint32_t it = 0;
    uint32_t sync_phase = 0;
    bool alive = true;
    // Bounded rendezvous of the consumer warps (an mbarrier, so a sibling that gave up on a
    // timed-out wait cannot leave the others blocked for ever).
    auto consumers_sync = [&]() -> bool {
        __syncwarp();
        if (lane == 0) mbar_arrive(sync_bar);
        const bool ok = mbar_wait_bounded(sync_bar, sync_phase);
        sync_phase ^= 1u;
        return ok;
    };
    // Unit start: this warp's Q rows, the rows' visibility masks, state reset.  Returns false
    // when a bounded rendezvous gave up.
    auto unit_start = [&](const TileMeta& m) -> bool {
            // ---- unit start: load this warp's Q rows, visibility masks, reset state -------
            Lpre = m.L_tot - a.n_q;
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int R = m.rb * kRowsPerBlock + mt * 16 + gid + r * 8;
                row_ok[r] = R < a.rows_total;
                const int i = row_ok[r] ? R / a.G : 0;
                vis[r] = step_visibility(a, m.b, i);
                m_r[r] = -INFINITY;
                l_r[r] = 0.f;
            }
#pragma unroll
            for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
            if constexpr (QS) {
                // every warp is past the previous unit's reads of these rows; each consumer thread
                // widens quarter rows (32 dims) of the unit's Q into shared memory
                if (!consumers_sync()) return false;
                for (int w = threadIdx.x; w < NMT * 16 * 4; w += NWC * 32) {
                    const int row = w >> 2, part = w & 3;
                    const int R = m.rb * kRowsPerBlock + row;
                    uint32_t h[16];
                    if (R < a.rows_total) {
                        const int i = R / a.G, g = R - (R / a.G) * a.G;
                        const uint4* src = reinterpret_cast<const uint4*>(
                            a.q + (((size_t)m.b * a.n_q + i) * a.Hq + (size_t)m.h * a.G + g) * kD + 32 * part);
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint4 v = __ldg(src + k);
                            h[4 * k] = bf16x2_to_f16x2(v.x);
                            h[4 * k + 1] = bf16x2_to_f16x2(v.y);
                            h[4 * k + 2] = bf16x2_to_f16x2(v.z);
                            h[4 * k + 3] = bf16x2_to_f16x2(v.w);
                        }
                    } else {
#pragma unroll
                        for (int k = 0; k < 16; ++k) h[k] = 0u;
                    }
                    const uint32_t dst = smem_addr(smem + L::kQOff) + (uint32_t)(row * L::kQStride + 64 * part);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};"
                                     :: "r"(dst + 16u * k), "r"(h[4 * k]), "r"(h[4 * k + 1]),
                                        "r"(h[4 * k + 2]), "r"(h[4 * k + 3]) : "memory");
                }
                if (!consumers_sync()) return false;
            } else {
            const uint32_t* q32[2];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int R = m.rb * kRowsPerBlock + mt * 16 + gid + r * 8;
                const int i = R / a.G, g = R - (R / a.G) * a.G;
                q32[r] = reinterpret_cast<const uint32_t*>(
                    a.q + (((size_t)m.b * a.n_q + i) * a.Hq + (size_t)m.h * a.G + g) * kD);
            }
            if (KV8) {
                // fp16 A-fragments with the k order of the fp8 K fragments: k slots (2 tig, +1)
                // and (2 tig + 8, +9) of step ks hold dims 16 ks + 4 tig + (0, 1) and (2, 3)
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const int c = ks * 8 + 2 * tig;
                    qa[ks][0] = row_ok[0] ? bf16x2_to_f16x2(__ldg(q32[0] + c)) : 0u;
                    qa[ks][1] = row_ok[1] ? bf16x2_to_f16x2(__ldg(q32[1] + c)) : 0u;
                    qa[ks][2] = row_ok[0] ? bf16x2_to_f16x2(__ldg(q32[0] + c + 1)) : 0u;
                    qa[ks][3] = row_ok[1] ? bf16x2_to_f16x2(__ldg(q32[1] + c + 1)) : 0u;
                }
            } else {
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const int c = ks * 8 + tig;     // 32-bit word index of dims (16 ks + 2 tig)
                    qa[ks][0] = row_ok[0] ? __ldg(q32[0] + c) : 0u;
                    qa[ks][1] = row_ok[1] ? __ldg(q32[1] + c) : 0u;
                    qa[ks][2] = row_ok[0] ? __ldg(q32[0] + c + 4) : 0u;
                    qa[ks][3] = row_ok[1] ? __ldg(q32[1] + c + 4) : 0u;
                }
            }
            }
                return true;
    };
    if (t_begin < t_end) {
        // the first unit is known from the plan, so its Q loads overlap the first tile's TMA
        TileMeta m0;
        if (CL) {
            int ty0 = 0, tz0 = 0;
            s_walk.describe(a, (int)t_begin, (int)t_begin, (int)t_end, m0, ty0, tz0);
        } else {
            unit_of_tile(a, plan_tiles, plan_len, t_begin, m0);
        }
        if (!unit_start(m0)) alive = false;
        if (warp == 0 && lane == 0) WMTP_TRACE_AT(12);
    }
    for (long long t = t_begin; t < t_end && alive; ++t, ++it) {
        const int stage = (int)(it % NSTAGE);
        const uint32_t phase = (it / NSTAGE) & 1u;
        if (!mbar_wait_bounded(&full_bar[stage], phase)) { alive = false; break; }
        if (warp == 0 && lane == 0) WMTP_TRACE_TILE(1, it);
        const TileMeta m = meta[stage];
        bool patched = false;
        if (CL && a.n_new > 0 && m.nvalid > 0) {
            // fused append: the call's new positions [L_old, L_tot) that fall in this warp's keys
            // of the tile are copied from k_new / v_new over the (stale) ring rows the TMA
            // brought, and into the ring itself (once per unit)
            const int L_old = m.L_tot - a.n_new;
            const int k_hi = key0 + KPW < m.nvalid ? key0 + KPW : m.nvalid;
            const int p_lo = max(m.pos0 + key0, L_old);
            const int p_hi = min(m.pos0 + k_hi, m.L_tot);
            if (p_lo < p_hi) {
                patched = true;
                constexpr int kChunks = KV8 ? 8 : 16;          // 16-byte pieces of a row
                const uint32_t kb = smem_addr(smem + (size_t)stage * kStage);
                const uint32_t vb = kb + (KV8 ? kTileBytes8 : kTileBytes);
                for (int p = p_lo; p < p_hi; ++p) {
                    const int row = p - m.pos0;
                    if (lane < 2 * kChunks) {
                        const bool isv = lane >= kChunks;
                        const int c = isv ? lane - kChunks : lane;
                        const size_t src_row = ((size_t)m.b * a.n_new + (p - L_old)) * a.Hkv + m.h;
                        const uint4 val = __ldg((isv ? a.v_new : a.k_new) + src_row * kChunks + c);
                        const uint32_t base = isv ? vb : kb;
                        const uint32_t dst = KV8 ? tile8_chunk_addr(base, row, c) : tile_chunk_addr(base, row, c);
                        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};"
                                     :: "r"(dst), "r"(val.x), "r"(val.y), "r"(val.z), "r"(val.w) : "memory");
                        if (mt == 0 && m.rb == 0) {
                            const size_t slot = (size_t)(m.b * a.Hkv + m.h) * a.capacity + m.slot0 + row;
                            (isv ? a.ring_vw : a.ring_kw)[slot * kChunks + c] = val;
                        }
                    }
                }
                __syncwarp();
            }
        }

        if ((m.flags & kFirst) && it != 0) {
            if (!unit_start(m)) { alive = false; break; }
        }

        if (warp == 0 && lane == 0 && (m.flags & kFirst)) WMTP_TRACE_AT(11);
        if (m.nvalid > 0) {
            const uint32_t kbase = smem_addr(smem + (size_t)stage * kStage);
            const uint32_t vbase = kbase + (KV8 ? kTileBytes8 : kTileBytes);
            // ---- S = Q K^T over this warp's KPW keys -------------------------------------
            float s[NT][4];
#pragma unroll
            for (int n = 0; n < NT; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
            if (KV8) {
                // matrix (lane / 8): key octet 2 np + (lane / 8) % 2, dim chunk 2 kp + lane / 16
                const int r8 = (lane & 7) + (((lane >> 3) & 1) << 3);
                const int c8 = lane >> 4;
#pragma unroll
                for (int kp = 0; kp < 4; ++kp) {
                    // A fragments of k-steps 2 kp, 2 kp + 1 (QS: from the shared fp16 rows, dims
                    // 16 ks + 4 tig .. + 3 of rows gid and gid + 8)
                    uint32_t qs[2][4];
                    if constexpr (QS) {
#pragma unroll
                        for (int kss = 0; kss < 2; ++kss) {
                            const uint32_t q0 = smem_addr(smem + L::kQOff) +
                                                (uint32_t)((mt * 16 + gid) * L::kQStride + 32 * (2 * kp + kss) + 8 * tig);
                            const uint32_t q1 = q0 + 8u * L::kQStride;
                            asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];"
                                         : "=r"(qs[kss][0]), "=r"(qs[kss][2]) : "r"(q0));
                            asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];"
                                         : "=r"(qs[kss][1]), "=r"(qs[kss][3]) : "r"(q1));
                        }
                    }
                    const uint32_t* A0 = QS ? qs[0] : qa[2 * kp];
                    const uint32_t* A1 = QS ? qs[1] : qa[2 * kp + 1];
#pragma unroll
                    for (int np = 0; np < NT / 2; ++np) {
                        uint32_t r0, r1, r2, r3;
                        ldsm_x4(tile8_chunk_addr(kbase, key0 + np * 16 + r8, 2 * kp + c8), r0, r1, r2, r3);
                        uint32_t b[8];
                        e4m3x4_to_f16x2x2(r0, b[0], b[1]);
                        e4m3x4_to_f16x2x2(r1, b[2], b[3]);
                        e4m3x4_to_f16x2x2(r2, b[4], b[5]);
                        e4m3x4_to_f16x2x2(r3, b[6], b[7]);
                        mma_f16_16816(s[2 * np], A0, b[0], b[1]);
                        mma_f16_16816(s[2 * np + 1], A0, b[2], b[3]);
                        mma_f16_16816(s[2 * np], A1, b[4], b[5]);
                        mma_f16_16816(s[2 * np + 1], A1, b[6], b[7]);
                    }
                }
            } else if constexpr (SRC == kSrcRing && NT <= 2) {
                // ring source (the windowed draft, whose few tiles per CTA make the consumer's
                // latency the pace), 16 keys per warp: odd k-steps accumulate into a second
                // set, so the dependent MMA chains are four long instead of eight
                float s2[NT][4];
#pragma unroll
                for (int n = 0; n < NT; ++n) s2[n][0] = s2[n][1] = s2[n][2] = s2[n][3] = 0.f;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
                    for (int np = 0; np < NT / 2; ++np) {
                        uint32_t b0a, b1a, b0b, b1b;
                        ldsm_x4(tile_chunk_addr(kbase, key0 + np * 16 + k_row_l, ks * 2 + k_chk_l),
                                b0a, b1a, b0b, b1b);
                        float (*acc)[4] = (ks & 1) ? s2 : s;
                        mma_bf16_16816(acc[2 * np], qa[ks], b0a, b1a);
                        mma_bf16_16816(acc[2 * np + 1], qa[ks], b0b, b1b);
                    }
                }
#pragma unroll
                for (int n = 0; n < NT; ++n)
#pragma unroll
                    for (int e = 0; e < 4; ++e) s[n][e] += s2[n][e];
            } else {
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
                    for (int np = 0; np < NT / 2; ++np) {
                        uint32_t b0a, b1a, b0b, b1b;
                        ldsm_x4(tile_chunk_addr(kbase, key0 + np * 16 + k_row_l, ks * 2 + k_chk_l),
                                b0a, b1a, b0b, b1b);
                        mma_bf16_16816(s[2 * np], qa[ks], b0a, b1a);
                        mma_bf16_16816(s[2 * np + 1], qa[ks], b0b, b1b);
                    }
                }
            }
            // ---- mask: ragged tile end, in-step (causal / tree) keys ----------------------
            const bool need_mask = (m.nvalid < kTileKeys) || (m.pos0 + kTileKeys > Lpre);
            if (need_mask) {
#pragma unroll
                for (int n = 0; n < NT; ++n) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int kr = key0 + n * 8 + 2 * tig + (e & 1);
                        const int pos = m.pos0 + kr;
                        const int off = pos - Lpre;
                        const unsigned long long vm = vis[e >> 1];
                        const bool ok = kr < m.nvalid &&
                                        (off < 0 || (off < 64 && ((vm >> off) & 1ull)));
                        if (!ok) s[n][e] = -INFINITY;
                    }
                }
            }
            // ---- online softmax (base 2) -------------------------------------------------
            float m_use[2], alpha[2];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                float mx = -INFINITY;
#pragma unroll
                for (int n = 0; n < NT; ++n) mx = fmaxf(mx, fmaxf(s[n][2 * r], s[n][2 * r + 1]));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                const float m_new = fmaxf(m_r[r], mx * a.scale_log2);
                m_use[r] = (m_new == -INFINITY) ? 0.f : m_new;
                alpha[r] = fast_exp2(m_r[r] - m_use[r]);
                m_r[r] = m_new;
                l_r[r] *= alpha[r];
            }
            // the running maxima rarely move after the first tiles: skip the O rescale when no
            // row of this warp changed
            if (__any_sync(0xffffffffu, alpha[0] != 1.f || alpha[1] != 1.f)) {
#pragma unroll
                for (int n = 0; n < 16; ++n) {
                    o[n][0] *= alpha[0]; o[n][1] *= alpha[0];
                    o[n][2] *= alpha[1]; o[n][3] *= alpha[1];
                }
            }
            uint32_t pa[NT / 2][4];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    const float p0 = fast_exp2(fmaf(s[n][2 * r], a.scale_log2, -m_use[r]));
                    const float p1 = fast_exp2(fmaf(s[n][2 * r + 1], a.scale_log2, -m_use[r]));
                    // fp16 (fp8 KV) or bf16 weights for PV; the row sum over the fp32 weights (the
                    // rounded weights would cost two unpacks a pair; the sums differ by at most
                    // 2^-9 of a weight, within the tolerance, and it measured ~1 % faster in the
                    // power-capped step)
                    const uint32_t pk = KV8 ? pack_f16x2(p0, p1) : pack_bf16x2(p0, p1);
                    l_r[r] += p0 + p1;
                    pa[n >> 1][r + 2 * (n & 1)] = pk;
                }
            }
            // ---- O += P V ------------------------------------------------------------------
            const bool ragged = m.nvalid < kTileKeys;
#pragma unroll
            for (int kk = 0; kk < NT / 2; ++kk) {
                const int krow = key0 + kk * 16;
                uint32_t lo_keep = 0xffffffffu, hi_keep = 0xffffffffu;   // keys 2tig(+1), +8
                if (ragged) {
                    const int k0 = krow + 2 * tig;
                    lo_keep = (k0 < m.nvalid ? 0x0000ffffu : 0u) | (k0 + 1 < m.nvalid ? 0xffff0000u : 0u);
                    hi_keep = (k0 + 8 < m.nvalid ? 0x0000ffffu : 0u) | (k0 + 9 < m.nvalid ? 0xffff0000u : 0u);
                }
                if (KV8) {
                    // matrix (lane / 8): key octet (lane / 8) % 2, dim chunk 2 jp + lane / 16.
                    // Widened, each matrix is two 8x8 fp16 matrices (dims 16 j + 4 c + {0, 1} and
                    // + {2, 3}); transposed, they are the B fragments of output tiles 2 j, 2 j + 1.
                    const int r8 = (lane & 7) + (((lane >> 3) & 1) << 3);
                    const int c8 = lane >> 4;
#pragma unroll
                    for (int jp = 0; jp < 4; ++jp) {
                        uint32_t r[4];
                        ldsm_x4(tile8_chunk_addr(vbase, krow + r8, 2 * jp + c8), r[0], r[1], r[2], r[3]);
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int j = 2 * jp + h;
                            uint32_t x00, x01, x10, x11;
                            e4m3x4_to_f16x2x2(r[2 * h], x00, x01);
                            e4m3x4_to_f16x2x2(r[2 * h + 1], x10, x11);
                            uint32_t b00 = movmatrix_trans(x00);
                            uint32_t b10 = movmatrix_trans(x10);
                            uint32_t b01 = movmatrix_trans(x01);
                            uint32_t b11 = movmatrix_trans(x11);
                            if (ragged) {
                                b00 &= lo_keep; b01 &= lo_keep;
                                b10 &= hi_keep; b11 &= hi_keep;
                            }
                            mma_f16_16816(o[2 * j], pa[kk], b00, b10);
                            mma_f16_16816(o[2 * j + 1], pa[kk], b01, b11);
                        }
                    }
                } else {
#pragma unroll
                    for (int dp = 0; dp < 8; ++dp) {
                        uint32_t b0a, b1a, b0b, b1b;
                        ldsm_x4_trans(tile_chunk_addr(vbase, krow + v_row_l, dp * 2 + v_chk_l),
                                      b0a, b1a, b0b, b1b);
                        if (ragged) {
                            b0a &= lo_keep; b0b &= lo_keep;
                            b1a &= hi_keep; b1b &= hi_keep;
                        }
                        mma_bf16_16816(o[2 * dp], pa[kk], b0a, b1a);
                        mma_bf16_16816(o[2 * dp + 1], pa[kk], b0b, b1b);
                    }
                }
            }
        }
        // generic-proxy writes to the stage (the append patch) before the producer's next TMA
        // write into it
        if (CL && patched) fence_proxy_async();
        __syncwarp();
        // MS: a unit's last stage is released after the key-group merge that goes through it
        const bool hold_stage = MS && NKG > 1 && (m.flags & kLast);
        if (lane == 0 && !hold_stage) mbar_arrive(&empty_bar[stage]);
        if (warp == 0 && lane == 0) WMTP_TRACE_TILE(2, it);

        if (m.flags & kLast) {
            // ---- unit end: combine key groups, then write the result or a partial ----------
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                l_r[r] += __shfl_xor_sync(0xffffffffu, l_r[r], 1);
                l_r[r] += __shfl_xor_sync(0xffffffffu, l_r[r], 2);
            }
            if (QS && NKG > 1) {
                // one m-tile at a time through the shared Q rows' space, once every warp is past
                // its last reads of them
                if (!consumers_sync()) { alive = false; break; }
#pragma unroll 1
                for (int mt2 = 0; mt2 < NMT; ++mt2) {
                    if (mt == mt2 && kg > 0) {
                        float* mo = merge_o + ((size_t)(kg - 1) * 16) * L::kMergeStride;
                        float* ml = merge_ml + ((size_t)(kg - 1) * 16) * 2;
#pragma unroll
                        for (int r = 0; r < 2; ++r) {
                            const int row = gid + 8 * r;
#pragma unroll
                            for (int n = 0; n < 16; ++n)
                                *reinterpret_cast<float2*>(mo + row * L::kMergeStride + n * 8 + 2 * tig) =
                                    make_float2(o[n][2 * r], o[n][2 * r + 1]);
                            if (tig == 0) { ml[row * 2] = m_r[r]; ml[row * 2 + 1] = l_r[r]; }
                        }
                    }
                    if (!consumers_sync()) { alive = false; break; }
                    if (mt == mt2 && kg == 0) {
#pragma unroll 1
                        for (int g2 = 1; g2 < NKG; ++g2) {
                            const float* mo = merge_o + ((size_t)(g2 - 1) * 16) * L::kMergeStride;
                            const float* ml = merge_ml + ((size_t)(g2 - 1) * 16) * 2;
#pragma unroll
                            for (int r = 0; r < 2; ++r) {
                                const int row = gid + 8 * r;
                                const float m2 = ml[row * 2], l2 = ml[row * 2 + 1];
                                const float mn = fmaxf(m_r[r], m2);
                                const float mu = (mn == -INFINITY) ? 0.f : mn;
                                const float w1 = fast_exp2(m_r[r] - mu), w2 = fast_exp2(m2 - mu);
                                l_r[r] = l_r[r] * w1 + l2 * w2;
                                m_r[r] = mn;
#pragma unroll
                                for (int n = 0; n < 16; ++n) {
                                    const float2 v2 = *reinterpret_cast<const float2*>(
                                        mo + row * L::kMergeStride + n * 8 + 2 * tig);
                                    o[n][2 * r] = o[n][2 * r] * w1 + v2.x * w2;
                                    o[n][2 * r + 1] = o[n][2 * r + 1] * w1 + v2.y * w2;
                                }
                            }
                        }
                    }
                    if (!consumers_sync()) { alive = false; break; }
                }
                if (!alive) break;
            } else if (NKG > 1) {
                float* const mrg_o = MS ? reinterpret_cast<float*>(smem + (size_t)stage * kStage) : merge_o;
                float* const mrg_ml = MS ? mrg_o + L::kMergeFloats : merge_ml;
                // MS: every warp is past its reads of the stage's K and V before it is overwritten
                if (MS && !consumers_sync()) { alive = false; break; }
                if (kg > 0) {
                    float* mo = mrg_o + ((size_t)((kg - 1) * NMT + mt) * 16) * L::kMergeStride;
                    float* ml = mrg_ml + ((size_t)((kg - 1) * NMT + mt) * 16) * 2;
#pragma unroll
                    for (int r = 0; r < 2; ++r) {
                        if (CL && !row_ok[r]) continue;     // (cluster mode: rows past the unit's)
                        const int row = gid + 8 * r;
#pragma unroll
                        for (int n = 0; n < 16; ++n)
                            *reinterpret_cast<float2*>(mo + row * L::kMergeStride + n * 8 + 2 * tig) =
                                make_float2(o[n][2 * r], o[n][2 * r + 1]);
                        if (tig == 0) { ml[row * 2] = m_r[r]; ml[row * 2 + 1] = l_r[r]; }
                    }
                }
                if (!consumers_sync()) { alive = false; break; }
                if (kg == 0) {
#pragma unroll 1
                    for (int g2 = 1; g2 < NKG; ++g2) {
                        const float* mo = mrg_o + ((size_t)((g2 - 1) * NMT + mt) * 16) * L::kMergeStride;
                        const float* ml = mrg_ml + ((size_t)((g2 - 1) * NMT + mt) * 16) * 2;
#pragma unroll
                        for (int r = 0; r < 2; ++r) {
                            if (CL && !row_ok[r]) continue;
                            const int row = gid + 8 * r;
                            const float m2 = ml[row * 2], l2 = ml[row * 2 + 1];
                            const float mn = fmaxf(m_r[r], m2);
                            const float mu = (mn == -INFINITY) ? 0.f : mn;
                            const float w1 = fast_exp2(m_r[r] - mu), w2 = fast_exp2(m2 - mu);
                            l_r[r] = l_r[r] * w1 + l2 * w2;
                            m_r[r] = mn;
#pragma unroll
                            for (int n = 0; n < 16; ++n) {
                                const float2 v2 = *reinterpret_cast<const float2*>(
                                    mo + row * L::kMergeStride + n * 8 + 2 * tig);
                                o[n][2 * r] = o[n][2 * r] * w1 + v2.x * w2;
                                o[n][2 * r + 1] = o[n][2 * r + 1] * w1 + v2.y * w2;
                            }
                        }
                    }
                }
                // the merge space is free again for the CTA's next unit (a cluster CTA has one)
                if ((!CL || MS) && !consumers_sync()) { alive = false; break; }
                // every warp has read the merge rows: the stage goes back to the producer
                if (MS && lane == 0) mbar_arrive(&empty_bar[stage]);
            }
            if (CL && NKG == 1) {
                // every consumer warp is past its last reads of the stage space the partial takes
                if (!consumers_sync()) { alive = false; break; }
            }
            if (kg == 0) {
                const int slot = (int)blockIdx.x + m.unit;
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    if (!row_ok[r]) continue;
                    const int rr = mt * 16 + gid + 8 * r;            // row within the block
                    const int R = m.rb * kRowsPerBlock + rr;
                    const float l = l_r[r];
                    const float inv = l > 0.f ? a.v_scale / l : 0.f;
                    const float lse2 = l > 0.f ? m_r[r] + __log2f(l) : -INFINITY;
                    if (CL) {
                        float* po = reinterpret_cast<float*>(smem + L::kPartOff) + (size_t)rr * kD;
#pragma unroll
                        for (int n = 0; n < 16; ++n)
                            *reinterpret_cast<float2*>(po + out_dim(n, tig)) =
                                make_float2(o[n][2 * r] * inv, o[n][2 * r + 1] * inv);
                        if (tig == 0) reinterpret_cast<float*>(smem + L::kPartLseOff)[rr] = lse2;
                    } else if (m.flags & kWhole) {
                        const int i = R / a.G, g = R - (R / a.G) * a.G;
                        const size_t orow = ((size_t)m.b * a.n_q + i) * a.Hq + (size_t)m.h * a.G + g;
                        uint32_t* op = reinterpret_cast<uint32_t*>(a.out + orow * kD);
#pragma unroll
                        for (int n = 0; n < 16; ++n)
                            op[out_dim(n, tig) >> 1] = pack_bf16x2(o[n][2 * r] * inv, o[n][2 * r + 1] * inv);
                        if (a.lse != nullptr && tig == 0) a.lse[orow] = lse2 * kLn2;
                    } else {
                        float* wo = a.ws_o + ((size_t)slot * a.rows_blk + rr) * kD;
#pragma unroll
                        for (int n = 0; n < 16; ++n)
                            *reinterpret_cast<float2*>(wo + out_dim(n, tig)) =
                                make_float2(o[n][2 * r] * inv, o[n][2 * r + 1] * inv);
                        if (tig == 0) a.ws_lse[(size_t)slot * a.rows_blk + rr] = lse2;
                    }
                }
            }
        }
    }
    if (warp == 0 && lane == 0) WMTP_TRACE_AT(28);
    if (warp == 0 && lane == 0) WMTP_TRACE_MAX(43);
    if (CL) {
        __syncwarp();
        cluster_merge_rows<NMT, NKG, NSTAGE, KV8, QS>(a, smem, s_walk, s_peff, warp, lane);
        if (warp == 0 && lane == 0) WMTP_TRACE_AT(31);
    }
}

// ---------------------------------------------------------------------------------------------
// lse_merge_kernel: combines the split partials of units that span several CTAs, and writes
// empty units (no keys at all) as out = 0, lse = -inf.  Grid (units, rows per block, C head-dim
// chunks of 128 / C dims), 256 threads.  Partial s has weight 2^(lse_s - M) with M the largest
// partial LSE; empty partials have lse = -inf and weight 0.
// The plan (which CTAs hold the unit's partials) needs only the request lengths, which the
// attention kernel before this one does not write and which were final before it let this kernel
// launch (it triggers after its own wait), so it is computed before this kernel's wait.  After the
// wait, thread t takes partials t / F, t / F + 256 / F, ... (F = 32 / C float4 per partial chunk)
// and float4 t % F of each, issues the LSE and 16-byte partial loads of kMergeBatch partials at
// once and folds them into a running (max, sum, O); the threads' states are combined per head dim
// in shared memory.  The host picks C so that one round of loads covers the expected partials (a
// 128K-key verify unit has ~150: one L2 round trip).
constexpr int kMaxParts = 1024;
constexpr int kMergeThreads = 256;
constexpr int kMergeBatch = 6;

template <int SRC>
__global__ void __launch_bounds__(kMergeThreads)
lse_merge_kernel(const AttnArgs a, int P_launch) {
    pdl_launch_dependents();
    if (threadIdx.x == 0) WMTP_TRACE_AT(48);
    const int u = blockIdx.x;
    const int rr = blockIdx.y;
    const int rb = u % a.n_rb;
    const int h = (u / a.n_rb) % a.Hkv;
    const int b = u / (a.n_rb * a.Hkv);
    const int R = rb * kRowsPerBlock + rr;
    if (R >= a.rows_total) return;

    __shared__ int s_info[3];           // unit tiles, first and last CTA of the unit
    if (threadIdx.x == 0) {
        long long T = 0, start = 0;
        int nt_u = 0;
        for (int bb = 0; bb < a.B; ++bb) {
            const int nt = request_tiles<SRC>(a, request_len<SRC>(a, bb));
            if (bb == b) { start = T + (long long)(h * a.n_rb + rb) * nt; nt_u = nt; }
            T += (long long)nt * a.Hkv * a.n_rb;
        }
        s_info[0] = nt_u;
        if (nt_u > 0) {
            const int peff = plan_ctas(T, P_launch, a.min_tiles_per_cta);
            s_info[1] = cta_of_tile(start, T, peff);
            s_info[2] = cta_of_tile(start + nt_u - 1, T, peff);
        }
    }
    __syncthreads();
    const int nt_u = s_info[0];
    const int i = R / a.G, g = R - (R / a.G) * a.G;
    const size_t orow = ((size_t)b * a.n_q + i) * a.Hq + (size_t)h * a.G + g;
    const int tid = threadIdx.x;
    const int C = gridDim.z, F = (kD / 4) / C, dims = kD / C, d_lo = blockIdx.z * dims;
    pdl_wait();
    if (threadIdx.x == 0) WMTP_TRACE_AT(49);
    if (nt_u == 0) {
        if (tid < dims) a.out[orow * kD + d_lo + tid] = __float2bfloat16_rn(0.f);
        if (a.lse != nullptr && tid == 0 && blockIdx.z == 0) a.lse[orow] = -INFINITY;
        return;
    }
    const int c_lo = s_info[1], c_hi = s_info[2];
    if (c_lo == c_hi) return;           // finished inside one CTA
    const int np = c_hi - c_lo + 1;     // <= peff <= P_launch <= kMaxParts (host-checked)
    const int lanes = kMergeThreads / F;          // partials per load step
    const int qk = tid / F, f4 = tid - qk * F;
    const float* lse_base = a.ws_lse + (size_t)(c_lo + u) * a.rows_blk + rr;
    const float4* o_base = reinterpret_cast<const float4*>(
        a.ws_o + ((size_t)(c_lo + u) * a.rows_blk + rr) * kD + d_lo) + f4;
    const size_t kSlotStride4 = (size_t)a.rows_blk * (kD / 4);
    float m_t = -INFINITY, s_t = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int k0 = qk; k0 < np; k0 += kMergeBatch * lanes) {
        float lv[kMergeBatch];
        float4 x[kMergeBatch];
#pragma unroll
        for (int j = 0; j < kMergeBatch; ++j) {
            const int k = k0 + j * lanes;
            lv[j] = k < np ? __ldcg(lse_base + (size_t)k * a.rows_blk) : -INFINITY;
            x[j] = k < np ? __ldcg(o_base + (size_t)k * kSlotStride4) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        float mb = lv[0];
#pragma unroll
        for (int j = 1; j < kMergeBatch; ++j) mb = fmaxf(mb, lv[j]);
        if (mb > m_t) {
            const float f = (m_t == -INFINITY) ? 0.f : exp2f(m_t - mb);
            acc.x *= f; acc.y *= f; acc.z *= f; acc.w *= f;
            s_t *= f;
            m_t = mb;
        }
        if (m_t == -INFINITY) continue;
#pragma unroll
        for (int j = 0; j < kMergeBatch; ++j) {
            const float w = (lv[j] == -INFINITY) ? 0.f : exp2f(lv[j] - m_t);
            acc.x += w * x[j].x; acc.y += w * x[j].y; acc.z += w * x[j].z; acc.w += w * x[j].w;
            s_t += w;
        }
    }
    if (threadIdx.x == 0) WMTP_TRACE_AT(50);
    // the threads of one partial lane (same qk) folded the same partials: one (max, sum) per
    // lane, kept by its first thread; warp 0 turns them into weights once
    __shared__ float4 s_acc[kMergeThreads];
    __shared__ float s_m[32], s_s[32], s_f[32], s_wt;
    __shared__ float s_M;
    s_acc[tid] = acc;
    if (f4 == 0) {
        s_m[qk] = m_t;
        s_s[qk] = s_t;
    }
    __syncthreads();
    if (tid < 32) {
        const float mq = tid < lanes ? s_m[tid] : -INFINITY;
        float M = mq;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        const float f = (mq == -INFINITY) ? 0.f : exp2f(mq - M);
        float wt = tid < lanes ? f * s_s[tid] : 0.f;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) wt += __shfl_xor_sync(0xffffffffu, wt, off);
        s_f[tid] = f;
        if (tid == 0) {
            s_M = M;
            s_wt = wt;
        }
    }
    __syncthreads();
    if (tid >= dims) return;
    // thread d combines head dim d_lo + d over the partial lanes
    const int fd = tid >> 2, cd = tid & 3;
    float accd = 0.f;
    for (int q = 0; q < lanes; ++q)
        accd += s_f[q] * reinterpret_cast<const float*>(&s_acc[q * F + fd])[cd];
    const float wt = s_wt, M = s_M;
    const float res = wt > 0.f ? accd / wt : 0.f;
    a.out[orow * kD + d_lo + tid] = __float2bfloat16_rn(res);
    if (a.lse != nullptr && tid == 0 && blockIdx.z == 0)
        a.lse[orow] = wt > 0.f ? (M + log2f(wt)) * kLn2 : -INFINITY;
    if (threadIdx.x == 0) WMTP_TRACE_AT(51);
}

}  // namespace wmtp
