// ring_accept_kernels.cuh -- the draft-KV ring append and greedy acceptance for sm_100a.
#pragma once

#include "device_common.cuh"

namespace wmtp {

// ---------------------------------------------------------------------------------------------
// Ring append (Windowed-MTP, arXiv 2607.21535; Pith verdict, referee_report.minor_comments,
// App. A pseudocode: the draft KV ring is addressed as ring_base(r) + logical_pos).
// Slot of position p: p for p < n_sink, else n_sink + (p - n_sink) mod (C - n_sink).
// Of the call's positions [L_old, L_new) only the survivors are copied: the sink positions
// (p < n_sink) and the last C - n_sink positions; an earlier position that a later one of the
// same call would overwrite is never written, so no two threads write one slot.
// Grid (chunks, B), 256 threads; each thread moves 16-byte pieces of rows of CH pieces (16 for
// bf16 rows of 256 bytes, 8 for fp8 rows of 128 bytes).
__device__ __forceinline__ long long ring_slot_of(long long p, int s, int C) {
    return p < s ? p : (long long)s + (p - s) % (long long)(C - s);
}

template <int CH>
__global__ void __launch_bounds__(256)
ring_append_kernel(uint4* __restrict__ ring_k, uint4* __restrict__ ring_v, long long* ring_len,
                   const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                   int n_new, int Hkv, int n_sink, int C, int update_len_here) {
    pdl_launch_dependents();
    pdl_wait();
    const int b = blockIdx.y;
    const long long L_old = ring_len[b];
    const long long L_new = L_old + n_new;
    // survivors: tokens [0, e1) are sink positions, tokens [s2, n_new) are the ring's tail
    long long e1 = (long long)n_sink - L_old;
    e1 = e1 < 0 ? 0 : (e1 > n_new ? n_new : e1);
    long long s2 = (long long)n_new - (C - n_sink);
    if (s2 < e1) s2 = e1;
    const long long n_surv = e1 + (n_new - s2);
    constexpr int kChunks = CH;                              // 16-byte pieces per row
    const long long work = n_surv * Hkv * kChunks;
    for (long long w = (long long)blockIdx.x * blockDim.x + threadIdx.x; w < work;
         w += (long long)gridDim.x * blockDim.x) {
        const int chunk = (int)(w % kChunks);
        const long long row = w / kChunks;
        const int h = (int)(row % Hkv);
        const long long j = row / Hkv;
        const long long t = j < e1 ? j : s2 + (j - e1);
        const long long slot = ring_slot_of(L_old + t, n_sink, C);
        const size_t src = (((size_t)b * n_new + (size_t)t) * Hkv + h) * kChunks + chunk;
        const size_t dst = (((size_t)b * Hkv + h) * (size_t)C + (size_t)slot) * kChunks + chunk;
        ring_k[dst] = k_new[src];
        ring_v[dst] = v_new[src];
    }
    if (update_len_here) {
        __syncthreads();                   // every thread of this (only) CTA has read L_old
        if (threadIdx.x == 0) ring_len[b] = L_new;
    }
}

// Length update for appends spread over several CTAs per request (runs after them on the
// same stream).
__global__ void ring_len_add_kernel(long long* ring_len, int B, int n_new) {
    pdl_launch_dependents();
    pdl_wait();
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b < B) ring_len[b] += n_new;
}

// ---------------------------------------------------------------------------------------------
// Greedy acceptance (AI field-notes abstract for 2607.21535: the target decides every accepted
// token; Pith verdict, pith_extraction.forward_implications: greedy-exact).
// One CTA per request; warps take nodes, each lane scans a strided slice of the vocabulary with
// a strict '>' (its lowest index among equal maxima), then a warp reduction keeps the larger
// value and, on equal values, the lower index.  Thread 0 then walks the chain or tree.
__global__ void __launch_bounds__(256)
accept_greedy_kernel(const float* __restrict__ logits, const int* __restrict__ tokens,
                     const int* __restrict__ tree_parent, int n_q, int V,
                     int* __restrict__ accepted, int* __restrict__ n_accepted) {
    __shared__ int t_arg[64];
    pdl_launch_dependents();
    pdl_wait();
    const int b = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = warp; i < n_q; i += blockDim.x >> 5) {
        const float* row = logits + ((size_t)b * n_q + i) * (size_t)V;
        float best = -INFINITY;
        int idx = -1;
        for (int v = lane; v < V; v += 32) {
            const float x = row[v];
            if (idx < 0 || x > best) { best = x; idx = v; }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ob = __shfl_xor_sync(0xffffffffu, best, off);
            const int oi = __shfl_xor_sync(0xffffffffu, idx, off);
            const bool take = oi >= 0 && (idx < 0 || ob > best || (ob == best && oi < idx));
            if (take) { best = ob; idx = oi; }
        }
        if (lane == 0) t_arg[i] = idx;
    }
    __syncthreads();
    if (threadIdx.x != 0) return;
    const int* tok = tokens + (size_t)b * n_q;
    int* acc = accepted + (size_t)b * n_q;
    int n = 0;
    if (tree_parent == nullptr) {
        int a = 0;
        while (a + 1 < n_q && tok[a + 1] == t_arg[a]) ++a;
        for (int j = 1; j <= a; ++j) acc[n++] = tok[j];
        acc[n++] = t_arg[a];
    } else {
        const int* par = tree_parent + (size_t)b * n_q;
        int cur = 0;
        for (int depth = 0; depth + 1 < n_q; ++depth) {   // a root path has at most n_q - 1 drafts
            int next = -1;
            for (int c = 1; c < n_q; ++c)
                if (par[c] == cur && tok[c] == t_arg[cur]) { next = c; break; }
            if (next < 0) break;
            acc[n++] = tok[next];
            cur = next;
        }
        acc[n++] = t_arg[cur];
    }
    for (int j = n; j < n_q; ++j) acc[j] = -1;
    n_accepted[b] = n;
}

}  // namespace wmtp

namespace wmtp {

// ---------------------------------------------------------------------------------------------
// Stochastic acceptance (AI field-notes abstract for 2607.21535: the target's verified output
// distribution is preserved; Pith verdict, referee_report.significance: the standard
// speculative-decoding theorem).  The standard rejection rule (Leviathan, Kalman and Matias,
// ICML 2023; Chen et al., 2023): draft i is kept with probability min(1, p_{i-1}(x) / q_{i-1}(x));
// at the first rejection a token is drawn from norm(max(0, p_{i-1} - q_{i-1})); after all gamma
// drafts a bonus token is drawn from p_gamma.  Randomness comes in as integers and every
// decision is exact: keep iff u * q(x) < p(x) * 2^24 (u < 2^24; both products exact in double);
// a draw over weights w uses m(v) = floor(w(v) * 2^40) (64-bit integers), M = sum m,
// t = floor(u_sample * M / 2^32) and picks the smallest v whose running sum of m exceeds t.
// With no residual mass (M = 0) the draw uses p; with none there either it emits token 0.
// One CTA per request: thread 0 walks the drafts; the draw is a block-wide integer scan
// (each thread owns a contiguous chunk of the vocabulary), so the result does not depend on
// the summation order.
__device__ __forceinline__ unsigned long long fix40(float w) {
    if (!(w > 0.f)) return 0ull;
    return (unsigned long long)((double)w * 1099511627776.0);      // 2^40, truncating
}

// w(v) = max(0, a[v] - b[v]) when b != nullptr, else a[v].
__device__ __forceinline__ float draw_weight(const float* a, const float* b, int v) {
    if (b == nullptr) return a[v];
    const float d = __fsub_rn(a[v], b[v]);
    return d > 0.f ? d : 0.f;
}

template <int NT>
__device__ int block_draw(const float* a, const float* b, int V, unsigned int u_sample,
                          unsigned long long* s_warp, int* s_y) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int chunk = (V + NT - 1) / NT;
    const int v0 = tid * chunk;
    const int v1 = min(V, v0 + chunk);
    unsigned long long local = 0;
    for (int v = v0; v < v1; ++v) local += fix40(draw_weight(a, b, v));
    // block-wide exclusive scan of the per-thread sums (integers: exact in any order)
    unsigned long long incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const unsigned long long o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) s_warp[warp] = incl;
    if (tid == 0) *s_y = -1;
    __syncthreads();
    unsigned long long base = 0, M = 0;
    for (int w = 0; w < NT / 32; ++w) {
        if (w < warp) base += s_warp[w];
        M += s_warp[w];
    }
    const unsigned long long excl = base + incl - local;
    if (M != 0) {
        const unsigned long long t =
            (unsigned long long)u_sample * (M >> 32) + (((unsigned long long)u_sample * (M & 0xffffffffull)) >> 32);
        if (excl <= t && t < excl + local) {
            unsigned long long c = excl;
            for (int v = v0; v < v1; ++v) {
                c += fix40(draw_weight(a, b, v));
                if (c > t) { *s_y = v; break; }
            }
        }
    }
    __syncthreads();
    const int y = *s_y;
    __syncthreads();                       // s_warp / s_y may be reused by the next draw
    return y;
}

template <int NT>
__global__ void __launch_bounds__(NT)
accept_stochastic_kernel(const float* __restrict__ p, const float* __restrict__ q,
                         const int* __restrict__ tokens, const unsigned int* __restrict__ u_accept,
                         const unsigned int* __restrict__ u_sample, int n_q, int V,
                         int* __restrict__ accepted, int* __restrict__ n_accepted) {
    __shared__ unsigned long long s_warp[NT / 32];
    __shared__ int s_y, s_rej, s_n;
    pdl_launch_dependents();
    pdl_wait();
    const int b = blockIdx.x;
    const int* tok = tokens + (size_t)b * n_q;
    if (threadIdx.x == 0) {
        int n = 0, rej = -1;
        for (int i = 1; i < n_q; ++i) {
            const int x = tok[i];
            double px = 0.0, qx = 0.0;
            if (x >= 0 && x < V) {
                px = (double)p[((size_t)b * n_q + (i - 1)) * (size_t)V + x];
                qx = (double)q[((size_t)b * (n_q - 1) + (i - 1)) * (size_t)V + x];
            } else {
                flag_status(kStatusDeviceIndex);
            }
            const double u = (double)u_accept[(size_t)b * (n_q - 1) + (i - 1)];
            if (u * qx < px * 16777216.0) {
                ++n;
            } else {
                rej = i;
                break;
            }
        }
        s_n = n;
        s_rej = rej;
    }
    __syncthreads();
    const int n = s_n, rej = s_rej;
    int y;
    if (rej > 0) {
        const float* pr = p + ((size_t)b * n_q + (rej - 1)) * (size_t)V;
        const float* qr = q + ((size_t)b * (n_q - 1) + (rej - 1)) * (size_t)V;
        y = block_draw<NT>(pr, qr, V, u_sample[b], s_warp, &s_y);
        if (y < 0) y = block_draw<NT>(pr, nullptr, V, u_sample[b], s_warp, &s_y);
    } else {
        y = block_draw<NT>(p + ((size_t)b * n_q + (n_q - 1)) * (size_t)V, nullptr, V, u_sample[b],
                           s_warp, &s_y);
    }
    if (threadIdx.x == 0) {
        int* acc = accepted + (size_t)b * n_q;
        for (int j = 0; j < n; ++j) acc[j] = tok[j + 1];
        acc[n] = y < 0 ? 0 : y;
        for (int j = n + 1; j < n_q; ++j) acc[j] = -1;
        n_accepted[b] = n + 1;
    }
}

}  // namespace wmtp
