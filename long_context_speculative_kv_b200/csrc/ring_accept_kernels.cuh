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
// Grid (chunks, B), 256 threads; each thread moves 16-byte pieces of 256-byte rows.
__device__ __forceinline__ long long ring_slot_of(long long p, int s, int C) {
    return p < s ? p : (long long)s + (p - s) % (long long)(C - s);
}

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
    constexpr int kChunks = 256 / 16;                        // 16-byte pieces per row
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
