// loop_kernels.cuh -- device-side bookkeeping of the speculative decode loop: the ring append
// at a device-given position (which is also the rollback of rejected draft rows) and the commit
// of accepted tokens into the per-request state, so that a whole decode step runs without the
// host reading anything back (and can be captured as one CUDA graph).
#pragma once

#include "device_common.cuh"
#include "ring_accept_kernels.cuh"

namespace wmtp {

// ---------------------------------------------------------------------------------------------
// Ring append at a position (Windowed-MTP, arXiv 2607.21535; Pith verdict,
// referee_report.minor_comments on the App. A pseudocode: ring slots with "+d slack").
// Request b writes rows t in [0, n_new[b]) of k_new/v_new [B, n_max, Hkv, 128] at positions
// pos[b] + t and sets ring_len[b] = pos[b] + n_new[b].  Positions at or past pos[b] that earlier
// calls wrote (draft rows of a rejected speculation) are thereby rolled back: the attention
// calls only read the positions below ring_len.  Only survivors are copied (see
// ring_append_kernel).  pos and n_new are read, ring_len only written, so every CTA may store
// the (same) new length.  A bad pos/n_new (negative, n_new > n_max) flags kStatusDeviceIndex
// and the request is skipped.
__global__ void __launch_bounds__(256)
ring_append_at_kernel(uint4* __restrict__ ring_k, uint4* __restrict__ ring_v,
                      long long* __restrict__ ring_len, const uint4* __restrict__ k_new,
                      const uint4* __restrict__ v_new, const long long* __restrict__ pos,
                      const int* __restrict__ n_new_b, int n_max, int Hkv, int n_sink, int C) {
    pdl_launch_dependents();
    pdl_wait();
    const int b = blockIdx.y;
    const long long L_old = pos[b];
    const int n_new = n_new_b[b];
    if (L_old < 0 || n_new < 0 || n_new > n_max) {
        if (blockIdx.x == 0 && threadIdx.x == 0) flag_status(kStatusDeviceIndex);
        return;
    }
    long long e1 = (long long)n_sink - L_old;
    e1 = e1 < 0 ? 0 : (e1 > n_new ? n_new : e1);
    long long s2 = (long long)n_new - (C - n_sink);
    if (s2 < e1) s2 = e1;
    const long long n_surv = e1 + (n_new - s2);
    constexpr int kChunks = 256 / 16;
    const long long work = n_surv * Hkv * kChunks;
    for (long long w = (long long)blockIdx.x * blockDim.x + threadIdx.x; w < work;
         w += (long long)gridDim.x * blockDim.x) {
        const int chunk = (int)(w % kChunks);
        const long long row = w / kChunks;
        const int h = (int)(row % Hkv);
        const long long j = row / Hkv;
        const long long t = j < e1 ? j : s2 + (j - e1);
        const long long slot = ring_slot_of(L_old + t, n_sink, C);
        const size_t src = (((size_t)b * n_max + (size_t)t) * Hkv + h) * kChunks + chunk;
        const size_t dst = (((size_t)b * Hkv + h) * (size_t)C + (size_t)slot) * kChunks + chunk;
        ring_k[dst] = k_new[src];
        ring_v[dst] = v_new[src];
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) ring_len[b] = L_old + n_new;
}

// ---------------------------------------------------------------------------------------------
// Commit of one verify step's accepted tokens (the greedy rule's output: n_accepted[b] tokens,
// the accepted drafts and the bonus token).  Per request, with T the committed token count:
//   history[b, T + j] = accepted[b, j] for j < n;   append_pos[b] = T;  n_append[b] = n;
//   T += n;  verify_len[b] = T - 1 + n_q_verify;    draft_len[j][b] = T + j (j <= n_draft - 1).
// The last committed token is the next step's verify node 0, which sits at cache position
// T - 1 (the target cache holds the T - 1 tokens before it), hence verify_len.  The next
// step's draft context pass appends the n newly committed tokens' draft rows at append_pos,
// which rolls back the draft forwards' rows of this step.  A count outside [1, n_q] or a
// history overflow flags kStatusDeviceIndex and leaves the request unchanged.
__global__ void __launch_bounds__(128)
spec_commit_kernel(const int* __restrict__ accepted, const int* __restrict__ n_accepted, int B,
                   int n_q, int* __restrict__ history, long long max_tokens,
                   long long* __restrict__ n_tokens, long long* __restrict__ append_pos,
                   int* __restrict__ n_append, int* __restrict__ verify_len, int n_q_verify,
                   int* __restrict__ draft_len, int n_draft) {
    pdl_launch_dependents();
    pdl_wait();
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= B) return;
    const int n = n_accepted[b];
    const long long T = n_tokens[b];
    if (n < 1 || n > n_q || T < 1 || T + n > max_tokens) {
        flag_status(kStatusDeviceIndex);
        return;
    }
    for (int j = 0; j < n; ++j)
        history[(size_t)b * (size_t)max_tokens + (size_t)(T + j)] = accepted[(size_t)b * n_q + j];
    const long long Tn = T + n;
    append_pos[b] = T;
    n_append[b] = n;
    n_tokens[b] = Tn;
    if (verify_len != nullptr) verify_len[b] = (int)(Tn - 1 + n_q_verify);
    if (draft_len != nullptr)
        for (int j = 0; j < n_draft; ++j) draft_len[(size_t)j * B + b] = (int)(Tn + j);
}

}  // namespace wmtp
