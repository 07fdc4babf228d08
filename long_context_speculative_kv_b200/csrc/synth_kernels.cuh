// synth_kernels.cuh -- a synthetic stand-in for the target's and the draft's language-model
// heads, so that the decode loop runs with real acceptance decisions and no trained weights.
// None of this is part of the Windowed-MTP method; it replaces the models whose logits the
// method's acceptance rule consumes.
//
// Target: the logits for the token after a prefix are a fixed function of a seed, the prefix's
// last four tokens and its length (counter-based, through splitmix64: Steele, Lea and Flood,
// "Fast splittable pseudorandom number generators", OOPSLA 2014, the mixing function of their
// SplitMix generator with the golden-ratio increment):
//   h = mix(seed);  h = mix(h ^ (uint32)(t + 1)) for the last four tokens t (oldest first,
//   missing ones = -1);  h = mix(h ^ length);  logit[v] = 2 * (mix(h ^ v) >> 40) / 2^24 - 1,
// which is exact in float32.
// Draft: proposal j extends the prefix by the target's greedy token with probability
// agree24 / 2^24, decided by z = mix(mix(draft_seed ^ length) ^ (uint32)(last + 1)), and by
// (greedy + 1 + mix(z) mod (V - 1)) mod V otherwise.
#pragma once

#include "device_common.cuh"

namespace wmtp {
namespace synth {

__device__ __forceinline__ unsigned long long mix(unsigned long long x) {
    unsigned long long z = x + 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

__device__ __forceinline__ unsigned long long path_hash(unsigned long long seed, const int (&last4)[4],
                                                        long long len) {
    unsigned long long h = mix(seed);
#pragma unroll
    for (int i = 0; i < 4; ++i) h = mix(h ^ (unsigned long long)(unsigned int)(last4[i] + 1));
    return mix(h ^ (unsigned long long)len);
}

__device__ __forceinline__ float logit_of(unsigned long long h, int v) {
    const int k = (int)(mix(h ^ (unsigned long long)v) >> 40);      // 24-bit uniform
    return (float)(2 * k - (1 << 24)) * 5.9604644775390625e-08f;    // exact: |2k - 2^24| < 2^24
}

// Token at offset `back` (1 = last) of the path history[b, :T] ++ ext[0 : n_ext], or -1 before
// its start.
__device__ __forceinline__ int path_token(const int* hist_b, long long T, const int* ext, int n_ext,
                                          int back) {
    if (back <= n_ext) return ext[n_ext - back];
    const long long i = T - (back - n_ext);
    return i >= 0 ? hist_b[i] : -1;
}

// Block-wide argmax of the target logits for hash h: largest value, lowest index on ties.
// 256 threads; red_v/red_i hold 8 entries.
__device__ __forceinline__ int block_argmax(unsigned long long h, int V, float* red_v, int* red_i) {
    float best = -INFINITY;
    int idx = -1;
    for (int v = threadIdx.x; v < V; v += blockDim.x) {
        const float x = logit_of(h, v);
        if (idx < 0 || x > best) { best = x; idx = v; }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, best, off);
        const int oi = __shfl_xor_sync(0xffffffffu, idx, off);
        if (oi >= 0 && (idx < 0 || ob > best || (ob == best && oi < idx))) { best = ob; idx = oi; }
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) { red_v[warp] = best; red_i[warp] = idx; }
    __syncthreads();
    int r = -1;
    if (threadIdx.x == 0) {
        float bv = -INFINITY;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
            const int oi = red_i[w];
            if (oi >= 0 && (r < 0 || red_v[w] > bv || (red_v[w] == bv && oi < r))) { bv = red_v[w]; r = oi; }
        }
    }
    __syncthreads();                       // red_* may be reused by the next call
    return r;                              // valid in thread 0 only
}

// Draft proposals: one CTA (256 threads) per request.  tokens[b, 0] = last committed token,
// tokens[b, 1 + j] = proposal j (j < gamma).
__global__ void __launch_bounds__(256)
draft_tokens_kernel(const int* __restrict__ history, const long long* __restrict__ n_tokens,
                    long long max_tokens, int gamma, int V, unsigned long long target_seed,
                    unsigned long long draft_seed, unsigned int agree24, int* __restrict__ tokens) {
    __shared__ float red_v[8];
    __shared__ int red_i[8];
    __shared__ int ext[WMTP_MAX_QUERIES];
    pdl_launch_dependents();
    pdl_wait();
    const int b = blockIdx.x;
    const long long T = n_tokens[b];
    int* out = tokens + (size_t)b * (gamma + 1);
    if (T < 1 || T > max_tokens) {
        if (threadIdx.x == 0) flag_status(kStatusDeviceIndex);
        for (int j = threadIdx.x; j <= gamma; j += blockDim.x) out[j] = 0;
        return;
    }
    const int* hist_b = history + (size_t)b * (size_t)max_tokens;
    for (int j = 0; j < gamma; ++j) {
        int last4[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) last4[i] = path_token(hist_b, T, ext, j, 4 - i);
        const long long len = T + j;
        const unsigned long long h = path_hash(target_seed, last4, len);
        const int greedy = block_argmax(h, V, red_v, red_i);
        if (threadIdx.x == 0) {
            const unsigned long long z =
                mix(mix(draft_seed ^ (unsigned long long)len) ^ (unsigned long long)(unsigned int)(last4[3] + 1));
            const bool agree = (unsigned int)(z >> 40) < agree24;
            const int r = (int)(mix(z) % (unsigned long long)(V - 1));
            ext[j] = agree ? greedy : (greedy + 1 + r) % V;
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) out[0] = hist_b[T - 1];
    for (int j = threadIdx.x; j < gamma; j += blockDim.x) out[1 + j] = ext[j];
}

// Target logits of every verify node: grid (n_q, B), 256 threads.  Node 0 is the last committed
// token (prefix = history[b, :T]); node i > 0 extends its parent's prefix by tokens[b, i]
// (chain: parent i - 1).  logits [B, n_q, V].
__global__ void __launch_bounds__(256)
target_logits_kernel(const int* __restrict__ history, const long long* __restrict__ n_tokens,
                     long long max_tokens, const int* __restrict__ tokens,
                     const int* __restrict__ tree_parent, int n_q, int V,
                     unsigned long long target_seed, float* __restrict__ logits) {
    __shared__ unsigned long long s_h;
    pdl_launch_dependents();
    pdl_wait();
    const int i = blockIdx.x, b = blockIdx.y;
    const long long T = n_tokens[b];
    float* row = logits + ((size_t)b * n_q + i) * (size_t)V;
    if (T < 1 || T > max_tokens) {
        if (threadIdx.x == 0) flag_status(kStatusDeviceIndex);
        for (int v = threadIdx.x; v < V; v += blockDim.x) row[v] = 0.f;
        return;
    }
    if (threadIdx.x == 0) {
        // the path's own tokens after history[:T], root-side first
        int path[WMTP_MAX_QUERIES];
        int n = 0;
        int cur = i;
        bool bad = false;
        while (cur > 0 && n < WMTP_MAX_QUERIES) {
            path[n++] = tokens[(size_t)b * n_q + cur];
            const int p = tree_parent ? tree_parent[(size_t)b * n_q + cur] : cur - 1;
            if (p < 0 || p >= cur) { bad = true; break; }
            cur = p;
        }
        if (bad) flag_status(kStatusDeviceIndex);
        for (int a = 0, z = n - 1; a < z; ++a, --z) { const int t = path[a]; path[a] = path[z]; path[z] = t; }
        const int* hist_b = history + (size_t)b * (size_t)max_tokens;
        int last4[4];
        for (int k = 0; k < 4; ++k) last4[k] = path_token(hist_b, T, path, n, 4 - k);
        s_h = path_hash(target_seed, last4, T + n);
    }
    __syncthreads();
    const unsigned long long h = s_h;
    for (int v = threadIdx.x; v < V; v += blockDim.x) row[v] = logit_of(h, v);
}

}  // namespace synth
}  // namespace wmtp
