/*
 * oracle.c -- plain, slow, fp64 CPU oracle for the Windowed-MTP decode-attention path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the benchmark's CPU
 * baseline leg may load this library.  The CUDA library never links, includes or calls it,
 * and this file includes nothing from the CUDA library: the two share no code.
 *
 * Sources (web pages on arXiv 2607.21535, "Windowed-MTP: Removing the Full-Context Draft-KV
 * Tax at Million-Token Context"):
 *   [verdict]  the Pith verdict page for 2607.21535; the field named after it.
 *   [notes]    the Weekly Paper Notes post "windowed-mtp-draft-kv-tax", TL;DR.
 *   [abstract] the AI field-notes entry for the paper, English abstract.
 *
 * Everything here is the plain definition written out: every output element is an explicit
 * loop over the keys of its key set, with no blocking, splitting or fusion.  Inputs are bf16
 * bit patterns (uint16) widened exactly to double; all arithmetic is double.
 *
 * Parity pins: every function below is pinned by the CPU tests (closed forms, brute force on
 * tiny inputs, invariants).  No function here is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_ERR_ARG -1

/* Exact widening of a bf16 bit pattern: the bf16 bits are the top half of an IEEE float. */
static double bf16_to_double(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------------------------------
 * Ring slot mapping.
 * [verdict, referee_report.minor_comments (App. A pseudocode)]: the windowed draft cache keeps
 * each request's draft KV in a compact ring addressed as "ring_base(r) + logical_pos".  Reading
 * adopted: the first n_sink slots hold the sink positions for good; positions past the sink
 * cycle through the remaining capacity - n_sink slots, so
 *     slot(p) = p                                   if p < n_sink
 *             = n_sink + ((p - n_sink) mod (C - n_sink))   otherwise.
 * ring_base(r) is the request's own [Hkv, C, D] block, so it is an array index below.
 * ---------------------------------------------------------------------------------------- */
long long orc_ring_slot(long long p, int n_sink, int capacity) {
    if (p < 0 || n_sink < 0 || capacity <= n_sink) return -1;
    if (p < n_sink) return p;
    return (long long)n_sink + (p - n_sink) % (long long)(capacity - n_sink);
}

/* Appends n_new tokens per request, ONE AT A TIME IN POSITION ORDER, each to slot(p).
 * Later positions overwrite earlier ones that map to the same slot: that is the definition of
 * a ring, and the survivors emerge from it rather than being computed.
 *   ring_k, ring_v : [B, Hkv, C, D] bf16 bits   (in/out)
 *   ring_len       : [B] logical length before the call; updated to length after it
 *   k_new, v_new   : [B, n_new, Hkv, D] bf16 bits                                        */
int orc_ring_kv_append(uint16_t* ring_k, uint16_t* ring_v, long long* ring_len,
                       const uint16_t* k_new, const uint16_t* v_new,
                       int B, int n_new, int Hkv, int D, int n_sink, int capacity) {
    if (B < 0 || n_new < 0 || Hkv <= 0 || D <= 0 || n_sink < 0 || capacity <= n_sink) return ORC_ERR_ARG;
    for (int b = 0; b < B; ++b) {
        long long L0 = ring_len[b];
        if (L0 < 0) return ORC_ERR_ARG;
        for (int t = 0; t < n_new; ++t) {
            long long p = L0 + t;
            long long slot = orc_ring_slot(p, n_sink, capacity);
            for (int h = 0; h < Hkv; ++h) {
                size_t dst = (((size_t)b * Hkv + h) * (size_t)capacity + (size_t)slot) * (size_t)D;
                size_t src = (((size_t)b * n_new + t) * (size_t)Hkv + h) * (size_t)D;
                for (int d = 0; d < D; ++d) {
                    ring_k[dst + d] = k_new[src + d];
                    ring_v[dst + d] = v_new[src + d];
                }
            }
        }
        ring_len[b] = L0 + n_new;
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------------------------
 * Key sets.
 * [verdict, pith_extraction.key_machinery]: the draft's per-request KV index is truncated to
 * "the first n_sink tokens plus the last W tokens"; the target's verification keeps full
 * attention.  Query i of a call with n_q queries sits at position p_i = L_tot - n_q + i, where
 * L_tot is the request's KV length including this call's tokens, and never sees keys after
 * itself.
 * ---------------------------------------------------------------------------------------- */

/* Window membership of key position j for a request of logical length L_tot (before the
 * causal cut): j in [0, L_tot) and (j < n_sink or j >= L_tot - window). */
int orc_window_member(long long L_tot, long long j, int n_sink, int window) {
    if (j < 0 || j >= L_tot) return 0;
    return (j < (long long)n_sink) || (j >= L_tot - (long long)window);
}

/* Tree visibility inside a verify step: node j is visible from node i when j is i or one of
 * i's ancestors (walk parent links from i to the root; parent[0] = -1, parent[k] < k).
 * [verdict, pith_extraction.forward_implications]: windowing composes with tree-shaped
 * speculation; the verifier attends along the tree's root paths. */
int orc_tree_visible(const int* parent, int n_q, int i, int j) {
    int cur = i;
    int guard = 0;
    while (cur >= 0 && guard <= n_q) {
        if (cur == j) return 1;
        cur = parent[cur];
        ++guard;
    }
    return 0;
}

/* Key-set membership for one (request, query) pair.
 *   mode 0: causal full attention   (native full-context draft; chain verification)
 *   mode 1: sink + recent window, then causal   (windowed draft)
 *   mode 2: tree verification: the committed prefix [0, L) plus the node's root path      */
#define ORC_MODE_CAUSAL 0
#define ORC_MODE_WINDOW 1
#define ORC_MODE_TREE 2
int orc_key_visible(int mode, long long L_tot, int n_q, int i, long long j,
                    int n_sink, int window, const int* parent) {
    long long p_i = L_tot - n_q + i;
    if (j < 0 || j > p_i || j >= L_tot) return 0;
    if (mode == ORC_MODE_CAUSAL) return 1;
    if (mode == ORC_MODE_WINDOW) return orc_window_member(L_tot, j, n_sink, window);
    if (mode == ORC_MODE_TREE) {
        long long L = L_tot - n_q;            /* committed prefix length */
        if (j < L) return 1;
        return orc_tree_visible(parent, n_q, i, (int)(j - L));
    }
    return 0;
}

/* ------------------------------------------------------------------------------------------
 * Attention over a key set, in fp64.
 * For query head h (kv head floor(h / G), G = Hq / Hkv) and query i:
 *     s_j   = sm_scale * <q_h, k_j>               for j in K(i)
 *     o_h   = sum_j exp(s_j - m) v_j / sum_j exp(s_j - m),   m = max_j s_j
 *     lse_h = m + ln sum_j exp(s_j - m)
 * An empty key set yields o = 0 and lse = -inf.
 * [verdict, pith_extraction.key_machinery]: windowing changes only the key set; the keys carry
 * their rotary phase already, so no position-dependent transform is applied here.
 *
 *   q      : [B, n_q, Hq, D] bf16 bits
 *   k, v   : [B, Hkv, Lmax, D] bf16 bits, the LOGICAL key sequence of every request
 *   kv_len : [B] L_tot per request (<= Lmax), including this call's n_q positions
 *   rows   : optional list of n_rows (b, i, h) triples to compute; NULL computes all
 *   out    : [B, n_q, Hq, D] doubles;  lse: [B, n_q, Hq] doubles (only listed rows written)
 * ---------------------------------------------------------------------------------------- */
static void attention_row(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                          const long long* kv_len, long long Lmax, int n_q, int Hq, int Hkv, int D,
                          int mode, int n_sink, int window, const int* tree_parent, double sm_scale,
                          int b, int i, int h, double* out, double* lse, double* s_buf) {
    int G = Hq / Hkv;
    int hk = h / G;
    long long L_tot = kv_len[b];
    const uint16_t* qrow = q + (((size_t)b * n_q + i) * (size_t)Hq + h) * (size_t)D;
    const uint16_t* kbase = k + ((size_t)b * Hkv + hk) * (size_t)Lmax * (size_t)D;
    const uint16_t* vbase = v + ((size_t)b * Hkv + hk) * (size_t)Lmax * (size_t)D;
    const int* parent = tree_parent ? tree_parent + (size_t)b * n_q : NULL;
    double* o = out + (((size_t)b * n_q + i) * (size_t)Hq + h) * (size_t)D;

    double m = -INFINITY;
    for (long long j = 0; j < L_tot; ++j) {
        s_buf[j] = -INFINITY;
        if (!orc_key_visible(mode, L_tot, n_q, i, j, n_sink, window, parent)) continue;
        double dot = 0.0;
        for (int d = 0; d < D; ++d)
            dot += bf16_to_double(qrow[d]) * bf16_to_double(kbase[(size_t)j * D + d]);
        s_buf[j] = sm_scale * dot;
        if (s_buf[j] > m) m = s_buf[j];
    }
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    double* l_out = lse + ((size_t)b * n_q + i) * (size_t)Hq + h;
    if (m == -INFINITY) {               /* empty key set */
        *l_out = -INFINITY;
        return;
    }
    double l = 0.0;
    for (long long j = 0; j < L_tot; ++j) {
        if (s_buf[j] == -INFINITY) continue;
        double w = exp(s_buf[j] - m);
        l += w;
        for (int d = 0; d < D; ++d) o[d] += w * bf16_to_double(vbase[(size_t)j * D + d]);
    }
    for (int d = 0; d < D; ++d) o[d] /= l;
    *l_out = m + log(l);
}

int orc_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                  const long long* kv_len, long long Lmax, int B, int n_q, int Hq, int Hkv, int D,
                  int mode, int n_sink, int window, const int* tree_parent, double sm_scale,
                  const int* rows, int n_rows, double* out, double* lse, int n_threads) {
    if (B <= 0 || n_q <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || Hq % Hkv != 0) return ORC_ERR_ARG;
    if (mode == ORC_MODE_TREE && tree_parent == NULL) return ORC_ERR_ARG;
    for (int b = 0; b < B; ++b)
        if (kv_len[b] < 0 || kv_len[b] > Lmax) return ORC_ERR_ARG;
    long long total = rows ? (long long)n_rows : (long long)B * n_q * Hq;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
    int failed = 0;
#pragma omp parallel
    {
        double* s_buf = (double*)malloc(sizeof(double) * (size_t)(Lmax > 0 ? Lmax : 1));
        if (!s_buf) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (long long r = 0; r < total; ++r) {
                int b, i, h;
                if (rows) {
                    b = rows[3 * r]; i = rows[3 * r + 1]; h = rows[3 * r + 2];
                } else {
                    b = (int)(r / ((long long)n_q * Hq));
                    i = (int)((r / Hq) % n_q);
                    h = (int)(r % Hq);
                }
                attention_row(q, k, v, kv_len, Lmax, n_q, Hq, Hkv, D, mode, n_sink, window,
                              tree_parent, sm_scale, b, i, h, out, lse, s_buf);
            }
            free(s_buf);
        }
    }
    return failed ? ORC_ERR_ARG : ORC_OK;
}

/* ------------------------------------------------------------------------------------------
 * Greedy acceptance.
 * [abstract]; [verdict, pith_extraction.forward_implications]: the full-attention target
 * decides every accepted token; under greedy decoding the output equals the target's own
 * greedy output whatever the draft proposes.
 *   t_i = argmax_v logits[i][v], the lowest index on ties (a strict '>' scan from v = 0).
 *   tokens[0] is the last committed token (the root); tokens[1..] are the drafted tokens.
 *   Chain (tree_parent == NULL): a = largest k with tokens[j] == t_{j-1} for all 1 <= j <= k;
 *     emit tokens[1..a] then the bonus t_a;  n_accepted = a + 1.
 *   Tree: from the root, while some child c has tokens[c] == t_cur, step to the lowest-index
 *     such c; emit the path's tokens then t_cur.
 *   accepted: [B, n_q] padded with -1.
 * ---------------------------------------------------------------------------------------- */
static int argmax_lowest(const float* row, int V) {
    int best = 0;
    float bv = row[0];
    for (int x = 1; x < V; ++x)
        if (row[x] > bv) { bv = row[x]; best = x; }
    return best;
}

int orc_accept_greedy(const float* logits, const int* tokens, const int* tree_parent,
                      int B, int n_q, int V, int* accepted, int* n_accepted) {
    if (B <= 0 || n_q <= 0 || V <= 0) return ORC_ERR_ARG;
    int* t = (int*)malloc(sizeof(int) * (size_t)n_q);
    if (!t) return ORC_ERR_ARG;
    for (int b = 0; b < B; ++b) {
        for (int i = 0; i < n_q; ++i)
            t[i] = argmax_lowest(logits + ((size_t)b * n_q + i) * (size_t)V, V);
        const int* tok = tokens + (size_t)b * n_q;
        int* acc = accepted + (size_t)b * n_q;
        for (int i = 0; i < n_q; ++i) acc[i] = -1;
        int n = 0;
        if (tree_parent == NULL) {
            int a = 0;
            while (a + 1 < n_q && tok[a + 1] == t[a]) ++a;
            for (int j = 1; j <= a; ++j) acc[n++] = tok[j];
            acc[n++] = t[a];
        } else {
            const int* par = tree_parent + (size_t)b * n_q;
            int cur = 0;
            for (;;) {
                int next = -1;
                for (int c = 1; c < n_q; ++c)
                    if (par[c] == cur && tok[c] == t[cur]) { next = c; break; }
                if (next < 0) break;
                acc[n++] = tok[next];
                cur = next;
            }
            acc[n++] = t[cur];
        }
        n_accepted[b] = n;
    }
    free(t);
    return ORC_OK;
}

/* ------------------------------------------------------------------------------------------
 * Stochastic (rejection-sampling) acceptance of a drafted chain.
 * [abstract]: windowing preserves the target's verified output DISTRIBUTION; [verdict,
 * referee_report.significance]: the losslessness is the standard speculative-decoding theorem.
 * The pages do not restate the rule; this is the standard one (Leviathan, Kalman and Matias,
 * "Fast Inference from Transformers via Speculative Decoding", ICML 2023, Algorithm 1; Chen et
 * al., "Accelerating Large Language Model Decoding with Speculative Sampling", 2023):
 *   for drafted token i = 1 .. n_q - 1 (x = tokens[i], proposed from the draft distribution
 *   q_{i-1} = q[i - 1]; the target's distribution at that position is p_{i-1} = p[i - 1]):
 *     accept x with probability min(1, p_{i-1}(x) / q_{i-1}(x));
 *     on the first rejection emit a token drawn from norm(max(0, p_{i-1} - q_{i-1})) and stop;
 *   when every draft is accepted, emit a token drawn from p_{n_q - 1} (the bonus).
 * Randomness is an input and every decision is exact integer/fp64 arithmetic, so two
 * implementations agree bit for bit:
 *   acceptance: u = u_accept[i - 1] in [0, 2^24); accept iff u * q(x) < p(x) * 2^24, both
 *     products exact in double (a 24-bit integer times a float32);
 *   a draw from weights w(v) (w = max(0, p - q) computed in float32, or p): m(v) =
 *     floor(w(v) * 2^40) as a 64-bit integer, M = sum_v m(v), t = floor(u_sample * M / 2^32)
 *     with u_sample a 32-bit integer; emit the smallest v with m(0) + ... + m(v) > t.  If the
 *     residual has M = 0 the draw uses p instead; if that is 0 too it emits token 0.
 * Inputs: p [B, n_q, V] and q [B, n_q - 1, V] float32 probabilities (entries in [0, 1]);
 * tokens [B, n_q] (tokens[0] = last committed token); u_accept [B, n_q - 1] (< 2^24);
 * u_sample [B].  Outputs as orc_accept_greedy.
 * ---------------------------------------------------------------------------------------- */
#define ORC_FIX_SCALE 1099511627776.0   /* 2^40 */

static uint64_t fix40(float w) {
    if (!(w > 0.0f)) return 0;
    return (uint64_t)((double)w * ORC_FIX_SCALE);     /* truncation = floor for w >= 0 */
}

/* The inverse-CDF draw described above over weights w; returns -1 when every m(v) is 0. */
static int draw_fixed(const float* w, int V, uint32_t u_sample) {
    uint64_t M = 0;
    for (int v = 0; v < V; ++v) M += fix40(w[v]);
    if (M == 0) return -1;
    const unsigned __int128 prod = (unsigned __int128)u_sample * (unsigned __int128)M;
    const uint64_t t = (uint64_t)(prod >> 32);
    uint64_t c = 0;
    for (int v = 0; v < V; ++v) {
        c += fix40(w[v]);
        if (c > t) return v;
    }
    return V - 1;   /* not reached: t < M */
}

int orc_accept_stochastic(const float* p, const float* q, const int* tokens,
                          const uint32_t* u_accept, const uint32_t* u_sample,
                          int B, int n_q, int V, int* accepted, int* n_accepted) {
    if (B <= 0 || n_q <= 0 || V <= 0) return ORC_ERR_ARG;
    float* w = (float*)malloc(sizeof(float) * (size_t)V);
    if (!w) return ORC_ERR_ARG;
    for (int b = 0; b < B; ++b) {
        const int* tok = tokens + (size_t)b * n_q;
        int* acc = accepted + (size_t)b * n_q;
        for (int i = 0; i < n_q; ++i) acc[i] = -1;
        int n = 0, rejected_at = -1;
        for (int i = 1; i < n_q; ++i) {
            const int x = tok[i];
            const float* pr = p + ((size_t)b * n_q + (i - 1)) * (size_t)V;
            const float* qr = q + ((size_t)b * (n_q - 1) + (i - 1)) * (size_t)V;
            const double px = (x >= 0 && x < V) ? (double)pr[x] : 0.0;
            const double qx = (x >= 0 && x < V) ? (double)qr[x] : 0.0;
            const double u = (double)u_accept[(size_t)b * (n_q - 1) + (i - 1)];
            if (u * qx < px * 16777216.0) {
                acc[n++] = x;
            } else {
                rejected_at = i;
                break;
            }
        }
        int y;
        if (rejected_at > 0) {
            const float* pr = p + ((size_t)b * n_q + (rejected_at - 1)) * (size_t)V;
            const float* qr = q + ((size_t)b * (n_q - 1) + (rejected_at - 1)) * (size_t)V;
            for (int v = 0; v < V; ++v) {
                const float d = pr[v] - qr[v];
                w[v] = d > 0.0f ? d : 0.0f;
            }
            y = draw_fixed(w, V, u_sample[b]);
            if (y < 0) y = draw_fixed(pr, V, u_sample[b]);
        } else {
            y = draw_fixed(p + ((size_t)b * n_q + (n_q - 1)) * (size_t)V, V, u_sample[b]);
        }
        acc[n++] = y < 0 ? 0 : y;
        n_accepted[b] = n;
    }
    free(w);
    return ORC_OK;
}

/* ------------------------------------------------------------------------------------------
 * fp8 (E4M3) KV.  [verdict, pith_extraction.forward_implications[4]]: windowing composes with
 * KV quantisation (fp8).  The format is OCP 8-bit floating point E4M3 (the "OFP8" specification,
 * 2023): 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent field 0 encodes
 * subnormals (m / 8) * 2^-6; S.1111.111 is NaN; there are no infinities; the largest finite
 * magnitude is 448.  A cached key or value is k_scale (v_scale) times its decoded code; the
 * oracle decodes exactly and folds the scales into sm_scale and the output.
 * ---------------------------------------------------------------------------------------- */
double orc_e4m3_value(unsigned int code) {
    const unsigned int s = (code >> 7) & 1u, e = (code >> 3) & 15u, m = code & 7u;
    double mag;
    if (e == 15u && m == 7u) return NAN;
    if (e == 0u) mag = ldexp((double)m / 8.0, -6);
    else mag = ldexp(1.0 + (double)m / 8.0, (int)e - 7);
    return s ? -mag : mag;
}

void orc_e4m3_decode(const uint8_t* in, size_t n, double* out) {
    for (size_t i = 0; i < n; ++i) out[i] = orc_e4m3_value(in[i]);
}

/* Number of OpenMP threads the oracle would use (1 without OpenMP). */
int orc_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
