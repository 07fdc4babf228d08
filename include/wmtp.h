/*
 * wmtp.h -- C ABI of libwmtp.so: the per-step decode attention of Windowed-MTP speculative
 * decoding on one B200 (sm_100a).
 *
 * Sources (web pages on arXiv 2607.21535, "Windowed-MTP: Removing the Full-Context Draft-KV Tax
 * at Million-Token Context"):
 *   [verdict]  Pith verdict page for 2607.21535, the JSON field named;
 *   [abstract] AI field-notes entry for the paper, English abstract;
 *   [notes]    Weekly Paper Notes post "windowed-mtp-draft-kv-tax", TL;DR.
 *
 * Conventions shared by every call
 *   - Pointers are DEVICE pointers unless stated.  The caller owns all memory; the library
 *     allocates nothing and keeps no state except the device status word (wmtp_device_status).
 *   - bf16 tensors are passed as their 16-bit patterns (wmtp_bf16).  All attention arithmetic
 *     accumulates in fp32; outputs are bf16 (round to nearest even) plus optional fp32 LSE.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the legacy default stream)
 *     and never synchronizes.  Arguments are checked on the host before any launch; a bad
 *     argument returns a negative status and launches nothing.  Launch failures return
 *     WMTP_ERR_CUDA.  Nothing is thrown across the ABI.
 *   - Layouts (row-major, innermost last; D = head_dim = 128):
 *       q, out          [B, n_q, Hq, D]            query head h uses kv head h / (Hq / Hkv)
 *       lse             [B, n_q, Hq]   float       natural-log sum of exp of scaled scores
 *       paged K/V pool  [num_pages, Hkv, P, D]     P = page_size = 64; one 16 KiB block per
 *                                                  (page, kv head)
 *       page_table      [B, max_pages] int32       logical page t of request b -> physical page
 *       ring K/V        [B, Hkv, C, D]             C = ring capacity
 *   - Alignment: every tensor pointer 16-byte aligned; the workspace 256-byte aligned.
 *   - Device-side index problems (a page id outside [0, num_pages)) never trap: the tile is
 *     skipped as if empty and the device status word records WMTP_ERR_DEVICE_INDEX.
 *   - An empty key set (a query whose window or causal cut keeps no key) yields out = 0 and
 *     lse = -inf.
 */
#ifndef WMTP_H
#define WMTP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define WMTP_API __attribute__((visibility("default")))
#else
#define WMTP_API
#endif

typedef uint16_t wmtp_bf16;                 /* bf16 bit pattern */
typedef struct CUstream_st* wmtp_stream_t;  /* identical to cudaStream_t */

enum wmtp_status {
    WMTP_OK = 0,
    WMTP_ERR_ARG = -1,           /* null pointer, negative size, n_sink >= capacity, ...      */
    WMTP_ERR_SHAPE = -2,         /* unsupported shape: D != 128, P != 64, Hq % Hkv != 0, ...  */
    WMTP_ERR_ALIGN = -3,         /* pointer not 16-byte aligned (workspace: 256-byte)        */
    WMTP_ERR_WORKSPACE = -4,     /* workspace smaller than wmtp_workspace_bytes(...)         */
    WMTP_ERR_CUDA = -5,          /* a CUDA runtime/driver call or launch failed              */
    WMTP_ERR_DEVICE_INDEX = -6,  /* (device status only) a page id was out of range          */
    WMTP_ERR_UNSUPPORTED = -7,   /* the current device is not an sm_100 GPU                  */
    WMTP_ERR_TIMEOUT = -8,       /* (device status only) a bounded wait in a kernel gave up   */
    WMTP_ERR_SCRATCH_LIMIT = -9  /* shape needs more scratch than the built-in array holds    */
};

/* Limits checked on the host. */
#define WMTP_HEAD_DIM 128
#define WMTP_PAGE_SIZE 64
#define WMTP_MAX_GROUP 16        /* Hq / Hkv */
#define WMTP_MAX_QUERIES 64      /* n_q per call (chain gamma + 1, or tree nodes) */

/* Human-readable name of a status code (static string; never NULL). */
WMTP_API const char* wmtp_status_string(int status);

/* Bytes of device workspace the attention calls need for this shape on the CURRENT device
 * (a 256-byte control block, then split-KV partial results: one (o, lse) block per CTA per
 * request-head it touches).  The same workspace may be reused by consecutive calls on one
 * stream; calls that may run concurrently need separate workspaces.  Returns 0 for invalid
 * shapes.
 * The control block (the workspace's first 256 bytes) must be zero before the workspace's first
 * use by draft_attn_window_append (allocate it zeroed, e.g. with cudaMemset); every call leaves
 * it zero.  After a call whose device status reports WMTP_ERR_TIMEOUT, zero it again. */
WMTP_API size_t wmtp_workspace_bytes(int B, int n_q, int Hq, int Hkv, int D);

/* ---------------------------------------------------------------------------------------------
 * ring_kv_append -- write new draft K/V rows into the compact per-request ring buffer.
 * [verdict, referee_report.minor_comments (App. A pseudocode)]: the draft KV lives in a ring
 * addressed as ring_base(r) + logical_pos, sized for the sink plus the window (+ slack);
 * [abstract]: the unread draft KV is reclaimed by this compact ring.
 *   Position p of request b goes to slot(p) = p for p < n_sink, else
 *   n_sink + (p - n_sink) mod (capacity - n_sink).  The call appends positions
 *   [L_old, L_old + n_new) with L_old = ring_len[b], writes only the rows that survive the call
 *   (a later position of the same call overwriting a slot wins), and sets
 *   ring_len[b] = L_old + n_new.  n_new larger than capacity - n_sink is legal.
 *   ring_k, ring_v  [B, Hkv, capacity, D] bf16   in/out
 *   ring_len        [B] int64                    in/out (device)
 *   k_new, v_new    [B, n_new, Hkv, D] bf16      in
 *   Errors: WMTP_ERR_ARG (null pointers, n_new < 0, n_sink < 0, capacity <= n_sink),
 *           WMTP_ERR_SHAPE (D != 128), WMTP_ERR_ALIGN, WMTP_ERR_CUDA.  n_new == 0 is a no-op. */
WMTP_API int ring_kv_append(wmtp_bf16* ring_k, wmtp_bf16* ring_v, int64_t* ring_len,
                   const wmtp_bf16* k_new, const wmtp_bf16* v_new,
                   int B, int n_new, int Hkv, int D, int n_sink, int capacity,
                   wmtp_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * draft_attn_window -- the draft head's attention over the attention sink plus the recent
 * window, read from the ring (never a dense mask: at most three contiguous slot ranges).
 * [verdict, pith_extraction.key_machinery]: the draft's per-request KV index keeps the first
 * n_sink tokens plus the last W tokens; keys carry their rotary phase already (or none: NoPE),
 * so the kept scores are unchanged.  [verdict, one_line_summary]: a "4K sink-plus-recent window".
 *   With L_tot = ring_len[b] (the request's draft length INCLUDING this call's n_q positions,
 *   i.e. after ring_kv_append), query i sits at position p_i = L_tot - n_q + i and attends to
 *   keys j <= p_i with j < n_sink or j >= L_tot - window.
 *   Requires window <= capacity - n_sink (the ring must hold the window).
 *   q          [B, n_q, Hq, D] bf16;  ring_k/ring_v [B, Hkv, capacity, D] bf16
 *   ring_len   [B] int64 (device)
 *   out        [B, n_q, Hq, D] bf16;  lse [B, n_q, Hq] float or NULL
 *   ws         device workspace of ws_bytes >= wmtp_workspace_bytes(B, n_q, Hq, Hkv, D)
 *   Errors: WMTP_ERR_ARG, WMTP_ERR_SHAPE (D != 128, Hq % Hkv, G > 16, n_q > 64),
 *           WMTP_ERR_ALIGN, WMTP_ERR_WORKSPACE, WMTP_ERR_CUDA. */
WMTP_API int draft_attn_window(const wmtp_bf16* q, const wmtp_bf16* ring_k, const wmtp_bf16* ring_v,
                      const int64_t* ring_len,
                      int B, int n_q, int Hq, int Hkv, int D, int n_sink, int window,
                      int capacity, float sm_scale,
                      wmtp_bf16* out, float* lse, void* ws, size_t ws_bytes,
                      wmtp_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * draft_attn_window_append -- one draft forward in one launch: ring_kv_append of the call's new
 * rows followed by draft_attn_window, with identical results.
 * [verdict, pith_extraction.key_machinery]: each draft forward writes its token's draft KV and
 * attends over the sink plus the last W tokens (t_fwd_draft in Eq. 1); [verdict,
 * referee_report.minor_comments (App. A pseudocode)]: the KV goes to the compact ring.
 *   Appends positions [L_old, L_old + n_new) (L_old = ring_len[b]) from k_new / v_new
 *   [B, n_new, Hkv, D] exactly as ring_kv_append does, sets ring_len[b] = L_old + n_new, and
 *   computes draft_attn_window with L_tot = L_old + n_new.  Usually n_new = n_q (the forward's
 *   own tokens).  When 0 < n_new <= window the append happens inside the attention kernel (the
 *   new rows are in the key set, so the CTA that holds a new row's slot writes it); a larger
 *   n_new runs ring_kv_append as a separate kernel first.
 *   ring_k, ring_v, ring_len are in/out; ws as for draft_attn_window, and its control block must
 *   be zero (see wmtp_workspace_bytes).
 *   Errors: those of ring_kv_append and draft_attn_window. */
WMTP_API int draft_attn_window_append(const wmtp_bf16* q, wmtp_bf16* ring_k, wmtp_bf16* ring_v,
                                      int64_t* ring_len, const wmtp_bf16* k_new,
                                      const wmtp_bf16* v_new, int n_new,
                                      int B, int n_q, int Hq, int Hkv, int D, int n_sink, int window,
                                      int capacity, float sm_scale,
                                      wmtp_bf16* out, float* lse, void* ws, size_t ws_bytes,
                                      wmtp_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * draft_attn_full -- the native MTP draft attention it replaces: causal attention over the
 * request's whole paged KV cache.
 * [abstract]; [verdict, pith_extraction.core_discovery]: the shipping draft head runs full
 * attention over the entire KV cache at every draft step, so its read grows with context.
 *   With L_tot = kv_len[b] (including this call's n_q positions), query i attends to keys
 *   j <= L_tot - n_q + i.
 *   k_pool, v_pool  [num_pages, Hkv, 64, D] bf16
 *   page_table      [B, max_pages] int32; kv_len [B] int32 (device)
 *   other arguments as draft_attn_window.
 *   Errors: as draft_attn_window, plus WMTP_ERR_SHAPE for page_size != 64. */
WMTP_API int draft_attn_full(const wmtp_bf16* q, const wmtp_bf16* k_pool, const wmtp_bf16* v_pool,
                    const int32_t* page_table, const int32_t* kv_len,
                    int B, int n_q, int Hq, int Hkv, int D, int page_size, int max_pages,
                    int num_pages, float sm_scale,
                    wmtp_bf16* out, float* lse, void* ws, size_t ws_bytes,
                    wmtp_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * verify_attn -- one target attention layer verifying the drafted tokens with full attention.
 * [verdict, pith_extraction.key_machinery]: the target's verification is untouched by
 * windowing (t_verify in t_step = t_verify + t_ctx_draft + gamma * t_fwd_draft, Eq. 1);
 * [verdict, pith_extraction.forward_implications]: composes with tree-shaped speculation.
 *   The cache already holds the n_q step rows at positions L .. L + n_q - 1, L = kv_len[b] - n_q.
 *   Node i attends to the prefix [0, L) plus the nodes on its root path (itself included).
 *   tree_parent [B, n_q] int32 with parent[0] = -1 and parent[i] < i, or NULL for a chain
 *   (node i's parent is i - 1: plain causal attention).
 *   Other arguments and errors as draft_attn_full. */
WMTP_API int verify_attn(const wmtp_bf16* q, const wmtp_bf16* k_pool, const wmtp_bf16* v_pool,
                const int32_t* page_table, const int32_t* kv_len, const int32_t* tree_parent,
                int B, int n_q, int Hq, int Hkv, int D, int page_size, int max_pages,
                int num_pages, float sm_scale,
                wmtp_bf16* out, float* lse, void* ws, size_t ws_bytes,
                wmtp_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * accept_greedy -- lossless greedy acceptance of a chain or tree of drafted tokens.
 * [abstract]: the full-attention target decides every accepted token; windowing changes only
 * which tokens are proposed.  [verdict, pith_extraction.forward_implications]: greedy-exact.
 *   t_i = argmax_v logits[b, i, v] (lowest index on ties).  tokens[b, 0] is the last committed
 *   token (the root); tokens[b, i > 0] are drafted.  Chain (tree_parent NULL): keep drafts while
 *   tokens[i] == t_{i-1}; tree: from the root, step to the lowest-index child c with
 *   tokens[c] == t_cur.  Emits the kept drafts then the target's token at the last kept node.
 *   logits      [B, n_q, V] float;  tokens [B, n_q] int32;  tree_parent [B, n_q] int32 or NULL
 *   accepted    [B, n_q] int32 out (-1 padded);  n_accepted [B] int32 out (1 .. n_q)
 *   Errors: WMTP_ERR_ARG (null pointers, B/n_q/V < 1, n_q > 64), WMTP_ERR_ALIGN, WMTP_ERR_CUDA. */
WMTP_API int accept_greedy(const float* logits, const int32_t* tokens, const int32_t* tree_parent,
                  int B, int n_q, int V, int32_t* accepted, int32_t* n_accepted,
                  wmtp_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * accept_stochastic -- lossless acceptance of a drafted chain under sampling (rejection rule).
 * [abstract]: the target's verified output distribution is preserved; [verdict,
 * referee_report.significance]: the losslessness is the standard speculative-decoding theorem.
 * The pages do not restate the rule; this is the standard one (Leviathan, Kalman and Matias,
 * ICML 2023; Chen et al., 2023): draft i (x = tokens[b, i], proposed from q[b, i-1, :]) is kept
 * with probability min(1, p[b, i-1, x] / q[b, i-1, x]); at the first rejection one token is drawn
 * from norm(max(0, p[b, i-1, :] - q[b, i-1, :])); when all n_q - 1 drafts are kept, a bonus token
 * is drawn from p[b, n_q-1, :].  The emitted tokens then follow the target's distributions.
 *   Randomness is an input, and every decision is exact integer/double arithmetic (so results
 *   are reproducible bit for bit):  keep iff u_accept[b, i-1] * q(x) < p(x) * 2^24, with
 *   u_accept < 2^24;  a draw over weights w takes m(v) = floor(w(v) * 2^40) as 64-bit integers,
 *   M = sum_v m(v), t = floor(u_sample[b] * M / 2^32), and emits the smallest v whose running sum
 *   m(0) + ... + m(v) exceeds t (weights below 2^-40 are never drawn).  max(0, p - q) is computed
 *   in float32.  A rejection with no residual mass (possible only when p and q do not sum to the
 *   same total) draws from p instead; a row with no mass at all emits token 0.
 *   p         [B, n_q, V] float   target probabilities (entries in [0, 1]) at the n_q positions
 *   q         [B, n_q - 1, V] float   draft probabilities of the drafted positions (NULL if n_q = 1)
 *   tokens    [B, n_q] int32      tokens[b, 0] = last committed token, then the drafts
 *   u_accept  [B, n_q - 1] uint32 (NULL if n_q = 1);  u_sample [B] uint32
 *   accepted  [B, n_q] int32 out (-1 padded);  n_accepted [B] int32 out (1 .. n_q)
 *   A drafted token outside [0, V) is rejected and recorded as WMTP_ERR_DEVICE_INDEX in the
 *   device status word.
 *   Errors: WMTP_ERR_ARG (null pointers, B < 1, n_q < 1, n_q > 64, V < 1, V >= 2^24),
 *           WMTP_ERR_ALIGN, WMTP_ERR_CUDA. */
WMTP_API int accept_stochastic(const float* p, const float* q, const int32_t* tokens,
                               const uint32_t* u_accept, const uint32_t* u_sample,
                               int B, int n_q, int V, int32_t* accepted, int32_t* n_accepted,
                               wmtp_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * fp8 (E4M3) KV variants.  [verdict, pith_extraction.forward_implications[4]]: windowing
 * composes with KV quantisation (fp8), which halves the bytes every attention call streams.
 *   K and V hold OCP E4M3 codes (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; no
 *   infinities), one byte per element, in the layouts of the bf16 calls:
 *       ring K/V [B, Hkv, capacity, 128] uint8;  pools [num_pages, Hkv, 64, 128] uint8.
 *   A key is k_scale times its code's value, a value v_scale times its code's value (one
 *   scale per tensor, > 0).  q, out, lse, the workspace and every other argument are those of
 *   the bf16 call of the same name; the workspace size is the same.  The kernels widen codes
 *   and queries to fp16 exactly and accumulate in fp32, so results match attention over the
 *   dequantised cache to the tolerance of the bf16 calls.  Codes of NaN (S.1111.111) must not
 *   occur in keys or values that a query can see.
 *   Errors: those of the bf16 call, plus WMTP_ERR_ARG for a scale <= 0 or not finite.
 * ring_kv_append_fp8: ring_kv_append on fp8 rows (128 bytes per row and head). */
WMTP_API int ring_kv_append_fp8(uint8_t* ring_k, uint8_t* ring_v, int64_t* ring_len,
                                const uint8_t* k_new, const uint8_t* v_new,
                                int B, int n_new, int Hkv, int D, int n_sink, int capacity,
                                wmtp_stream_t stream);
WMTP_API int draft_attn_window_fp8(const wmtp_bf16* q, const uint8_t* ring_k, const uint8_t* ring_v,
                                   const int64_t* ring_len,
                                   int B, int n_q, int Hq, int Hkv, int D, int n_sink, int window,
                                   int capacity, float sm_scale, float k_scale, float v_scale,
                                   wmtp_bf16* out, float* lse, void* ws, size_t ws_bytes,
                                   wmtp_stream_t stream);
/* draft_attn_window_append_fp8: draft_attn_window_append on fp8 rings and fp8 new rows. */
WMTP_API int draft_attn_window_append_fp8(const wmtp_bf16* q, uint8_t* ring_k, uint8_t* ring_v,
                                          int64_t* ring_len, const uint8_t* k_new,
                                          const uint8_t* v_new, int n_new,
                                          int B, int n_q, int Hq, int Hkv, int D, int n_sink,
                                          int window, int capacity, float sm_scale, float k_scale,
                                          float v_scale, wmtp_bf16* out, float* lse, void* ws,
                                          size_t ws_bytes, wmtp_stream_t stream);
WMTP_API int draft_attn_full_fp8(const wmtp_bf16* q, const uint8_t* k_pool, const uint8_t* v_pool,
                                 const int32_t* page_table, const int32_t* kv_len,
                                 int B, int n_q, int Hq, int Hkv, int D, int page_size, int max_pages,
                                 int num_pages, float sm_scale, float k_scale, float v_scale,
                                 wmtp_bf16* out, float* lse, void* ws, size_t ws_bytes,
                                 wmtp_stream_t stream);
WMTP_API int verify_attn_fp8(const wmtp_bf16* q, const uint8_t* k_pool, const uint8_t* v_pool,
                             const int32_t* page_table, const int32_t* kv_len,
                             const int32_t* tree_parent,
                             int B, int n_q, int Hq, int Hkv, int D, int page_size, int max_pages,
                             int num_pages, float sm_scale, float k_scale, float v_scale,
                             wmtp_bf16* out, float* lse, void* ws, size_t ws_bytes,
                             wmtp_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * draft_attn_window_noalloc -- draft_attn_window without a caller-supplied workspace.
 * The paper has no counterpart: this entry point exists for callers that cannot allocate device
 * memory on their decode path -- engines that plan every buffer at start-up and forbid later
 * allocations, or latency-critical loops that cannot afford cudaMalloc's implicit device
 * synchronisation -- and so cannot provide the workspace the other attention calls take.
 *   Arguments, layouts and results are those of draft_attn_window, minus ws / ws_bytes.  The
 *   split partials go to a scratch array compiled into the library: WMTP_NOALLOC_SCRATCH_BYTES
 *   (8 MiB) of device memory that every GPU which loads the library holds until the process
 *   exits.  The call allocates nothing.
 *   Limit: the shape must fit the scratch: (CTAs the call launches, one or two per SM, plus
 *   B * Hkv * ceil(n_q * Hq / Hkv / 64)) partial slots of rows * 516 bytes each, rows =
 *   min(64, n_q * Hq / Hkv).  On a 148-SM B200 a one-query call with 8 query heads per kv head
 *   fits B * Hkv <= 1736, a 4-query call (32 rows) B * Hkv <= 212.  Larger shapes return
 *   WMTP_ERR_SCRATCH_LIMIT and launch nothing.
 *   The first call on each device looks up the scratch array's device address (with that device
 *   current); make that first call before any stream capture.
 *   All calls on one device share the one scratch array and leave their partials in it.  Nothing
 *   in it has to start at zero (each call writes every partial it reads), but two calls whose
 *   kernels overlap on the GPU (different streams, no ordering between them) race on it and
 *   give wrong results: order such calls, or use draft_attn_window with separate workspaces. */
#define WMTP_NOALLOC_SCRATCH_BYTES (8u << 20)
WMTP_API int draft_attn_window_noalloc(const wmtp_bf16* q, const wmtp_bf16* ring_k,
                                       const wmtp_bf16* ring_v, const int64_t* ring_len,
                                       int B, int n_q, int Hq, int Hkv, int D, int n_sink,
                                       int window, int capacity, float sm_scale,
                                       wmtp_bf16* out, float* lse, wmtp_stream_t stream);

/* Number of kernels this library has launched in this process (all devices), for launch
 * accounting by benchmarks.  Never resets. */
WMTP_API uint64_t wmtp_launch_count(void);

/* Reads and clears the device status word on the current device (synchronizes `stream`).
 * Returns WMTP_OK, WMTP_ERR_DEVICE_INDEX, WMTP_ERR_TIMEOUT, or WMTP_ERR_CUDA if the read itself
 * failed. */
WMTP_API int wmtp_device_status(wmtp_stream_t stream);

/* ---------------------------------------------------------------------------------------------
 * wmtp_selftest_wait_timeout -- exercises the library's failure path without a fault (not part
 * of the method).  Launches one CTA whose thread waits on a shared-memory mbarrier that nothing
 * arrives on, with the same bounded spin the kernels use but a limit of `limit_ns` nanoseconds
 * (1 ms .. 2 s); it then sets the timeout bit of the device status word and returns, so the next
 * wmtp_device_status reports WMTP_ERR_TIMEOUT and the context stays usable.
 *   Errors: WMTP_ERR_ARG for a limit outside [1e6, 2e9] ns; WMTP_ERR_CUDA for a launch failure. */
WMTP_API int wmtp_selftest_wait_timeout(uint64_t limit_ns, wmtp_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* WMTP_H */
