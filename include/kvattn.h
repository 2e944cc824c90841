/*
 * kvattn.h -- C ABI of the B200 (sm_100a) RoPE + grouped-query KV-cache
 * attention library (libkvattn.so).
 *
 * Scope: causal attention of new queries over a KV cache, with RoPE applied
 * to q and k only (plain, PI, NTK, YaRN and dynamic-NTK frequency scaling and
 * the YaRN cos/sin temperature), MHA / GQA / MQA head grouping, the
 * lightning-indexer top-k + sparse latent-row decode, and the block-level
 * (4-token group) indexer + sparse GQA decode.  Sources are cited per
 * entry point by page title and section:
 *   "Agentic RL 入门3：transformer 架构"        (RoPE §1.1-1.2, GQA §2.1, DSA §2.2, MLA §2.3)
 *   "注意力变体与 MoE"                         (KV cache, decode roofline, GQA attention())
 *   "attention"                               (GroupQueryAttention; DSA ①②③; QSA §3)
 *   "注意力机制进化史：从MHA、MQA、GQA、MLA到NSA、MoBA！" (KV cache append, layer_past)
 *
 * Conventions (all entry points):
 *  - Tensors are caller-owned DEVICE memory unless stated otherwise.  The
 *    library never allocates or frees device memory; scratch space is the
 *    caller's `workspace`, sized by the matching *_workspace_bytes() query.
 *  - bf16 values are passed as their 16-bit patterns (kvattn_bf16).
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the
 *    legacy default stream) and never synchronises the host.
 *  - Every pointer to a tensor must be 16-byte aligned; the innermost
 *    dimension is contiguous.  Shapes are in elements.
 *  - Return value: KVATTN_OK (0) or a negative KVATTN_ERR_* code, with a
 *    message in kvattn_last_error_string() (thread-local).  Argument errors
 *    are detected on the host before anything is launched; on error nothing
 *    is written.
 *  - Values that only the device can see (positions, sequence lengths, top-k
 *    indices) are range-checked inside the kernels: an out-of-range value is
 *    never dereferenced; it is clamped or skipped as each entry point states,
 *    and, when `dev_status` is non-NULL, the matching KVATTN_STATUS_* bit is
 *    OR-ed into *dev_status (a device int32 the caller zeroes).
 *  - Inputs are read-only unless the entry point says it writes them.
 */
#ifndef KVATTN_H
#define KVATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t kvattn_bf16; /* bf16 bit pattern */

/* ---- status ------------------------------------------------------------ */
#define KVATTN_OK 0
#define KVATTN_ERR_NULL (-1)        /* a required pointer is NULL */
#define KVATTN_ERR_ALIGN (-2)       /* a pointer or stride breaks the 16-byte rule */
#define KVATTN_ERR_SHAPE (-3)       /* inconsistent or out-of-range sizes */
#define KVATTN_ERR_UNSUPPORTED (-4) /* valid but not implemented (e.g. head_dim) */
#define KVATTN_ERR_CUDA (-5)        /* a CUDA runtime/driver call failed */
#define KVATTN_ERR_WORKSPACE (-6)   /* workspace NULL or smaller than required */

/* Device-side status bits (OR-ed into *dev_status). */
#define KVATTN_STATUS_BAD_POSITION 0x1 /* a RoPE position outside [0, max_pos) */
#define KVATTN_STATUS_BAD_LENGTH 0x2   /* a sequence length outside [0, T_max] */
#define KVATTN_STATUS_BAD_INDEX 0x4    /* a top-k index outside [-1, L_max) */
#define KVATTN_STATUS_NAN_SCORE 0x8    /* an indexer score was NaN */
#define KVATTN_STATUS_TIMEOUT 0x10     /* a pipeline wait ran out of time; outputs are invalid */

/* Message for the last error on the calling thread ("" when none). */
const char* kvattn_last_error_string(void);

/* Library version string. */
const char* kvattn_version(void);

/*
 * Failure-detection testing.  The pages have no counterpart: this hook exists
 * so that a test can make a pipeline wait run out on the GPU without a fault.
 * Every wait inside the kernels is bounded (about a second of %globaltimer);
 * when one runs out the kernel stops using its pipeline, ORs
 * KVATTN_STATUS_TIMEOUT into *dev_status and returns, and the CUDA context
 * stays usable.  After this call, decode calls made by the calling thread
 * (attn_decode_gqa, attn_decode_gqa_rope, attn_decode_gqa_rope_window) whose
 * group size is at most 32, or whose head_dim is 64, bound each pipeline wait
 * by wait_limit_ns instead (0 = the default), and, when drop_tile >= 0, the
 * first persistent CTA never issues the loads of its tile number drop_tile,
 * so the waits for that tile run out: the call then reports
 * KVATTN_STATUS_TIMEOUT, its outputs are invalid, and the workspace's counter
 * region must be cleared before the workspace is used again.  Nothing is
 * loaded and abandoned; every copy issued completes before the kernel returns.
 * kvattn_test_decode_stall(-1, 0) restores normal operation.
 * Errors: KVATTN_ERR_SHAPE (drop_tile < -1, or a limit outside 0 .. 10 s).
 */
int kvattn_test_decode_stall(int drop_tile, long long wait_limit_ns);

/* ---- RoPE ----------------------------------------------------------------
 * "Agentic RL 入门3：transformer 架构" §1.1 (rotation R(m, theta_i),
 * theta_i = base^(-2i/d)), §1.2 ① PI, ② NTK-aware, ③ YaRN (NTK-by-parts
 * ramp and attention temperature), ④ dynamic NTK.
 */
#define KVATTN_ROPE_NONE 0    /* theta_i = base^(-2i/d) */
#define KVATTN_ROPE_PI 1      /* position m -> m / s */
#define KVATTN_ROPE_NTK 2     /* base -> base * s^(d/(d-2)) */
#define KVATTN_ROPE_YARN 3    /* ramp-blended theta, cos/sin x (0.1 ln s + 1) */
#define KVATTN_ROPE_DYN_NTK 4 /* NTK with s = max(1, L_cur / L_train) */

typedef struct kvattn_rope_params {
    int head_dim;   /* d: even, 4 .. 256 */
    int scaling;    /* KVATTN_ROPE_* */
    int pair_style; /* 0: pairs (2i, 2i+1) (default); 1: pairs (i, i + d/2) */
    int reserved;   /* must be 0 */
    double base;    /* RoPE base b (10000, 500000, ...) */
    double s;       /* extension factor s = L_new / L_train (PI, NTK, YaRN); >= 1 */
    double L_train; /* training length (YaRN ramp, dynamic NTK) */
    double alpha;   /* YaRN ramp lower edge (default 1): gamma = 0 for r <= alpha */
    double beta;    /* YaRN ramp upper edge (default 32): gamma = 1 for r > beta */
    double L_cur;   /* current length (dynamic NTK only) */
} kvattn_rope_params;

/*
 * Build the cos/sin table: cos_out[m*(d/2) + i] = mag * cos((m/pdiv) * theta_i),
 * sin_out likewise, for m in [0, max_pos), i in [0, d/2).  theta_i, the
 * position divisor pdiv (s for PI, else 1) and the magnitude mag
 * (0.1 ln s + 1 for YaRN, else 1) follow the scaling mode.  Angles are formed
 * and evaluated in fp64 on the device; the table is stored as fp32.
 * cos_out, sin_out: device fp32 [max_pos][d/2], written.  Errors:
 * KVATTN_ERR_NULL, _SHAPE (max_pos < 1, bad d, s < 1, beta <= alpha,
 * L_train <= 0 where needed), _UNSUPPORTED (unknown scaling or pair_style).
 */
int rope_table_build(const kvattn_rope_params* params, int max_pos, float* cos_out, float* sin_out,
                     void* stream);

/*
 * Rotate q and k IN PLACE with a table from rope_table_build (v is never
 * rotated: position enters only the score, §1.1 last paragraph).
 * Each of q and k is a 4-D view [nb][nt][nh][d] with element (b,t,h,j) at
 * x[b*sb + t*st + h*sh + j] (strides in elements, multiples of 8), and
 * positions pos[b*nt + t] (device int32).  Examples: decode queries
 * [B][H][d] -> (B, 1, H, d, H*d, 0, d); a cache [B][Hk][T][d] ->
 * (B, T, Hk, d, Hk*T*d, d, T*d); prefill queries [B][T][H][d] ->
 * (B, T, H, d, T*H*d, H*d, d).  Either of q or k may be NULL (skipped).
 * For pair (a, b) with table entries (c, s): (x_a, x_b) ->
 * (x_a c - x_b s, x_a s + x_b c), computed in fp32, stored as bf16 (RNE).
 * A position outside [0, max_pos) leaves that vector unchanged and sets
 * KVATTN_STATUS_BAD_POSITION.  head_dim: multiple of 16, <= 256; each of q and k
 * fewer than 2^31 chunks of 8 elements (KVATTN_ERR_SHAPE otherwise).
 */
int rope_apply_qk(kvattn_bf16* q, int q_nb, int q_nt, int q_nh, int64_t q_sb, int64_t q_st,
                  int64_t q_sh, const int32_t* q_pos, kvattn_bf16* k, int k_nb, int k_nt, int k_nh,
                  int64_t k_sb, int64_t k_st, int64_t k_sh, const int32_t* k_pos,
                  const float* cos_tab, const float* sin_tab, int max_pos, int head_dim,
                  int pair_style, int32_t* dev_status, void* stream);

/* ---- decode over a KV cache -----------------------------------------------
 * One new query per sequence attends to every cached row: "注意力变体与 MoE"
 * (decode reads all cached K/V; GQA attention()), "注意力机制进化史" (KV cache
 * layer_past append), "attention" GroupQueryAttention (query head h uses KV
 * head h / g, g = n_head / n_kv_head; n_kv_head = n_head is MHA, 1 is MQA).
 *
 * q [B][n_head][d]; k_cache, v_cache [B][n_kv_head][T_max][d] with rows
 * 0 .. seq_lens[b]-1 valid (rows past the length are never used, whatever
 * they hold); seq_lens device int32 [B].
 * out [B][n_head][d] bf16 = softmax(scale * q k^T) v;
 * lse [B][n_head] fp32 (natural log of the sum of exp(scale * q.k)), or NULL.
 * A sequence of length 0 gives out = 0 and lse = -inf.  A length outside
 * [0, T_max] is clamped into it and sets KVATTN_STATUS_BAD_LENGTH.
 * workspace: device scratch of attn_decode_gqa_workspace_bytes(...) bytes
 * (256-byte aligned).  Its first KVATTN_DECODE_WS_ZERO_BYTES bytes hold one
 * counter per (batch, KV head) pair -- how many pieces of a split pair have
 * finished, so that the CTA finishing the last one merges the pair -- and
 * must be zero before the first call on the workspace (cudaMemsetAsync once);
 * every call leaves them zero again, except one that sets
 * KVATTN_STATUS_TIMEOUT, after which they must be cleared before reuse.  The
 * rest of the workspace needs no initialisation.  Calls that share a
 * workspace must be ordered (one stream, or events).
 * Supported: head_dim in {64, 128}; n_head % n_kv_head == 0 with
 * g = n_head / n_kv_head in {1, 2, 4, 8, 16, 32, 64}; T_max >= 1;
 * B * n_kv_head <= KVATTN_DECODE_WS_ZERO_BYTES / 4.
 */
#define KVATTN_DECODE_WS_ZERO_BYTES (64u << 10)
size_t attn_decode_gqa_workspace_bytes(int B, int n_head, int n_kv_head, int head_dim, int T_max);

int attn_decode_gqa(const kvattn_bf16* q, const kvattn_bf16* k_cache, const kvattn_bf16* v_cache,
                    const int32_t* seq_lens, int B, int n_head, int n_kv_head, int head_dim,
                    int T_max, float scale, kvattn_bf16* out, float* lse, void* workspace,
                    size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * attn_decode_gqa on queries that are not yet rotated: q [B][n_head][d] holds
 * the raw projections, and each sequence's query is rotated inside the decode
 * kernel at position q_pos[b] (device int32 [B]) with the tables of
 * rope_table_build (cos_tab, sin_tab [max_pos][d/2], pair_style as in
 * rope_apply_qk) -- RoPE on q only, never on v ("Agentic RL 入门3" §1.1), the
 * cached keys having been rotated when they were written.  q is not modified.
 * The rotation is bit-identical to rope_apply_qk's, so the result equals
 * rope_apply_qk on q followed by attn_decode_gqa, in one launch.  A position
 * outside [0, max_pos) sets KVATTN_STATUS_BAD_POSITION and that sequence's
 * query is used unrotated.  Workspace, outputs and limits as attn_decode_gqa;
 * the tables must be 16-byte aligned.
 */
int attn_decode_gqa_rope(const kvattn_bf16* q, const int32_t* q_pos, const float* cos_tab,
                         const float* sin_tab, int max_pos, int pair_style, const kvattn_bf16* k_cache,
                         const kvattn_bf16* v_cache, const int32_t* seq_lens, int B, int n_head,
                         int n_kv_head, int head_dim, int T_max, float scale, kvattn_bf16* out,
                         float* lse, void* workspace, size_t workspace_bytes, int32_t* dev_status,
                         void* stream);

/*
 * Append the new token's key and value to the cache: "注意力机制进化史" (KV
 * cache: the new k, v are concatenated to layer_past) with the key rotated at
 * its own position first ("Agentic RL 入门3" §1.1: RoPE on k, not on v).
 * k_new, v_new [B][n_kv_head][d] bf16; pos device int32 [B]: the slot the
 * token takes, which is also its rotation position (normally the length before
 * the append).  Writes k_cache[b][h][pos[b]] = RoPE(k_new[b][h], pos[b]) and
 * v_cache[b][h][pos[b]] = v_new[b][h] for every KV head; nothing else in the
 * caches changes.  The rotation is bit-identical to rope_apply_qk's.  A slot
 * outside [0, T_max) or a position outside [0, max_pos) sets
 * KVATTN_STATUS_BAD_POSITION and that sequence is left as it was.  The caller
 * advances its lengths.  head_dim a multiple of 16, at most 256; all pointers
 * 16-byte aligned.
 */
int kv_append_rope(const kvattn_bf16* k_new, const kvattn_bf16* v_new, const int32_t* pos, int B,
                   int n_kv_head, int head_dim, kvattn_bf16* k_cache, kvattn_bf16* v_cache, int T_max,
                   const float* cos_tab, const float* sin_tab, int max_pos, int pair_style,
                   int32_t* dev_status, void* stream);

/* ---- sliding window with attention sinks over a rolling cache ----------------
 * "Agentic RL 入门3" §1 (sliding-window attention: a query sees the last w
 * keys; the first s tokens kept as attention sinks), the band mask of the
 * "attention" page: the query at position i sees keys j with i - w < j <= i
 * and the s first tokens.  A rolling cache of capacity T_max >= n_sink + window
 * rows per (batch, KV head) keeps the token at position p in slot p if
 * p < n_sink, else in slot n_sink + (p - n_sink) mod window; after len tokens
 * its first min(len, n_sink + window) slots hold tokens 0 .. n_sink-1 and the
 * last window tokens (each key rotated at its own position, so slot order does
 * not matter to attention).
 *
 * kv_append_rope_ring: kv_append_rope into that layout (pos[b] = the token's
 * position; its slot follows from it).
 * attn_decode_gqa_rope_window: attn_decode_gqa_rope over such a cache, with
 * seq_lens[b] = tokens appended so far (any value >= 0, not limited by T_max):
 * attention runs over the min(seq_lens[b], n_sink + window) filled slots.
 * Both: n_sink >= 0, window >= 1, n_sink + window <= T_max; otherwise as their
 * linear-cache counterparts.
 */
int kv_append_rope_ring(const kvattn_bf16* k_new, const kvattn_bf16* v_new, const int32_t* pos, int n_sink,
                        int window, int B, int n_kv_head, int head_dim, kvattn_bf16* k_cache,
                        kvattn_bf16* v_cache, int T_max, const float* cos_tab, const float* sin_tab,
                        int max_pos, int pair_style, int32_t* dev_status, void* stream);

int attn_decode_gqa_rope_window(const kvattn_bf16* q, const int32_t* q_pos, const float* cos_tab,
                                const float* sin_tab, int max_pos, int pair_style, const kvattn_bf16* k_cache,
                                const kvattn_bf16* v_cache, const int32_t* seq_lens, int n_sink, int window,
                                int B, int n_head, int n_kv_head, int head_dim, int T_max, float scale,
                                kvattn_bf16* out, float* lse, void* workspace, size_t workspace_bytes,
                                int32_t* dev_status, void* stream);

/*
 * attn_decode_gqa for callers that cannot allocate device memory.  The pages
 * have no counterpart to this entry point; it exists for callers that cannot
 * give the library a workspace: code running inside another runtime's fixed
 * memory pool (which owns the device and forbids cudaMalloc behind its back),
 * code on a latency-critical path where cudaMalloc would implicitly
 * synchronise the device, and plain C callers with no allocator of their own.
 * Same arguments, layout and results as attn_decode_gqa, minus the workspace:
 * the scratch lives in a file-scope device array of
 * KVATTN_NOALLOC_SCRATCH_BYTES that every GPU loading the library holds until
 * the process exits.  The call allocates nothing (no cudaMalloc, cudaFree or
 * allocating library routine).  A shape whose scratch need
 * (attn_decode_gqa_workspace_bytes) exceeds the array is rejected with
 * KVATTN_ERR_WORKSPACE.  The first call on a device looks the array's device
 * address up (cudaGetSymbolAddress); make that first call before any stream
 * capture.  All calls on a device share the one array: it starts zeroed, as
 * the counter region at its start requires, and every call leaves that region
 * zero, except one that reports KVATTN_STATUS_TIMEOUT: after it, call
 * attn_decode_gqa_noalloc_reset before the next call on that device.  Calls
 * that can overlap on the GPU -- different streams, or graphs replayed
 * concurrently -- race and corrupt each other's results.
 */
#define KVATTN_NOALLOC_SCRATCH_BYTES (8u << 20)

/*
 * Zero the counter region (the first KVATTN_DECODE_WS_ZERO_BYTES) of the
 * static array that attn_decode_gqa_noalloc uses, on the current device, as an
 * asynchronous memset on `stream`; it allocates nothing.  Needed only after a
 * call that reported KVATTN_STATUS_TIMEOUT.  The array's device address is
 * looked up once per device and kept for the life of the process, so neither
 * entry point may be used on a device after cudaDeviceReset.
 */
int attn_decode_gqa_noalloc_reset(void* stream);

int attn_decode_gqa_noalloc(const kvattn_bf16* q, const kvattn_bf16* k_cache, const kvattn_bf16* v_cache,
                            const int32_t* seq_lens, int B, int n_head, int n_kv_head, int head_dim,
                            int T_max, float scale, kvattn_bf16* out, float* lse, int32_t* dev_status,
                            void* stream);

/* ---- causal prefill ---------------------------------------------------------
 * softmax(scale * q k^T + M) v with the lower-triangular mask M (key j is
 * visible to query i iff j <= i): "注意力变体与 MoE" attention() (triu(1)
 * filled with -inf), grouped as in decode.
 * q [B][T][n_head][d]; k, v [B][n_kv_head][T][d]; out [B][T][n_head][d] bf16;
 * lse [B][n_head][T] fp32 or NULL.  Supported: head_dim 128; g as in decode.
 */
int attn_prefill_causal(const kvattn_bf16* q, const kvattn_bf16* k, const kvattn_bf16* v, int B,
                        int T, int n_head, int n_kv_head, int head_dim, float scale,
                        kvattn_bf16* out, float* lse, void* stream);

/* ---- merge of decode results over disjoint key sets ---------------------------
 * The softmax over a union of key sets from the softmax over each set: with
 * LSE = ln sum_j exp(lse_j), out = sum_j exp(lse_j - LSE) o_j and lse = LSE (the
 * split/merge identity the split-K decode uses inside one call).  This is the last
 * step of a sequence-sharded decode: each GPU (or each call) runs attn_decode_gqa
 * over one slice of a long cache, the slices' (out, lse) are exchanged once
 * (all-gather), and every rank merges them.  A part with no keys (lse = -inf)
 * has weight 0; if every part is empty, out = 0 and lse = -inf.
 * o_parts [n_parts][B][n_head][head_dim] bf16 (16-byte aligned); lse_parts
 * [n_parts][B][n_head] fp32; out [B][n_head][head_dim] bf16; lse [B][n_head] fp32
 * or NULL.  Supported: head_dim in {64, 128}.
 */
int attn_merge_lse(const kvattn_bf16* o_parts, const float* lse_parts, int n_parts, int B, int n_head, int head_dim,
                   kvattn_bf16* out, float* lse, void* stream);

/*
 * attn_prefill_causal with a sliding window and attention sinks (the band
 * mask of the "attention" page, "Agentic RL 入门3" §1 sinks): query row i sees
 * key j iff j <= i and (j > i - window or j < n_sink).  Key tiles entirely
 * outside every row's set are skipped.  window >= 1, n_sink >= 0; otherwise as
 * attn_prefill_causal.
 */
int attn_prefill_causal_window(const kvattn_bf16* q, const kvattn_bf16* k, const kvattn_bf16* v, int B,
                               int T, int n_head, int n_kv_head, int head_dim, int n_sink, int window,
                               float scale, kvattn_bf16* out, float* lse, void* stream);

/* ---- lightning indexer + top-k ---------------------------------------------
 * "Agentic RL 入门3" §2.2 (1): s_{b,t} = sum_{j < H_I} w[b][j] *
 * ReLU(q_idx[b][j] . k_idx[b][t]) (no scale, no RoPE); §2.2 (2): S_b =
 * TopK_t(s_{b,t}); "attention" DSA ① (64 heads, one key shared by all heads).
 * q_idx [B][H_I][d_I] bf16; w [B][H_I] fp32; k_idx [B][L_max][d_I] bf16;
 * seq_lens device int32 [B] or NULL (= L_max for every row).
 * topk_idx [B][k] int32: the k largest scores of row b under the order
 * (score descending, index ascending) -- ties go to the lower index --
 * listed in increasing index order; min(k, len) entries, then -1.  The
 * selection is made on the fp32 scores the kernel computed; scores_out
 * [B][L_max] fp32 receives them (-inf past each length) when non-NULL.
 * workspace: dsa_index_topk_workspace_bytes(...) bytes, 256-byte aligned, always
 * required.  Its first 8 KiB per row (B * 2048 counters, the histogram of the top-k's
 * first radix digit, which the indexer fills as it scores and the top-k reads instead
 * of a pass of its own) and the B counters after them (rounded up to 256 bytes: the key
 * tiles of each row the indexer's CTAs have claimed) must be zero before the first call
 * on the workspace (cudaMemsetAsync once); every call leaves them zero, except one that
 * sets KVATTN_STATUS_TIMEOUT.  The rest (the scores, when scores_out is NULL) needs no
 * initialisation.  Calls that share a workspace must be ordered.
 * Supported: H_I = 64, d_I = 128, 1 <= k <= 2048, 1 <= L_max <= 131072.
 */
size_t dsa_index_topk_workspace_bytes(int B, int L_max, int k);

int dsa_index_topk(const kvattn_bf16* q_idx, const float* w, const kvattn_bf16* k_idx,
                   const int32_t* seq_lens, int B, int n_idx_head, int idx_dim, int L_max, int k,
                   int32_t* topk_idx, float* scores_out, void* workspace, size_t workspace_bytes,
                   int32_t* dev_status, void* stream);

/* ---- the lightning indexer sharded over L ------------------------------------------
 * "稀疏注意力：省了什么，没省什么" (改进一: the indexer still scores every earlier token,
 * O(L) per query -- the part of DSA that grows with the context) and "Agentic RL 入门3"
 * §2.2 (2) (S = TopK(s)).  With the keys of a row cut into slices, slice p holding
 * global positions [p * S, p * S + L_slice), each slice keeps its own top-k
 * (dsa_index_topk over its keys) and the global top-k is the top-k of the union of
 * those candidates: an element of the global top-k is beaten by fewer than k keys of
 * its own slice.  The scores of a token do not depend on the slicing, so the merged
 * selection is the one dsa_index_topk makes over the whole row, ties included.
 *
 * dsa_topk_candidates: one slice's selection as (score, global index) pairs:
 * scores [B][L_slice] (that call's scores_out), topk_idx [B][k] (its selection, local
 * indices) -> cand_scores [B][k] = scores[b][topk_idx], cand_idx [B][k] = topk_idx +
 * idx_offset; -1 entries give (-inf, -1).
 * dsa_topk_merge: cand_scores, cand_idx [n_parts][B][k] (the slices' candidates in
 * slice order, as an all-gather concatenates them) -> topk_idx [B][k]: the k best
 * valid candidates of each row under (score descending, index ascending), listed in
 * increasing index order, -1 padded -- exactly dsa_index_topk's output format.  The
 * parts must come in increasing slice order, each part's indices in increasing order
 * (as dsa_index_topk emits them).  NaN scores are never selected (KVATTN_STATUS_NAN_SCORE).
 * Limits: 1 <= k <= 2048, n_parts * k <= 49152.
 */
int dsa_topk_candidates(const float* scores, const int32_t* topk_idx, int B, int L_slice, int k, int idx_offset,
                        float* cand_scores, int32_t* cand_idx, void* stream);

int dsa_topk_merge(const float* cand_scores, const int32_t* cand_idx, int n_parts, int B, int k,
                   int32_t* topk_idx, int32_t* dev_status, void* stream);

/* ---- sparse latent-row decode -------------------------------------------------
 * "Agentic RL 入门3" §2.2 (2) o = MLA(q, {k_j, v_j : j in S}); "attention"
 * DSA ② (after weight absorption every query head reads the same single-head
 * latent rows: MQA over the selected rows) and the "乘法结合律" note
 * ([1,128,576] queries).  Key row j = latent[b][j][0 .. Dk-1]; value row
 * j = latent[b][j][0 .. Dv-1] (K and V share the latent, §2.3.5).
 * q [B][Hq][Dk] bf16; latent [B][L_max][Dk] bf16; topk_idx [B][k] int32
 * (-1 = unused slot; other values outside [0, L_max) are skipped and set
 * KVATTN_STATUS_BAD_INDEX).  out [B][Hq][Dv] bf16; lse [B][Hq] fp32 or NULL.
 * A row with no valid index gives out = 0, lse = -inf.
 * workspace: attn_decode_sparse_workspace_bytes(...) bytes (0 when k <= 128),
 * 256-byte aligned; its first 8 * B bytes hold per-row counters that must be zero
 * before the first call on the workspace (cudaMemsetAsync once) -- every call leaves
 * them zero, except one that sets KVATTN_STATUS_TIMEOUT -- and the rest needs no
 * initialisation.  Calls that share a workspace must be ordered.
 * Supported: Dk = 576, Dv = 512, Hq in {64, 128}, 1 <= k <= 2048, B <= 65535.
 */
size_t attn_decode_sparse_workspace_bytes(int B, int Hq, int Dv, int k);

int attn_decode_sparse(const kvattn_bf16* q, const kvattn_bf16* latent, const int32_t* topk_idx,
                       int B, int Hq, int Dk, int Dv, int L_max, int k, float scale,
                       kvattn_bf16* out, float* lse, void* workspace, size_t workspace_bytes,
                       int32_t* dev_status, void* stream);

/* ---- FP8 (E4M3) latent cache and indexer keys -----------------------------------
 * "稀疏注意力：省了什么，没省什么", 改进一: a DeepSeek-V3.2 cache keeps per token and
 * layer 656 bytes -- FP8 latent + scale + the bf16 RoPE part -- plus an indexer
 * key of about 132 bytes; "Agentic RL 入门3" §2.2 (1): the indexer runs stably in
 * fp8.  The pages give the byte budget and no rounding rule; the reading taken:
 * each group of 128 values gets one fp32 scale s = absmax / 448 (448 = the
 * largest finite E4M3 value) and codes E4M3(x / s) -- IEEE fp32 division,
 * round-to-nearest-even, saturating at +-448, the sign of zero kept; an all-zero
 * group has s = 0 and codes 0.  E4M3 = the OCP 8-bit format with 4 exponent bits
 * (bias 7), 3 mantissa bits, no infinities.
 *
 * Packed latent row (656 bytes, 16-byte aligned rows): bytes 0..511 the codes of
 * latent[0..511] (groups 0..3 of 128), bytes 512..527 the 4 fp32 scales
 * (little-endian), bytes 528..655 latent[512..575] as bf16, unchanged.
 * FP8 indexer key: 128 codes in codes[t][0..127] plus one fp32 scale scales[t]
 * (132 bytes per token, kept as two arrays so that the codes stay TMA-aligned).
 *
 * latent_quant_fp8: latent [n_rows][576] bf16 -> packed [n_rows][656] uint8.
 * idx_key_quant_fp8: k_idx [n_rows][128] bf16 -> codes [n_rows][128] uint8 and
 * scales [n_rows] fp32.  Both quantise row by row (a cache built once, or the new
 * token's row appended at each step: pass pointers to that row, n_rows = 1).
 * Non-finite inputs are not supported.  Errors: KVATTN_ERR_NULL, _SHAPE
 * (n_rows < 0), _ALIGN (16 bytes; scales 4).
 *
 * attn_decode_sparse_fp8: attn_decode_sparse over packed FP8 latent rows
 * latent_fp8 [B][L_max][656]: key row j = the dequantised row
 * (value(code) * scale, rounded to bf16, then the RoPE part), value row j its
 * first 512 entries.  Arguments, limits, workspace
 * (attn_decode_sparse_workspace_bytes) and results otherwise as
 * attn_decode_sparse.
 */
int latent_quant_fp8(const kvattn_bf16* latent, long long n_rows, uint8_t* packed, void* stream);

/*
 * dsa_index_topk in fp8 ("Agentic RL 入门3" §2.2 (1): the indexer runs stably in fp8;
 * its product runs on E4M3 operands): k_codes [B][L_max][128] uint8 and k_scales
 * [B][L_max] fp32 are the keys (idx_key_quant_fp8); each 128-wide query head
 * q_idx[b][j] (bf16) is quantised inside the call with the same rule (scale qs_j =
 * absmax / 448).  The scores are the indexer formula on the dequantised operands,
 * s_{b,t} = sum_j w[b][j] * ReLU(qhat_j . khat_t) = ks_t * sum_j (w_j qs_j) *
 * ReLU(qcode_j . kcode_t) (the scales are >= 0), the code products exact and summed
 * in fp32 on the tensor cores.  HBM bytes per token: 132 instead of 256.  Everything
 * else (selection, order, -1 padding, scores_out, workspace, limits) as dsa_index_topk.
 */
int dsa_index_topk_fp8(const kvattn_bf16* q_idx, const float* w, const uint8_t* k_codes,
                       const float* k_scales, const int32_t* seq_lens, int B, int n_idx_head,
                       int idx_dim, int L_max, int k, int32_t* topk_idx, float* scores_out,
                       void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream);

int idx_key_quant_fp8(const kvattn_bf16* k_idx, long long n_rows, uint8_t* codes, float* scales, void* stream);

int attn_decode_sparse_fp8(const kvattn_bf16* q, const uint8_t* latent_fp8, const int32_t* topk_idx, int B,
                           int Hq, int Dk, int Dv, int L_max, int k, float scale, kvattn_bf16* out,
                           float* lse, void* workspace, size_t workspace_bytes, int32_t* dev_status,
                           void* stream);

/* ---- block-level indexer over 4-token groups ----------------------------------
 * "attention" page, "Qwen Sparse Attention (QSA)" §3 ①–④: the visible prefix is
 * cut into groups of 4 tokens; each complete group gets one block key (the mean of
 * its 4 indexer keys, normalised, rotated at the group's first position); blocks
 * are scored like the lightning indexer and the best n_top kept; the kept groups
 * are unpacked into their 4 token positions and the 0..3 tokens of the trailing
 * incomplete group are appended; standard GQA attention then runs over those
 * tokens of the full-precision cache (at most 4 n_top + 3 of them: 2048..2051 for
 * n_top = 512).  Readings where the section is silent: the normalisation is RMS
 * without a gain, x / sqrt(mean(x^2) + eps); the rotation is RoPE over all 128
 * dimensions with the caller's table at position 4j; the lightning indexer's head
 * weights w are kept (all ones gives the section's plain head sum); one selection
 * per sequence serves every KV head.
 *
 * qsa_block_keys: block key of group j of row b, for j in [block_from[b],
 * min(seq_lens[b] / 4, block_from[b] + max_new)) -- a decode step that completes a
 * group builds just that one (block_from = its index, max_new = 1); block_from
 * NULL = 0; max_new <= 0 = no limit.  k_idx [B][L_max][128] bf16 (the indexer
 * keys, unrotated); seq_lens device int32 [B] (tokens; outside [0, L_max]: clamped,
 * KVATTN_STATUS_BAD_LENGTH); cos_tab / sin_tab [max_pos][64] fp32 from
 * rope_table_build (position 4j >= max_pos: the key is stored unrotated and
 * KVATTN_STATUS_BAD_POSITION set); pair_style as rope_apply_qk; eps >= 0.
 * block_keys [B][L_max / 4][128] bf16 (written; other groups untouched).  The
 * arithmetic is fp32, rounded once to bf16.  Supported: L_max a multiple of 4,
 * B <= 65535.
 */
int qsa_block_keys(const kvattn_bf16* k_idx, const int32_t* seq_lens, const int32_t* block_from, int max_new, int B,
                   int idx_dim, int L_max, const float* cos_tab, const float* sin_tab, int max_pos, int pair_style,
                   float eps, kvattn_bf16* block_keys, int32_t* dev_status, void* stream);

/*
 * qsa_select: score the seq_lens[b] / 4 complete groups of row b, s_j = sum_h
 * w[b][h] * ReLU(q_idx[b][h] . block_keys[b][j]) in fp32, keep the n_top best
 * (ties to the lower group; the decision is taken on those fp32 scores) and expand.
 * q_idx [B][64][128] bf16 (rotated at the query's position by the caller);
 * w [B][64] fp32; block_keys [B][L_max / 4][128] bf16 (qsa_block_keys);
 * seq_lens device int32 [B] (tokens).  tok_idx [B][4 n_top + 3] int32: the
 * selected token positions in increasing order, -1 padded; tok_count [B] int32:
 * how many (4 min(L / 4, n_top) + L mod 4).  scores_out [B][L_max / 4] fp32 (the
 * group scores, -inf past each row's groups) or NULL.  workspace:
 * qsa_select_workspace_bytes(...) bytes, 256-byte aligned, with the zero-between-calls
 * histogram region of dsa_index_topk at its start (zero before the first call).
 * Supported: 64 indexer heads of width 128, L_max a multiple of 4 with
 * L_max / 4 <= 131072, 1 <= n_top <= 2048.
 */
size_t qsa_select_workspace_bytes(int B, int L_max, int n_top);

int qsa_select(const kvattn_bf16* q_idx, const float* w, const kvattn_bf16* block_keys, const int32_t* seq_lens, int B,
               int n_idx_head, int idx_dim, int L_max, int n_top, int32_t* tok_idx, int32_t* tok_count,
               float* scores_out, void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream);

/*
 * attn_decode_gqa_sparse: attn_decode_gqa over a per-sequence list of cache rows
 * ("Qwen Sparse Attention (QSA)" ③–④: the selected tokens' K and V are fetched
 * from the full cache by index, then softmax(scale q K_sel^T) V_sel per query head,
 * query head h reading KV head h / g).  tok_idx [B][n_idx] int32 cache rows (any
 * order); the first tok_count[b] entries of row b are used (tok_count device int32
 * [B], or NULL = all n_idx; a count outside [0, n_idx] is clamped and sets
 * KVATTN_STATUS_BAD_LENGTH); an entry -1 is skipped, any other entry outside
 * [0, T_max) is skipped and sets KVATTN_STATUS_BAD_INDEX.  A sequence with no used
 * row gives out = 0, lse = -inf.  q, k_cache, v_cache, out, lse, workspace and its
 * zero counter region as attn_decode_gqa (attn_decode_gqa_sparse_workspace_bytes).
 * Supported: head_dim 64 (g <= 64) or 128 (g <= 32), g as attn_decode_gqa.
 */
size_t attn_decode_gqa_sparse_workspace_bytes(int B, int n_head, int n_kv_head, int head_dim, int n_idx);

int attn_decode_gqa_sparse(const kvattn_bf16* q, const kvattn_bf16* k_cache, const kvattn_bf16* v_cache,
                           const int32_t* tok_idx, const int32_t* tok_count, int n_idx, int B, int n_head,
                           int n_kv_head, int head_dim, int T_max, float scale, kvattn_bf16* out, float* lse,
                           void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* KVATTN_H */
