// kernels.h -- internal launch interface between the C-ABI layer (api.cu)
// and the kernel files.  Not installed; not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/kvattn.h"

namespace kvattn {

// Launch `kernel` on `stream` with programmatic stream serialisation (the
// kernel calls pdl_wait() before reading what earlier kernels wrote).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Record an error message for kvattn_last_error_string() and return `code`.
int record_error(int code, const char* fmt, ...);

// ---- RoPE ----
cudaError_t launch_rope_table(const kvattn_rope_params& p, int max_pos, float* cos_out, float* sin_out,
                              cudaStream_t stream);

struct RopeApplyArgs {
    kvattn_bf16* q;
    int q_nb, q_nt, q_nh;
    int64_t q_sb, q_st, q_sh;
    const int32_t* q_pos;
    kvattn_bf16* k;
    int k_nb, k_nt, k_nh;
    int64_t k_sb, k_st, k_sh;
    const int32_t* k_pos;
    const float* cos_tab;
    const float* sin_tab;
    int max_pos, head_dim, pair_style;
    int32_t* dev_status;
    int num_sms;
};
cudaError_t launch_rope_apply(const RopeApplyArgs& a, cudaStream_t stream);

struct KvAppendArgs {
    const kvattn_bf16* k_new;  // [B][Hk][d]
    const kvattn_bf16* v_new;  // [B][Hk][d]
    const int32_t* pos;        // [B] cache slot = rotation position
    kvattn_bf16* k_cache;      // [B][Hk][T_max][d]
    kvattn_bf16* v_cache;
    const float* cos_tab;
    const float* sin_tab;
    int B, Hk, head_dim, T_max, max_pos, pair_style;
    int n_sink, window;        // window > 0: rolling cache, slot of position p >= n_sink is
                               // n_sink + (p - n_sink) % window; window == 0: slot = position
    int32_t* dev_status;
};
cudaError_t launch_kv_append(const KvAppendArgs& a, cudaStream_t stream);

// ---- split-K decode ----
constexpr int DECODE_MAX_B = 1024;

struct DecodeArgs {
    const kvattn_bf16* q;
    const int32_t* seq_lens;
    kvattn_bf16* out;
    float* lse;
    float* part_o;   // [slots][g][d]  unnormalised partial outputs
    float* part_ml;  // [slots][g][2]  (running max in log2 units, sum of exponentials)
    int2* unit_info; // [B*Hk]         (first slot, number of pieces) of every non-empty unit
    int* unit_cnt;   // [B*Hk]         pieces of a split unit finished so far (zero between calls)
    // RoPE of the queries inside the kernel (cos_tab null: q is used as given)
    const int32_t* q_pos;  // [B] position of each sequence's query
    const float* cos_tab;  // [max_pos][d/2]
    const float* sin_tab;
    int max_pos, pair_style;
    int len_cap;           // > 0: a sequence of length len uses min(len, len_cap) cache rows
                           // (a rolling cache holding the sinks and the window)
    // Gather mode (idx non-null): the rows of unit (b, kv-head) are the cache rows
    // idx[b][0 .. n_b - 1], n_b = seq_lens[b] (n_idx when seq_lens is null); an
    // entry outside [0, T_max) is skipped (-1 silently, any other value flagged).
    const int32_t* idx;    // [B][n_idx]
    int n_idx;
    const kvattn_bf16* k_cache;  // [B][Hk][T_max][d], read by row in gather mode
    const kvattn_bf16* v_cache;
    int32_t* dev_status;
    int B, H, Hk, g, d, T_max;
    float scale;
    int grid;        // persistent CTAs (also the number of tile ranges)
    // Failure-detection testing (mma.sync kernel, tensor-map mode): each pipeline wait
    // gives up after wait_ns (0: WAIT_LIMIT_NS), and CTA 0 issues no loads for its
    // tile number drop_it (-1: none), so that its consumers' waits run out.
    unsigned long long wait_ns = 0;
    int drop_it = -1;
};
// Number of partial slots the decode kernel may write for a given grid.
long long decode_max_slots(int B, int Hk, int grid);
// Persistent CTAs per launch for this device.
int decode_grid(int num_sms);
// Runs the tcgen05 kernel for the groups decode_tc_supported() accepts, the
// mma.sync kernel otherwise, then the merge of split units.
cudaError_t launch_decode(const DecodeArgs& a, const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                          const CUtensorMap& tm_v, cudaStream_t stream);
bool decode_tc_supported(int d, int g);
cudaError_t launch_decode_tc(const DecodeArgs& a, const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                             const CUtensorMap& tm_v, cudaStream_t stream);
cudaError_t launch_decode_merge(const DecodeArgs& a, cudaStream_t stream);

// ---- merge of decode results over disjoint key sets ----
struct MergeArgs {
    const kvattn_bf16* o_parts;  // [n][B][H][d]
    const float* lse_parts;      // [n][B][H]
    kvattn_bf16* out;            // [B][H][d]
    float* lse;                  // [B][H] or null
    int n, B, H, d;
};
cudaError_t launch_merge_lse(const MergeArgs& a, cudaStream_t stream);

// ---- lightning indexer + top-k ----
struct DsaIndexArgs {
    const float* w;
    const int32_t* seq_lens;
    float* scores;      // [B][L_max] fp32 (caller's scores_out or workspace)
    int32_t* topk_idx;  // [B][k]
    int32_t* dev_status;
    int B, L_max, k, num_sms;
    int len_shift = 0;  // row b has seq_lens[b] >> len_shift keys (2: the 4-token block keys)
    // Groups mode (tok_idx non-null): key j stands for the 1 << len_shift tokens of group j;
    // the selection is written as token positions (increasing) followed by the row's
    // trailing tokens past its last complete group, -1 padded to (k << len_shift) +
    // (1 << len_shift) - 1 entries, with the count in tok_count; topk_idx is not written.
    int32_t* tok_idx = nullptr;
    int32_t* tok_count = nullptr;
    int L_tok = 0;  // token capacity of a row (seq_lens beyond it are clamped and flagged)
    // FP8 (kscale non-null): tm_k maps the key codes [B][L_max][128] uint8 with a {128, 128, 1}
    // box and 128-byte swizzle, kscale [B][L_max] fp32 holds each key's scale; the launch
    // first quantises the query heads into q8 / q8_scale, which tm_q maps ({128, 64, 1} box).
    const float* kscale = nullptr;
    const kvattn_bf16* q_idx = nullptr;  // FP8: the bf16 query heads [B][64][128], quantised into q8 / q8_scale
    uint8_t* q8 = nullptr;               // FP8: [B][64][128] codes (tm_q maps them)
    float* q8_scale = nullptr;           // FP8: [B][64]
    // [B][2048] first-digit counts of the top-k: zero on entry, the indexer adds to them, the
    // top-k reads them instead of its first pass and leaves them zero; null = the top-k counts
    uint32_t* hist = nullptr;
};
size_t dsa_scores_bytes(int B, int L_max);
size_t dsa_hist_bytes(int B);  // the [B][2048] first-digit counts
cudaError_t launch_dsa_index_topk(const DsaIndexArgs& a, const CUtensorMap& tm_k, const CUtensorMap& tm_q,
                                  cudaStream_t stream);

// ---- top-k over the candidates of several key slices (sharded indexer) ----
constexpr int TOPK_MERGE_MAX = 48 * 1024;  // candidates per row (n_parts * k) held in shared memory
cudaError_t launch_topk_candidates(const float* scores, const int32_t* idx, int B, int L_slice, int k, int offset,
                                   float* cand_score, int32_t* cand_idx, cudaStream_t stream);
cudaError_t launch_topk_merge(const float* cand_score, const int32_t* cand_idx, int n_parts, int B, int k,
                              int32_t* topk_idx, int32_t* dev_status, cudaStream_t stream);

// ---- block-level indexer (4-token groups) ----
constexpr int QSA_BLOCK = 4;
struct QsaKeysArgs {
    const kvattn_bf16* k_idx;   // [B][L_max][128]
    const int32_t* seq_lens;    // [B] tokens
    const int32_t* block_from;  // [B] first block to build, or null (0)
    const float* cos_tab;
    const float* sin_tab;
    kvattn_bf16* block_keys;    // [B][L_max / 4][128]
    int32_t* dev_status;
    int B, L_max, max_pos, pair_style, max_new;
    float eps;
};
cudaError_t launch_qsa_block_keys(const QsaKeysArgs& a, cudaStream_t stream);

// ---- sparse latent attention ----
struct SparseLaunch {
    const kvattn_bf16* q;
    const void* latent;  // bf16 [B][L_max][576], or packed FP8 rows [B][L_max][656] when fp8
    const int32_t* idx;
    kvattn_bf16* out;
    float* lse;
    void* workspace;     // several chunks: per-row counters (zero between calls), bf16 parts
                         // [B][chunks][Hq][512], their fp32 lse [B][chunks][Hq]; null for one chunk
    int32_t* dev_status;
    int B, Hq, L_max, k;
    float scale;
    bool fp8 = false;
    int num_sms = 0;     // the grid merges its parts itself when B * chunks <= num_sms
};
int sparse_chunks(int k);
size_t sparse_part_o_bytes(int B, int Hq, int k);
size_t sparse_partial_bytes(int B, int Hq, int k);
// tm_q: 3-D map over q [B][Hq][576] with a {64, Hq, 1} box (128-byte swizzle).
// tm_o: 3-D map with a {64, Hq, 1} box over the output [B][Hq][512] when k <= 128
// (one chunk), else over the workspace's bf16 parts [B * chunks][Hq][512]
// (sparse_counter_bytes(B) bytes into the workspace).
size_t sparse_counter_bytes(int B);
cudaError_t launch_sparse_attn(const SparseLaunch& l, const CUtensorMap& tm_q, const CUtensorMap& tm_o,
                               const CUtensorMap& tm_pm, cudaStream_t stream);

// ---- FP8 (E4M3) quantisation of latent rows and indexer keys ----
cudaError_t launch_latent_quant_fp8(const kvattn_bf16* src, long long n_rows, uint8_t* dst, cudaStream_t stream);
cudaError_t launch_idx_key_quant_fp8(const kvattn_bf16* src, long long n_rows, uint8_t* codes, float* scales,
                                     cudaStream_t stream);

// ---- causal prefill ----
constexpr int PREFILL_Q_ROWS = 128;  // rows of a Q tile (box height of tm_q)
constexpr int PREFILL_KV_ROWS = 128;  // keys of a K/V tile (box height of tm_k, tm_v)
struct PrefillLaunch {
    kvattn_bf16* out;
    float* lse;
    int32_t* dev_status;
    int B, T, H, Hk;
    float scale;
    int n_sink = 0, window = 0;  // window > 0: sliding window with n_sink sink tokens
};
cudaError_t launch_prefill(const PrefillLaunch& l, const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                           const CUtensorMap& tm_v, cudaStream_t stream);

}  // namespace kvattn
