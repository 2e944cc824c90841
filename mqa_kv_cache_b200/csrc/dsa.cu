// dsa.cu -- DeepSeek-V3.2-style lightning indexer and top-k selection.
//
// Indexer ("Agentic RL 入门3：transformer 架构" §2.2 (1); "attention", DSA ①):
//   s_{b,t} = sum_{j<64} w[b][j] * ReLU(q_idx[b][j] . k_idx[b][t])
// with 64 indexer heads sharing one 128-wide key per token.  Per batch row this
// is a [L x 128] x [128 x 64] contraction followed by a ReLU-weighted reduction
// over the 64 heads, so it runs on the tensor cores: tcgen05.mma with the 128
// tokens of a tile as M, the 64 heads as N and K = 128, the fp32 accumulator
// in TMEM (four 64-column buffers so the epilogue of one tile overlaps the MMAs
// of the next ones), and the head reduction fused into the TMEM read-out.  It is
// bound by the one read of k_idx from HBM (intensity ~63 FLOP/byte).
//
// Top-k (§2.2 (2): S = TopK_t(s_t), ties to the lower index): one cluster of
// 8 CTAs per batch row, each holding its slice of order-preserving 32-bit keys
// of the fp32 scores in shared memory, runs an exact 3-digit (11/11/10-bit)
// radix select; every CTA sums the cluster's histograms through distributed
// shared memory and finds the digit itself.  An ordered compaction then writes
// the selected indices straight out in increasing index order.
#include <cooperative_groups.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace kvattn {

namespace {

// ---- indexer ------------------------------------------------------------------

// Order-preserving 32-bit key of an fp32 score (larger score, larger key);
// -0 is first made +0 so that it ties with +0; NaN maps to 0 (never selected
// ahead of a number) and is reported.
__device__ __forceinline__ uint32_t score_key(float f, bool& nan)
{
    uint32_t u = __float_as_uint(f);
    if ((u & 0x7fffffffu) > 0x7f800000u) {
        nan = true;
        return 0u;
    }
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The first radix digit of the top-k (the key's top 11 bits).  The indexers count the
// digits of every row's valid scores as they produce them (a shared-memory histogram per
// CTA and row, flushed into the row's histogram in global memory when the CTA is done with
// the row), so that the top-k starts at its second digit.
constexpr int TK_DIGITS0 = 2048;
constexpr int TK_SHIFT0 = 21;


constexpr int IX_TOK = 128;   // tokens per tile (MMA M)
constexpr int IX_HEADS = 64;  // indexer heads (MMA N)
constexpr int IX_DIM = 128;   // key width (MMA K)
constexpr int IX_BOX = IX_TOK * 128;          // one 128-byte-wide SW128 box of a key tile (16 KB)
constexpr int IX_QBOX = IX_HEADS * 128;       // one 128-byte-wide box of the query heads (8 KB)
constexpr int IX_THREADS = 320;               // warp 0 TMA, warp 1 MMA + TMEM, warps 2..9 epilogue
constexpr int IX_EPI = 256;                   // two groups of four warps, alternate tiles
constexpr int IX_NACC = 4;                    // 64-column accumulators in flight (the MMA-to-epilogue
                                              // round trip is ~1 us)
constexpr int IX_TMEM_COLS = IX_NACC * 64;
constexpr int IX_IQ = 4;     // work items in the producer's hand-out ring
constexpr int IX_CLAIM = 4;  // key tiles per claim

// bf16 keys: a tile is two 64-column boxes, 6 in flight, K = 128 in eight K = 16 steps
// (kind::f16); FP8 ("the indexer runs stably in fp8", "Agentic RL 入门3" §2.2 (1)): the
// query heads and keys are E4M3 codes, a tile is one 128-code box, 12 in flight, K = 128
// in four K = 32 steps on kind::f8f6f4 (exact code products, fp32 sums); the query head's
// scale is folded into its weight and the key's scale multiplies the score, which is
// exact algebra since ReLU(qs ks x) = qs ks ReLU(x) for scales >= 0.
template <bool FP8>
struct IxCfg {
    static constexpr int KBOX = FP8 ? 1 : 2;            // boxes per key tile (and per query)
    static constexpr int TILE = KBOX * IX_BOX;
    static constexpr int STAGES = FP8 ? 12 : 6;
    static constexpr int QBYTES = KBOX * IX_QBOX;
    static constexpr int KSTEPS = FP8 ? 4 : 8;
    static constexpr int OFF_Q = STAGES * TILE;
    static constexpr int OFF_W = OFF_Q + QBYTES;
    static constexpr int OFF_HIST = OFF_W + IX_HEADS * 4;   // [2048] digit counts of the current row
    static constexpr int OFF_ITEMS = OFF_HIST + 2048 * 4;     // [IX_IQ][3] (row, first tile, end tile); [3] the epilogue's
    static constexpr int OFF_BAR = OFF_ITEMS + (IX_IQ + 1) * 3 * 4 + 4;
    // full[S], empty[S], q_full, q_empty, acc_full[NACC], acc_empty[NACC], mma_done, item_full[IQ], item_empty[IQ]
    static constexpr int NBAR = 2 * STAGES + 3 + 2 * IX_NACC + 2 * IX_IQ;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int SMEM = OFF_MISC + 32 + 1024;
    static_assert(SMEM <= 232448, "shared memory");
    static constexpr uint32_t IDESC = FP8 ? ((1u << 4) | (static_cast<uint32_t>(IX_HEADS >> 3) << 17) |
                                             (static_cast<uint32_t>(IX_TOK >> 4) << 24))  // E4M3 x E4M3 -> fp32
                                          : umma_idesc_bf16(IX_TOK, IX_HEADS);
};

struct IndexerArgs {
    const float* w;
    const int32_t* seq_lens;
    const float* kscale;  // FP8: [B][L_max] key scales
    const float* qscale;  // FP8: [B][64] query-head scales
    float* scores;
    uint32_t* hist;       // [B][2048] first-digit counts of the valid scores (added to; zero on entry)
    int* row_ctr;         // [B] key tiles of each row claimed so far (zero on entry; the top-k clears them)
    int32_t* dev_status;
    int B, L_max, tiles_per_b;  // tiles_per_b: tiles of a full row (L_max); a row's claims stop at its length
    int len_shift;  // row b scores seq_lens[b] >> len_shift keys (2: 4-token groups)
};

// Rows served by CTA c of G: with G >= B the CTAs are split over the rows (row c B / G),
// each row's tiles (up to its length) claimed IX_CLAIM at a time from its counter by
// whichever of its CTAs is ready, so that faster CTAs take more (going on to other rows
// once a row is done was measured slower); with G < B, rows c, c + G, ...
__device__ __forceinline__ int ix_rows(int c, int G, int B) { return G >= B ? 1 : (B - c + G - 1) / G; }
__device__ __forceinline__ int ix_row(int c, int G, int B, int r)
{
    return G >= B ? static_cast<int>(static_cast<long long>(c) * B / G) : c + r * G;
}

__device__ __forceinline__ void tc_mma_f8(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

template <bool FP8>
__global__ void __launch_bounds__(IX_THREADS, 1)
    indexer_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q, IndexerArgs a)
{
    using C = IxCfg<FP8>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* full = bars;
    uint64_t* empty = bars + C::STAGES;
    uint64_t* q_full = bars + 2 * C::STAGES;
    uint64_t* q_empty = q_full + 1;
    uint64_t* acc_full = q_full + 2;
    uint64_t* acc_empty = acc_full + IX_NACC;
    uint64_t* mma_done = acc_empty + IX_NACC;
    // The producer hands out work items (row b, key tiles [t0, t1)) through a ring; an item
    // with t0 == t1 closes row b, and b < 0 ends the stream.
    uint64_t* item_full = mma_done + 1;        // [IQ]
    uint64_t* item_empty = item_full + IX_IQ;  // [IQ]: read by the MMA thread and the epilogue
    int* s_items = reinterpret_cast<int*>(smem + C::OFF_ITEMS);
    volatile int* s_cur = reinterpret_cast<volatile int*>(s_items + IX_IQ * 3);  // the epilogue's current item
    float* s_w = reinterpret_cast<float*>(smem + C::OFF_W);
    uint32_t* s_hist = reinterpret_cast<uint32_t*>(smem + C::OFF_HIST);
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = static_cast<int>(gridDim.x), cta = static_cast<int>(blockIdx.x);

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int i = 0; i < IX_NACC; ++i) {
            mbar_init(&acc_full[i], 1);
            mbar_init(&acc_empty[i], 4);
        }
        mbar_init(mma_done, 1);
        for (int i = 0; i < IX_IQ; ++i) {
            mbar_init(&item_full[i], 1);
            mbar_init(&item_empty[i], 2);
        }
        *s_abort = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_q);
    }
    if (warp == 1) {
        tmem_alloc(s_tmem, IX_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    pdl_wait();
    pdl_trigger();

    if (warp == 0) {
        // ===== TMA producer: each row's query heads, then the key tiles it claims =====
        if (lane == 0) {
            int it = 0, n = 0, nq = 0;
            auto push = [&](int b, int t0, int t1) {
                const int slot = n % IX_IQ;
                if (n >= IX_IQ && !mbar_wait(&item_empty[slot], ((n / IX_IQ) - 1) & 1)) return false;
                s_items[3 * slot] = b;
                s_items[3 * slot + 1] = t0;
                s_items[3 * slot + 2] = t1;
                mbar_arrive(&item_full[slot]);
                ++n;
                return true;
            };
            bool ok = true;
            // the keys are read once: evict them from L2 first, so that the scores (and their
            // histograms) this kernel writes are still there for the top-k
            const uint64_t k_pol = l2_evict_first_policy();
            const int n_rows = ix_rows(cta, G, a.B);
            for (int r = 0; ok && r < n_rows && !*s_abort; ++r) {
                const int b = ix_row(cta, G, a.B, r);
                // the row's tiles up to its length (the epilogue writes -inf past it within the last)
                const int len_raw = a.seq_lens ? (__ldg(a.seq_lens + b) >> a.len_shift) : a.L_max;
                const int T = (min(max(len_raw, 0), a.L_max) + IX_TOK - 1) / IX_TOK;
                if (r > 0 && __ldcg(a.row_ctr + b) >= T) continue;  // nothing left there
                // the first claim comes before the row's query heads: a row this CTA gets no tiles of
                // loads nothing and hands out nothing (every query load is waited for by the MMA)
                int t0 = atomicAdd(a.row_ctr + b, IX_CLAIM);
                if (t0 >= T) continue;
                // the row's query heads, once the S MMAs of the previous row are done with its own
                if (nq > 0 && !mbar_wait(q_empty, (nq - 1) & 1)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(q_full, C::QBYTES);
#pragma unroll
                for (int i = 0; i < C::KBOX; ++i) tma_load_3d(smem + C::OFF_Q + i * IX_QBOX, &tm_q, q_full, 64 * i, 0, b);
                ++nq;
                while (ok) {
                    const int t1 = min(t0 + IX_CLAIM, T);
                    if (!(ok = push(b, t0, t1))) break;
                    for (int t = t0; t < t1; ++t, ++it) {
                        const int s = it % C::STAGES;
                        if (it >= C::STAGES && (*s_abort || !mbar_wait(&empty[s], ((it / C::STAGES) - 1) & 1))) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&full[s], C::TILE);
                        uint8_t* dst = smem + s * C::TILE;
#pragma unroll
                        for (int i = 0; i < C::KBOX; ++i)
                            tma_load_3d_hint(dst + i * IX_BOX, &tm_k, &full[s], 64 * i, t * IX_TOK, b, k_pol);
                    }
                    if (!ok) break;
                    t0 = atomicAdd(a.row_ctr + b, IX_CLAIM);
                    if (t0 >= T) break;
                }
                if (ok) ok = push(b, 0, 0);  // row b closed
            }
            if (!ok) *s_abort = 1;
            push(-1, 0, 0);  // the end (bounded wait; after a timeout the consumers' own waits end them)
            if (*s_abort) report_status(a.dev_status, KVATTN_STATUS_TIMEOUT);
            // copies still in flight complete before the CTA leaves (bounded waits)
            if (nq > 0) mbar_wait(q_full, (nq - 1) & 1);
            for (int j = it - C::STAGES > 0 ? it - C::STAGES : 0; j < it; ++j)
                mbar_wait(&full[j % C::STAGES], (j / C::STAGES) & 1);
        }
    } else if (warp == 1) {
        // ===== MMA issuer (one thread) =====
        if (lane == 0) {
            const uint32_t q_addr = smem_u32(smem + C::OFF_Q);
            int it = 0, nq = 0, cur_b = -1;
            for (int n = 0; !*s_abort; ++n) {
                const int slot = n % IX_IQ;
                if (!mbar_wait(&item_full[slot], (n / IX_IQ) & 1)) {
                    *s_abort = 1;
                    break;
                }
                const int b = s_items[3 * slot], t0 = s_items[3 * slot + 1], t1 = s_items[3 * slot + 2];
                mbar_arrive(&item_empty[slot]);
                if (b < 0) break;
                if (t0 == t1) {  // row b closed: every S of it is issued, its query heads may go
                    tc_commit(q_empty);
                    cur_b = -1;
                    continue;
                }
                if (b != cur_b) {  // the row's query heads have landed
                    if (!mbar_wait(q_full, nq & 1)) {
                        *s_abort = 1;
                        break;
                    }
                    ++nq;
                    cur_b = b;
                }
                for (int t = t0; t < t1; ++t, ++it) {
                    const int s = it % C::STAGES;
                    const int buf = it % IX_NACC;
                    if (*s_abort || !mbar_wait(&full[s], (it / C::STAGES) & 1) ||
                        (it >= IX_NACC && !mbar_wait(&acc_empty[buf], ((it / IX_NACC) - 1) & 1))) {
                        *s_abort = 1;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t k_addr = smem_u32(smem + s * C::TILE);
                    const uint32_t d_addr = tmem + buf * IX_HEADS;
#pragma unroll
                    for (int ks = 0; ks < C::KSTEPS; ++ks) {
                        // 32 bytes of K per step (16 bf16 or 32 codes) of a 128-byte row
                        const uint32_t off = (ks >> 2) * IX_BOX + (ks & 3) * 32;
                        const uint64_t ad = umma_desc_k_sw128(k_addr + off);
                        const uint64_t bd = umma_desc_k_sw128(q_addr + (ks >> 2) * IX_QBOX + (ks & 3) * 32);
                        if constexpr (FP8)
                            tc_mma_f8(d_addr, ad, bd, C::IDESC, ks > 0 ? 1u : 0u);
                        else
                            tc_mma_bf16(d_addr, ad, bd, C::IDESC, ks > 0 ? 1u : 0u);
                    }
                    tc_commit(&empty[s]);
                    tc_commit(&acc_full[buf]);
                }
            }
            // every issued MMA has finished before the accumulators are released
            tc_commit(mma_done);
            mbar_wait(mma_done, 0);
            if (*s_abort) report_status(a.dev_status, KVATTN_STATUS_TIMEOUT);
        }
    } else {
        // ===== epilogue: TMEM -> ReLU, weight, sum over heads -> scores; two groups of
        // four warps take alternate tiles (a tile's read-out and sums are serial work) =====
        const int quarter = warp & 3;  // TMEM lanes this warp may read
        const int grp = (warp - 2) >> 2;
        const int row = quarter * 32 + lane;
        const int ep = threadIdx.x - 64;
        for (int i = ep; i < TK_DIGITS0; i += IX_EPI) s_hist[i] = 0u;  // ordered by the item's first barrier
        int tc = 0, cur_b = -1, len = 0;
        for (int n = 0;; ++n) {
            // one thread takes the item from the ring (bounded wait; b < 0 ends) and every
            // epilogue thread reads it between two barriers, so that all meet the same barriers
            if (ep == 0) {
                const int slot = n % IX_IQ;
                if (!*s_abort && mbar_wait(&item_full[slot], (n / IX_IQ) & 1)) {
                    s_cur[0] = s_items[3 * slot];
                    s_cur[1] = s_items[3 * slot + 1];
                    s_cur[2] = s_items[3 * slot + 2];
                } else {
                    *s_abort = 1;
                    s_cur[0] = -1;
                }
                mbar_arrive(&item_empty[slot]);
            }
            named_bar_sync(2, IX_EPI);
            const int b = s_cur[0], t0 = s_cur[1], t1 = s_cur[2];
            named_bar_sync(2, IX_EPI);
            if (b < 0) break;
            if (t0 == t1) {  // row b closed: its counts into the row's histogram, the shared one back to zero
                if (a.hist) {
                    uint32_t* gh = a.hist + static_cast<long long>(b) * TK_DIGITS0;
                    for (int i = ep; i < TK_DIGITS0; i += IX_EPI) {
                        const uint32_t v = s_hist[i];
                        if (v) {
                            atomicAdd(gh + i, v);
                            s_hist[i] = 0u;
                        }
                    }
                }
                cur_b = -1;
                continue;  // the next item's barriers order these before any new count
            }
            if (b != cur_b) {
                const int len_raw = a.seq_lens ? (a.seq_lens[b] >> a.len_shift) : a.L_max;
                len = min(max(len_raw, 0), a.L_max);
                if (len != len_raw && ep == 0) report_status(a.dev_status, KVATTN_STATUS_BAD_LENGTH);
                if (ep < IX_HEADS) {
                    const long long wi = static_cast<long long>(b) * IX_HEADS + ep;
                    s_w[ep] = FP8 ? a.w[wi] * a.qscale[wi] : a.w[wi];
                }
                named_bar_sync(2, IX_EPI);
                cur_b = b;
            }
            float* out = a.scores + static_cast<long long>(b) * a.L_max;
            for (int t = t0; t < t1; ++t, ++tc) {
                if ((tc & 1) != grp) continue;
                const int buf = tc % IX_NACC;
                const int tok = t * IX_TOK + row;
                const float kscale = FP8 && tok < a.L_max ? __ldg(a.kscale + static_cast<long long>(b) * a.L_max + tok) : 1.f;
                // on an abort the loops still run to the end (without waiting or
                // working) so that all four warps meet at the same named barriers
                if (!warp_wait(&acc_full[buf], (tc / IX_NACC) & 1, s_abort)) continue;
                tc_fence_after();
                const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + buf * IX_HEADS;
                uint32_t v0[32], v1[32];
                tmem_ld32(taddr, v0);
                tmem_ld32(taddr + 32, v1);
                tmem_wait_ld();
                tmem_regs_ready(v0);
                tmem_regs_ready(v1);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[buf]);
                // four independent chains over the heads (a 64-deep chain is latency-bound)
                float accs[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int j = 0; j < 32; ++j) accs[j & 3] = fmaf(s_w[j], fmaxf(__uint_as_float(v0[j]), 0.f), accs[j & 3]);
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    accs[j & 3] = fmaf(s_w[32 + j], fmaxf(__uint_as_float(v1[j]), 0.f), accs[j & 3]);
                float acc = (accs[0] + accs[1]) + (accs[2] + accs[3]);
                if (FP8) acc *= kscale;
                if (acc != acc) report_status(a.dev_status, KVATTN_STATUS_NAN_SCORE);
                if (tok < a.L_max) out[tok] = tok < len ? acc : -INFINITY;
                // the score's first top-k digit, counted once per warp and digit
                const bool in = a.hist != nullptr && tok < len;
                bool nan_key = false;
                const uint32_t digit = in ? score_key(acc, nan_key) >> TK_SHIFT0 : 0xffffffffu;
                const uint32_t same = __match_any_sync(0xffffffffu, digit);
                if (in && lane == __ffs(same) - 1) atomicAdd(&s_hist[digit], static_cast<uint32_t>(__popc(same)));
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, IX_TMEM_COLS);
    }
}

// ---- top-k --------------------------------------------------------------------

constexpr int TK_CL = 8;  // CTAs per batch row (one cluster)
constexpr int TK_THREADS = 1024;

// Block-wide inclusive scan (sum) of one value per thread; TK_THREADS threads.
__device__ __forceinline__ int block_incl_scan(int v, int* s_warp)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
    }
    if (lane == 31) s_warp[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int w = s_warp[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += t;
        }
        s_warp[lane] = w;
    }
    __syncthreads();
    const int r = v + (warp > 0 ? s_warp[warp - 1] : 0);
    __syncthreads();
    return r;
}

// An exact block-wide (TK_THREADS threads) selection among n values x_i = v[i] (~v[i]
// with invert), of those with f[i] == fval when f is given and with x_i & known == prefix:
// the need-th largest, its digits below `known` found by passes of 11 bits from bit
// `top` down (the last pass takes what is left).  Returns it; *left = how many values
// equal to it are still needed, *n_eq = how many equal it.
__device__ uint32_t block_select(const uint32_t* v, bool invert, const uint32_t* f, uint32_t fval, int n,
                                 uint32_t prefix, uint32_t known, int need, int top, uint32_t* hist, int* s_warp,
                                 uint32_t* s_sel, int* left, int* n_eq)
{
    const int tid = threadIdx.x;
    int eq = 0;
    for (int sh = top; sh > -11; sh -= 11) {
        const int lo_bit = sh < 0 ? 0 : sh;
        const int nb = 1 << (sh < 0 ? 11 + sh : 11);
        const uint32_t mask = static_cast<uint32_t>(nb - 1);
        for (int i = tid; i < nb; i += TK_THREADS) hist[i] = 0u;
        __syncthreads();
        for (int i = tid; i < n; i += TK_THREADS) {
            const uint32_t x = invert ? ~v[i] : v[i];
            if ((x & known) == prefix && (f == nullptr || f[i] == fval)) atomicAdd(&hist[(x >> lo_bit) & mask], 1u);
        }
        __syncthreads();
        const int d0 = nb - 1 - 2 * tid, d1 = d0 - 1;
        const int c0 = d0 >= 0 ? static_cast<int>(hist[d0]) : 0, c1 = d1 >= 0 ? static_cast<int>(hist[d1]) : 0;
        const int incl = block_incl_scan(c0 + c1, s_warp);
        const int before = incl - c0 - c1;
        if (d0 >= 0 && before < need && before + c0 >= need) {
            s_sel[0] = static_cast<uint32_t>(d0);
            s_sel[1] = static_cast<uint32_t>(need - before);
        } else if (d1 >= 0 && before + c0 < need && before + c0 + c1 >= need) {
            s_sel[0] = static_cast<uint32_t>(d1);
            s_sel[1] = static_cast<uint32_t>(need - before - c0);
        }
        __syncthreads();
        prefix |= s_sel[0] << lo_bit;
        known |= mask << lo_bit;
        need = static_cast<int>(s_sel[1]);
        eq = static_cast<int>(hist[s_sel[0]]);
        __syncthreads();  // hist is cleared by the next pass
        if (lo_bit == 0) break;
    }
    *left = need;
    *n_eq = eq;
    return prefix;
}

struct TopkArgs;
__device__ void write_tail(const TopkArgs& a, int row, int rank, int len, int n_sel, int32_t* out, int32_t* tout,
                           int width, int gs);

struct TopkArgs {
    const float* scores;
    const int32_t* seq_lens;
    uint32_t* hist;      // [B][2048] first-digit counts from the indexer (zeroed here after use), or null
    int32_t* out;
    int32_t* dev_status;
    int L_max, k;
    int len_shift;
    int32_t* tok_out;    // groups mode (see DsaIndexArgs), else null
    int32_t* tok_count;
    int L_tok;
    int* row_ctr;        // [B] the indexer's claim counters: cleared here for the next call (null: none)
    float* fill;         // scores, writable: -inf is written past each row's length (null: none)
};

constexpr int TK_SLICE_MAX = 16384;  // keys per CTA held in shared memory
// Keys of the row whose first digit is the threshold's, gathered into rank 0's shared
// memory (key, index) for the rest of the selection; more than this many take the
// cluster-wide passes instead.
constexpr int TK_CAND_MAX = 16384;
// Key i of the slice sits at word i + i / 16: a thread's run of 16 keys then
// starts in its own bank, so the runs of a warp are read without conflicts.
__device__ __forceinline__ int kpad(int i) { return i + (i >> 4); }
constexpr int TK_SLICE_WORDS = TK_SLICE_MAX + TK_SLICE_MAX / 16;

// Words of a CTA's key slice (kpad layout) for rows of L_max scores.
__host__ __device__ constexpr int slice_words(int L_max)
{
    return (L_max + TK_CL - 1) / TK_CL + ((L_max + TK_CL - 1) / TK_CL >> 4) + 1;
}

// After the n_sel selected entries of a row: -1 (fewer than k only when NaN scores were
// skipped); in groups mode the row's trailing tokens come first.  Rank 0 writes it.
__device__ void write_tail(const TopkArgs& a, int row, int rank, int len, int n_sel, int32_t* out, int32_t* tout,
                           int width, int gs)
{
    if (rank != 0) return;
    const int tid = threadIdx.x;
    if (tout) {
        const int tok_raw = a.seq_lens[row];
        const int tok_len = min(max(tok_raw, 0), a.L_tok);
        if (tok_len != tok_raw && tid == 0) report_status(a.dev_status, KVATTN_STATUS_BAD_LENGTH);
        const int tail0 = len * gs, n_tail = max(tok_len - tail0, 0), first = n_sel * gs;
        for (int j = first + tid; j < width; j += TK_THREADS) tout[j] = j - first < n_tail ? tail0 + (j - first) : -1;
        if (tid == 0) a.tok_count[row] = first + n_tail;
    } else {
        for (int j = n_sel + tid; j < a.k; j += TK_THREADS) out[j] = -1;
    }
}

__global__ void __launch_bounds__(TK_THREADS, 1) topk_kernel(TopkArgs a)
{
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = static_cast<int>(cluster.block_rank());
    const int row = blockIdx.x / TK_CL;
    const int tid = threadIdx.x, lane = tid & 31;

    extern __shared__ uint32_t s_keys[];  // this CTA's slice as keys (TK_SLICE_MAX at most), kpad layout
    __shared__ uint32_t hist2[2][2048];  // per-pass histograms, alternating (see below)
    __shared__ int s_warp[32];
    __shared__ uint32_t s_sel[2];    // threshold digit, keys still needed from it
    __shared__ int s_counts[2];      // this CTA's (#key > T, #key == T)
    __shared__ int s_nan;

    pdl_wait();
    pdl_trigger();
    if (a.row_ctr && rank == 0 && tid == 0) a.row_ctr[row] = 0;  // the indexer is done with it

    const int len_raw = a.seq_lens ? (a.seq_lens[row] >> a.len_shift) : a.L_max;
    const int len = min(max(len_raw, 0), a.L_max);
    if (len != len_raw && rank == 0 && tid == 0) report_status(a.dev_status, KVATTN_STATUS_BAD_LENGTH);
    const int kk = min(a.k, len);
    const int slice = (len + TK_CL - 1) / TK_CL;
    const int lo = min(rank * slice, len), hi = min(lo + slice, len);
    const int n_mine = hi - lo;
    const float* sc = a.scores + static_cast<long long>(row) * a.L_max;
    if (a.fill) {
        // the indexer scored whole tiles up to the length only: the rest of the row is -inf (in
        // the workspace nothing reads it; a caller's scores_out gets -inf past the length)
        float* f = a.fill + static_cast<long long>(row) * a.L_max;
        for (int i = len + rank * TK_THREADS + tid; i < a.L_max; i += TK_CL * TK_THREADS) f[i] = -INFINITY;
    }
    if (tid == 0) s_nan = 0;
    bool nan = false;
    // the candidate counter in rank 0 is zero before any CTA of the cluster counts into it
    __shared__ int s_cand_n;
    __shared__ int s_gt1[TK_CL];       // rank 0: per rank, its keys above the threshold's first digit
    __shared__ int s_rsel[TK_CL];      // rank 0: per rank, its selected candidates
    __shared__ uint32_t s_bcast[4];    // from rank 0: T, last index taken among keys == T, first position, total
    if (tid == 0) s_cand_n = 0;
    __syncthreads();
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
    // keys of the slice -> shared memory (one read of the scores, 16 loads in flight per thread)
    constexpr int TK_U = 16;
    for (int base = 0; base < n_mine; base += TK_THREADS * TK_U) {
        float v[TK_U];
#pragma unroll
        for (int u = 0; u < TK_U; ++u) {
            const int i = base + u * TK_THREADS + tid;
            v[u] = i < n_mine ? __ldcg(sc + lo + i) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < TK_U; ++u) {
            const int i = base + u * TK_THREADS + tid;
            if (i < n_mine) s_keys[kpad(i)] = score_key(v[u], nan);
        }
    }
    __syncthreads();
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");

    // ---- radix select: the (k)-th largest key T, and how many keys equal to T to take ----
    uint32_t prefix = 0u, known = 0u;
    int k_rem = kk;
    if (len > a.k) {
        for (int p = 0; p < 3; ++p) {
            // digits of 11, 11 and 10 bits from the top
            const int sh = p == 0 ? 21 : (p == 1 ? 10 : 0), nb = p == 2 ? 1024 : 2048;
            // Pass p clears and fills buffer p & 1.  Buffer p & 1 was last read by the other CTAs in
            // pass p - 2, before they reached pass p - 1's cluster barrier, which this CTA has passed:
            // one cluster barrier per pass suffices.
            uint32_t* hist = hist2[p & 1];
            const int d0 = nb - 1 - 2 * tid, d1 = d0 - 1;
            int c0 = 0, c1 = 0;
            if (p == 0 && a.hist) {
                // the indexer counted the first digits of the row: every CTA reads them
                const uint32_t* gh = a.hist + static_cast<long long>(row) * TK_DIGITS0;
                if (d0 >= 0) c0 = static_cast<int>(__ldcg(gh + d0));
                if (d1 >= 0) c1 = static_cast<int>(__ldcg(gh + d1));
            } else {
                for (int i = tid; i < nb; i += TK_THREADS) hist[i] = 0u;
                __syncthreads();
                // scores bunch into few top digits: lanes with equal digits add once per warp
                for (int base = 0; base < n_mine; base += TK_THREADS) {
                    const int i = base + tid;
                    const uint32_t key = i < n_mine ? s_keys[kpad(i)] : 0u;
                    const bool in = i < n_mine && (key & known) == prefix;
                    const uint32_t digit = in ? (key >> sh) & (nb - 1) : 0xffffffffu;
                    const uint32_t same = __match_any_sync(0xffffffffu, digit);
                    if (in && (tid & 31) == __ffs(same) - 1)
                        atomicAdd(&hist[digit], static_cast<uint32_t>(__popc(same)));
                }
                cluster.sync();
                // every CTA sums the cluster's histograms and finds the digit itself:
                // thread t owns digits nb-1-2t and nb-2-2t (largest first)
                if (d0 >= 0) {
#pragma unroll
                    for (int q = 0; q < TK_CL; ++q) {
                        const uint32_t* hq = cluster.map_shared_rank(hist, q);
                        c0 += static_cast<int>(hq[d0]);
                        if (d1 >= 0) c1 += static_cast<int>(hq[d1]);
                    }
                }
            }
            const int incl = block_incl_scan(c0 + c1, s_warp);
            const int before = incl - c0 - c1;
            if (d0 >= 0 && before < k_rem && before + c0 >= k_rem) {
                s_sel[0] = static_cast<uint32_t>(d0);
                s_sel[1] = static_cast<uint32_t>(k_rem - before);
            } else if (d1 >= 0 && before + c0 < k_rem && before + c0 + c1 >= k_rem) {
                s_sel[0] = static_cast<uint32_t>(d1);
                s_sel[1] = static_cast<uint32_t>(k_rem - before - c0);
            }
            __syncthreads();  // s_sel is written
            prefix |= s_sel[0] << sh;
            k_rem = static_cast<int>(s_sel[1]);
            known |= static_cast<uint32_t>(nb - 1) << sh;
            if (p == 0) {
                // ---- the keys with the threshold's first digit, (key, index), into rank 0 ----
                const uint32_t b1 = prefix >> TK_SHIFT0;
                const int key_words = slice_words(a.L_max);
                uint32_t* cand_key = s_keys + key_words;
                uint32_t* cand_idx = cand_key + TK_CAND_MAX;
                int* cnt0 = cluster.map_shared_rank(&s_cand_n, 0);
                uint32_t* ck0 = cluster.map_shared_rank(cand_key, 0);
                uint32_t* ci0 = cluster.map_shared_rank(cand_idx, 0);
                // two passes over the slice: count per warp, one remote add per warp for its
                // place in rank 0's list, then the stores
                int n_gt1 = 0, w_total = 0;
                for (int base = 0; base < n_mine; base += TK_THREADS) {
                    const int i = base + tid;
                    const uint32_t d = i < n_mine ? s_keys[kpad(i)] >> TK_SHIFT0 : 0u;
                    n_gt1 += i < n_mine && d > b1;
                    w_total += __popc(__ballot_sync(0xffffffffu, i < n_mine && d == b1));
                }
                int w_pos = 0;
                if (lane == 0 && w_total > 0) w_pos = atomicAdd(cnt0, w_total);
                w_pos = __shfl_sync(0xffffffffu, w_pos, 0);
                for (int base = 0; base < n_mine && w_total > 0; base += TK_THREADS) {
                    const int i = base + tid;
                    const uint32_t key = i < n_mine ? s_keys[kpad(i)] : 0u;
                    const bool in = i < n_mine && (key >> TK_SHIFT0) == b1;
                    const uint32_t m = __ballot_sync(0xffffffffu, in);
                    const int pos = w_pos + __popc(m & ((1u << lane) - 1u));
                    if (in && pos < TK_CAND_MAX) {
                        ck0[pos] = key;
                        ci0[pos] = static_cast<uint32_t>(lo + i);
                    }
                    w_pos += __popc(m);
                }
                const int gt_all = block_incl_scan(n_gt1, s_warp);
                if (tid == TK_THREADS - 1) *cluster.map_shared_rank(&s_gt1[rank], 0) = gt_all;
                cluster.sync();
                const int n_c = *cnt0;
                if (n_c <= TK_CAND_MAX) {
                    // every CTA has read the row's first-digit counts: leave them zero
                    if (a.hist && rank == 0)
                        for (int i = tid; i < TK_DIGITS0; i += TK_THREADS)
                            a.hist[static_cast<long long>(row) * TK_DIGITS0 + i] = 0u;
                    if (rank == 0) {
                        // T = the k_rem-th largest candidate; among the candidates equal to T
                        // (T != 0: NaN keys are 0 and never taken) the `left` lowest indices
                        int left = 0, n_eq = 0, l2 = 0, e2 = 0;
                        const uint32_t T = block_select(cand_key, false, nullptr, 0u, n_c, prefix, known, k_rem,
                                                        TK_SHIFT0 - 11, hist2[0], s_warp, s_sel, &left, &n_eq);
                        uint32_t cut = 0x7fffffffu;  // last index taken among the keys equal to T
                        if (T != 0u && left < n_eq)
                            cut = ~block_select(cand_idx, true, cand_key, T, n_c, 0x80000000u, 0x80000000u, left, 20,
                                                hist2[1], s_warp, s_sel, &l2, &e2);
                        if (tid < TK_CL) s_rsel[tid] = 0;
                        __syncthreads();
                        for (int i = tid; i < n_c; i += TK_THREADS) {
                            const uint32_t key = cand_key[i], idx = cand_idx[i];
                            if (key > T || (T != 0u && key == T && idx <= cut))
                                atomicAdd(&s_rsel[static_cast<int>(idx) / slice], 1);
                        }
                        __syncthreads();
                        if (tid == 0) {
                            uint32_t first = 0u;
                            for (int q = 0; q < TK_CL; ++q) first += static_cast<uint32_t>(s_gt1[q] + s_rsel[q]);
                            const uint32_t total = first;
                            first = 0u;
                            for (int q = 0; q < TK_CL; ++q) {
                                uint32_t* bq = cluster.map_shared_rank(s_bcast, q);
                                bq[0] = T;
                                bq[1] = cut;
                                bq[2] = first;
                                bq[3] = total;
                                first += static_cast<uint32_t>(s_gt1[q] + s_rsel[q]);
                            }
                        }
                    }
                    cluster.sync();
                    // ---- ordered compaction: each thread owns a contiguous run of the slice ----
                    const uint32_t Tf = s_bcast[0], cut = s_bcast[1];
                    const int run = (n_mine + TK_THREADS - 1) / TK_THREADS;
                    const int r0 = min(tid * run, n_mine), r1 = min(r0 + run, n_mine);
                    int n_take = 0;
                    for (int i = r0; i < r1; ++i) {
                        const uint32_t key = s_keys[kpad(i)];
                        n_take += key > Tf || (Tf != 0u && key == Tf && static_cast<uint32_t>(lo + i) <= cut);
                    }
                    const int inc = block_incl_scan(n_take, s_warp);
                    int pos = static_cast<int>(s_bcast[2]) + inc - n_take;
                    const int gs = 1 << a.len_shift;
                    const int width = a.k * gs + gs - 1;
                    int32_t* out = a.out ? a.out + static_cast<long long>(row) * a.k : nullptr;
                    int32_t* tout = a.tok_out ? a.tok_out + static_cast<long long>(row) * width : nullptr;
                    for (int i = r0; i < r1; ++i) {
                        const uint32_t key = s_keys[kpad(i)];
                        if (key > Tf || (Tf != 0u && key == Tf && static_cast<uint32_t>(lo + i) <= cut)) {
                            if (tout) {
                                for (int r = 0; r < gs; ++r) tout[pos * gs + r] = (lo + i) * gs + r;
                            } else {
                                out[pos] = lo + i;
                            }
                            ++pos;
                        }
                    }
                    write_tail(a, row, rank, len, static_cast<int>(s_bcast[3]), out, tout, width, gs);
                    if (nan) s_nan = 1;
                    __syncthreads();
                    if (s_nan && tid == 0) report_status(a.dev_status, KVATTN_STATUS_NAN_SCORE);
                    return;
                }
            }
        }
    }
    // With len <= k everything is taken: T = 0 selects every number (NaN keys are 0).
    const uint32_t T = len > a.k ? prefix : 0u;

    // ---- ordered compaction: each thread owns a contiguous run of the slice ----
    const int run = (n_mine + TK_THREADS - 1) / TK_THREADS;
    const int r0 = min(tid * run, n_mine), r1 = min(r0 + run, n_mine);
    int n_gt = 0, n_eq = 0;
    for (int i = r0; i < r1; ++i) {
        const uint32_t key = s_keys[kpad(i)];
        n_gt += key > T;
        n_eq += key == T && T != 0u;
    }
    const int inc_gt = block_incl_scan(n_gt, s_warp);
    const int inc_eq = block_incl_scan(n_eq, s_warp);
    if (tid == TK_THREADS - 1) {
        s_counts[0] = inc_gt;
        s_counts[1] = inc_eq;
    }
    cluster.sync();
    int gt_before = 0, eq_before = 0, gt_total = 0, eq_total = 0;
#pragma unroll
    for (int q = 0; q < TK_CL; ++q) {
        const int* cq = cluster.map_shared_rank(s_counts, q);
        if (q < rank) {
            gt_before += cq[0];
            eq_before += cq[1];
        }
        gt_total += cq[0];
        eq_total += cq[1];
    }
    const int take_eq = kk - gt_total;  // keys equal to T still needed (lowest indices first)
    // selected entries before this thread's run, in index order
    int g_rank = gt_before + inc_gt - n_gt;
    int e_rank = eq_before + inc_eq - n_eq;
    int pos = g_rank + min(e_rank, max(take_eq, 0));
    const int gs = 1 << a.len_shift;  // tokens per key in groups mode
    const int width = a.k * gs + gs - 1;
    int32_t* out = a.out ? a.out + static_cast<long long>(row) * a.k : nullptr;
    int32_t* tout = a.tok_out ? a.tok_out + static_cast<long long>(row) * width : nullptr;
    for (int i = r0; i < r1; ++i) {
        const uint32_t key = s_keys[kpad(i)];
        bool take = key > T;
        if (key == T && T != 0u) {
            take = e_rank < take_eq;
            ++e_rank;
        }
        if (take) {
            if (tout) {
                for (int r = 0; r < gs; ++r) tout[pos * gs + r] = (lo + i) * gs + r;
            } else {
                out[pos] = lo + i;
            }
            ++pos;
        }
    }
    write_tail(a, row, rank, len, gt_total + min(max(take_eq, 0), eq_total), out, tout, width, gs);
    if (nan) s_nan = 1;
    __syncthreads();
    if (s_nan && tid == 0) report_status(a.dev_status, KVATTN_STATUS_NAN_SCORE);
    cluster.sync();  // no CTA leaves while others may still read its shared memory
    // every CTA has read the row's first-digit counts (before its first cluster barrier):
    // leave them zero for the next call
    if (a.hist && rank == 0)
        for (int i = tid; i < TK_DIGITS0; i += TK_THREADS) a.hist[static_cast<long long>(row) * TK_DIGITS0 + i] = 0u;
}

// ---- top-k over the candidates of several key slices -----------------------------------
// Sharding the indexer over L ("稀疏注意力：省了什么，没省什么": the indexer stays O(L) per
// query, the cost that grows with the context): part p scores keys [p S, (p + 1) S) and
// keeps its own top-k.  Every element of the global top-k is in its part's top-k (fewer
// than k keys of its part beat it), so the top-k of the union of the parts' candidates is
// the global top-k, and with the same order (score desc, index asc) it is the same set.

// (score, global index) pairs of one part's selection: cand_idx = local index + offset.
__global__ void topk_candidates_kernel(const float* scores, const int32_t* idx, int B, int L_slice, int k, int offset,
                                       float* cand_score, int32_t* cand_idx)
{
    const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= static_cast<long long>(B) * k) return;
    const int b = static_cast<int>(i / k);
    const int j = idx[i];
    const bool ok = j >= 0 && j < L_slice;
    cand_score[i] = ok ? scores[static_cast<long long>(b) * L_slice + j] : -INFINITY;
    cand_idx[i] = ok ? j + offset : -1;
}

struct MergeTopkArgs {
    const float* cand_score;  // [n_parts][B][k]
    const int32_t* cand_idx;  // [n_parts][B][k]; -1 = no candidate
    int32_t* out;             // [B][k]
    int32_t* dev_status;
    int n_parts, B, k;
};

// One CTA per batch row: the row's n_parts * k candidates, in part order (part p's
// indices all below part p + 1's, each part's in increasing order), as keys in shared
// memory; an exact 3-digit radix select of the k-th largest key among the valid ones,
// then an ordered compaction that takes the keys above it and the lowest-index keys
// equal to it, written in increasing index order.
__global__ void __launch_bounds__(TK_THREADS) topk_merge_kernel(MergeTopkArgs a)
{
    extern __shared__ uint32_t s_ck[];  // [n] keys (0: no candidate, or a NaN score)
    __shared__ uint32_t hist[2048];
    __shared__ int s_warp[32];
    __shared__ uint32_t s_sel[2];
    __shared__ int s_n;
    const int row = blockIdx.x, tid = threadIdx.x;
    const int n = a.n_parts * a.k;
    pdl_wait();
    pdl_trigger();
    int n_valid_mine = 0;
    bool nan = false;
    for (int i = tid; i < n; i += TK_THREADS) {
        const int p = i / a.k, j = i - p * a.k;
        const long long off = (static_cast<long long>(p) * a.B + row) * a.k + j;
        const int ci = a.cand_idx[off];
        uint32_t key = 0u;
        if (ci >= 0) {
            key = score_key(a.cand_score[off], nan);  // 0 only for NaN: never selected
            n_valid_mine += key != 0u;
        }
        s_ck[i] = key;
    }
    if (tid == 0) s_n = 0;
    __syncthreads();
    atomicAdd(&s_n, n_valid_mine);
    __syncthreads();
    const int n_valid = s_n;
    const int kk = min(a.k, n_valid);
    uint32_t prefix = 0u, known = 0u;
    int k_rem = kk;
    if (n_valid > a.k) {
        const int shifts[3] = {21, 10, 0};
        const int widths[3] = {11, 11, 10};
        for (int pass = 0; pass < 3; ++pass) {
            const int sh = shifts[pass], nb = 1 << widths[pass];
            for (int i = tid; i < nb; i += TK_THREADS) hist[i] = 0u;
            __syncthreads();
            for (int i = tid; i < n; i += TK_THREADS) {
                const uint32_t key = s_ck[i];
                if (key != 0u && (key & known) == prefix) atomicAdd(&hist[(key >> sh) & (nb - 1)], 1u);
            }
            __syncthreads();
            // thread t owns digits nb-1-2t and nb-2-2t (largest first)
            const int d0 = nb - 1 - 2 * tid, d1 = d0 - 1;
            const int c0 = d0 >= 0 ? static_cast<int>(hist[d0]) : 0, c1 = d1 >= 0 ? static_cast<int>(hist[d1]) : 0;
            const int incl = block_incl_scan(c0 + c1, s_warp);
            const int before = incl - c0 - c1;
            if (d0 >= 0 && before < k_rem && before + c0 >= k_rem) {
                s_sel[0] = static_cast<uint32_t>(d0);
                s_sel[1] = static_cast<uint32_t>(k_rem - before);
            } else if (d1 >= 0 && before + c0 < k_rem && before + c0 + c1 >= k_rem) {
                s_sel[0] = static_cast<uint32_t>(d1);
                s_sel[1] = static_cast<uint32_t>(k_rem - before - c0);
            }
            __syncthreads();
            prefix |= s_sel[0] << sh;
            k_rem = static_cast<int>(s_sel[1]);
            known |= static_cast<uint32_t>(nb - 1) << sh;
            __syncthreads();
        }
    }
    // with n_valid <= k every valid candidate is taken
    const uint32_t T = prefix;
    const int take_eq = n_valid > a.k ? k_rem : 0;
    const int run = (n + TK_THREADS - 1) / TK_THREADS;
    const int r0 = min(tid * run, n), r1 = min(r0 + run, n);
    int n_gt = 0, n_eq = 0;
    for (int i = r0; i < r1; ++i) {
        const uint32_t key = s_ck[i];
        n_gt += n_valid > a.k ? key > T : key != 0u;
        n_eq += n_valid > a.k && key == T;
    }
    const int inc_gt = block_incl_scan(n_gt, s_warp);
    const int inc_eq = block_incl_scan(n_eq, s_warp);
    int e_rank = inc_eq - n_eq;
    int pos = (inc_gt - n_gt) + min(e_rank, take_eq);
    int32_t* out = a.out + static_cast<long long>(row) * a.k;
    for (int i = r0; i < r1; ++i) {
        const uint32_t key = s_ck[i];
        bool take = n_valid > a.k ? key > T : key != 0u;
        if (n_valid > a.k && key == T) {
            take = e_rank < take_eq;
            ++e_rank;
        }
        if (take) {
            const int p = i / a.k, j = i - p * a.k;
            out[pos++] = a.cand_idx[(static_cast<long long>(p) * a.B + row) * a.k + j];
        }
    }
    for (int j = kk + tid; j < a.k; j += TK_THREADS) out[j] = -1;
    if (nan) report_status(a.dev_status, KVATTN_STATUS_NAN_SCORE);
}

}  // namespace

size_t dsa_scores_bytes(int B, int L_max) { return static_cast<size_t>(B) * L_max * sizeof(float); }

// [B][2048] first-digit counts, then [B] claim counters of the indexer's rows
size_t dsa_hist_bytes(int B)
{
    return static_cast<size_t>(B) * TK_DIGITS0 * sizeof(uint32_t) + (static_cast<size_t>(B) * 4 + 255) / 256 * 256;
}

cudaError_t launch_dsa_index_topk(const DsaIndexArgs& a, const CUtensorMap& tm_k, const CUtensorMap& tm_q,
                                  cudaStream_t stream)
{
    static bool attr_set[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 64 && !attr_set[dev]) {
        e = cudaFuncSetAttribute(indexer_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, IxCfg<false>::SMEM);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(indexer_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, IxCfg<true>::SMEM);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    const bool fp8 = a.kscale != nullptr;
    if (fp8) {
        // the query heads as E4M3 codes and scales, with the keys' rule, once per call
        e = launch_idx_key_quant_fp8(a.q_idx, static_cast<long long>(a.B) * IX_HEADS, a.q8, a.q8_scale, stream);
        if (e != cudaSuccess) return e;
    }
    if (!a.hist) return cudaErrorInvalidValue;  // the workspace's zero region holds the claim counters
    IndexerArgs ia{};
    ia.hist = a.hist;
    ia.kscale = a.kscale;
    ia.qscale = a.q8_scale;
    ia.w = a.w;
    ia.seq_lens = a.seq_lens;
    ia.scores = a.scores;
    ia.dev_status = a.dev_status;
    ia.B = a.B;
    ia.L_max = a.L_max;
    ia.len_shift = a.len_shift;
    ia.tiles_per_b = (a.L_max + IX_TOK - 1) / IX_TOK;
    ia.row_ctr = reinterpret_cast<int*>(a.hist + static_cast<size_t>(a.B) * TK_DIGITS0);
    // every SM, but no more CTAs than claims
    const long long claims = static_cast<long long>(a.B) * ((ia.tiles_per_b + IX_CLAIM - 1) / IX_CLAIM);
    const int grid = claims < a.num_sms ? static_cast<int>(claims) : a.num_sms;
    e = fp8 ? launch_pdl(indexer_kernel<true>, dim3(grid), dim3(IX_THREADS), IxCfg<true>::SMEM, stream, tm_k, tm_q, ia)
            : launch_pdl(indexer_kernel<false>, dim3(grid), dim3(IX_THREADS), IxCfg<false>::SMEM, stream, tm_k, tm_q, ia);
    if (e != cudaSuccess) return e;

    TopkArgs ta{a.scores, a.seq_lens, a.hist, a.tok_idx ? nullptr : a.topk_idx, a.dev_status, a.L_max, a.k,
                a.len_shift, a.tok_idx, a.tok_count, a.L_tok, ia.row_ctr, a.scores};
    const size_t key_bytes = static_cast<size_t>(slice_words(a.L_max) + 2 * TK_CAND_MAX) * sizeof(uint32_t);
    static bool tk_attr[64] = {};
    if (dev < 64 && !tk_attr[dev]) {
        e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (TK_SLICE_WORDS + 1 + 2 * TK_CAND_MAX) * static_cast<int>(sizeof(uint32_t)));
        if (e != cudaSuccess) return e;
        tk_attr[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.B * TK_CL);
    cfg.blockDim = dim3(TK_THREADS);
    cfg.dynamicSmemBytes = key_bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = TK_CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, topk_kernel, ta);
}

}  // namespace kvattn

namespace kvattn {

cudaError_t launch_topk_candidates(const float* scores, const int32_t* idx, int B, int L_slice, int k, int offset,
                                   float* cand_score, int32_t* cand_idx, cudaStream_t stream)
{
    const long long n = static_cast<long long>(B) * k;
    topk_candidates_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, stream>>>(scores, idx, B, L_slice, k,
                                                                                         offset, cand_score, cand_idx);
    return cudaGetLastError();
}

cudaError_t launch_topk_merge(const float* cand_score, const int32_t* cand_idx, int n_parts, int B, int k,
                              int32_t* topk_idx, int32_t* dev_status, cudaStream_t stream)
{
    const size_t smem = static_cast<size_t>(n_parts) * k * sizeof(uint32_t);
    static bool attr[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 64 && !attr[dev]) {
        e = cudaFuncSetAttribute(topk_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        if (e != cudaSuccess) return e;
        attr[dev] = true;
    }
    MergeTopkArgs a{cand_score, cand_idx, topk_idx, dev_status, n_parts, B, k};
    return launch_pdl(topk_merge_kernel, dim3(B), dim3(TK_THREADS), smem, stream, a);
}

}  // namespace kvattn
