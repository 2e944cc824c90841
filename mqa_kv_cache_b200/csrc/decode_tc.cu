// decode_tc.cu -- decode over a KV cache for groups of 64 query heads (MQA at
// n_head = 64) on the tcgen05 tensor cores.
//
// Same method, plan and merge as decode.cu (softmax(scale q k^T) v, query head
// h reading KV head h / g; "注意力变体与 MoE": each K/V tile read once for the
// whole group).  With g = 64 (MQA at n_head = 64) every byte of K/V feeds 64
// heads, 64 FLOP/byte: streaming at HBM speed needs ~0.3 PFLOP/s of bf16 MMA,
// which is the tcgen05 rate, not the mma.sync one.
//
// Per 64-key tile: S = Q K^T with M = 64 heads (rows in TMEM lanes 0-15 of
// each 32-lane quarter), N = 64 keys, K = 128, in one of three TMEM buffers so
// that the next tiles' scores are computed while this one's softmax runs; the
// softmax (four warps reading their 16 lanes with the 16x256b shape, so that
// all 32 threads work: a head's keys spread over a lane quad, two heads per
// thread) writes P as bf16 into a swizzled shared-memory tile and O += P V runs
// as a second MMA into a 128-column TMEM accumulator.  Warp 0 streams Q (per
// piece) and the K tiles, warp 7 the V tiles, through separate TMA rings (a K
// slot is released as soon as its S MMA is done, a V slot after its P V, one
// tile later: with one producer for both, a full V ring would hold back K);
// warp 1 issues the S MMAs (and owns TMEM), warp 6 the P V MMAs, so neither
// waits for the other's operands.
#include "common.cuh"
#include "decode_plan.cuh"
#include "kernels.h"

namespace kvattn {

namespace {

constexpr int TC_T = DEC_TILE;            // keys per tile (64)
constexpr int TC_D = 128;                 // head dim
constexpr int TC_M = 64;                  // query heads per MMA
constexpr int TC_KS = 5;                  // K ring slots
constexpr int TC_VS = 5;                  // V ring slots
constexpr int TC_BOX = TC_T * 128;        // 8 KB: 64 rows x one 64-wide d block
constexpr int TC_TILE = 2 * TC_BOX;       // 16 KB: a K or V tile [64 x 128]
constexpr int TC_QBOX = TC_M * 128;       // 8 KB
constexpr int TC_PBYTES = TC_M * 128;     // 8 KB: P tile [64 heads x 64 keys] bf16
constexpr int TC_THREADS = 256;           // w0 Q + K loads, w1 S MMAs + TMEM, w2-5 softmax, w6 P V MMAs, w7 V loads
constexpr int TC_NB = 3;                  // S and P buffers
constexpr int TC_TMEM_COLS = 512;         // S0 | S1 | S2 (64 columns each) | O (128), rounded up to a power of 2
constexpr int TC_OCOL = TC_NB * TC_T;
constexpr uint32_t TC_IDESC_S = umma_idesc_bf16(TC_M, TC_T);             // Q x K^T
constexpr uint32_t TC_IDESC_O = umma_idesc_bf16(TC_M, TC_D, false, true);  // P x V (V MN-major)
constexpr float kLog2e = 1.44269504088896340736f;
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kRescaleThreshold = 8.0f;

constexpr int TC_OFF_K = 0;
constexpr int TC_OFF_V = TC_OFF_K + TC_KS * TC_TILE;
constexpr int TC_OFF_Q = TC_OFF_V + TC_VS * TC_TILE;
constexpr int TC_OFF_P = TC_OFF_Q + 2 * TC_QBOX;                  // TC_NB P tiles
constexpr int TC_OFF_CS = TC_OFF_P + TC_NB * TC_PBYTES;          // cos row | sin row of the query position
constexpr int TC_OFF_QPOS = TC_OFF_CS + 2 * (TC_D / 2) * 4;       // [DECODE_MAX_B] query positions
constexpr int TC_OFF_N = TC_OFF_QPOS + DECODE_MAX_B * 4;
constexpr int TC_OFF_UB = TC_OFF_N + DECODE_MAX_B * 4;
constexpr int TC_OFF_LEN = TC_OFF_UB + (DECODE_MAX_B + 1) * 4;
constexpr int TC_OFF_BAR = (TC_OFF_LEN + DECODE_MAX_B * 4 + 7) / 8 * 8;
// kfull[KS], kempty[KS], vfull[VS], vempty[VS], q_full, q_empty, s_full[NB], p_full[NB], pv_done[NB], done[2]
constexpr int TC_NBAR = 2 * TC_KS + 2 * TC_VS + 2 + 3 * TC_NB + 2 + 1;  // + q_rot
constexpr int TC_OFF_MISC = TC_OFF_BAR + TC_NBAR * 8;
constexpr int TC_SMEM = TC_OFF_MISC + 32 + 1024;
static_assert(TC_SMEM <= 232448, "shared memory");

// The tiles of one CTA in stream order, with the piece they belong to.
struct TileStream {
    Walk w;
    long long t_cur = 0, t_end = 0;
    int piece = -1;
    __device__ bool next(long long lo, long long hi, int B, int Hk, const int* s_n, long long N, int G,
                         bool& first)
    {
        if (t_cur >= t_end) {
            // the next unit holding tiles of the range
            for (bool moved = piece < 0;; moved = false) {
                if (!moved) walk_next(w, B, Hk, s_n, N, G);
                if (!(w.U < hi && w.b < B)) return false;
                if (piece_tiles(w, s_n[w.b], lo, hi, t_cur, t_end)) break;
            }
            ++piece;
            first = true;
        } else {
            first = false;
        }
        ++t_cur;
        return true;
    }
};

// RoPE of the 64 query rows of a piece in place, in their two 128-byte-swizzled
// boxes (box k: dims 64k .. 64k+63, row h at h * 128 bytes, 16-byte chunk j of a
// row at ((j ^ (h & 7)) << 4)).  nthr threads take chunks.
__device__ __forceinline__ void rope_q_swizzled(uint8_t* q, const float* cs, const float* sn, int pair_style,
                                                int tid, int nthr)
{
    if (pair_style == 0) {
        // chunk (box k, j) holds pairs 32k + 4j .. 32k + 4j + 3
        for (int i = tid; i < TC_M * 16; i += nthr) {
            const int h = i >> 4, k = (i >> 3) & 1, j = i & 7;
            const int p0 = 32 * k + 4 * j;
            const float cc[4] = {cs[p0], cs[p0 + 1], cs[p0 + 2], cs[p0 + 3]};
            const float ss[4] = {sn[p0], sn[p0 + 1], sn[p0 + 2], sn[p0 + 3]};
            uint4* p = reinterpret_cast<uint4*>(q + k * TC_QBOX + swz128(h, j));
            *p = rope_chunk_adjacent(*p, cc, ss);
        }
    } else {
        // element e of chunk j in box 0 pairs with the same element in box 1: pair 8j + e
        for (int i = tid; i < TC_M * 8; i += nthr) {
            const int h = i >> 3, j = i & 7;
            float cc[8], ss[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                cc[e] = cs[8 * j + e];
                ss[e] = sn[8 * j + e];
            }
            uint4* pa = reinterpret_cast<uint4*>(q + swz128(h, j));
            uint4* pb = reinterpret_cast<uint4*>(q + TC_QBOX + swz128(h, j));
            uint4 ra = *pa, rb = *pb;
            rope_chunk_half(ra, rb, cc, ss);
            *pa = ra;
            *pb = rb;
        }
    }
}

__global__ void __launch_bounds__(TC_THREADS, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, DecodeArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    int* s_n = reinterpret_cast<int*>(smem + TC_OFF_N);
    int* s_Ub = reinterpret_cast<int*>(smem + TC_OFF_UB);
    int* s_len = reinterpret_cast<int*>(smem + TC_OFF_LEN);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + TC_OFF_BAR);
    uint64_t* kfull = bars;
    uint64_t* kempty = kfull + TC_KS;
    uint64_t* vfull = kempty + TC_KS;
    uint64_t* vempty = vfull + TC_VS;
    uint64_t* q_full = vempty + TC_VS;
    uint64_t* q_empty = q_full + 1;
    // Every barrier below is indexed by the tile's buffer i % TC_NB and waited with
    // phase (i / TC_NB) & 1, so that no waiter is ever more than one phase behind it
    // (the S and P buffers bound the lag).
    uint64_t* s_full = q_full + 2;               // [NB]: S of tile i ready in S buffer i % NB
    uint64_t* p_full = s_full + TC_NB;           // [NB]: P of tile i ready (S buffer i % NB read)
    uint64_t* pv_done = p_full + TC_NB;          // [NB]: P V of tile i finished (P buffer free, O updated)
    uint64_t* done = pv_done + TC_NB;            // [2]: all S MMAs / all P V MMAs finished
    uint64_t* q_rot = done + 2;                  // with RoPE: the piece's Q rows rotated (4 warps)
    float* sCos = reinterpret_cast<float*>(smem + TC_OFF_CS);
    float* sSin = sCos + TC_D / 2;
    int* s_qpos = reinterpret_cast<int*>(smem + TC_OFF_QPOS);
    const bool rope = a.cos_tab != nullptr;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + TC_OFF_MISC);
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem + TC_OFF_MISC + 4);
    int* s_acc = reinterpret_cast<int*>(smem + TC_OFF_MISC + 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < TC_KS; ++s) {
            mbar_init(&kfull[s], 1);
            mbar_init(&kempty[s], 1);
        }
        for (int s = 0; s < TC_VS; ++s) {
            mbar_init(&vfull[s], 1);
            mbar_init(&vempty[s], 1);
        }
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        mbar_init(q_rot, 4);
        for (int x = 0; x < TC_NB; ++x) {
            mbar_init(&s_full[x], 1);
            mbar_init(&p_full[x], 4);
            mbar_init(&pv_done[x], 1);
        }
        for (int x = 0; x < 2; ++x) mbar_init(&done[x], 1);
        *s_abort = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    if (warp == 1) {
        tmem_alloc(s_tmem, TC_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    pdl_wait();
    pdl_trigger();

    const long long N = plan_prefix(a.seq_lens, a.B, a.Hk, a.T_max, s_len, s_n, s_Ub, a.dev_status,
                                    blockIdx.x == 0, rope ? a.q_pos : nullptr, s_qpos,
                                    a.len_cap);
    const int G = static_cast<int>(N < a.grid ? N : a.grid), c = blockIdx.x;
    const bool active = N > 0 && c < G;
    long long lo = 0, hi = 0;
    Walk w_start{0, 0, 0, 0};
    if (active) {
        lo = range_start(c, N, G);
        hi = range_start(c + 1, N, G);
        w_start = walk_from(lo, a.B, a.Hk, s_n, s_Ub, 0);
    }
    // slots_before synchronises the whole CTA: every thread takes part
    const int S0 = slots_before(active ? w_start.b * a.Hk + w_start.kvh : 0, a.Hk, s_n, s_Ub, N > 0 ? N : 1,
                                G > 0 ? G : 1, s_acc);
    w_start.S = S0;

    if (active && warp == 0) {
        // ===== TMA producer: Q of each piece, then K of each tile (warp 7 loads V) =====
        if (lane == 0) {
            const uint64_t pol = l2_evict_first_policy();  // K and V are read once
            Walk w = w_start;
            int it = 0, np = 0;
            bool ok = true;
            for (; ok && w.U < hi && w.b < a.B; walk_next(w, a.B, a.Hk, s_n, N, G)) {
                long long tb, te;
                if (!piece_tiles(w, s_n[w.b], lo, hi, tb, te)) continue;
                const int z = w.b * a.Hk + w.kvh;
                if (np > 0 && !mbar_wait(q_empty, (np - 1) & 1)) {
                    ok = false;
                    break;
                }
                // with RoPE, the cos and sin rows of the query's position come along
                const int qp = rope ? s_qpos[w.b] : -1;
                const bool rot = rope && qp >= 0 && qp < a.max_pos;
                mbar_arrive_expect_tx(q_full, 2 * TC_QBOX + (rot ? TC_D * 4 : 0));
                tma_load_3d(smem + TC_OFF_Q, &tm_q, q_full, 0, 0, z);
                tma_load_3d(smem + TC_OFF_Q + TC_QBOX, &tm_q, q_full, 64, 0, z);
                if (rot) {
                    bulk_load(sCos, a.cos_tab + static_cast<long long>(qp) * (TC_D / 2), TC_D * 2, q_full);
                    bulk_load(sSin, a.sin_tab + static_cast<long long>(qp) * (TC_D / 2), TC_D * 2, q_full);
                }
                for (long long t = tb; t < te; ++t, ++it) {
                    const int ks = it % TC_KS;
                    const int row = static_cast<int>(t * TC_T);
                    if (it >= TC_KS && (*s_abort || !mbar_wait(&kempty[ks], ((it / TC_KS) - 1) & 1))) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&kfull[ks], TC_TILE);
                    uint8_t* kd = smem + TC_OFF_K + ks * TC_TILE;
                    tma_load_3d_hint(kd, &tm_k, &kfull[ks], 0, row, z, pol);
                    tma_load_3d_hint(kd + TC_BOX, &tm_k, &kfull[ks], 64, row, z, pol);
                }
                ++np;
            }
            if (!ok) {
                *s_abort = 1;
                report_status(a.dev_status, KVATTN_STATUS_TIMEOUT);
            }
            // copies still in flight complete before the CTA leaves (bounded waits)
            for (int j = it - TC_KS > 0 ? it - TC_KS : 0; j < it; ++j) mbar_wait(&kfull[j % TC_KS], (j / TC_KS) & 1);
        }
    } else if (active && warp == 7) {
        // ===== V loads: their own ring and pace (a V slot frees one tile later than a K slot,
        // after the P V; tied to the K loads, V would hold back K) =====
        if (lane == 0) {
            const uint64_t pol = l2_evict_first_policy();
            TileStream ts{w_start};
            bool ok = true, first = false;
            int it = 0;
            for (; ts.next(lo, hi, a.B, a.Hk, s_n, N, G, first); ++it) {
                const int vs = it % TC_VS;
                if (it >= TC_VS && (*s_abort || !mbar_wait(&vempty[vs], ((it / TC_VS) - 1) & 1))) {
                    ok = false;
                    break;
                }
                const int z = ts.w.b * a.Hk + ts.w.kvh;
                const int row = static_cast<int>((ts.t_cur - 1) * TC_T);
                mbar_arrive_expect_tx(&vfull[vs], TC_TILE);
                uint8_t* vd = smem + TC_OFF_V + vs * TC_TILE;
                tma_load_3d_hint(vd, &tm_v, &vfull[vs], 0, row, z, pol);
                tma_load_3d_hint(vd + TC_BOX, &tm_v, &vfull[vs], 64, row, z, pol);
            }
            if (!ok) {
                *s_abort = 1;
                report_status(a.dev_status, KVATTN_STATUS_TIMEOUT);
            }
            for (int j = it - TC_VS > 0 ? it - TC_VS : 0; j < it; ++j) mbar_wait(&vfull[j % TC_VS], (j / TC_VS) & 1);
        }
    } else if (active && warp == 1) {
        // ===== S = Q K^T issuer =====
        if (lane == 0) {
            const uint32_t sq = smem_u32(smem + TC_OFF_Q);
            TileStream ts{w_start};
            bool ok = true, first = false;
            int piece_s = -1;
            for (int i = 0; ok && ts.next(lo, hi, a.B, a.Hk, s_n, N, G, first); ++i) {
                if (ts.piece != piece_s) {
                    if (piece_s >= 0) tc_commit(q_empty);  // every S of the previous piece is issued
                    // the piece's Q has landed (and, with RoPE, been rotated by the softmax warps)
                    if (!(ok = mbar_wait(rope ? q_rot : q_full, ts.piece & 1))) break;
                    piece_s = ts.piece;
                }
                const int ks = i % TC_KS;
                // S buffer i % NB was read by the softmax of tile i - NB
                if (i >= TC_NB && !(ok = mbar_wait(&p_full[i % TC_NB], ((i / TC_NB) - 1) & 1))) break;
                if (!(ok = mbar_wait(&kfull[ks], (i / TC_KS) & 1))) break;
                tc_fence_after();
                const uint32_t kt = smem_u32(smem + TC_OFF_K + ks * TC_TILE);
                const uint32_t d = tmem + (i % TC_NB) * TC_T;
#pragma unroll
                for (int kk = 0; kk < TC_D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * TC_BOX + (kk & 3) * 32;
                    tc_mma_bf16(d, umma_desc_k_sw128(sq + off), umma_desc_k_sw128(kt + off), TC_IDESC_S,
                                kk > 0 ? 1u : 0u);
                }
                tc_commit(&kempty[ks]);
                tc_commit(&s_full[i % TC_NB]);
            }
            if (!ok) {
                *s_abort = 1;
                report_status(a.dev_status, KVATTN_STATUS_TIMEOUT);
            }
            tc_commit(&done[0]);
            mbar_wait(&done[0], 0);
        }
    } else if (active && warp == 6) {
        // ===== O += P V issuer =====
        if (lane == 0) {
            const uint32_t sp = smem_u32(smem + TC_OFF_P);
            TileStream ts{w_start};
            bool ok = true, first = false;
            for (int i = 0; ok && ts.next(lo, hi, a.B, a.Hk, s_n, N, G, first); ++i) {
                const int vs = i % TC_VS;
                if (!(ok = mbar_wait(&p_full[i % TC_NB], (i / TC_NB) & 1))) break;
                if (!(ok = mbar_wait(&vfull[vs], (i / TC_VS) & 1))) break;
                tc_fence_after();
                const uint32_t vt = smem_u32(smem + TC_OFF_V + vs * TC_TILE);
                const uint32_t pa = sp + (i % TC_NB) * TC_PBYTES;
#pragma unroll
                for (int kk = 0; kk < TC_T / 16; ++kk) {
                    const uint64_t bd = umma_desc_mn_sw128(vt + kk * 2048, TC_BOX, 1024);
                    tc_mma_bf16(tmem + TC_OCOL, umma_desc_k_sw128(pa + kk * 32), bd, TC_IDESC_O,
                                (!first || kk > 0) ? 1u : 0u);
                }
                tc_commit(&vempty[vs]);
                tc_commit(&pv_done[i % TC_NB]);
            }
            if (!ok) {
                *s_abort = 1;
                report_status(a.dev_status, KVATTN_STATUS_TIMEOUT);
            }
            tc_commit(&done[1]);
            mbar_wait(&done[1], 0);
        }
    } else if (active && warp >= 2 && warp <= 5) {
        // ===== softmax + epilogue: 16 heads per warp, read with the 16-lane TMEM shape =====
        // Thread t of quarter q holds heads h0 = 16q + t/4 and h1 = h0 + 8 (g = 64: every
        // row is a head) and, of each 8-key chunk j, keys 8j + cq and 8j + cq + 1 with
        // cq = 2 (t % 4); a head's 64 scores are spread over one lane quad.
        const int quarter = warp & 3;
        const int h0 = quarter * 16 + (lane >> 2), h1 = h0 + 8;
        const int cq = 2 * (lane & 3);
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t o_addr = tmem + lane_off + TC_OCOL;
        const float sl2 = a.scale * kLog2e;
        const float2 sc2 = make_float2(sl2, sl2);
        uint8_t* sP0 = smem + TC_OFF_P;
        Walk w = w_start;
        int i = 0, pc = 0;
        for (; w.U < hi && w.b < a.B; walk_next(w, a.B, a.Hk, s_n, N, G)) {
            const int n = s_n[w.b];
            const int len = s_len[w.b];
            long long tb, te;
            if (!piece_tiles(w, n, lo, hi, tb, te)) continue;
            const int count = unit_count(w.U, n, N, G);
            const int slot = w.S + (c - unit_first_owner(w.U, N, G));
            if (rope) {
                // rotate the piece's 64 Q rows in their swizzled boxes, then release the S MMAs
                // (bad positions: flagged, Q left as given)
                const int qp = s_qpos[w.b];
                if (warp_wait(q_full, pc & 1, s_abort)) {
                    if (qp >= 0 && qp < a.max_pos)
                        rope_q_swizzled(smem + TC_OFF_Q, sCos, sSin, a.pair_style, (warp - 2) * 32 + lane, 128);
                    else if (tb == 0 && warp == 2 && lane == 0)
                        report_status(a.dev_status, KVATTN_STATUS_BAD_POSITION);
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(q_rot);
            }
            ++pc;
            float m0 = -INFINITY, m1 = -INFINITY;  // running max (log2 units) of h0, h1
            float2 l2 = make_float2(0.f, 0.f);      // this thread's share of their sums
            for (long long t = tb; t < te; ++t, ++i) {
                const bool first = t == tb;
                if (!warp_wait(&s_full[i % TC_NB], (i / TC_NB) & 1, s_abort)) continue;
                // P buffer i % NB is free once the P V of tile i - NB has finished (the
                // previous piece's epilogue waited for all of its P V)
                if (t - tb >= TC_NB && !warp_wait(&pv_done[i % TC_NB], ((i / TC_NB) - 1) & 1, s_abort)) continue;
                tc_fence_after();
                const int n_valid = len - static_cast<int>(t) * TC_T;  // >= 1
                uint32_t sv[32];
                tmem_ld_16x256b_x8(tmem + lane_off + (i % TC_NB) * TC_T, sv);
                tmem_wait_ld();
                if (n_valid < TC_T) {  // tail tile (warp-uniform): keys past the length -> -inf
#pragma unroll
                    for (int x = 0; x < 32; ++x)
                        if (8 * (x >> 2) + cq + (x & 1) >= n_valid) sv[x] = 0xff800000u;
                }
                // row maxima: two 3-input chains per head, then across the quad
                float ma0 = -INFINITY, mb0 = -INFINITY, ma1 = -INFINITY, mb1 = -INFINITY;
#pragma unroll
                for (int j = 0; j < 8; j += 2) {
                    ma0 = fmax3(ma0, __uint_as_float(sv[4 * j]), __uint_as_float(sv[4 * j + 1]));
                    mb0 = fmax3(mb0, __uint_as_float(sv[4 * j + 4]), __uint_as_float(sv[4 * j + 5]));
                    ma1 = fmax3(ma1, __uint_as_float(sv[4 * j + 2]), __uint_as_float(sv[4 * j + 3]));
                    mb1 = fmax3(mb1, __uint_as_float(sv[4 * j + 6]), __uint_as_float(sv[4 * j + 7]));
                }
                float mx0 = fmaxf(ma0, mb0), mx1 = fmaxf(ma1, mb1);
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2)) * sl2;
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2)) * sl2;
                const bool mv0 = mx0 > m0 + kRescaleThreshold || m0 == -INFINITY;
                const bool mv1 = mx1 > m1 + kRescaleThreshold || m1 == -INFINITY;
                const float n0 = mv0 ? fmaxf(mx0, m0) : m0, n1 = mv1 ? fmaxf(mx1, m1) : m1;
                const bool rs0 = mv0 && m0 != -INFINITY && !first, rs1 = mv1 && m1 != -INFINITY && !first;
                if (__any_sync(0xffffffffu, rs0 || rs1)) {
                    // O must be stable: wait for the P V of the previous tile
                    if (!warp_wait(&pv_done[(i - 1) % TC_NB], ((i - 1) / TC_NB) & 1, s_abort)) continue;
                    tc_fence_after();
                    const float al0 = rs0 ? fast_exp2(m0 - n0) : 1.f, al1 = rs1 ? fast_exp2(m1 - n1) : 1.f;
                    l2.x *= al0;
                    l2.y *= al1;
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        uint32_t ov[32];
                        tmem_ld_16x256b_x8(o_addr + half * 64, ov);
                        tmem_wait_ld();
#pragma unroll
                        for (int x = 0; x < 32; ++x)
                            ov[x] = __float_as_uint(__uint_as_float(ov[x]) * ((x & 2) ? al1 : al0));
                        tmem_st_16x256b_x8(o_addr + half * 64, ov);
                    }
                    tmem_wait_st();
                }
                m0 = n0;
                m1 = n1;
                const float2 nmu0 = make_float2(m0 == -INFINITY ? 0.f : -m0, m0 == -INFINITY ? 0.f : -m0);
                const float2 nmu1 = make_float2(m1 == -INFINITY ? 0.f : -m1, m1 == -INFINITY ? 0.f : -m1);
                // a tail tile's V rows are zeroed below: its load must have landed first
                if (n_valid < TC_T && !warp_wait(&vfull[i % TC_VS], (i / TC_VS) & 1, s_abort)) continue;
                // P -> 128-byte swizzled rows h0, h1 of P tile i % NB (4 bytes per chunk and head)
                uint8_t* pt = sP0 + (i % TC_NB) * TC_PBYTES + cq * 2;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float2 x0 = __ffma2_rn(make_float2(__uint_as_float(sv[4 * j]), __uint_as_float(sv[4 * j + 1])),
                                                 sc2, nmu0);
                    const float2 x1 = __ffma2_rn(
                        make_float2(__uint_as_float(sv[4 * j + 2]), __uint_as_float(sv[4 * j + 3])), sc2, nmu1);
                    const float2 p0 = make_float2(fast_exp2(x0.x), fast_exp2(x0.y));
                    float2 p1;
                    if ((j & 1) == 0) {
                        p1 = exp2_fma2(x1);  // a quarter of the exponentials off the MUFU pipe
                    } else {
                        p1.x = fast_exp2(x1.x);
                        p1.y = fast_exp2(x1.y);
                    }
                    l2.x += p0.x + p0.y;
                    l2.y += p1.x + p1.y;
                    *reinterpret_cast<uint32_t*>(pt + swz128(h0, j)) = pack_bf16x2(p0.x, p0.y);
                    *reinterpret_cast<uint32_t*>(pt + swz128(h1, j)) = pack_bf16x2(p1.x, p1.y);
                }
                // rows of a tail tile past the length may hold anything: zero them in V so
                // that 0 * garbage cannot reach O (the V slot is not read before p_full);
                // thread (q, t) clears half (t % 2) of key row 16q + t/2
                if (n_valid < TC_T) {
                    const int vr = quarter * 16 + (lane >> 1);
                    if (vr >= n_valid) {
                        uint8_t* vrow = smem + TC_OFF_V + (i % TC_VS) * TC_TILE + (lane & 1) * TC_BOX + vr * 128;
#pragma unroll
                        for (int ch = 0; ch < 8; ++ch) *reinterpret_cast<uint4*>(vrow + ch * 16) = make_uint4(0, 0, 0, 0);
                    }
                }
                // make the shared-memory writes visible to the tensor cores
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[i % TC_NB]);
            }
            // ---- end of the piece: O (and m, l) out once its last P V has finished ----
            float l0 = l2.x, l1 = l2.y;
            l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
            l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
            l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
            l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
            if (warp_wait(&pv_done[(i - 1) % TC_NB], ((i - 1) / TC_NB) & 1, s_abort)) {
                tc_fence_after();
                const bool fin = count == 1;
                const long long bh0 = static_cast<long long>(w.b) * a.H + static_cast<long long>(w.kvh) * a.g + h0;
                const float inv0 = l0 > 0.f ? 1.f / l0 : 0.f, inv1 = l1 > 0.f ? 1.f / l1 : 0.f;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t ov[32];
                    tmem_ld_16x256b_x8(o_addr + half * 64, ov);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int col = half * 64 + 8 * j + cq;
                        const float o00 = __uint_as_float(ov[4 * j]), o01 = __uint_as_float(ov[4 * j + 1]);
                        const float o10 = __uint_as_float(ov[4 * j + 2]), o11 = __uint_as_float(ov[4 * j + 3]);
                        if (fin) {
                            __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(a.out) + bh0 * TC_D + col;
                            *reinterpret_cast<uint32_t*>(o) = pack_bf16x2(o00 * inv0, o01 * inv0);
                            *reinterpret_cast<uint32_t*>(o + 8 * TC_D) = pack_bf16x2(o10 * inv1, o11 * inv1);
                        } else {
                            float* po = a.part_o + (static_cast<long long>(slot) * a.g + h0) * TC_D + col;
                            *reinterpret_cast<float2*>(po) = make_float2(o00, o01);
                            *reinterpret_cast<float2*>(po + 8 * TC_D) = make_float2(o10, o11);
                        }
                    }
                }
                if ((lane & 3) == 0) {
                    if (fin) {
                        if (a.lse) {
                            a.lse[bh0] = l0 > 0.f ? (m0 + __log2f(l0)) * kLn2 : -INFINITY;
                            a.lse[bh0 + 8] = l1 > 0.f ? (m1 + __log2f(l1)) * kLn2 : -INFINITY;
                        }
                    } else {
                        const long long pi = static_cast<long long>(slot) * a.g + h0;
                        a.part_ml[pi * 2] = m0 == -INFINITY ? 0.f : m0;
                        a.part_ml[pi * 2 + 1] = l0;
                        a.part_ml[(pi + 8) * 2] = m1 == -INFINITY ? 0.f : m1;
                        a.part_ml[(pi + 8) * 2 + 1] = l1;
                    }
                }
                if (tb == 0 && warp == 2 && lane == 0) a.unit_info[w.b * a.Hk + w.kvh] = make_int2(w.S, count);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, TC_TMEM_COLS);
    }
}

}  // namespace

bool decode_tc_supported(int d, int g) { return d == TC_D && g == TC_M; }

cudaError_t launch_decode_tc(const DecodeArgs& a, const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                             const CUtensorMap& tm_v, cudaStream_t stream)
{
    static bool attr_set[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 64 && !attr_set[dev]) {
        e = cudaFuncSetAttribute(decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, TC_SMEM);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    e = launch_pdl(decode_tc_kernel, dim3(a.grid), dim3(TC_THREADS), TC_SMEM, stream, tm_q, tm_k, tm_v, a);
    if (e != cudaSuccess) return e;
    return launch_decode_merge(a, stream);
}

}  // namespace kvattn
