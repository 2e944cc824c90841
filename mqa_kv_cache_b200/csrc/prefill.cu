// prefill.cu -- causal attention over a whole prompt on the tcgen05 tensor cores.
//
// Method: O_i = sum_{j <= i} softmax_j(scale q_i . k_j) v_j per query head,
// query head h reading KV head h / g ("注意力变体与 MoE", attention(): the
// lower-triangular mask fills triu(1) with -inf; "attention",
// GroupQueryAttention).  Both contractions (Q K^T and P V) are dense, so they
// run on tcgen05 with fp32 accumulators in tensor memory, FlashAttention-style
// (scores never leave the SM; "Agentic RL 入门3" §2.4: the matmul parts on tensor
// cores, the sequential softmax parts between chunks).
//
// CTA = (batch, query head, block of 256 query rows) = two 128-row Q tiles that
// share every K/V tile, so the softmax of one tile overlaps the MMAs of the
// other.  Warps 0-3 / 4-7: softmax of Q tile 0 / 1, one thread per query row
// (a full score row per thread, all 128 scores in registers: row max and sum need
// no shuffles and the scores are read from TMEM once); warp 8: the single
// MMA-issuing thread; warp 9: TMA loads (Q once, then K_j, V_j through a 4-slot
// ring); warps 10-11 idle, so that warps 8-11 form a warpgroup that hands its
// registers to the softmax warpgroups (setmaxnreg).  TMEM (512 columns):
// S0 | S1 | O0 | O1, 128 columns each.
// The softmax writes P (bf16, two per 32-bit column) over the first 64 columns
// of its S buffer and the P V product takes P straight from TMEM.  The running
// max is only moved (and O rescaled) when it grows by more than 2^8, so most
// tiles never touch O.  Blocks of the longest query rows launch first.
#include "common.cuh"
#include "kernels.h"

namespace kvattn {

namespace {

constexpr int PF_D = 128;     // head dim
constexpr int PF_BM = 128;    // query rows per Q tile
constexpr int PF_BN = 128;    // keys per K/V tile
static_assert(PF_BM == PREFILL_Q_ROWS && PF_BN == PREFILL_KV_ROWS, "tensor map boxes");
constexpr int PF_SLOTS = 4;   // K/V ring slots (one tile each)
constexpr int PF_THREADS = 384;  // w0-7 softmax, w8 MMA, w9 TMA, w10-11 idle (a whole warpgroup for setmaxnreg)
constexpr int PF_TILE = PF_BN * PF_D * 2;  // 32 KB: one K or V tile, two 64-column SW128 boxes
constexpr int PF_BOX = PF_BN * 128;        // 16 KB
constexpr int PF_OFF_Q = 0;                // two Q tiles
constexpr int PF_OFF_KV = 2 * PF_TILE;
constexpr int PF_OFF_BAR = PF_OFF_KV + PF_SLOTS * PF_TILE;
// kv_full[4], kv_empty[4], q_full, s_full[2], p_full[2], pv_done[2], mma_done
constexpr int PF_NBAR = 2 * PF_SLOTS + 8;
constexpr int PF_OFF_MISC = PF_OFF_BAR + PF_NBAR * 8;
constexpr int PF_SMEM = PF_OFF_MISC + 32 + 1024;
constexpr uint32_t PF_IDESC_S = umma_idesc_bf16(PF_BM, PF_BN);             // Q (K-major) x K (K-major)
constexpr uint32_t PF_IDESC_O = umma_idesc_bf16(PF_BM, PF_D, false, true);  // P (tmem) x V (MN-major)
constexpr float kLog2e = 1.44269504088896340736f;
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct PrefillArgs {
    kvattn_bf16* out;  // [B][T][H][d]
    float* lse;        // [B][H][T] or null
    int32_t* dev_status;
    int B, T, H, Hk, g, n_qblk;
    int n_sink, window;  // window > 0: query i sees keys j <= i with j > i - window or j < n_sink
    float scale;
};

// WINDOW: a sliding window with sinks is in effect (a.window > 0); the plain causal
// kernel is compiled without the band test.
template <bool WINDOW>
__global__ void __launch_bounds__(PF_THREADS, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, PrefillArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + PF_OFF_BAR);
    uint64_t* kv_full = bars;
    uint64_t* kv_empty = bars + PF_SLOTS;
    uint64_t* q_full = bars + 2 * PF_SLOTS;
    uint64_t* s_full = q_full + 1;
    uint64_t* p_full = q_full + 3;
    uint64_t* pv_done = q_full + 5;
    uint64_t* mma_done = q_full + 7;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + PF_OFF_MISC);
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem + PF_OFF_MISC + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // work item: longest query blocks first
    const int bh_count = a.B * a.H;
    const int qblk = a.n_qblk - 1 - static_cast<int>(blockIdx.x) / bh_count;
    const int bh = static_cast<int>(blockIdx.x) % bh_count;
    const int b = bh / a.H, h = bh - b * a.H;
    const int kvh = h / a.g;
    const int q0 = qblk * 2 * PF_BM;
    const int n_qt = (a.T - q0) > PF_BM ? 2 : 1;   // Q tiles in this block
    // Key tiles.  Q tile t sees tiles 0 .. diag(t) (its diagonal tile); with a window, only the
    // sink tiles [0, ns) and the band tiles [lo(t), diag(t)].  The CTA walks the union of its Q
    // tiles' sets in increasing order (lo(0) <= lo(1), diag(1) = diag(0) + 1); each Q tile counts
    // its own steps, which set its barrier phases.
    const int ns = WINDOW ? (a.n_sink + PF_BN - 1) / PF_BN : 0;
    auto diag_of = [&](int t) { return (q0 + t * PF_BM) / PF_BN; };
    auto lo_of = [&](int t) {
        const int first_key = q0 + t * PF_BM - a.window + 1;  // lowest band key of the tile's first row
        return (WINDOW && first_key > 0) ? first_key / PF_BN : 0;
    };
    auto first_in = [&](int lo) { return (ns > 0 || lo == 0) ? 0 : lo; };
    auto next_in = [&](int lo, int j) { return (j + 1 < ns || j + 1 >= lo) ? j + 1 : lo; };
    auto in_t = [&](int t, int j) { return t < n_qt && j <= diag_of(t) && (j < ns || j >= lo_of(t)); };
    const int lo_u = lo_of(0), d_u = diag_of(n_qt - 1);
    const int n_kv0 = q0 / PF_BN + 1;  // plain causal: Q tile t sees tiles 0 .. n_kv0 - 1 + t
    const int n_kv = n_kv0 + (n_qt - 1);

    if (threadIdx.x == 0) {
        for (int i = 0; i < PF_SLOTS; ++i) {
            mbar_init(&kv_full[i], 1);
            mbar_init(&kv_empty[i], 1);
        }
        mbar_init(q_full, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], 4);
            mbar_init(&pv_done[i], 1);
        }
        mbar_init(mma_done, 1);
        *s_abort = 0;
        fence_barrier_init();
    }
    if (warp == 9 && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    if (warp == 8) {
        tmem_alloc(s_tmem, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    pdl_wait();
    pdl_trigger();

    // registers: the softmax warpgroups take 216 each thread, the MMA / TMA warpgroup keeps 64
    // (2 x 128 x 216 + 128 x 64 = 63488 of the 384 x 168 = 64512 the block is launched with;
    // per SM sub-partition 2 x 32 x 216 + 32 x 64 = 15872 of 16384)
    if (warp == 9) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 64;" ::: "memory");
        // ===== TMA loads =====
        if (lane == 0) {
            mbar_arrive_expect_tx(q_full, n_qt * PF_TILE);
            for (int t = 0; t < n_qt; ++t) {
                uint8_t* dst = smem + PF_OFF_Q + t * PF_TILE;
                tma_load_4d(dst, &tm_q, q_full, 0, h, q0 + t * PF_BM, b);
                tma_load_4d(dst + PF_BOX, &tm_q, q_full, 64, h, q0 + t * PF_BM, b);
            }
            const int z = b * a.Hk + kvh;
            int u = 0;
            if constexpr (WINDOW) {
                // ring sequence: K_j, V_j for the CTA's key tiles j in increasing order
                for (int j = first_in(lo_u); j <= d_u && !*s_abort; j = next_in(lo_u, j)) {
                    for (int kv = 0; kv < 2; ++kv, ++u) {
                        const int slot = u % PF_SLOTS;
                        if (u >= PF_SLOTS && !mbar_wait(&kv_empty[slot], ((u / PF_SLOTS) - 1) & 1)) {
                            *s_abort = 1;
                            break;
                        }
                        mbar_arrive_expect_tx(&kv_full[slot], PF_TILE);
                        uint8_t* dst = smem + PF_OFF_KV + slot * PF_TILE;
                        const CUtensorMap* m = kv == 0 ? &tm_k : &tm_v;
                        tma_load_3d(dst, m, &kv_full[slot], 0, j * PF_BN, z);
                        tma_load_3d(dst + PF_BOX, m, &kv_full[slot], 64, j * PF_BN, z);
                    }
                }
            } else {
                // ring sequence: K_0, V_0, K_1, V_1, ...
                for (int j = 0; j < n_kv && !*s_abort; ++j) {
                    for (int kv = 0; kv < 2; ++kv, ++u) {
                        const int slot = u % PF_SLOTS;
                        if (u >= PF_SLOTS && !mbar_wait(&kv_empty[slot], ((u / PF_SLOTS) - 1) & 1)) {
                            *s_abort = 1;
                            break;
                        }
                        mbar_arrive_expect_tx(&kv_full[slot], PF_TILE);
                        uint8_t* dst = smem + PF_OFF_KV + slot * PF_TILE;
                        const CUtensorMap* m = kv == 0 ? &tm_k : &tm_v;
                        tma_load_3d(dst, m, &kv_full[slot], 0, j * PF_BN, z);
                        tma_load_3d(dst + PF_BOX, m, &kv_full[slot], 64, j * PF_BN, z);
                    }
                }
            }
            if (*s_abort) report_status(a.dev_status, KVATTN_STATUS_TIMEOUT);
            for (int x = u - PF_SLOTS > 0 ? u - PF_SLOTS : 0; x < u; ++x)
                mbar_wait(&kv_full[x % PF_SLOTS], (x / PF_SLOTS) & 1);
        }
    } else if (warp == 8) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 64;" ::: "memory");
        // ===== MMA issue (one thread) =====
        if (lane == 0) {
            const uint32_t sq = smem_u32(smem + PF_OFF_Q);
            const uint32_t skv = smem_u32(smem + PF_OFF_KV);
            bool ok = mbar_wait(q_full, 0);
            int u = 0;
            auto issue_s = [&](int t, uint32_t kslot_addr) {
                const uint32_t d = tmem + t * PF_BN;  // S_t
                const uint32_t qa = sq + t * PF_TILE;
#pragma unroll
                for (int ks = 0; ks < PF_D / 16; ++ks) {
                    const uint32_t off = (ks >> 2) * PF_BOX + (ks & 3) * 32;
                    tc_mma_bf16(d, umma_desc_k_sw128(qa + off), umma_desc_k_sw128(kslot_addr + off), PF_IDESC_S,
                                ks > 0 ? 1u : 0u);
                }
                tc_commit(&s_full[t]);
            };
            auto issue_pv = [&](int t, bool acc, uint32_t vslot_addr) {
                const uint32_t d = tmem + 256 + t * PF_D;  // O_t
                const uint32_t pa = tmem + t * PF_BN;      // P_t over S_t, bf16 pairs
#pragma unroll
                for (int ks = 0; ks < PF_BN / 16; ++ks) {
                    // V tile [keys][d]: 16 keys = 2 eight-row atoms (2 KB); the two 64-wide d blocks 16 KB apart
                    const uint64_t bd = umma_desc_mn_sw128(vslot_addr + ks * 2048, PF_BOX, 1024);
                    tc_mma_bf16_ts(d, pa + ks * 8, bd, PF_IDESC_O, (acc || ks > 0) ? 1u : 0u);
                }
                tc_commit(&pv_done[t]);
            };
            if constexpr (WINDOW) {
                // scores of the first key tile for the Q tiles that see it
                int cnt[2] = {0, 0};  // P V products issued per Q tile
                int kslot = 0;
                int j = first_in(lo_u);
                if (ok) {
                    kslot = u % PF_SLOTS;
                    ok = mbar_wait(&kv_full[kslot], (u / PF_SLOTS) & 1);
                    ++u;
                }
                if (ok) {
                    tc_fence_after();
                    const uint32_t ka = skv + kslot * PF_TILE;
                    for (int t = 0; t < 2; ++t)
                        if (in_t(t, j)) issue_s(t, ka);
                    tc_commit(&kv_empty[kslot]);
                }
                // per key tile: each Q tile's P V, then at once its next scores (as in the plain loop)
                for (; j <= d_u && ok;) {
                    const int jn = next_in(lo_u, j);
                    const int vslot = u % PF_SLOTS;
                    ok = mbar_wait(&kv_full[vslot], (u / PF_SLOTS) & 1);
                    ++u;
                    if (!ok) break;
                    const uint32_t va = skv + vslot * PF_TILE;
                    const bool more = jn <= d_u;
                    uint32_t ka = 0;
                    for (int t = 0; t < 2 && ok; ++t) {
                        if (in_t(t, j)) {
                            ok = mbar_wait(&p_full[t], cnt[t] & 1);
                            if (!ok) break;
                            tc_fence_after();
                            issue_pv(t, cnt[t] > 0, va);
                            ++cnt[t];
                        }
                        if (more && t == 0) {
                            kslot = u % PF_SLOTS;
                            ok = mbar_wait(&kv_full[kslot], (u / PF_SLOTS) & 1);
                            ++u;
                            if (!ok) break;
                            ka = skv + kslot * PF_TILE;
                        }
                        if (more && in_t(t, jn)) {
                            // P_t (read by this Q tile's last P V) shares columns with S_t: wait for it
                            if (cnt[t] > 0) {
                                ok = mbar_wait(&pv_done[t], (cnt[t] - 1) & 1);
                                if (!ok) break;
                                tc_fence_after();
                            }
                            issue_s(t, ka);
                        }
                    }
                    if (!ok) break;
                    tc_commit(&kv_empty[vslot]);
                    if (more) tc_commit(&kv_empty[kslot]);
                    j = jn;
                }
            } else {
                // S for tile 0 of every Q tile
                int kslot = 0;
                if (ok) {
                    kslot = u % PF_SLOTS;
                    ok = mbar_wait(&kv_full[kslot], (u / PF_SLOTS) & 1);
                    ++u;
                }
                if (ok) {
                    tc_fence_after();
                    const uint32_t ka = skv + kslot * PF_TILE;
                    if (n_kv0 > 0) issue_s(0, ka);
                    if (n_qt > 1) issue_s(1, ka);
                    tc_commit(&kv_empty[kslot]);
                }
                // Per key tile j: each Q tile's P V, then at once its next scores (S_t shares its
                // columns with P_t, so the scores wait for that P V), so that Q tile 0's next
                // scores never wait for Q tile 1's softmax.
                for (int j = 0; j < n_kv && ok; ++j) {
                    const int vslot = u % PF_SLOTS;
                    ok = mbar_wait(&kv_full[vslot], (u / PF_SLOTS) & 1);
                    ++u;
                    if (!ok) break;
                    const uint32_t va = skv + vslot * PF_TILE;
                    const bool more = j + 1 < n_kv;
                    uint32_t ka = 0;
                    for (int t = 0; t < n_qt && ok; ++t) {
                        if (j < n_kv0 + t) {  // Q tile 0 stops one tile earlier
                            ok = mbar_wait(&p_full[t], j & 1);
                            if (!ok) break;
                            tc_fence_after();
                            issue_pv(t, j > 0, va);
                        }
                        if (more && t == 0) {
                            kslot = u % PF_SLOTS;
                            ok = mbar_wait(&kv_full[kslot], (u / PF_SLOTS) & 1);
                            ++u;
                            if (!ok) break;
                            ka = skv + kslot * PF_TILE;
                        }
                        if (more && j + 1 < n_kv0 + t) {
                            // P_t (read by the P V just issued) shares columns with S_t: wait for it
                            ok = mbar_wait(&pv_done[t], j & 1);
                            if (!ok) break;
                            tc_fence_after();
                            issue_s(t, ka);
                        }
                    }
                    if (!ok) break;
                    tc_commit(&kv_empty[vslot]);
                    if (more) tc_commit(&kv_empty[kslot]);
                }
            }
            if (!ok) {
                *s_abort = 1;
                report_status(a.dev_status, KVATTN_STATUS_TIMEOUT);
            }
            tc_commit(mma_done);
            mbar_wait(mma_done, 0);
        }
    } else if (warp < 8) {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 216;" ::: "memory");
        // ===== softmax + epilogue: warps 0-3 -> Q tile 0, warps 4-7 -> Q tile 1 =====
        const int t = warp >> 2;
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;  // query row in the tile = TMEM lane
        const int qrow = q0 + t * PF_BM + row;
        const int lo_t = lo_of(t), dg = diag_of(t);
        // keys <= qrow - window (and not sinks) are outside the band; only tiles whose lowest key
        // can fall that low for the tile's last row need the test
        const int band_top = q0 + t * PF_BM + PF_BM - 1 - a.window;
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t s_addr = tmem + lane_off + t * PF_BN;
        const uint32_t o_addr = tmem + lane_off + 256 + t * PF_D;
        const float sl2 = a.scale * kLog2e;
        float m_run = -INFINITY, l_run = 0.f;
        if (t < n_qt) {
            int k = 0;  // steps of this Q tile
            for (int j = WINDOW ? first_in(lo_t) : 0; j <= dg; j = WINDOW ? next_in(lo_t, j) : j + 1, ++k) {
                if (!warp_wait(&s_full[t], k & 1, s_abort)) continue;
                tc_fence_after();
                const bool diag = j == dg;  // keys j*128 .. : the diagonal tile
                const bool band = WINDOW && j * PF_BN <= band_top;
                const int kbase = j * PF_BN;
                // The row's 128 raw scores in registers (four 32-column loads in flight, one wait):
                // the row max (scale > 0 commutes with the max), then the exponentials from the
                // same registers.
                uint32_t sv[4][32];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(s_addr + c * 32, sv[c]);
                tmem_wait_ld();
                float mxc[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};  // four independent chains
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    tmem_regs_ready(sv[c]);
                    if constexpr (WINDOW) {
                        if (diag || band) {
#pragma unroll
                            for (int i = 0; i < 32; ++i) {
                                const int key = kbase + c * 32 + i;
                                // -inf: key after the query, or below its band and not a sink
                                if (key > qrow || (band && key <= qrow - a.window && key >= a.n_sink))
                                    sv[c][i] = 0xff800000u;
                            }
                        }
                    } else if (diag) {
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (c * 32 + i > row) sv[c][i] = 0xff800000u;  // -inf: key after the query
                    }
#pragma unroll
                    for (int i = 0; i < 32; i += 2)
                        mxc[c] = fmax3(mxc[c], __uint_as_float(sv[c][i]), __uint_as_float(sv[c][i + 1]));
                }
                float mx = fmaxf(fmaxf(mxc[0], mxc[1]), fmaxf(mxc[2], mxc[3])) * sl2;
                // Move this row's reference max only when it grows by more than 2^8.
                // The O rescale uses warp-collective TMEM loads/stores, so the
                // warp takes that path together (alpha = 1 for rows that keep
                // their reference).
                const bool move = mx > m_run + kRescaleThreshold || m_run == -INFINITY;
                const float m_new = move ? fmaxf(mx, m_run) : m_run;
                const bool rescale = move && m_run != -INFINITY && k > 0;
                if (__any_sync(0xffffffffu, rescale)) {
                    const float alpha = rescale ? fast_exp2(m_run - m_new) : 1.f;
                    l_run *= alpha;
#pragma unroll 1
                    for (int c = 0; c < 4; ++c) {
                        uint32_t ov[32];
                        tmem_ld32(o_addr + c * 32, ov);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
                        tmem_st32(o_addr + c * 32, ov);
                    }
                }
                m_run = m_new;
                const float mu = m_run == -INFINITY ? 0.f : m_run;
                const float2 sc2 = make_float2(sl2, sl2), nmu = make_float2(-mu, -mu);
                float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                                 make_float2(0.f, 0.f)};  // four independent sums
                // p = 2^(s * scale * log2 e - m) -> bf16 P over the first 64 S columns (chunk c's
                // P lands in columns 16c..16c+15; every score is already in registers)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float2 x = __ffma2_rn(
                            make_float2(__uint_as_float(sv[c][2 * i]), __uint_as_float(sv[c][2 * i + 1])), sc2, nmu);
                        float2 pr;
                        if ((i & 3) == 0) {
                            pr = exp2_fma2(x);  // a quarter of the exponentials off the MUFU pipe
                        } else {
                            pr.x = fast_exp2(x.x);
                            pr.y = fast_exp2(x.y);
                        }
                        acc[i & 3] = __fadd2_rn(acc[i & 3], pr);
                        pk[i] = pack_bf16x2(pr.x, pr.y);
                    }
                    asm volatile(
                        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
                        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(
                            s_addr + c * 16),
                        "r"(pk[0]), "r"(pk[1]), "r"(pk[2]), "r"(pk[3]), "r"(pk[4]), "r"(pk[5]), "r"(pk[6]),
                        "r"(pk[7]), "r"(pk[8]), "r"(pk[9]), "r"(pk[10]), "r"(pk[11]), "r"(pk[12]), "r"(pk[13]),
                        "r"(pk[14]), "r"(pk[15])
                        : "memory");
                }
                const float2 a01 = __fadd2_rn(acc[0], acc[1]), a23 = __fadd2_rn(acc[2], acc[3]);
                const float ls = (a01.x + a01.y) + (a23.x + a23.y);
                l_run += ls;
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[t]);
            }
            // ---- epilogue: O / l -> bf16 rows, lse ----
            if (warp_wait(&pv_done[t], (k - 1) & 1, s_abort)) {
                tc_fence_after();
                const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
                __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.out) +
                                      ((static_cast<long long>(b) * a.T + qrow) * a.H + h) * PF_D;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t ov[32];
                    tmem_ld32(o_addr + c * 32, ov);
                    tmem_wait_ld();
                    if (qrow < a.T) {
#pragma unroll
                        for (int i = 0; i < 32; i += 8) {
                            uint4 w;
                            w.x = pack_bf16x2(__uint_as_float(ov[i]) * inv, __uint_as_float(ov[i + 1]) * inv);
                            w.y = pack_bf16x2(__uint_as_float(ov[i + 2]) * inv, __uint_as_float(ov[i + 3]) * inv);
                            w.z = pack_bf16x2(__uint_as_float(ov[i + 4]) * inv, __uint_as_float(ov[i + 5]) * inv);
                            w.w = pack_bf16x2(__uint_as_float(ov[i + 6]) * inv, __uint_as_float(ov[i + 7]) * inv);
                            *reinterpret_cast<uint4*>(orow + c * 32 + i) = w;
                        }
                    }
                }
                if (a.lse && qrow < a.T)
                    a.lse[(static_cast<long long>(b) * a.H + h) * a.T + qrow] =
                        l_run > 0.f ? (m_run + __log2f(l_run)) * kLn2 : -INFINITY;
            }
        }
    } else {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 64;" ::: "memory");  // warps 10-11: idle
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 8) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace

cudaError_t launch_prefill(const PrefillLaunch& l, const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                           const CUtensorMap& tm_v, cudaStream_t stream)
{
    static bool attr_set[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 64 && !attr_set[dev]) {
        e = cudaFuncSetAttribute(prefill_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, PF_SMEM);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(prefill_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, PF_SMEM);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    PrefillArgs a{};
    a.out = l.out;
    a.lse = l.lse;
    a.dev_status = l.dev_status;
    a.B = l.B;
    a.T = l.T;
    a.H = l.H;
    a.Hk = l.Hk;
    a.g = l.H / l.Hk;
    a.n_qblk = (l.T + 2 * PF_BM - 1) / (2 * PF_BM);
    a.scale = l.scale;
    a.n_sink = l.n_sink;
    a.window = l.window;
    const long long grid = static_cast<long long>(a.n_qblk) * l.B * l.H;
    return launch_pdl(a.window > 0 ? prefill_kernel<true> : prefill_kernel<false>, dim3(static_cast<unsigned>(grid)), dim3(PF_THREADS), PF_SMEM, stream, tm_q,
                      tm_k, tm_v, a);
}

}  // namespace kvattn
