// decode.cu -- one new query per sequence over a bf16 KV cache, all query
// heads of a KV group served by a single read of each K/V tile.
//
// Method: softmax(scale q k^T) v per query head, query head h reading KV head
// h / g ("注意力变体与 MoE", GQA attention(): the g heads of a group share one
// K/V and a real kernel reads the shared block once; "attention",
// GroupQueryAttention).  The cache is read exactly once: decode is bound by
// HBM, with g FLOP per byte (same page, decode roofline).
//
// Work split (ragged, balanced by tiles, computed on the device from the
// lengths): the cache rows of every (batch, kv-head) unit are cut into tiles
// of 64 rows; all tiles of all units form one ordered list of N tiles; CTA c
// of G = min(grid, N) CTAs owns tiles x with floor(x G / N) == c, a
// contiguous range.  Where a range crosses units it produces one "piece" per
// unit.  A unit that lies inside one CTA is finished there; otherwise every
// piece writes an unnormalised partial (O, running max, sum) and a second
// kernel merges the partials of the unit (the split-softmax identity).
//
// CTA: 4 consumer warps + 1 TMA producer warp.  K and V tiles [64 x d] land in
// shared memory through a 3-D tensor map (d, T_max, B*Hk) with 128-byte
// swizzle, STAGES deep, one mbarrier pair per stage.  Consumers run bf16
// mma.sync m16n8k16 with the query heads of the group as the M rows (a group
// of g <= 16 heads is one M tile, zero-padded; g = 32/64 use 2/4 M tiles),
// fp32 accumulation, online softmax in base 2 with quad shuffles.
//
// Gather mode (a sparse token list per sequence, "attention" page, "Qwen Sparse
// Attention (QSA)" ③–④: the selected tokens' full-precision K/V are fetched from
// the cache by index and standard GQA attention runs over them): a unit's rows
// are the listed cache rows.  GATHER_WARPS producer warps copy each 64-row tile
// with 16-byte cp.async (a 256-byte row = 16 lanes; each warp its share of the
// rows, with the row indices staged in shared memory) into the same swizzled
// layout as the tiled loads, each lane arriving asynchronously on the stage
// barrier once its copies land, and the first one passes the tile's valid-row
// bitmask (skipped entries, the tail) along.  Row gathers through the copy engine
// (per-row bulk copies, tile::gather4) were measured slower: the engine sustains
// few small copies in flight per SM.
#include <type_traits>

#include "common.cuh"
#include "decode_plan.cuh"
#include "kernels.h"

namespace kvattn {

namespace {

constexpr int TILE = DEC_TILE;  // cache rows per pipeline stage
constexpr int CWARPS = 4;  // consumer warps
constexpr int THREADS = 32 * (CWARPS + 1);
constexpr int GATHER_WARPS = 2;  // gather mode: producer warps
constexpr int IDX_TILES = GATHER_WARPS <= 2 ? 8 : 4;  // tiles whose row indices a producer warp stages at once
constexpr int threads_of(bool gather) { return 32 * (CWARPS + (gather ? GATHER_WARPS : 1)); }
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kLog2e = 1.44269504088896340736f;

template <int D, int NMT, bool GATHER>
struct Cfg {
    static constexpr int STAGES = D == 128 ? 5 : 8;
    static constexpr int HALVES = D / 64;  // 128-byte column blocks per row
    static constexpr int TILE_BYTES = TILE * D * 2;
    static constexpr int STAGE_BYTES = 2 * TILE_BYTES;  // K tile + V tile
    static constexpr int SCR_STRIDE = D + 8;            // floats per scratch row
    static constexpr int OFF_SCR_O = STAGES * STAGE_BYTES;
    static constexpr int OFF_SCR_ML = OFF_SCR_O + CWARPS * 16 * SCR_STRIDE * 4;
    static constexpr int OFF_Q = OFF_SCR_ML + CWARPS * 16 * 2 * 4;  // q rows of the next piece
    static constexpr int Q_BYTES = NMT * 16 * D * 2;
    static constexpr int OFF_CS = OFF_Q + Q_BYTES;                   // cos row | sin row of its position
    static constexpr int OFF_QPOS = OFF_CS + 2 * (D / 2) * 4;        // [DECODE_MAX_B] query positions
    static constexpr int OFF_N = OFF_QPOS + DECODE_MAX_B * 4;
    static constexpr int OFF_UB = OFF_N + DECODE_MAX_B * 4;
    static constexpr int OFF_LEN = OFF_UB + (DECODE_MAX_B + 1) * 4;
    static constexpr int OFF_BAR = ((OFF_LEN + DECODE_MAX_B * 4) + 7) / 8 * 8;
    static constexpr int OFF_MISC = OFF_BAR + (2 * STAGES + 2) * 8;
    static constexpr int OFF_MASK = OFF_MISC + 64;                  // [STAGES] valid rows (gather mode)
    static constexpr int OFF_IDX = (OFF_MASK + STAGES * 8 + 15) / 16 * 16;  // [GATHER_WARPS][IDX_TILES * TILE] rows
    static constexpr int SMEM = OFF_IDX + (GATHER ? GATHER_WARPS * IDX_TILES * TILE * 4 : 0) + 1024;  // + slack
    static_assert(SMEM <= 232448, "shared memory");
};

// Byte offset of the 16-byte chunk holding dims dim .. dim+7 of row `tok` in a K or V
// tile of 128-byte-swizzled 64-column blocks.
__device__ __forceinline__ uint32_t tile_off(int tok, int dim)
{
    return static_cast<uint32_t>((dim >> 6) * (TILE * 128)) + swz128(tok, (dim & 63) >> 3);
}

__device__ __forceinline__ uint32_t ld_u32(const kvattn_bf16* p)
{
    return *reinterpret_cast<const uint32_t*>(p);
}

// ---- RoPE of query rows held in shared memory ------------------------------------
// rows [rows][D] bf16, contiguous; cos/sin rows of D/2 entries.  nthr threads each
// take 8-element chunks (adjacent pairs) or pairs of chunks d/2 apart (half-split).
__device__ __forceinline__ void rope_rows_smem(uint8_t* rows, int nrows, int D, const float* cs, const float* sn,
                                               int pair_style, int tid, int nthr)
{
    __nv_bfloat16* q = reinterpret_cast<__nv_bfloat16*>(rows);
    if (pair_style == 0) {
        const int per = D / 8;
        for (int i = tid; i < nrows * per; i += nthr) {
            const int r = i / per, ch = i - r * per;
            const float cc[4] = {cs[4 * ch], cs[4 * ch + 1], cs[4 * ch + 2], cs[4 * ch + 3]};
            const float ss[4] = {sn[4 * ch], sn[4 * ch + 1], sn[4 * ch + 2], sn[4 * ch + 3]};
            uint4* p = reinterpret_cast<uint4*>(q + r * D + ch * 8);
            *p = rope_chunk_adjacent(*p, cc, ss);
        }
    } else {
        const int per = D / 16, half = D / 2;
        for (int i = tid; i < nrows * per; i += nthr) {
            const int r = i / per, ch = i - r * per;
            float cc[8], ss[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                cc[j] = cs[8 * ch + j];
                ss[j] = sn[8 * ch + j];
            }
            uint4* pa = reinterpret_cast<uint4*>(q + r * D + ch * 8);
            uint4* pb = reinterpret_cast<uint4*>(q + r * D + half + ch * 8);
            uint4 ra = *pa, rb = *pb;
            rope_chunk_half(ra, rb, cc, ss);
            *pa = ra;
            *pb = rb;
        }
    }
}

// ---- merge of a split unit ------------------------------------------------------
// The softmax over a union of key sets is the max-shifted mix of its parts: with
// M = max_j m_j, L = sum_j 2^(m_j - M) l_j and w_j = 2^(m_j - M) / L,
// out = sum_j w_j O_j and lse = ln 2 (M + log2 L).  Thread items are (head,
// 4 dims); an item requests every slot's (m, l) and O chunk at once, so the merge
// costs one memory round trip (the weights are recomputed per item).
constexpr int MERGE_MAX_BATCH = 8;

template <int D>
__device__ void merge_unit(const DecodeArgs& a, int u, int S, int count, int tid, int nthr)
{
    const int g = a.g;
    const int b = u / a.Hk, kvh = u - b * a.Hk;
    const long long bh0 = static_cast<long long>(b) * a.H + static_cast<long long>(kvh) * g;
    constexpr int Q4 = D / 4;
    const long long ml_step = g;                              // float2 per slot
    const long long o_step = static_cast<long long>(g) * Q4;  // float4 per slot
    for (int idx = tid; idx < g * Q4; idx += nthr) {
        const int h = idx / Q4, q4 = idx - h * Q4;
        const float2* ml = reinterpret_cast<const float2*>(a.part_ml) + static_cast<long long>(S) * g + h;
        const float4* o = reinterpret_cast<const float4*>(a.part_o + (static_cast<long long>(S) * g + h) * D) + q4;
        float M = -INFINITY, L = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j0 = 0; j0 < count; j0 += MERGE_MAX_BATCH) {
            float2 mlv[MERGE_MAX_BATCH];
            float4 ov[MERGE_MAX_BATCH];
#pragma unroll
            for (int j = 0; j < MERGE_MAX_BATCH; ++j) {
                if (j0 + j < count) {
                    mlv[j] = __ldcg(ml + (j0 + j) * ml_step);
                    ov[j] = __ldcg(o + (j0 + j) * o_step);
                }
            }
            float Mb = M;
#pragma unroll
            for (int j = 0; j < MERGE_MAX_BATCH; ++j)
                if (j0 + j < count) Mb = fmaxf(Mb, mlv[j].x);
            const float r = M == -INFINITY ? 0.f : fast_exp2(M - Mb);
            L *= r;
            acc.x *= r;
            acc.y *= r;
            acc.z *= r;
            acc.w *= r;
            M = Mb;
#pragma unroll
            for (int j = 0; j < MERGE_MAX_BATCH; ++j) {
                if (j0 + j < count) {
                    // a piece whose rows were all skipped (gather mode) has m = -inf, l = 0
                    const float e = mlv[j].x == -INFINITY ? 0.f : fast_exp2(mlv[j].x - M);
                    L += e * mlv[j].y;
                    acc.x += e * ov[j].x;
                    acc.y += e * ov[j].y;
                    acc.z += e * ov[j].z;
                    acc.w += e * ov[j].w;
                }
            }
        }
        const float inv = L > 0.f ? 1.f / L : 0.f;
        *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(a.out) + (bh0 + h) * D + 4 * q4) =
            make_uint2(pack_bf16x2(acc.x * inv, acc.y * inv), pack_bf16x2(acc.z * inv, acc.w * inv));
        if (q4 == 0 && a.lse) a.lse[bh0 + h] = L > 0.f ? (M + __log2f(L)) * kLn2 : -INFINITY;
    }
}

// ---- the decode kernel ---------------------------------------------------------

static_assert(TILE == 64, "gather mode passes a tile's valid rows as one 64-bit mask");

template <int D, int NMT, bool GATHER>
__global__ void __launch_bounds__(threads_of(GATHER), 1)
    decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v, DecodeArgs a)
{
    using C = Cfg<D, NMT, GATHER>;
    constexpr int WPM = CWARPS / NMT;  // warps sharing one M tile (split the tile's rows)
    constexpr int TPW = TILE / WPM;    // cache rows per warp per tile
    constexpr int NT = TPW / 8;        // score n-tiles per warp
    constexpr int KS = D / 16;         // k-steps of q.k
    constexpr int DT = D / 8;          // output n-tiles

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* scr_o = reinterpret_cast<float*>(smem + C::OFF_SCR_O);
    float* scr_ml = reinterpret_cast<float*>(smem + C::OFF_SCR_ML);
    int* s_n = reinterpret_cast<int*>(smem + C::OFF_N);
    int* s_Ub = reinterpret_cast<int*>(smem + C::OFF_UB);
    int* s_len = reinterpret_cast<int*>(smem + C::OFF_LEN);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* empty = full + C::STAGES;
    uint64_t* q_full = empty + C::STAGES;
    uint64_t* q_empty = q_full + 1;
    uint8_t* sQ = smem + C::OFF_Q;
    float* sCos = reinterpret_cast<float*>(smem + C::OFF_CS);
    float* sSin = sCos + D / 2;
    int* s_qpos = reinterpret_cast<int*>(smem + C::OFF_QPOS);
    const bool rope = a.cos_tab != nullptr;
    int* s_misc = reinterpret_cast<int*>(smem + C::OFF_MISC);
    volatile int* s_abort = s_misc + 1;
    int* s_merge = s_misc + 4;  // [0] = split pieces made here, then (unit, first slot, pieces) x 2
    uint64_t* s_mask = reinterpret_cast<uint64_t*>(smem + C::OFF_MASK);  // valid rows of each stage (gather)
    int* s_idx = reinterpret_cast<int*>(smem + C::OFF_IDX);  // staged row indices, per producer warp (gather)

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const unsigned long long wlim = a.wait_ns ? a.wait_ns : WAIT_LIMIT_NS;
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            // gather mode: every producer lane arrives once its copies land, plus the mask arrival
            mbar_init(&full[s], GATHER ? 32 * GATHER_WARPS + 1 : 1);
            mbar_init(&empty[s], CWARPS);
        }
        mbar_init(q_full, 1);
        mbar_init(q_empty, CWARPS);
        *s_abort = 0;
        s_merge[0] = 0;
        fence_barrier_init();
    }
    if (warp == CWARPS && lane == 0) {
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    // everything above overlaps the previous kernel of the stream
    pdl_wait();
    pdl_trigger();
    const long long N = plan_prefix(a.seq_lens, a.B, a.Hk, GATHER ? a.n_idx : a.T_max, s_len, s_n, s_Ub,
                                    a.dev_status, blockIdx.x == 0, rope ? a.q_pos : nullptr, s_qpos,
                                    a.len_cap);
    // empty sequences have no tiles: their heads get zeros and lse = -inf here
    for (int b = blockIdx.x; b < a.B; b += gridDim.x) {
        if (s_len[b] != 0) continue;
        __nv_bfloat16* ob = reinterpret_cast<__nv_bfloat16*>(a.out) + static_cast<long long>(b) * a.H * D;
        for (int i = threadIdx.x; i < a.H * D; i += blockDim.x) ob[i] = __float2bfloat16_rn(0.f);
        if (a.lse)
            for (int h = threadIdx.x; h < a.H; h += blockDim.x) a.lse[static_cast<long long>(b) * a.H + h] = -INFINITY;
    }
    if (N == 0) return;
    // With fewer tiles than CTAs only the first N CTAs take part, so that every
    // participating CTA owns at least one tile and the CTAs owning a unit's
    // tiles are consecutive (the piece count of a unit is then exact).
    const int G = static_cast<int>(N < a.grid ? N : a.grid), c = blockIdx.x;
    if (c >= G) return;
    const long long lo = range_start(c, N, G), hi = range_start(c + 1, N, G);

    // the unit holding tile `lo`, and the partial slots of the units before it
    Walk w_start = walk_from(lo, a.B, a.Hk, s_n, s_Ub, 0);
    w_start.S = slots_before(w_start.b * a.Hk + w_start.kvh, a.Hk, s_n, s_Ub, N, G, s_misc + 2);

    if (warp >= CWARPS) {
        // ===== producer: streams K/V tiles of every piece in order (one thread with
        // the tensor maps; GATHER_WARPS whole warps in gather mode) =====
        if (!GATHER && lane != 0) return;
        const int pw = warp - CWARPS;  // producer warp (gather mode)
        int* my_idx = s_idx + pw * (IDX_TILES * TILE);
        // gather mode: a warp-wide copy instruction moves RPI rows (CPR lanes x 16 bytes
        // each); lane group my_r copies rows my_r * NI .. my_r * NI + NI - 1 of a tile,
        // producer warp pw the NIW of them starting at pw * NIW
        constexpr int CPR = D / 8;
        constexpr int RPI = 32 / CPR;
        constexpr int NI = TILE / RPI;
        constexpr int NIW = NI / GATHER_WARPS;
        static_assert(NIW % 4 == 0, "row indices are read four at a time");
        const int my_r = lane / CPR, my_ch = lane % CPR;
        const uint32_t my_dst = (my_ch >> 3) * (TILE * 128);
        Walk w = w_start;
        int it = 0, np = 0;
        bool ok = true;
        const uint32_t q_bytes = static_cast<uint32_t>(a.g) * D * 2;
        const uint64_t pol = l2_evict_first_policy();  // K and V are read once
        for (; ok && w.U < hi && w.b < a.B; walk_next(w, a.B, a.Hk, s_n, N, G)) {
            long long tb, te;
            if (!piece_tiles(w, s_n[w.b], lo, hi, tb, te)) continue;
            const int z = w.b * a.Hk + w.kvh;
            // the piece's g query rows (contiguous), once the consumers hold the previous ones
            if (np > 0 && pw == 0) {
                const bool got = GATHER ? warp_wait(q_empty, (np - 1) & 1, s_abort, wlim)
                                        : (!*s_abort && mbar_wait(q_empty, (np - 1) & 1, wlim));
                if (!got) {
                    ok = false;
                    break;
                }
            }
            // with RoPE, the cos and sin rows of the query's position come along
            if (lane == 0 && pw == 0) {
                const int qp = rope ? s_qpos[w.b] : -1;
                const bool rot = rope && qp >= 0 && qp < a.max_pos;
                mbar_arrive_expect_tx(q_full, q_bytes + (rot ? D * 4 : 0));
                bulk_load(sQ, a.q + (static_cast<long long>(w.b) * a.H + static_cast<long long>(w.kvh) * a.g) * D,
                          q_bytes, q_full);
                if (rot) {
                    bulk_load(sCos, a.cos_tab + static_cast<long long>(qp) * (D / 2), D * 2, q_full);
                    bulk_load(sSin, a.sin_tab + static_cast<long long>(qp) * (D / 2), D * 2, q_full);
                }
            }
            ++np;
            // gather mode: the row indices of up to IDX_TILES tiles at a time are staged in
            // shared memory (all loads in flight together: one round trip per chunk)
            const int cnt = s_len[w.b];
            const int32_t* irow = GATHER ? a.idx + static_cast<long long>(w.b) * a.n_idx : nullptr;
            long long chunk_t0 = -IDX_TILES;
            for (long long t = tb; t < te; ++t, ++it) {
                if (GATHER && t >= chunk_t0 + IDX_TILES) {
                    chunk_t0 = t;
                    const int e0 = static_cast<int>(t) * TILE;
                    int v[IDX_TILES * TILE / 32];
#pragma unroll
                    for (int u = 0; u < IDX_TILES * TILE / 32; ++u) {
                        const int e = e0 + u * 32 + lane;
                        v[u] = e < cnt ? __ldg(irow + e) : -1;
                    }
                    __syncwarp();  // the previous chunk has been read by every lane
#pragma unroll
                    for (int u = 0; u < IDX_TILES * TILE / 32; ++u) my_idx[u * 32 + lane] = v[u];
                    __syncwarp();
                }
                const int s = it % C::STAGES;
                const uint32_t ph = (it / C::STAGES) & 1;
                if (it >= C::STAGES) {
                    const bool got = GATHER ? warp_wait(&empty[s], ph ^ 1, s_abort, wlim)
                                            : (!*s_abort && mbar_wait(&empty[s], ph ^ 1, wlim));
                    if (!got) {
                        ok = false;
                        break;
                    }
                }
                uint8_t* kd = smem + s * C::STAGE_BYTES;
                uint8_t* vd = kd + C::TILE_BYTES;
                if constexpr (!GATHER) {
                    if (blockIdx.x == 0 && it == a.drop_it) continue;  // testing: a tile never loaded
                    mbar_arrive_expect_tx(&full[s], C::STAGE_BYTES);
#pragma unroll
                    for (int h = 0; h < C::HALVES; ++h) {
                        tma_load_3d_hint(kd + h * (TILE * 128), &tm_k, &full[s], h * 64, static_cast<int>(t * TILE), z,
                                         pol);
                        tma_load_3d_hint(vd + h * (TILE * 128), &tm_v, &full[s], h * 64, static_cast<int>(t * TILE), z,
                                         pol);
                    }
                } else {
                    const int rb = static_cast<int>(t - chunk_t0) * TILE;
                    const int ia = my_idx[rb + lane], ib = my_idx[rb + 32 + lane];
                    const bool va = ia >= 0 && ia < a.T_max, vb = ib >= 0 && ib < a.T_max;
                    if (pw == 0 && (ia < -1 || ia >= a.T_max || ib < -1 || ib >= a.T_max))
                        report_status(a.dev_status, KVATTN_STATUS_BAD_INDEX);
                    const uint32_t ma = __ballot_sync(0xffffffffu, va), mb = __ballot_sync(0xffffffffu, vb);
                    const kvattn_bf16* kz = a.k_cache + static_cast<long long>(z) * a.T_max * D + my_ch * 8;
                    const kvattn_bf16* vz = a.v_cache + static_cast<long long>(z) * a.T_max * D + my_ch * 8;
                    const uint32_t sk = smem_u32(kd) + my_dst, sv = smem_u32(vd) + my_dst;
                    const int r0 = my_r * NI + pw * NIW;  // first row of the tile this lane copies
                    int rows[NIW];
#pragma unroll
                    for (int u = 0; u < NIW; u += 4) {
                        const int4 x4 = *reinterpret_cast<const int4*>(my_idx + rb + r0 + u);
                        rows[u] = x4.x;
                        rows[u + 1] = x4.y;
                        rows[u + 2] = x4.z;
                        rows[u + 3] = x4.w;
                    }
#pragma unroll
                    for (int u = 0; u < NIW; ++u) {
                        if (rows[u] >= 0 && rows[u] < a.T_max) {  // the row's mask bit
                            const long long off = static_cast<long long>(rows[u]) * D;
                            const uint32_t so = swz128(r0 + u, my_ch & 7);
                            cp_async16(sk + so, kz + off, 16);
                            cp_async16(sv + so, vz + off, 16);
                        }
                    }
                    cp_async_arrive_noinc(&full[s]);
                    if (pw == 0 && lane == 0) {
                        s_mask[s] = (static_cast<uint64_t>(mb) << 32) | ma;
                        mbar_arrive(&full[s]);
                    }
                }
            }
        }
        if (!ok && lane == 0) {
            *s_abort = 1;
            report_status(a.dev_status, KVATTN_STATUS_TIMEOUT);
        }
        // copies still in flight complete before the CTA leaves (bounded waits)
        if (GATHER) cp_async_wait<0>();
        if (lane == 0 && pw == 0) {
            for (int j = it - C::STAGES > 0 ? it - C::STAGES : 0; j < it; ++j)
                mbar_wait(&full[j % C::STAGES], (j / C::STAGES) & 1, wlim);
            if (np > 0) mbar_wait(q_full, (np - 1) & 1, wlim);
        }
        return;
    }

    // ===== consumers =====
    const int mt = warp / WPM, sub = warp % WPM;
    const int tok0 = sub * TPW;
    const int r0 = lane >> 2, cq = lane & 3;
    const int g = a.g;
    const float sl2 = a.scale * kLog2e;
    const int ctid = threadIdx.x;  // 0 .. 127
    const int rows_out = g < NMT * 16 ? g : NMT * 16;

    Walk w = w_start;
    int it = 0, piece = 0;
    for (; w.U < hi && w.b < a.B; walk_next(w, a.B, a.Hk, s_n, N, G)) {
        const int n = s_n[w.b];
        const int len = s_len[w.b];
        long long tb, te;
        if (!piece_tiles(w, n, lo, hi, tb, te)) continue;
        const int count = unit_count(w.U, n, N, G);
        const int slot = w.S + (c - unit_first_owner(w.U, N, G));

        // query fragments (A operand) from the prefetched rows: heads of the group, zero beyond g
        uint32_t qa[KS][4];
        {
            const bool have_q = warp_wait(q_full, piece & 1, s_abort, wlim);
            const uint8_t* qg = sQ;
            if (rope) {
                // rotate the piece's g query rows in place (bad positions: flagged, left as given)
                const int qp = s_qpos[w.b];
                if (qp >= 0 && qp < a.max_pos) {
                    if (have_q) rope_rows_smem(sQ, g, D, sCos, sSin, a.pair_style, ctid, CWARPS * 32);
                } else if (ctid == 0 && c == unit_first_owner(w.U, N, G)) {
                    report_status(a.dev_status, KVATTN_STATUS_BAD_POSITION);
                }
                // the rows are read below, and rewritten by the next bulk copy after q_empty
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                named_bar_sync(1, CWARPS * 32);
            }
            const int ra = mt * 16 + r0, rb = ra + 8;
            const bool va = have_q && ra < g, vb = have_q && rb < g;
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
                const int col = kk * 16 + 2 * cq;
                qa[kk][0] = va ? *reinterpret_cast<const uint32_t*>(qg + (ra * D + col) * 2) : 0u;
                qa[kk][1] = vb ? *reinterpret_cast<const uint32_t*>(qg + (rb * D + col) * 2) : 0u;
                qa[kk][2] = va ? *reinterpret_cast<const uint32_t*>(qg + (ra * D + col + 8) * 2) : 0u;
                qa[kk][3] = vb ? *reinterpret_cast<const uint32_t*>(qg + (rb * D + col + 8) * 2) : 0u;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(q_empty);
            ++piece;
        }
        float o[DT][4];
#pragma unroll
        for (int i = 0; i < DT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
        float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

        for (long long t = tb; t < te; ++t, ++it) {
            const int s = it % C::STAGES;
            const uint32_t ph = (it / C::STAGES) & 1;
            const bool have = warp_wait(&full[s], ph, s_abort, wlim);
            if (!have && lane == 0) report_status(a.dev_status, KVATTN_STATUS_TIMEOUT);
            if (have) {
                const uint32_t sK = smem_u32(smem + s * C::STAGE_BYTES);
                const uint32_t sV = sK + C::TILE_BYTES;
                const int n_valid = len - static_cast<int>(t) * TILE;  // >= 1
                // gather mode: bit r set = row r of the tile holds a listed cache row
                const uint64_t vm = GATHER ? s_mask[s] : ~0ull;

                // ---- S = Q K^T over this warp's rows of the tile ----
                float sc[NT][4];
#pragma unroll
                for (int i = 0; i < NT; ++i) sc[i][0] = sc[i][1] = sc[i][2] = sc[i][3] = 0.f;
                const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
                for (int kk = 0; kk < KS; ++kk) {
                    const int dim = kk * 16 + ((mi & 1) << 3);
#pragma unroll
                    for (int np = 0; np < NT / 2; ++np) {
                        const int tok = tok0 + np * 16 + rr + ((mi >> 1) << 3);
                        uint32_t b0, b1, b2, b3;
                        ldsm_x4(sK + tile_off(tok, dim), b0, b1, b2, b3);
                        mma_bf16_16816(sc[2 * np], qa[kk], b0, b1);
                        mma_bf16_16816(sc[2 * np + 1], qa[kk], b2, b3);
                    }
                }
                // ---- online softmax (base 2) ----
                float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
                for (int i = 0; i < NT; ++i) {
                    const int tk = tok0 + i * 8 + 2 * cq;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        float v = sc[i][e] * sl2;
                        if (GATHER ? ((vm >> (tk + (e & 1))) & 1ull) == 0ull : tk + (e & 1) >= n_valid)
                            v = -INFINITY;
                        sc[i][e] = v;
                    }
                    mx0 = fmaxf(mx0, fmaxf(sc[i][0], sc[i][1]));
                    mx1 = fmaxf(mx1, fmaxf(sc[i][2], sc[i][3]));
                }
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
                const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
                const float mu0 = mn0 == -INFINITY ? 0.f : mn0;
                const float mu1 = mn1 == -INFINITY ? 0.f : mn1;
                const float al0 = fast_exp2(m0 - mu0), al1 = fast_exp2(m1 - mu1);
                m0 = mn0;
                m1 = mn1;
                float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
                for (int i = 0; i < NT; ++i) {
                    sc[i][0] = fast_exp2(sc[i][0] - mu0);
                    sc[i][1] = fast_exp2(sc[i][1] - mu0);
                    sc[i][2] = fast_exp2(sc[i][2] - mu1);
                    sc[i][3] = fast_exp2(sc[i][3] - mu1);
                    ps0 += sc[i][0] + sc[i][1];
                    ps1 += sc[i][2] + sc[i][3];
                }
                l0 = l0 * al0 + ps0;
                l1 = l1 * al1 + ps1;
#pragma unroll
                for (int i = 0; i < DT; ++i) {
                    o[i][0] *= al0;
                    o[i][1] *= al0;
                    o[i][2] *= al1;
                    o[i][3] *= al1;
                }
                // ---- O += P V ----
                const bool tail = GATHER ? vm != ~0ull : n_valid < TILE;
#pragma unroll
                for (int j = 0; j < TPW / 16; ++j) {
                    uint32_t pa[4];
                    pa[0] = pack_bf16x2(sc[2 * j][0], sc[2 * j][1]);
                    pa[1] = pack_bf16x2(sc[2 * j][2], sc[2 * j][3]);
                    pa[2] = pack_bf16x2(sc[2 * j + 1][0], sc[2 * j + 1][1]);
                    pa[3] = pack_bf16x2(sc[2 * j + 1][2], sc[2 * j + 1][3]);
                    const int tok = tok0 + j * 16 + rr + ((mi & 1) << 3);
                    // rows this thread's V fragments hold (for the tail mask)
                    const int vt = tok0 + j * 16 + 2 * cq;
#pragma unroll
                    for (int dp = 0; dp < D / 16; ++dp) {
                        const int dim = dp * 16 + ((mi >> 1) << 3);
                        uint32_t v0, v1, v2, v3;
                        ldsm_x4_t(sV + tile_off(tok, dim), v0, v1, v2, v3);
                        if (tail) {
                            // rows past the length may hold anything (NaN included):
                            // zero them so that 0 * garbage cannot reach the sum
                            uint32_t k0, k1;
                            if constexpr (GATHER) {
                                const uint32_t bits = static_cast<uint32_t>(vm >> vt);
                                k0 = ((bits & 1u) ? 0x0000ffffu : 0u) | ((bits & 2u) ? 0xffff0000u : 0u);
                                k1 = ((bits & 0x100u) ? 0x0000ffffu : 0u) | ((bits & 0x200u) ? 0xffff0000u : 0u);
                            } else {
                                k0 = (vt < n_valid ? 0x0000ffffu : 0u) | (vt + 1 < n_valid ? 0xffff0000u : 0u);
                                k1 = (vt + 8 < n_valid ? 0x0000ffffu : 0u) | (vt + 9 < n_valid ? 0xffff0000u : 0u);
                            }
                            v0 &= k0;
                            v2 &= k0;
                            v1 &= k1;
                            v3 &= k1;
                        }
                        mma_bf16_16816(o[2 * dp], pa, v0, v1);
                        mma_bf16_16816(o[2 * dp + 1], pa, v2, v3);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }

        // ---- finish the piece: merge the warps of each M tile, then write ----
        l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
        l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
        {
            float* so = scr_o + warp * 16 * C::SCR_STRIDE;
#pragma unroll
            for (int i = 0; i < DT; ++i) {
                const int col = i * 8 + 2 * cq;
                *reinterpret_cast<float2*>(so + r0 * C::SCR_STRIDE + col) = make_float2(o[i][0], o[i][1]);
                *reinterpret_cast<float2*>(so + (r0 + 8) * C::SCR_STRIDE + col) = make_float2(o[i][2], o[i][3]);
            }
            if (cq == 0) {
                float* ml = scr_ml + warp * 32;
                ml[r0] = m0;
                ml[r0 + 8] = m1;
                ml[16 + r0] = l0;
                ml[16 + r0 + 8] = l1;
            }
        }
        named_bar_sync(1, CWARPS * 32);
        {
            const bool fin = count == 1;
            const long long bh = static_cast<long long>(w.b) * a.H + static_cast<long long>(w.kvh) * g;
            for (int idx = ctid; idx < rows_out * D; idx += CWARPS * 32) {
                const int row = idx / D, dim = idx - row * D;
                const int mtile = row >> 4, lr = row & 15;
                float M = -INFINITY;
#pragma unroll
                for (int j = 0; j < WPM; ++j) M = fmaxf(M, scr_ml[(mtile * WPM + j) * 32 + lr]);
                const float Mu = M == -INFINITY ? 0.f : M;
                float acc = 0.f, L = 0.f;
#pragma unroll
                for (int j = 0; j < WPM; ++j) {
                    const int wj = mtile * WPM + j;
                    const float wgt = fast_exp2(scr_ml[wj * 32 + lr] - Mu);
                    acc += wgt * scr_o[(wj * 16 + lr) * C::SCR_STRIDE + dim];
                    L += wgt * scr_ml[wj * 32 + 16 + lr];
                }
                if (fin) {
                    const long long oi = (bh + row) * D + dim;
                    reinterpret_cast<__nv_bfloat16*>(a.out)[oi] = __float2bfloat16_rn(L > 0.f ? acc / L : 0.f);
                    if (dim == 0 && a.lse) a.lse[bh + row] = L > 0.f ? (Mu + __log2f(L)) * kLn2 : -INFINITY;
                } else {
                    const long long pi = static_cast<long long>(slot) * g + row;
                    a.part_o[pi * D + dim] = acc;
                    if (dim == 0) {
                        a.part_ml[pi * 2] = M;  // -inf only for a piece whose rows were all skipped
                        a.part_ml[pi * 2 + 1] = L;
                    }
                }
            }
        }
        named_bar_sync(1, CWARPS * 32);
        if (count > 1 && ctid == 0 && s_merge[0] < 2) {  // a split piece: counted once the CTA is done
            const int k = s_merge[0]++;
            s_merge[1 + 3 * k] = w.b * a.Hk + w.kvh;
            s_merge[2 + 3 * k] = w.S;
            s_merge[3 + 3 * k] = count;
        }
    }

    // ---- count this CTA's split pieces (its range is contiguous: at most its first and
    // last units are split); the piece that completes a unit merges it ----
    if (ctid == 0) {
        int nm = 0;
        if (!*s_abort) {  // after a timeout nothing is counted or merged
            const int np = s_merge[0];
            __threadfence();  // every partial written here (barrier above) before the counts
            const int old0 = np > 0 ? atomicAdd(&a.unit_cnt[s_merge[1]], 1) : 0;
            const int old1 = np > 1 ? atomicAdd(&a.unit_cnt[s_merge[4]], 1) : 0;
            for (int k = 0; k < np; ++k) {
                if ((k == 0 ? old0 : old1) == s_merge[3 + 3 * k] - 1) {
                    a.unit_cnt[s_merge[1 + 3 * k]] = 0;  // complete: leave the counter as found
                    s_merge[1 + 3 * nm] = s_merge[1 + 3 * k];
                    s_merge[2 + 3 * nm] = s_merge[2 + 3 * k];
                    s_merge[3 + 3 * nm] = s_merge[3 + 3 * k];
                    ++nm;
                }
            }
            if (nm) __threadfence();
        }
        s_merge[0] = nm;
    }
    named_bar_sync(1, CWARPS * 32);
    for (int k = 0; k < s_merge[0]; ++k)
        merge_unit<D>(a, s_merge[1 + 3 * k], s_merge[2 + 3 * k], s_merge[3 + 3 * k], ctid, CWARPS * 32);
}

// ---- merge of split units --------------------------------------------------------
// One warp per query head.  With weights w_j = 2^(m_j - M) / sum_i 2^(m_i - M) l_i:
// out = sum_j w_j O_j and lse = ln 2 * (M + log2 sum_j 2^(m_j - M) l_j): the softmax
// over a union of key sets is the max-shifted mix of the parts.  Lane j holds
// (m_j, l_j) of slot j, and every slot's O row is requested together with them, so
// the merge costs two dependent memory round trips after the slot range is known.
constexpr int MERGE_WARPS = 8;
constexpr int MERGE_BATCH = 16;  // slots whose O rows are in flight together

template <int D>
__global__ void __launch_bounds__(MERGE_WARPS * 32) decode_combine_kernel(DecodeArgs a)
{
    constexpr int PL = D / 32;  // dims per lane
    using VecF = typename std::conditional<PL == 4, float4, float2>::type;
    pdl_wait();
    pdl_trigger();
    const int u = blockIdx.x;
    const int b = u / a.Hk, kvh = u - b * a.Hk;
    const int g = a.g;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.y * MERGE_WARPS + warp;
    if (row >= g) return;
    const int len_raw = a.seq_lens[b];
    const int2 info = a.unit_info[u];
    const long long bh = static_cast<long long>(b) * a.H + static_cast<long long>(kvh) * g + row;
    __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.out) + bh * D + lane * PL;
    if (min(max(a.len_cap > 0 && len_raw > a.len_cap ? a.len_cap : len_raw, 0), a.T_max) == 0) {
#pragma unroll
        for (int i = 0; i < PL; ++i) out[i] = __float2bfloat16_rn(0.f);
        if (lane == 0 && a.lse) a.lse[bh] = -INFINITY;
        return;
    }
    if (info.y <= 1) return;  // finished inside one CTA
    const int count = info.y;
    const long long base = static_cast<long long>(info.x) * g + row;  // row of slot 0
    float M = -INFINITY, L = 0.f;
    float acc[PL];
#pragma unroll
    for (int i = 0; i < PL; ++i) acc[i] = 0.f;
    for (int j0 = 0; j0 < count; j0 += 32) {
        // (m, l) of slots j0 + lane, and the O rows of the first MERGE_BATCH of them
        const int jl = j0 + lane;
        float2 ml = make_float2(-INFINITY, 0.f);
        if (jl < count) ml = __ldcg(reinterpret_cast<const float2*>(a.part_ml) + base + static_cast<long long>(jl) * g);
        const int nj = min(32, count - j0);
        VecF ov[MERGE_BATCH];
#pragma unroll
        for (int j = 0; j < MERGE_BATCH; ++j)
            if (j < nj)
                ov[j] = __ldcg(reinterpret_cast<const VecF*>(a.part_o + (base + static_cast<long long>(j0 + j) * g) * D) +
                               lane);
        // rescale what is accumulated so far to the new maximum
        float Mc = ml.x;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) Mc = fmaxf(Mc, __shfl_xor_sync(0xffffffffu, Mc, o));
        const float Mn = fmaxf(M, Mc);
        const float r = M == -INFINITY ? 0.f : fast_exp2(M - Mn);
        L *= r;
#pragma unroll
        for (int i = 0; i < PL; ++i) acc[i] *= r;
        M = Mn;
        const float wl = jl < count ? fast_exp2(ml.x - M) : 0.f;
        float Ls = wl * ml.y;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) Ls += __shfl_xor_sync(0xffffffffu, Ls, o);
        L += Ls;
#pragma unroll
        for (int j = 0; j < MERGE_BATCH; ++j) {
            const float wj = __shfl_sync(0xffffffffu, wl, j);
            if (j < nj) {
                const float* v = reinterpret_cast<const float*>(&ov[j]);
#pragma unroll
                for (int i = 0; i < PL; ++i) acc[i] += wj * v[i];
            }
        }
        for (int j = MERGE_BATCH; j < nj; ++j) {
            const float wj = __shfl_sync(0xffffffffu, wl, j);
            const VecF x = __ldcg(reinterpret_cast<const VecF*>(a.part_o + (base + static_cast<long long>(j0 + j) * g) * D) +
                                  lane);
            const float* v = reinterpret_cast<const float*>(&x);
#pragma unroll
            for (int i = 0; i < PL; ++i) acc[i] += wj * v[i];
        }
    }
    const float inv = 1.f / L;
    if (PL == 4) {
        *reinterpret_cast<uint2*>(out) = make_uint2(pack_bf16x2(acc[0] * inv, acc[1] * inv),
                                                    pack_bf16x2(acc[PL - 2] * inv, acc[PL - 1] * inv));
    } else {
        *reinterpret_cast<uint32_t*>(out) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
    }
    if (lane == 0 && a.lse) a.lse[bh] = (M + __log2f(L)) * kLn2;
}

template <int D, int NMT, bool GATHER>
cudaError_t launch_typed(const DecodeArgs& a, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                         cudaStream_t stream)
{
    static bool attr_set[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 64 && !attr_set[dev]) {
        e = cudaFuncSetAttribute(decode_kernel<D, NMT, GATHER>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Cfg<D, NMT, GATHER>::SMEM);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    // split units are merged inside the kernel, by the CTA that finishes their last piece
    return launch_pdl(decode_kernel<D, NMT, GATHER>, dim3(a.grid), dim3(threads_of(GATHER)), Cfg<D, NMT, GATHER>::SMEM,
                      stream, tm_k,
                      tm_v, a);
}

}  // namespace

cudaError_t launch_decode_merge(const DecodeArgs& a, cudaStream_t stream)
{
    const dim3 cgrid(a.B * a.Hk, (a.g + MERGE_WARPS - 1) / MERGE_WARPS);
    if (a.d == 128) return launch_pdl(decode_combine_kernel<128>, cgrid, dim3(MERGE_WARPS * 32), 0, stream, a);
    return launch_pdl(decode_combine_kernel<64>, cgrid, dim3(MERGE_WARPS * 32), 0, stream, a);
}

long long decode_max_slots(int B, int Hk, int grid)
{
    return static_cast<long long>(grid) + static_cast<long long>(B) * Hk;
}

int decode_grid(int num_sms) { return num_sms; }

cudaError_t launch_decode(const DecodeArgs& a, const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                          const CUtensorMap& tm_v, cudaStream_t stream)
{
    const int nmt = a.g <= 16 ? 1 : (a.g <= 32 ? 2 : 4);
    if (a.idx) {
        // gather mode: the mma.sync kernel (g <= 32 at d = 128)
        if (a.d == 128) {
            if (nmt == 1) return launch_typed<128, 1, true>(a, tm_k, tm_v, stream);
            if (nmt == 2) return launch_typed<128, 2, true>(a, tm_k, tm_v, stream);
            return cudaErrorInvalidValue;
        }
        if (nmt == 1) return launch_typed<64, 1, true>(a, tm_k, tm_v, stream);
        if (nmt == 2) return launch_typed<64, 2, true>(a, tm_k, tm_v, stream);
        return launch_typed<64, 4, true>(a, tm_k, tm_v, stream);
    }
    if (decode_tc_supported(a.d, a.g)) return launch_decode_tc(a, tm_q, tm_k, tm_v, stream);
    if (a.d == 128) {
        if (nmt == 1) return launch_typed<128, 1, false>(a, tm_k, tm_v, stream);
        // g = 64 at d = 128 is the tcgen05 kernel's
        return launch_typed<128, 2, false>(a, tm_k, tm_v, stream);
    }
    if (nmt == 1) return launch_typed<64, 1, false>(a, tm_k, tm_v, stream);
    if (nmt == 2) return launch_typed<64, 2, false>(a, tm_k, tm_v, stream);
    return launch_typed<64, 4, false>(a, tm_k, tm_v, stream);
}

}  // namespace kvattn
