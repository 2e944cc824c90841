// sparse.cu -- attention of all query heads over a gathered set of latent rows.
//
// "Agentic RL 入门3：transformer 架构" §2.2 (2): o_t = MLA(q_t, {k_j, v_j : j in
// S_t}); "attention", DSA ② and the "乘法结合律" note: after weight absorption
// every query head ([1, 128, 576]) scores the same single-head latent rows, so
// the step is multi-query attention over the selected rows, with the 576-wide
// row as key and its first 512 columns as value (§2.3.3, §2.3.5).
//
// Kernel (tcgen05): one CTA per (batch row, chunk of 128 selected rows), all
// query heads as the M = 128 rows of both MMAs.  320 threads:
//   - warps 0-7 gather the chunk's 128 latent rows with 16-byte cp.async into
//     nine 64-column blocks laid out as the tensor cores read them (128-byte
//     rows, 128-byte swizzle); each block is signalled as it lands.  Invalid
//     indices are zero-filled and their columns masked.  In the FP8 variant
//     (rows of 656 bytes: 512 E4M3 codes, 4 fp32 scales, 64 bf16 RoPE values;
//     "稀疏注意力：省了什么，没省什么", 改进一) the RoPE part lands directly in block
//     8, the codes land in the space of blocks 4-7 and are dequantised there,
//     block by block, into bf16 (value(code) * scale, rounded to bf16): blocks
//     0-3 while the rest is still in flight, blocks 4-7 from registers once every
//     code has been read.
//   - warp 8 streams the queries through a four-slot TMA ring, 64 columns at a
//     time, in the order the blocks land; warp 9 issues S = Q C^T (M = 128
//     heads, N = 128 rows, K = 576) into TMEM block by block.
//   - warps 0-7 take the row softmax of S in base 2: warp w reads head row
//     32 (w % 4) + lane (its TMEM lane), the first four warps key columns 0-63,
//     the other four 64-127; the two halves exchange their maxima and sums
//     through shared memory.  P is written as bf16 over two free query slots.
//   - warp 9 issues O = P V with V = the resident rows read as an MN-major
//     operand, N = 256 twice, into all 512 TMEM columns (S's columns are free by
//     then).
//   - the epilogue writes O in boxes of 64 columns, normalised by the chunk's own
//     softmax sum and rounded to bf16 into shared memory (over the row blocks
//     that half's P V has consumed), each box stored by TMA as soon as it is
//     staged; warps 0-3 take boxes 0-1 and warps 4-7 boxes 2-3 of each half, so
//     both groups start on a half as soon as its P V is done.  A row with one
//     chunk is written to the output directly; otherwise each chunk leaves its
//     normalised bf16 part and its log-sum-exp, and the parts are merged
//     (out = sum_c 2^(lse_c - LSE) o_c): when the whole grid fits on the GPU at
//     once (one CTA per SM), it is launched cooperatively and the CTAs of a row
//     merge its parts themselves -- each warp group counts its stored boxes on a
//     per-row counter (a release add), every CTA waits (bounded) for the row's
//     2 x chunks counts, then merges its share of the row's tiles of 64 columns
//     x 64 heads: every part's tile comes in by TMA, and meanwhile the parts'
//     lse give each head's weights once (four threads per head); otherwise a
//     second kernel merges them.
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.h"

namespace kvattn {

namespace {

constexpr int SP_DK = 576;
constexpr int SP_DV = 512;
constexpr int SP_ROWS = 128;                   // selected rows per CTA (N of S, K of P V)
constexpr int SP_M = 128;                      // query heads per MMA (rows past Hq are discarded)
constexpr int SP_KB = SP_DK / 64;              // 64-column blocks of a latent row (9)
constexpr int SP_BLOCK = SP_ROWS * 128;        // 16 KB: 128 rows x 64 columns
constexpr int SP_QBLOCK = SP_M * 128;          // 16 KB: 128 heads x 64 columns
constexpr int SP_GW = 8;                       // gather / softmax / epilogue warps
constexpr int SP_GT = SP_GW * 32;
constexpr int SP_THREADS = SP_GT + 64;         // + TMA warp + MMA warp
constexpr int SP_TMA_WARP = SP_GW, SP_MMA_WARP = SP_GW + 1;
constexpr int SP_QS = 4;                       // query slots
constexpr int SP_K_MAX = 2048;                 // selected rows per batch row (the entry points' limit)
constexpr int SP_MAXC = SP_K_MAX / SP_ROWS;    // chunks per batch row (16)
constexpr int SP_OFF_C = 0;                                  // 9 blocks of gathered rows
constexpr int SP_OFF_RAW = SP_OFF_C + 4 * SP_BLOCK;          // FP8: codes [8 blocks][128 rows][64 B] (blocks 4-7)
constexpr int SP_RAW_BLOCK = SP_ROWS * 64;
constexpr int SP_OFF_Q = SP_OFF_C + SP_KB * SP_BLOCK;        // SP_QS query slots
constexpr int SP_OFF_P = SP_OFF_Q;                           // P: 2 blocks of 64 keys, over slots 0-1 after S
constexpr int SP_OFF_SCL = SP_OFF_Q + SP_QS * SP_QBLOCK;     // FP8: [128 rows][4] fp32 scales
constexpr int SP_OFF_RED = SP_OFF_SCL + SP_ROWS * 16;        // [2][128] row maxima, [2][128] row sums
constexpr int SP_OFF_VALID = SP_OFF_RED + 4 * SP_M * 4;      // [4] bit masks: slot row holds a valid index
constexpr int SP_OFF_ROW = SP_OFF_VALID + 16;                // [128] latent row of each slot (-1: none)
constexpr int SP_OFF_BAR = SP_OFF_ROW + SP_ROWS * 4;
// c_full[9], q_full[4], q_empty[4], s_full, p_full, o_full[2], done
constexpr int SP_NBAR = SP_KB + SP_QS + SP_QS + 1 + 1 + 2 + 1 + 1;  // + m_full (merge tiles)
constexpr int SP_OFF_MISC = SP_OFF_BAR + SP_NBAR * 8;
constexpr int SP_SMEM = SP_OFF_MISC + 16 + 1024;  // + alignment slack
static_assert(SP_SMEM <= 232448, "shared memory");
static_assert(SP_OFF_RAW + 8 * SP_RAW_BLOCK == SP_OFF_C + 8 * SP_BLOCK, "codes fill blocks 4-7 exactly");
static_assert(SP_MAXC * (8192 + 64 * 4) <= SP_KB * SP_BLOCK, "a merge tile of every part and its weights fit in the row blocks");
constexpr int SP_FP8_ROW = 656;                // packed row: 512 codes, 4 fp32 scales, 64 bf16
constexpr int SP_FP8_SCL = 512, SP_FP8_ROPE = 528;
constexpr uint32_t SP_IDESC_S = umma_idesc_bf16(SP_M, SP_ROWS);              // Q x C^T, both K-major
constexpr uint32_t SP_IDESC_O = umma_idesc_bf16(SP_M, 256, false, true);     // P x V, V MN-major
constexpr float kLog2e = 1.44269504088896340736f;
constexpr float kLn2 = 0.69314718055994530942f;

struct SparseArgs {
    const void* latent;         // bf16 [B][L_max][576], or packed FP8 [B][L_max][656]
    const int32_t* idx;         // [B][k]
    kvattn_bf16* out;           // [B][Hq][512]
    float* lse;                 // [B][Hq] or null
    kvattn_bf16* part_o;        // [B][chunks][Hq][512] bf16, each chunk normalised by its own sum
    float* part_lse;            // [B][chunks][Hq], log2 units (-inf: the chunk has no valid row)
    int32_t* dev_status;
    int* row_arrive;            // [B] parts of the row written so far (merge in the kernel; zero between calls)
    int* row_done;              // [B] CTAs of the row done merging (zero between calls)
    int B, Hq, L_max, k, chunks;
    int fused_merge;            // 1: the row's CTAs merge its parts themselves (cooperative launch)
    float scale;
};

// The order in which the latent blocks are consumed: the FP8 variant's RoPE block
// lands first (with the scales), the bf16 variant's blocks in column order.
template <bool FP8>
__device__ __forceinline__ int block_at(int i)
{
    return FP8 ? (i == 0 ? SP_KB - 1 : i - 1) : i;
}

// cp.async groups still pending after block kb's group may be at most 8 - kb.
__device__ __forceinline__ void wait_groups_upto(int kb)
{
    switch (kb) {
    case 0: cp_async_wait<8>(); break;
    case 1: cp_async_wait<7>(); break;
    case 2: cp_async_wait<6>(); break;
    case 3: cp_async_wait<5>(); break;
    case 4: cp_async_wait<4>(); break;
    case 5: cp_async_wait<3>(); break;
    case 6: cp_async_wait<2>(); break;
    case 7: cp_async_wait<1>(); break;
    default: cp_async_wait<0>(); break;
    }
}

// Eight E4M3 codes (two 32-bit words) times a scale -> eight bf16 (one 16-byte
// chunk).  E4M3 -> f16 is exact; the product is rounded to fp32, then to bf16.
__device__ __forceinline__ uint4 dequant8(uint32_t w0, uint32_t w1, float s)
{
    uint32_t h[4];
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h[0]) : "h"(static_cast<uint16_t>(w0 & 0xffffu)));
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h[1]) : "h"(static_cast<uint16_t>(w0 >> 16)));
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h[2]) : "h"(static_cast<uint16_t>(w1 & 0xffffu)));
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h[3]) : "h"(static_cast<uint16_t>(w1 >> 16)));
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h[i]));
        o[i] = pack_bf16x2(f.x * s, f.y * s);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// 32 codes of one row (two 16-byte words) -> chunks 4 hh .. 4 hh + 3 of that row
// of a swizzled bf16 block.
__device__ __forceinline__ void dequant_store(uint8_t* blk, int r, int hh, uint4 c0, uint4 c1, float s)
{
    *reinterpret_cast<uint4*>(blk + swz128(r, 4 * hh + 0)) = dequant8(c0.x, c0.y, s);
    *reinterpret_cast<uint4*>(blk + swz128(r, 4 * hh + 1)) = dequant8(c0.z, c0.w, s);
    *reinterpret_cast<uint4*>(blk + swz128(r, 4 * hh + 2)) = dequant8(c1.x, c1.y, s);
    *reinterpret_cast<uint4*>(blk + swz128(r, 4 * hh + 3)) = dequant8(c1.z, c1.w, s);
}

// Tiled shared -> global store through the tensor map (bulk-group completion).
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int x, int y, int z)
{
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
                 : "memory");
}

// Add with release semantics at GPU scope: what this thread wrote or saw before is visible
// to a thread that reads the sum with acquire.
__device__ __forceinline__ void red_release_add(int* p, int v)
{
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// One (head, 16-byte column chunk) of the merge of a row's C parts: out = sum_c
// 2^(lse_c - LSE) o_c, LSE = log2 sum_c 2^lse_c (log2 units; lse written in natural log).
__device__ __forceinline__ void merge_one(const SparseArgs& a, int b, int h, int j)
{
    constexpr int MAXC = SP_MAXC;
    const int C = a.chunks;
    float ls[MAXC];
    uint4 ov[MAXC];
#pragma unroll
    for (int c = 0; c < MAXC; ++c) {
        if (c < C) {
            const long long row = (static_cast<long long>(b) * C + c) * a.Hq + h;
            ls[c] = __ldcg(a.part_lse + row);
            ov[c] = __ldcg(reinterpret_cast<const uint4*>(a.part_o + row * SP_DV) + j);
        }
    }
    float M = -INFINITY;
#pragma unroll
    for (int c = 0; c < MAXC; ++c)
        if (c < C) M = fmaxf(M, ls[c]);
    const float Mu = M == -INFINITY ? 0.f : M;
    float L = 0.f;
    float wgt[MAXC];
#pragma unroll
    for (int c = 0; c < MAXC; ++c) {
        wgt[c] = c < C ? fast_exp2(ls[c] - Mu) : 0.f;
        L += wgt[c];
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < MAXC; ++c) {
        if (c < C) {
            const float wc = wgt[c] * inv;
            const uint32_t w4[4] = {ov[c].x, ov[c].y, ov[c].z, ov[c].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                acc[2 * i] = fmaf(wc, bf16_lo(w4[i]), acc[2 * i]);
                acc[2 * i + 1] = fmaf(wc, bf16_hi(w4[i]), acc[2 * i + 1]);
            }
        }
    }
    const long long ob = (static_cast<long long>(b) * a.Hq + h) * SP_DV;
    reinterpret_cast<uint4*>(a.out + ob)[j] = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                                                         pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
    if (j == 0 && a.lse) a.lse[static_cast<long long>(b) * a.Hq + h] = L > 0.f ? (Mu + __log2f(L)) * kLn2 : -INFINITY;
}


template <bool FP8>
__global__ void __launch_bounds__(SP_THREADS, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_o,
                       const __grid_constant__ CUtensorMap tm_pm, SparseArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint32_t* s_vmask = reinterpret_cast<uint32_t*>(smem + SP_OFF_VALID);
    int* s_row = reinterpret_cast<int*>(smem + SP_OFF_ROW);
    float* s_scl = reinterpret_cast<float*>(smem + SP_OFF_SCL);
    float* s_max = reinterpret_cast<float*>(smem + SP_OFF_RED);
    float* s_sum = s_max + 2 * SP_M;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SP_OFF_BAR);
    uint64_t* c_full = bars;                 // [9]: block kb of the rows ready (SP_GT arrivals)
    uint64_t* q_full = c_full + SP_KB;       // [SP_QS]
    uint64_t* q_empty = q_full + SP_QS;      // [SP_QS]
    uint64_t* s_full = q_empty + SP_QS;      // S complete in TMEM
    uint64_t* p_full = s_full + 1;           // P written (S read), SP_GT arrivals
    uint64_t* o_full = p_full + 1;           // [2]: O columns 0-255 / 256-511 complete
    uint64_t* done = o_full + 2;             // every MMA finished
    uint64_t* m_full = done + 1;             // in-kernel merge: a tile of every part landed
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + SP_OFF_MISC);
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem + SP_OFF_MISC + 4);

    const int chunk = blockIdx.x, b = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int i = 0; i < SP_KB; ++i) mbar_init(&c_full[i], SP_GT);
        for (int i = 0; i < SP_QS; ++i) {
            mbar_init(&q_full[i], 1);
            mbar_init(&q_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) mbar_init(&o_full[i], 1);
        mbar_init(s_full, 1);
        mbar_init(p_full, SP_GT);
        mbar_init(done, 1);
        mbar_init(m_full, 1);
        *s_abort = 0;
        fence_barrier_init();
    }
    if (warp == SP_TMA_WARP && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_o);
        tma_prefetch_desc(&tm_pm);
    }
    if (warp == SP_MMA_WARP) {
        tmem_alloc(s_tmem, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    pdl_wait();
    pdl_trigger();

    if (warp < SP_GW) {
        const int t = tid;
        // ===== the chunk's row indices =====
        if (t < SP_ROWS) {
            const int slot = chunk * SP_ROWS + t;
            int j = slot < a.k ? a.idx[static_cast<long long>(b) * a.k + slot] : -1;
            if (j < -1 || j >= a.L_max) {
                report_status(a.dev_status, KVATTN_STATUS_BAD_INDEX);
                j = -1;
            }
            const uint32_t vm = __ballot_sync(0xffffffffu, j >= 0);
            if (lane == 0) s_vmask[warp] = vm;
            s_row[t] = j;
        }
        named_bar_sync(1, SP_GT);  // every slot's row is known
        const uint32_t c0 = smem_u32(smem + SP_OFF_C);
        if constexpr (!FP8) {
            // ===== gather: block kb of row r, 16-byte chunk ch: thread (r % 32) * 8 + ch =====
            const kvattn_bf16* lat = static_cast<const kvattn_bf16*>(a.latent) + static_cast<long long>(b) * a.L_max * SP_DK;
            const int ch = t & 7;
            int jr[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) jr[u] = s_row[(t >> 3) + 32 * u];
#pragma unroll
            for (int kb = 0; kb < SP_KB; ++kb) {
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int r = (t >> 3) + 32 * u;
                    const int j = jr[u];
                    cp_async16(c0 + kb * SP_BLOCK + swz128(r, ch),
                               lat + static_cast<long long>(j < 0 ? 0 : j) * SP_DK + kb * 64 + ch * 8, j < 0 ? 0u : 16u);
                }
                cp_async_commit();
            }
#pragma unroll
            for (int kb = 0; kb < SP_KB; ++kb) {
                wait_groups_upto(kb);
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                mbar_arrive(&c_full[kb]);
            }
        } else {
            // ===== gather of packed FP8 rows: group 0 = scales + the RoPE block, groups 1-8 = code blocks =====
            const uint8_t* lat = static_cast<const uint8_t*>(a.latent) + static_cast<long long>(b) * a.L_max * SP_FP8_ROW;
            auto row_ptr = [&](int j) { return lat + static_cast<long long>(j < 0 ? 0 : j) * SP_FP8_ROW; };
            if (t < SP_ROWS) {
                const int j = s_row[t];
                cp_async16(smem_u32(s_scl + t * 4), row_ptr(j) + SP_FP8_SCL, j < 0 ? 0u : 16u);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int r = (t >> 3) + 32 * u, ch = t & 7;
                const int j = s_row[r];
                cp_async16(c0 + (SP_KB - 1) * SP_BLOCK + swz128(r, ch), row_ptr(j) + SP_FP8_ROPE + ch * 16,
                           j < 0 ? 0u : 16u);
            }
            cp_async_commit();
            const uint32_t raw0 = smem_u32(smem + SP_OFF_RAW);
#pragma unroll
            for (int jb = 0; jb < 8; ++jb) {
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int r = (t >> 2) + 64 * u, ch = t & 3;
                    const int j = s_row[r];
                    cp_async16(raw0 + jb * SP_RAW_BLOCK + r * 64 + ch * 16, row_ptr(j) + jb * 64 + ch * 16,
                               j < 0 ? 0u : 16u);
                }
                cp_async_commit();
            }
            // the RoPE block is ready as it lands
            cp_async_wait<8>();
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            mbar_arrive(&c_full[SP_KB - 1]);
            // dequantisation: thread t takes row t / 2, codes 32 (t % 2) .. + 31 of each block
            const int r = t >> 1, hh = t & 1;
            const uint8_t* raw = smem + SP_OFF_RAW;
            // blocks 0-3: their codes sit in blocks 4-5's space, their output in blocks 0-3
#pragma unroll
            for (int jb = 0; jb < 4; ++jb) {
                wait_groups_upto(jb + 1);
                named_bar_sync(1, SP_GT);  // every thread's copies of the block (and the scales) are visible
                const uint8_t* src = raw + jb * SP_RAW_BLOCK + r * 64 + hh * 32;
                dequant_store(smem + SP_OFF_C + jb * SP_BLOCK, r, hh, *reinterpret_cast<const uint4*>(src),
                              *reinterpret_cast<const uint4*>(src + 16), s_scl[r * 4 + (jb >> 1)]);
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                mbar_arrive(&c_full[jb]);
            }
            // blocks 4-7 overwrite the space the codes occupy: read every code first
            cp_async_wait<0>();
            named_bar_sync(1, SP_GT);
            uint4 cr[4][2];
#pragma unroll
            for (int jb = 4; jb < 8; ++jb) {
                const uint8_t* src = raw + jb * SP_RAW_BLOCK + r * 64 + hh * 32;
                cr[jb - 4][0] = *reinterpret_cast<const uint4*>(src);
                cr[jb - 4][1] = *reinterpret_cast<const uint4*>(src + 16);
            }
            named_bar_sync(1, SP_GT);
#pragma unroll
            for (int jb = 4; jb < 8; ++jb) {
                dequant_store(smem + SP_OFF_C + jb * SP_BLOCK, r, hh, cr[jb - 4][0], cr[jb - 4][1],
                              s_scl[r * 4 + (jb >> 1)]);
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                mbar_arrive(&c_full[jb]);
            }
        }

        // ===== softmax of head row h over key columns 64 g .. 64 g + 63 =====
        const int g = warp >> 2, quarter = warp & 3;
        const int h = quarter * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
        const bool live = h < a.Hq;
        const float sl2 = a.scale * kLog2e;
        uint32_t sv[2][32];
        float mx = -INFINITY;
        const bool have_s = warp_wait(s_full, 0, s_abort);
        if (have_s) {
            tc_fence_after();
            tmem_ld32(tmem + lane_off + 64 * g, sv[0]);
            tmem_ld32(tmem + lane_off + 64 * g + 32, sv[1]);
            tmem_wait_ld();
            tmem_regs_ready(sv[0]);
            tmem_regs_ready(sv[1]);
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const uint32_t vm = s_vmask[2 * g + cc];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    if (!((vm >> i) & 1u)) sv[cc][i] = 0xff800000u;  // -inf: not a selected row
                    mx = fmaxf(mx, __uint_as_float(sv[cc][i]));
                }
            }
        }
        s_max[g * SP_M + h] = mx;
        named_bar_sync(2, SP_GT);
        const float m = fmaxf(s_max[h], s_max[SP_M + h]) * sl2;
        const float mu = m == -INFINITY ? 0.f : m;
        float l_half = 0.f;
        if (have_s) {
            const float2 sc2 = make_float2(sl2, sl2), nmu = make_float2(-mu, -mu);
            float2 acc = make_float2(0.f, 0.f);
            uint8_t* pblk = smem + SP_OFF_P + g * SP_BLOCK;
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {  // 8-key chunk (16 bytes of P) q of this 32-key group
                    uint32_t pk[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int i = q * 8 + 2 * e;
                        const float2 x = __ffma2_rn(
                            make_float2(__uint_as_float(sv[cc][i]), __uint_as_float(sv[cc][i + 1])), sc2, nmu);
                        float2 p;
                        if (e == 0) {
                            p = exp2_fma2(x);  // a quarter of the exponentials off the MUFU pipe
                        } else {
                            p.x = fast_exp2(x.x);
                            p.y = fast_exp2(x.y);
                        }
                        if (!live) p = make_float2(0.f, 0.f);
                        acc = __fadd2_rn(acc, p);
                        pk[e] = pack_bf16x2(p.x, p.y);
                    }
                    *reinterpret_cast<uint4*>(pblk + swz128(h, cc * 4 + q)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
            }
            l_half = acc.x + acc.y;
        }
        // S is read and P is written: the P V MMAs may reuse S's columns
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_fence_before();
        mbar_arrive(p_full);
        s_sum[g * SP_M + h] = l_half;
        named_bar_sync(2, SP_GT);
        const float l = s_sum[h] + s_sum[SP_M + h];
        if (g == 0 && live) {  // early: its stores are done by the time the part is announced
            const float lse2 = l > 0.f ? m + __log2f(l) : -INFINITY;
            if (a.chunks == 1) {
                if (a.lse) a.lse[static_cast<long long>(b) * a.Hq + h] = lse2 * kLn2;
            } else {
                a.part_lse[(static_cast<long long>(b) * a.chunks + chunk) * a.Hq + h] = lse2;
                __threadfence();  // before warps 0-3 count their boxes on the row's counter
            }
        }

        // ===== epilogue: O of head row h, normalised, as bf16 boxes of 64 columns; warps 0-3 take
        // boxes 0-1 and warps 4-7 boxes 2-3 of each 256-column half, so that both groups work on
        // a half as soon as its P V is done =====
        const bool one = a.chunks == 1;
        const float inv = l > 0.f ? 1.f / l : 0.f;
        const bool fused = !one && a.fused_merge;
        const bool store = quarter == 0 && lane == 0;
        const int z = one ? b : b * a.chunks + chunk;
        bool have_o = true;
#pragma unroll 1
        for (int hf = 0; hf < 2; ++hf) {
            if (!(have_o = warp_wait(&o_full[hf], 0, s_abort))) break;
            tc_fence_after();
#pragma unroll 1
            for (int j = 0; j < 2; ++j) {
                // box bx = O columns 64 bx .. 64 bx + 63, staged in row block bx (read by this half's P V)
                const int bx = 4 * hf + 2 * g + j;
                uint32_t ov[2][32];
                tmem_ld32(tmem + lane_off + 64 * bx, ov[0]);
                tmem_ld32(tmem + lane_off + 64 * bx + 32, ov[1]);
                tmem_wait_ld();
                tmem_regs_ready(ov[0]);
                tmem_regs_ready(ov[1]);
                uint8_t* box = smem + SP_OFF_C + bx * SP_BLOCK;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float* f = reinterpret_cast<const float*>(ov[i >> 2]) + 8 * (i & 3);
                    *reinterpret_cast<uint4*>(box + swz128(h, i)) =
                        make_uint4(pack_bf16x2(f[0] * inv, f[1] * inv), pack_bf16x2(f[2] * inv, f[3] * inv),
                                   pack_bf16x2(f[4] * inv, f[5] * inv), pack_bf16x2(f[6] * inv, f[7] * inv));
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                named_bar_sync(3 + g, 128);
                if (store && !*s_abort) {
                    tma_store_3d(&tm_o, box, 64 * bx, 0, z);
                    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                }
            }
        }
        if (store) {
            if (fused && have_o) {
                // the group's boxes are in global memory before the row's counter says so: each
                // group counts itself (the lse, written by warps 0-3, was fenced before their barriers)
                asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
                asm volatile("fence.proxy.async.global;" ::: "memory");
                if (!*s_abort) red_release_add(a.row_arrive + b, 1);
            } else {
                asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");  // shared memory read before exit
            }
        }
        if (fused) {
            // ===== merge in the kernel: every CTA of the row (all resident: cooperative
            // launch) waits for the row's 2 x chunks counts, then merges its tiles of the row =====
            if (t == 0 && !*s_abort) {
                const unsigned long long t0 = global_timer_ns();
                while (ld_acquire_gpu(a.row_arrive + b) < 2 * a.chunks) {
                    if (global_timer_ns() - t0 > WAIT_LIMIT_NS) {
                        *s_abort = 1;
                        report_status(a.dev_status, KVATTN_STATUS_TIMEOUT);
                        break;
                    }
                    __nanosleep(64);
                }
            }
            named_bar_sync(1, SP_GT);
            if (!*s_abort) {
                const int C = a.chunks;  // <= SP_K_MAX / SP_ROWS
                // this CTA is past the wait: the row's last one to get here leaves the counters zero
                // (nobody reads them any more); the atomic's answer is needed only at the end
                const int past = t == 32 ? atomicAdd(a.row_done + b, 1) : 0;
                // The row's merge as tiles of 64 columns x 64 heads (8 per 64 heads); this CTA's
                // tiles are chunk, chunk + C, ...  Every part's 8 KB of a tile comes in by TMA
                // (one round trip for all of them); meanwhile the parts' lse give each head's
                // weights 2^(lse_c - LSE), computed once per head: thread (head t / 4, t % 4) takes
                // parts t % 4, t % 4 + 4, ...
                uint8_t* mbuf = smem + SP_OFF_C;                                   // [C][64 heads][128 B]
                float* mw = reinterpret_cast<float*>(smem + SP_OFF_C + SP_MAXC * 8192);  // [C][64] weights
                const int n_tiles = 8 * ((a.Hq + 63) / 64);
                const int wh = t >> 2, wq = t & 3;
                int n_t = 0;
                for (int wt = chunk; wt < n_tiles; wt += C, ++n_t) {
                    const int cb = wt & 7, hb = wt >> 3;
                    const int whq = 64 * hb + wh;
                    float lv[SP_MAXC / 4];
#pragma unroll
                    for (int i = 0; i < SP_MAXC / 4; ++i) {
                        const int c = wq + 4 * i;
                        lv[i] = c < C && whq < a.Hq
                                    ? __ldcg(a.part_lse + (static_cast<long long>(b) * C + c) * a.Hq + whq)
                                    : -INFINITY;
                    }
                    if (lane == 0) {  // lane 0 of warp w loads parts w, w + 8
                        asm volatile("fence.proxy.async.global;" ::: "memory");  // the parts, seen through the counter
                        if (warp == 0) mbar_arrive_expect_tx(m_full, static_cast<uint32_t>(C) * 8192u);
                        for (int c = warp; c < C; c += SP_GW)
                            tma_load_3d(mbuf + c * 8192, &tm_pm, m_full, 64 * cb, 64 * hb, b * C + c);
                    }
                    float M = -INFINITY;
#pragma unroll
                    for (int i = 0; i < SP_MAXC / 4; ++i) M = fmaxf(M, lv[i]);
                    M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, 1));
                    M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, 2));
                    const float Mu = M == -INFINITY ? 0.f : M;
                    float L = 0.f;
#pragma unroll
                    for (int i = 0; i < SP_MAXC / 4; ++i) {
                        lv[i] = fast_exp2(lv[i] - Mu);
                        L += lv[i];
                    }
                    L += __shfl_xor_sync(0xffffffffu, L, 1);
                    L += __shfl_xor_sync(0xffffffffu, L, 2);
                    const float winv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
                    for (int i = 0; i < SP_MAXC / 4; ++i)
                        if (wq + 4 * i < C) mw[(wq + 4 * i) * 64 + wh] = lv[i] * winv;
                    if (cb == 0 && wq == 0 && whq < a.Hq && a.lse)
                        a.lse[static_cast<long long>(b) * a.Hq + whq] = L > 0.f ? (Mu + __log2f(L)) * kLn2 : -INFINITY;
                    named_bar_sync(1, SP_GT);  // the weights are written
                    if (!warp_wait(m_full, n_t & 1, s_abort)) break;
                    for (int it = t; it < 64 * 8; it += SP_GT) {
                        const int hh = it >> 3, ch = it & 7, hq = 64 * hb + hh;
                        if (hq >= a.Hq) continue;
                        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
                        for (int c = 0; c < C; ++c) {
                            const float wc = mw[c * 64 + hh];
                            const float2 w2 = make_float2(wc, wc);
                            const uint4 o = *reinterpret_cast<const uint4*>(mbuf + c * 8192 + swz128(hh, ch));
                            const uint32_t w4[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const float2 r = __ffma2_rn(w2, make_float2(bf16_lo(w4[i]), bf16_hi(w4[i])),
                                                            make_float2(acc[2 * i], acc[2 * i + 1]));
                                acc[2 * i] = r.x;
                                acc[2 * i + 1] = r.y;
                            }
                        }
                        const long long ob = (static_cast<long long>(b) * a.Hq + hq) * SP_DV + 64 * cb + 8 * ch;
                        *reinterpret_cast<uint4*>(a.out + ob) =
                            make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                                       pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
                    }
                    named_bar_sync(1, SP_GT);  // the buffers are read before the next tile's loads
                }
                if (t == 32 && past == C - 1) {
                    a.row_arrive[b] = 0;
                    a.row_done[b] = 0;
                }
            }
        }
    } else if (warp == SP_TMA_WARP) {
        // ===== queries: 64 columns at a time through SP_QS slots, in the blocks' order =====
        if (lane == 0) {
            bool ok = true;
            const uint32_t q_bytes = static_cast<uint32_t>(a.Hq) * 128;
            int i = 0;
            for (; i < SP_KB; ++i) {
                const int s = i % SP_QS;
                if (i >= SP_QS && !(ok = mbar_wait(&q_empty[s], ((i / SP_QS) - 1) & 1))) break;
                mbar_arrive_expect_tx(&q_full[s], q_bytes);
                tma_load_3d(smem + SP_OFF_Q + s * SP_QBLOCK, &tm_q, &q_full[s], block_at<FP8>(i) * 64, 0, b);
            }
            if (!ok) {
                *s_abort = 1;
                report_status(a.dev_status, KVATTN_STATUS_TIMEOUT);
            }
            // copies in flight complete before the CTA leaves (bounded waits)
            for (int j = i - SP_QS > 0 ? i - SP_QS : 0; j < i; ++j) mbar_wait(&q_full[j % SP_QS], (j / SP_QS) & 1);
        }
    } else {
        // ===== MMA issuer =====
        if (lane == 0) {
            bool ok = true;
            const uint32_t c0 = smem_u32(smem + SP_OFF_C), q0 = smem_u32(smem + SP_OFF_Q);
            const uint32_t p0 = smem_u32(smem + SP_OFF_P);
            for (int i = 0; i < SP_KB && ok; ++i) {
                const int kb = block_at<FP8>(i);
                if (!(ok = mbar_wait(&c_full[kb], 0))) break;
                if (!(ok = mbar_wait(&q_full[i % SP_QS], (i / SP_QS) & 1))) break;
                tc_fence_after();
                const uint32_t qs = q0 + (i % SP_QS) * SP_QBLOCK, cs = c0 + kb * SP_BLOCK;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc_mma_bf16(tmem, umma_desc_k_sw128(qs + kk * 32), umma_desc_k_sw128(cs + kk * 32), SP_IDESC_S,
                                (i | kk) ? 1u : 0u);
                tc_commit(&q_empty[i % SP_QS]);
            }
            if (ok) {
                tc_commit(s_full);
                ok = mbar_wait(p_full, 0);
            }
            if (ok) {
                tc_fence_after();
#pragma unroll 1
                for (int half = 0; half < 2; ++half) {
                    // V rows = the chunk's first 512 columns, blocks 4*half .. 4*half+3
#pragma unroll
                    for (int kk = 0; kk < SP_ROWS / 16; ++kk) {
                        const uint64_t ad = umma_desc_k_sw128(p0 + (kk >> 2) * SP_BLOCK + (kk & 3) * 32);
                        const uint64_t bd = umma_desc_mn_sw128(c0 + 4 * half * SP_BLOCK + kk * 2048, SP_BLOCK, 1024);
                        tc_mma_bf16(tmem + half * 256, ad, bd, SP_IDESC_O, kk > 0 ? 1u : 0u);
                    }
                    tc_commit(&o_full[half]);
                }
            }
            if (!ok) {
                *s_abort = 1;
                report_status(a.dev_status, KVATTN_STATUS_TIMEOUT);
            }
            tc_commit(done);
            mbar_wait(done, 0);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == SP_MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---- merge of the chunk parts ------------------------------------------------------
// CTA = (batch row, 4 heads), 64 threads per head, one 16-byte chunk (8 columns)
// each.  A thread loads every chunk's lse and its 16 bytes of every part at
// once (one round trip), then out = sum_c 2^(lse_c - LSE) o_c and
// LSE = log2 sum_c 2^lse_c (all in log2 units; lse is written in natural log).
constexpr int SPM_HEADS = 4;

__global__ void __launch_bounds__(SPM_HEADS * 64) sparse_merge_kernel(SparseArgs a)
{
    pdl_wait();
    pdl_trigger();
    const int b = blockIdx.y;
    const int h = blockIdx.x * SPM_HEADS + (threadIdx.x >> 6);
    if (h < a.Hq) merge_one(a, b, h, threadIdx.x & 63);
}

template <bool FP8>
cudaError_t set_smem_attr_once()
{
    static bool attr_set[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 64 && attr_set[dev]) return cudaSuccess;
    e = cudaFuncSetAttribute(sparse_attn_kernel<FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize, SP_SMEM);
    if (e == cudaSuccess && dev < 64) attr_set[dev] = true;
    return e;
}

}  // namespace

int sparse_chunks(int k) { return (k + SP_ROWS - 1) / SP_ROWS; }

// Workspace (several chunks): [0, 256 * ceil(8 B / 256)) the per-row counters, then the
// bf16 parts [B][chunks][Hq][512], then their lse [B][chunks][Hq].
size_t sparse_counter_bytes(int B) { return (static_cast<size_t>(B) * 2 * sizeof(int) + 255) / 256 * 256; }

size_t sparse_part_o_bytes(int B, int Hq, int k)
{
    const int c = sparse_chunks(k);
    if (c <= 1) return 0;
    return static_cast<size_t>(B) * c * Hq * SP_DV * sizeof(kvattn_bf16);
}

size_t sparse_partial_bytes(int B, int Hq, int k)
{
    const int c = sparse_chunks(k);
    if (c <= 1) return 0;
    return sparse_counter_bytes(B) + sparse_part_o_bytes(B, Hq, k) + static_cast<size_t>(B) * c * Hq * sizeof(float);
}

cudaError_t launch_sparse_attn(const SparseLaunch& l, const CUtensorMap& tm_q, const CUtensorMap& tm_o,
                               const CUtensorMap& tm_pm,
                               cudaStream_t stream)
{
    cudaError_t e = l.fp8 ? set_smem_attr_once<true>() : set_smem_attr_once<false>();
    if (e != cudaSuccess) return e;
    SparseArgs a{};
    a.latent = l.latent;
    a.idx = l.idx;
    a.out = l.out;
    a.lse = l.lse;
    a.B = l.B;
    a.Hq = l.Hq;
    a.L_max = l.L_max;
    a.k = l.k;
    a.chunks = sparse_chunks(l.k);
    a.scale = l.scale;
    a.dev_status = l.dev_status;
    if (a.chunks > 1) {
        uint8_t* ws = static_cast<uint8_t*>(l.workspace);
        a.row_arrive = reinterpret_cast<int*>(ws);
        a.row_done = a.row_arrive + l.B;
        a.part_o = reinterpret_cast<kvattn_bf16*>(ws + sparse_counter_bytes(l.B));
        a.part_lse = reinterpret_cast<float*>(ws + sparse_counter_bytes(l.B) + sparse_part_o_bytes(l.B, l.Hq, l.k));
        // one CTA per SM (its shared memory): the row's CTAs can wait for each other only
        // when the whole grid is resident at once
        a.fused_merge = static_cast<long long>(l.B) * a.chunks <= l.num_sms ? 1 : 0;
    }
    const dim3 grid(a.chunks, l.B);
    if (a.fused_merge) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = grid;
        cfg.blockDim = dim3(SP_THREADS);
        cfg.dynamicSmemBytes = SP_SMEM;
        cfg.stream = stream;
        // cooperative (the row's CTAs wait for each other) and, like the other kernels, a
        // programmatic dependent of the previous launch (its prologue overlaps that one's tail)
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        return l.fp8 ? cudaLaunchKernelEx(&cfg, sparse_attn_kernel<true>, tm_q, tm_o, tm_pm, a)
                     : cudaLaunchKernelEx(&cfg, sparse_attn_kernel<false>, tm_q, tm_o, tm_pm, a);
    }
    e = l.fp8 ? launch_pdl(sparse_attn_kernel<true>, grid, dim3(SP_THREADS), SP_SMEM, stream, tm_q, tm_o, tm_pm, a)
              : launch_pdl(sparse_attn_kernel<false>, grid, dim3(SP_THREADS), SP_SMEM, stream, tm_q, tm_o, tm_pm, a);
    if (e != cudaSuccess || a.chunks == 1) return e;
    return launch_pdl(sparse_merge_kernel, dim3((l.Hq + SPM_HEADS - 1) / SPM_HEADS, l.B), dim3(SPM_HEADS * 64), 0,
                      stream, a);
}

}  // namespace kvattn
