// sparse.cu -- attention of all query heads over a gathered set of latent rows.
//
// "Agentic RL 入门3：transformer 架构" §2.2 (2): o_t = MLA(q_t, {k_j, v_j : j in
// S_t}); "attention", DSA ② and the "乘法结合律" note: after weight absorption
// every query head ([1, 128, 576]) scores the same single-head latent rows, so
// the step is multi-query attention over the selected rows, with the 576-wide
// row as key and its first 512 columns as value (§2.3.3, §2.3.5).
//
// Kernel (tcgen05): one CTA per (batch row, chunk of 128 selected rows), all
// query heads as the M = 128 rows of both MMAs.
//   - warps 0-3 gather the chunk's 128 latent rows (cp.async, 16 bytes at a
//     time, eight lanes per 128-byte line so that every warp request covers
//     four whole lines) into nine 64-column blocks laid out as the tensor cores
//     read them (128-byte rows, 128-byte swizzle); each block is signalled as it
//     lands.  Invalid indices are zero-filled and their columns masked.
//   - warp 4 streams the queries through a four-slot TMA ring, 64 columns at a
//     time; warp 5 issues S = Q C^T (M = 128 heads, N = 128 rows, K = 576) into
//     TMEM, block by block as the gather lands.
//   - warps 0-3 (thread = head = TMEM lane) take the row softmax of S in base 2
//     and write P as bf16 into shared memory (over two query slots, free once S
//     is complete); warp 5 then issues O = P V with
//     V = the same resident rows read as an MN-major operand, N = 256 twice,
//     into all 512 TMEM columns (S's columns are free by then).
//   - warps 0-3 write O (normalised when the row has one chunk, else the
//     unnormalised partial with its running max and sum, stored column-major
//     [column][head] so that a warp's 32 heads fill one 128-byte line); the
//     first half is written while the second half's MMAs run.
// Chunks of one row are merged by a second kernel (the split-softmax identity).
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
constexpr int SP_THREADS = 192;                // w0-3 gather/softmax/epilogue, w4 TMA, w5 MMA + TMEM
constexpr int SP_OFF_C = 0;                              // 9 blocks of gathered rows
constexpr int SP_QS = 4;                                 // query slots
constexpr int SP_OFF_Q = SP_OFF_C + SP_KB * SP_BLOCK;    // SP_QS query slots
constexpr int SP_OFF_P = SP_OFF_Q;                       // P: 2 blocks of 64 rows, over slots 0-1 after S
constexpr int SP_OFF_VALID = SP_OFF_Q + SP_QS * SP_QBLOCK;  // [4] bit masks: slot row holds a valid index
constexpr int SP_OFF_ROW = SP_OFF_VALID + 16;            // [128] latent row of each slot (-1: none)
constexpr int SP_OFF_BAR = SP_OFF_ROW + SP_ROWS * 4;
// c_full[9], q_full[4], q_empty[4], s_full, p_full, o_full[2], done
constexpr int SP_NBAR = SP_KB + SP_QS + SP_QS + 1 + 1 + 2 + 1;
constexpr int SP_OFF_MISC = SP_OFF_BAR + SP_NBAR * 8;
constexpr int SP_SMEM = SP_OFF_MISC + 16 + 1024;  // + alignment slack
static_assert(SP_SMEM <= 232448, "shared memory");
constexpr uint32_t SP_IDESC_S = umma_idesc_bf16(SP_M, SP_ROWS);              // Q x C^T, both K-major
constexpr uint32_t SP_IDESC_O = umma_idesc_bf16(SP_M, 256, false, true);     // P x V, V MN-major
constexpr float kLog2e = 1.44269504088896340736f;
constexpr float kLn2 = 0.69314718055994530942f;

struct SparseArgs {
    const kvattn_bf16* latent;  // [B][L_max][576]
    const int32_t* idx;         // [B][k]
    kvattn_bf16* out;           // [B][Hq][512]
    float* lse;                 // [B][Hq] or null
    float* part_o;              // [B][chunks][512][Hq] (head fastest)
    float* part_ml;             // [B][chunks][Hq][2]
    int32_t* dev_status;
    int B, Hq, L_max, k, chunks;
    float scale;
};

// cp.async groups still pending after block kb's group may be at most 8 - kb.
__device__ __forceinline__ void wait_block_groups(int kb)
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

__global__ void __launch_bounds__(SP_THREADS, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tm_q, SparseArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint32_t* s_vmask = reinterpret_cast<uint32_t*>(smem + SP_OFF_VALID);
    int* s_row = reinterpret_cast<int*>(smem + SP_OFF_ROW);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SP_OFF_BAR);
    uint64_t* c_full = bars;                 // [9]: block kb of the rows landed (128 arrivals)
    uint64_t* q_full = c_full + SP_KB;       // [SP_QS]
    uint64_t* q_empty = q_full + SP_QS;      // [SP_QS]
    uint64_t* s_full = q_empty + SP_QS;      // S complete in TMEM
    uint64_t* p_full = s_full + 1;           // P written (S read), 128 arrivals
    uint64_t* o_full = p_full + 1;           // [2]: O columns 0-255 / 256-511 complete
    uint64_t* done = o_full + 2;             // every MMA finished
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + SP_OFF_MISC);
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem + SP_OFF_MISC + 4);

    const int chunk = blockIdx.x, b = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int i = 0; i < SP_KB; ++i) mbar_init(&c_full[i], 128);
        for (int i = 0; i < SP_QS; ++i) {
            mbar_init(&q_full[i], 1);
            mbar_init(&q_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) mbar_init(&o_full[i], 1);
        mbar_init(s_full, 1);
        mbar_init(p_full, 128);
        mbar_init(done, 1);
        *s_abort = 0;
        fence_barrier_init();
    }
    if (warp == 4 && lane == 0) tma_prefetch_desc(&tm_q);
    if (warp == 5) {
        tmem_alloc(s_tmem, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    pdl_wait();
    pdl_trigger();

    if (warp < 4) {
        // ===== gather: the chunk's selected rows, block by block =====
        const int t = tid;
        {
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
        named_bar_sync(1, 128);  // every slot's row is known
        // copy job i of a block: row i / 8, 16-byte chunk i % 8 (eight lanes per line)
        const kvattn_bf16* lat = a.latent + static_cast<long long>(b) * a.L_max * SP_DK;
        const uint32_t c0 = smem_u32(smem + SP_OFF_C);
        int jr[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) jr[u] = s_row[(t >> 3) + 16 * u];
#pragma unroll
        for (int kb = 0; kb < SP_KB; ++kb) {
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int r = (t >> 3) + 16 * u, ch = t & 7;
                const int j = jr[u];
                cp_async16(c0 + kb * SP_BLOCK + swz128(r, ch),
                           lat + static_cast<long long>(j < 0 ? 0 : j) * SP_DK + kb * 64 + ch * 8, j < 0 ? 0u : 16u);
            }
            cp_async_commit();
        }
#pragma unroll
        for (int kb = 0; kb < SP_KB; ++kb) {
            wait_block_groups(kb);
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            mbar_arrive(&c_full[kb]);
        }

        // ===== softmax of head row t (TMEM lane t) =====
        const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
        const bool live = t < a.Hq;
        const float sl2 = a.scale * kLog2e;
        float m = -INFINITY, l = 0.f;
        if (warp_wait(s_full, 0, s_abort)) {
            tc_fence_after();
            uint32_t sv[4][32];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) tmem_ld32(tmem + lane_off + cc * 32, sv[cc]);
            tmem_wait_ld();
            float mx = -INFINITY;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                const uint32_t vm = s_vmask[cc];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    if (!((vm >> i) & 1u)) sv[cc][i] = 0xff800000u;  // -inf: not a selected row
                    mx = fmaxf(mx, __uint_as_float(sv[cc][i]));
                }
            }
            m = mx * sl2;
            const float mu = m == -INFINITY ? 0.f : m;
            const float2 sc2 = make_float2(sl2, sl2), nmu = make_float2(-mu, -mu);
            float2 acc = make_float2(0.f, 0.f);
            uint8_t* prow = smem + SP_OFF_P;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {  // 8-row chunk (16 bytes of P) q of this 32-row group
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
                    const int col = cc * 32 + q * 8;  // first selected row of the 16-byte chunk
                    *reinterpret_cast<uint4*>(prow + (col >> 6) * SP_BLOCK + swz128(t, (col & 63) >> 3)) =
                        make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
            }
            l = acc.x + acc.y;
        }
        // S is read and P is written: the P V MMAs may reuse S's columns
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_fence_before();
        mbar_arrive(p_full);

        // ===== epilogue: O row t, half by half =====
        const bool one = a.chunks == 1;
        const long long bh = static_cast<long long>(b) * a.Hq + t;
        const long long pc = (static_cast<long long>(b) * a.chunks + chunk) * SP_DV;  // partial column 0
        const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
            if (!warp_wait(&o_full[half], 0, s_abort)) break;
            tc_fence_after();
#pragma unroll 1
            for (int cc = 0; cc < 8; ++cc) {
                uint32_t ov[32];
                tmem_ld32(tmem + lane_off + half * 256 + cc * 32, ov);
                tmem_wait_ld();
                if (!live) continue;
                const int col = half * 256 + cc * 32;
                if (one) {
                    __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(a.out) + bh * SP_DV + col;
#pragma unroll
                    for (int i = 0; i < 32; i += 8)
                        *reinterpret_cast<uint4*>(o + i) = make_uint4(
                            pack_bf16x2(__uint_as_float(ov[i]) * inv, __uint_as_float(ov[i + 1]) * inv),
                            pack_bf16x2(__uint_as_float(ov[i + 2]) * inv, __uint_as_float(ov[i + 3]) * inv),
                            pack_bf16x2(__uint_as_float(ov[i + 4]) * inv, __uint_as_float(ov[i + 5]) * inv),
                            pack_bf16x2(__uint_as_float(ov[i + 6]) * inv, __uint_as_float(ov[i + 7]) * inv));
                } else {
                    // [column][head]: the warp's 32 heads of one column are one 128-byte line
                    float* po = a.part_o + (pc + col) * a.Hq + t;
#pragma unroll
                    for (int i = 0; i < 32; ++i) po[static_cast<long long>(i) * a.Hq] = __uint_as_float(ov[i]);
                }
            }
        }
        if (live) {
            if (one) {
                if (a.lse) a.lse[bh] = l > 0.f ? (m + __log2f(l)) * kLn2 : -INFINITY;
            } else {
                const long long pr = (static_cast<long long>(b) * a.chunks + chunk) * a.Hq + t;
                a.part_ml[pr * 2] = m;  // log2 units; -inf when the chunk holds no valid row
                a.part_ml[pr * 2 + 1] = l;
            }
        }
    } else if (warp == 4) {
        // ===== queries: 64 columns at a time through SP_QS slots =====
        if (lane == 0) {
            bool ok = true;
            const uint32_t q_bytes = static_cast<uint32_t>(a.Hq) * 128;
            int kb = 0;
            for (; kb < SP_KB; ++kb) {
                const int s = kb % SP_QS;
                if (kb >= SP_QS && !(ok = mbar_wait(&q_empty[s], ((kb / SP_QS) - 1) & 1))) break;
                mbar_arrive_expect_tx(&q_full[s], q_bytes);
                tma_load_3d(smem + SP_OFF_Q + s * SP_QBLOCK, &tm_q, &q_full[s], kb * 64, 0, b);
            }
            if (!ok) {
                *s_abort = 1;
                report_status(a.dev_status, KVATTN_STATUS_TIMEOUT);
            }
            // copies in flight complete before the CTA leaves (bounded waits)
            for (int j = kb - SP_QS > 0 ? kb - SP_QS : 0; j < kb; ++j) mbar_wait(&q_full[j % SP_QS], (j / SP_QS) & 1);
        }
    } else {
        // ===== MMA issuer =====
        if (lane == 0) {
            bool ok = true;
            const uint32_t c0 = smem_u32(smem + SP_OFF_C), q0 = smem_u32(smem + SP_OFF_Q);
            const uint32_t p0 = smem_u32(smem + SP_OFF_P);
            for (int kb = 0; kb < SP_KB && ok; ++kb) {
                if (!(ok = mbar_wait(&c_full[kb], 0))) break;
                if (!(ok = mbar_wait(&q_full[kb % SP_QS], (kb / SP_QS) & 1))) break;
                tc_fence_after();
                const uint32_t qs = q0 + (kb % SP_QS) * SP_QBLOCK, cs = c0 + kb * SP_BLOCK;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc_mma_bf16(tmem, umma_desc_k_sw128(qs + kk * 32), umma_desc_k_sw128(cs + kk * 32), SP_IDESC_S,
                                (kb | kk) ? 1u : 0u);
                tc_commit(&q_empty[kb % SP_QS]);
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
    if (warp == 5) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ---- merge of the chunk partials ------------------------------------------------
// CTA = (batch row, 32 heads, 32 value columns), 256 threads: lane = head, warp w
// = columns 4w .. 4w+3.  Every thread derives its head's chunk weights from the
// (m, l) pairs and requests all chunks' values at once (one round trip); the
// 32 x 32 result is transposed through shared memory so that each head's 32
// columns are written as one 64-byte run.
constexpr int SPM_MAX_CHUNKS = 16;  // k <= 2048 in chunks of 128
constexpr int SPM_HEADS = 32, SPM_COLS = 32;

__global__ void __launch_bounds__(256) sparse_merge_kernel(SparseArgs a)
{
    __shared__ float s_o[SPM_HEADS][SPM_COLS + 1];
    __shared__ float s_lse[SPM_HEADS];
    pdl_wait();
    pdl_trigger();
    const int C = a.chunks;
    const int col0 = blockIdx.x * SPM_COLS, h0 = blockIdx.y * SPM_HEADS, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = h0 + lane;
    const long long mlrow = static_cast<long long>(b) * C * a.Hq + h;  // (m, l) row of chunk 0
    float2 ml[SPM_MAX_CHUNKS];
    float ov[SPM_MAX_CHUNKS][4];
#pragma unroll
    for (int c = 0; c < SPM_MAX_CHUNKS; ++c) {
        if (c < C) {
            ml[c] = __ldcg(reinterpret_cast<const float2*>(a.part_ml) + mlrow + static_cast<long long>(c) * a.Hq);
            const float* po = a.part_o + ((static_cast<long long>(b) * C + c) * SP_DV + col0 + 4 * warp) * a.Hq + h;
#pragma unroll
            for (int i = 0; i < 4; ++i) ov[c][i] = __ldcg(po + static_cast<long long>(i) * a.Hq);
        }
    }
    float M = -INFINITY;
#pragma unroll
    for (int c = 0; c < SPM_MAX_CHUNKS; ++c)
        if (c < C) M = fmaxf(M, ml[c].x);
    const float Mu = M == -INFINITY ? 0.f : M;
    float L = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < SPM_MAX_CHUNKS; ++c) {
        if (c < C) {
            const float w = fast_exp2(ml[c].x - Mu);
            L += w * ml[c].y;
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[i] += w * ov[c][i];
        }
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) s_o[lane][4 * warp + i] = acc[i] * inv;
    if (warp == 0) s_lse[lane] = L > 0.f ? (Mu + __log2f(L)) * kLn2 : -INFINITY;
    __syncthreads();
    // thread -> (head tid / 8, columns 4 (tid % 8) .. +3): eight threads per head's 64 bytes
    const int hh = threadIdx.x >> 3, cc = (threadIdx.x & 7) * 4;
    __nv_bfloat16* out =
        reinterpret_cast<__nv_bfloat16*>(a.out) + (static_cast<long long>(b) * a.Hq + h0 + hh) * SP_DV + col0 + cc;
    *reinterpret_cast<uint2*>(out) = make_uint2(pack_bf16x2(s_o[hh][cc], s_o[hh][cc + 1]),
                                                pack_bf16x2(s_o[hh][cc + 2], s_o[hh][cc + 3]));
    if (blockIdx.x == 0 && threadIdx.x < SPM_HEADS && a.lse)
        a.lse[static_cast<long long>(b) * a.Hq + h0 + threadIdx.x] = s_lse[threadIdx.x];
}

}  // namespace

int sparse_chunks(int k) { return (k + SP_ROWS - 1) / SP_ROWS; }

size_t sparse_partial_bytes(int B, int Hq, int k)
{
    const int c = sparse_chunks(k);
    if (c <= 1) return 0;
    return static_cast<size_t>(B) * c * Hq * (SP_DV + 2) * sizeof(float);
}

cudaError_t launch_sparse_attn(const SparseLaunch& l, const CUtensorMap& tm_q, cudaStream_t stream)
{
    static bool attr_set[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 64 && !attr_set[dev]) {
        e = cudaFuncSetAttribute(sparse_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SP_SMEM);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
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
    a.part_o = l.workspace;
    a.part_ml = l.workspace ? l.workspace + static_cast<size_t>(l.B) * a.chunks * l.Hq * SP_DV : nullptr;
    e = launch_pdl(sparse_attn_kernel, dim3(a.chunks, l.B), dim3(SP_THREADS), SP_SMEM, stream, tm_q, a);
    if (e != cudaSuccess || a.chunks == 1) return e;
    return launch_pdl(sparse_merge_kernel, dim3(SP_DV / SPM_COLS, l.Hq / SPM_HEADS, l.B), dim3(256), 0, stream, a);
}

}  // namespace kvattn
