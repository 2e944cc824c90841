// sparse.cu -- attention of all query heads over a gathered set of latent rows.
//
// "Agentic RL 入门3：transformer 架构" §2.2 (2): o_t = MLA(q_t, {k_j, v_j : j in
// S_t}); "attention", DSA ② and the "乘法结合律" note: after weight absorption
// every query head ([1, 128, 576]) scores the same single-head latent rows, so
// the step is multi-query attention over the selected rows, with the 576-wide
// row as key and its first 512 columns as value (§2.3.3, §2.3.5).
//
// Kernel: one CTA per (batch row, block of 64 heads, chunk of 256 selected
// rows).  The chunk's rows are gathered 64 at a time with 16-byte cp.async
// (double-buffered, XOR-swizzled 16-byte chunks so that ldmatrix is
// conflict-free; invalid indices are zero-filled and masked).  Eight warps:
// warp w owns 16 heads (w / 2) and half of the 512 value columns (w % 2); the
// scores S = Q K^T (K = 576) and the online softmax are computed by both warps
// of a pair, P V by each for its half.  bf16 mma.sync, fp32 accumulation.
// Chunks of one row are merged by a second kernel (the split-softmax identity).
#include "common.cuh"
#include "kernels.h"

namespace kvattn {

namespace {

constexpr int SP_DK = 576;
constexpr int SP_DV = 512;
constexpr int SP_ROWS = 64;                     // gathered rows per tile
constexpr int SP_CHUNK = 256;                   // selected rows per CTA
constexpr int SP_HB = 64;                       // query heads per CTA
constexpr int SP_WARPS = 8;
constexpr int SP_THREADS = SP_WARPS * 32;
constexpr int SP_RB = SP_DK * 2;                // bytes per row (1152)
constexpr int SP_CPR = SP_RB / 16;              // 16-byte chunks per row (72)
constexpr int SP_TILE_BYTES = SP_ROWS * SP_RB;  // 73728
constexpr int SP_Q_BYTES = SP_HB * SP_RB;       // 73728
constexpr int SP_OFF_TILE = SP_Q_BYTES;
constexpr int SP_OFF_IDX = SP_OFF_TILE + 2 * SP_TILE_BYTES;
constexpr int SP_SMEM = SP_OFF_IDX + 2 * SP_ROWS * 4 + 128;
constexpr float kLog2e = 1.44269504088896340736f;
constexpr float kLn2 = 0.69314718055994530942f;

// Byte offset of 16-byte chunk c of row r: chunks XOR-swizzled in groups of 8.
__device__ __forceinline__ uint32_t sp_off(int r, int c)
{
    return static_cast<uint32_t>(r * SP_RB + (((c & ~7) | ((c & 7) ^ (r & 7))) << 4));
}

struct SparseArgs {
    const kvattn_bf16* q;       // [B][Hq][576]
    const kvattn_bf16* latent;  // [B][L_max][576]
    const int32_t* idx;         // [B][k]
    kvattn_bf16* out;           // [B][Hq][512]
    float* lse;                 // [B][Hq] or null
    float* part_o;              // [B][chunks][Hq][512]
    float* part_ml;             // [B][chunks][Hq][2]
    int32_t* dev_status;
    int B, Hq, L_max, k, chunks;
    float scale;
};

__global__ void __launch_bounds__(SP_THREADS, 1) sparse_attn_kernel(SparseArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    const uint32_t sQ = smem_u32(smem);
    int* s_idx = reinterpret_cast<int*>(smem + SP_OFF_IDX);  // [2][SP_ROWS] validated row numbers (-1 = none)

    const int chunk = blockIdx.x, hblk = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int hg = warp >> 1, vh = warp & 1;
    const int r0 = lane >> 2, cq = lane & 3;
    const int row_lo = chunk * SP_CHUNK;
    const int row_hi = min(row_lo + SP_CHUNK, a.k);
    const int n_tiles = (row_hi - row_lo + SP_ROWS - 1) / SP_ROWS;
    const int h_base = hblk * SP_HB;
    const kvattn_bf16* lat = a.latent + static_cast<long long>(b) * a.L_max * SP_DK;
    pdl_wait();
    pdl_trigger();

    // queries of this head block -> shared memory (group 0)
    const kvattn_bf16* qb = a.q + (static_cast<long long>(b) * a.Hq + h_base) * SP_DK;
    for (int i = tid; i < SP_HB * SP_CPR; i += SP_THREADS) {
        const int r = i / SP_CPR, c = i - r * SP_CPR;
        cp_async16(sQ + sp_off(r, c), qb + r * SP_DK + c * 8, 16);
    }
    auto gather = [&](int t, int buf) {
        const uint32_t dst = smem_u32(smem + SP_OFF_TILE + buf * SP_TILE_BYTES);
        const int base = row_lo + t * SP_ROWS;
        if (tid < SP_ROWS) {
            int j = base + tid < row_hi ? a.idx[static_cast<long long>(b) * a.k + base + tid] : -1;
            if (j < -1 || j >= a.L_max) {
                report_status(a.dev_status, KVATTN_STATUS_BAD_INDEX);
                j = -1;
            }
            s_idx[buf * SP_ROWS + tid] = j;
        }
        __syncthreads();
        for (int i = tid; i < SP_ROWS * SP_CPR; i += SP_THREADS) {
            const int r = i / SP_CPR, c = i - r * SP_CPR;
            const int j = s_idx[buf * SP_ROWS + r];
            const kvattn_bf16* src = lat + static_cast<long long>(j < 0 ? 0 : j) * SP_DK + c * 8;
            cp_async16(dst + sp_off(r, c), src, j < 0 ? 0u : 16u);
        }
    };
    gather(0, 0);
    cp_async_commit();

    float o[SP_DV / 2 / 8][4];  // 16 heads x 256 value columns
#pragma unroll
    for (int i = 0; i < SP_DV / 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    const float sl2 = a.scale * kLog2e;
    const int mi = lane >> 3, rr = lane & 7;

    for (int t = 0; t < n_tiles; ++t) {
        const int buf = t & 1;
        if (t + 1 < n_tiles) gather(t + 1, buf ^ 1);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        const uint32_t sT = smem_u32(smem + SP_OFF_TILE + buf * SP_TILE_BYTES);
        // ---- S = Q K^T over the tile's 64 rows (K = 576) ----
        float sc[SP_ROWS / 8][4];
#pragma unroll
        for (int i = 0; i < SP_ROWS / 8; ++i) sc[i][0] = sc[i][1] = sc[i][2] = sc[i][3] = 0.f;
#pragma unroll 4
        for (int kk = 0; kk < SP_DK / 16; ++kk) {
            uint32_t qa[4];
            {
                const int r = hg * 16 + rr + ((mi & 1) << 3);
                const int c = kk * 2 + (mi >> 1);
                ldsm_x4(sQ + sp_off(r, c), qa[0], qa[1], qa[2], qa[3]);
            }
#pragma unroll
            for (int np = 0; np < SP_ROWS / 16; ++np) {
                const int r = np * 16 + rr + ((mi >> 1) << 3);
                const int c = kk * 2 + (mi & 1);
                uint32_t b0, b1, b2, b3;
                ldsm_x4(sT + sp_off(r, c), b0, b1, b2, b3);
                mma_bf16_16816(sc[2 * np], qa, b0, b1);
                mma_bf16_16816(sc[2 * np + 1], qa, b2, b3);
            }
        }
        // ---- online softmax over the 64 rows ----
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int i = 0; i < SP_ROWS / 8; ++i) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = i * 8 + 2 * cq + (e & 1);
                float v = sc[i][e] * sl2;
                if (s_idx[buf * SP_ROWS + r] < 0) v = -INFINITY;
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
        const float mu0 = mn0 == -INFINITY ? 0.f : mn0, mu1 = mn1 == -INFINITY ? 0.f : mn1;
        const float al0 = fast_exp2(m0 - mu0), al1 = fast_exp2(m1 - mu1);
        m0 = mn0;
        m1 = mn1;
        float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
        for (int i = 0; i < SP_ROWS / 8; ++i) {
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
        for (int i = 0; i < SP_DV / 16; ++i) {
            o[i][0] *= al0;
            o[i][1] *= al0;
            o[i][2] *= al1;
            o[i][3] *= al1;
        }
        // ---- O += P V for this warp's 256 value columns ----
#pragma unroll
        for (int j = 0; j < SP_ROWS / 16; ++j) {
            uint32_t pa[4];
            pa[0] = pack_bf16x2(sc[2 * j][0], sc[2 * j][1]);
            pa[1] = pack_bf16x2(sc[2 * j][2], sc[2 * j][3]);
            pa[2] = pack_bf16x2(sc[2 * j + 1][0], sc[2 * j + 1][1]);
            pa[3] = pack_bf16x2(sc[2 * j + 1][2], sc[2 * j + 1][3]);
            const int r = j * 16 + rr + ((mi & 1) << 3);
#pragma unroll
            for (int dp = 0; dp < SP_DV / 2 / 16; ++dp) {
                const int c = (vh * (SP_DV / 2) + dp * 16) / 8 + (mi >> 1);
                uint32_t v0, v1, v2, v3;
                ldsm_x4_t(sT + sp_off(r, c), v0, v1, v2, v3);
                mma_bf16_16816(o[2 * dp], pa, v0, v1);
                mma_bf16_16816(o[2 * dp + 1], pa, v2, v3);
            }
        }
        __syncthreads();  // the buffer is refilled by the next iteration's gather
    }
    cp_async_wait<0>();

    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    const int ha = h_base + hg * 16 + r0, hb = ha + 8;
    if (a.chunks == 1) {
        const float i0 = l0 > 0.f ? 1.f / l0 : 0.f, i1 = l1 > 0.f ? 1.f / l1 : 0.f;
        __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.out) + static_cast<long long>(b) * a.Hq * SP_DV;
#pragma unroll
        for (int i = 0; i < SP_DV / 16; ++i) {
            const int col = vh * (SP_DV / 2) + i * 8 + 2 * cq;
            *reinterpret_cast<uint32_t*>(out + static_cast<long long>(ha) * SP_DV + col) =
                pack_bf16x2(o[i][0] * i0, o[i][1] * i0);
            *reinterpret_cast<uint32_t*>(out + static_cast<long long>(hb) * SP_DV + col) =
                pack_bf16x2(o[i][2] * i1, o[i][3] * i1);
        }
        if (a.lse && vh == 0 && cq == 0) {
            const long long bh = static_cast<long long>(b) * a.Hq;
            a.lse[bh + ha] = l0 > 0.f ? (m0 + __log2f(l0)) * kLn2 : -INFINITY;
            a.lse[bh + hb] = l1 > 0.f ? (m1 + __log2f(l1)) * kLn2 : -INFINITY;
        }
    } else {
        const long long pbase = (static_cast<long long>(b) * a.chunks + chunk) * a.Hq;
        float* po = a.part_o + pbase * SP_DV;
#pragma unroll
        for (int i = 0; i < SP_DV / 16; ++i) {
            const int col = vh * (SP_DV / 2) + i * 8 + 2 * cq;
            *reinterpret_cast<float2*>(po + static_cast<long long>(ha) * SP_DV + col) = make_float2(o[i][0], o[i][1]);
            *reinterpret_cast<float2*>(po + static_cast<long long>(hb) * SP_DV + col) = make_float2(o[i][2], o[i][3]);
        }
        if (vh == 0 && cq == 0) {
            a.part_ml[(pbase + ha) * 2] = m0;
            a.part_ml[(pbase + ha) * 2 + 1] = l0;
            a.part_ml[(pbase + hb) * 2] = m1;
            a.part_ml[(pbase + hb) * 2 + 1] = l1;
        }
    }
}

// One warp per (batch row, head): merge the chunk partials.
__global__ void __launch_bounds__(256) sparse_merge_kernel(SparseArgs a)
{
    pdl_wait();
    pdl_trigger();
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    if (warp >= a.B * a.Hq) return;
    const int b = warp / a.Hq, h = warp - b * a.Hq;
    float M = -INFINITY;
    for (int c = 0; c < a.chunks; ++c) M = fmaxf(M, a.part_ml[((static_cast<long long>(b) * a.chunks + c) * a.Hq + h) * 2]);
    const float Mu = M == -INFINITY ? 0.f : M;
    float L = 0.f;
    float acc[SP_DV / 32];
#pragma unroll
    for (int i = 0; i < SP_DV / 32; ++i) acc[i] = 0.f;
    for (int c = 0; c < a.chunks; ++c) {
        const long long p = (static_cast<long long>(b) * a.chunks + c) * a.Hq + h;
        const float wgt = fast_exp2(a.part_ml[p * 2] - Mu);
        L += wgt * a.part_ml[p * 2 + 1];
        const float* po = a.part_o + p * SP_DV;
#pragma unroll
        for (int i = 0; i < SP_DV / 32; ++i) acc[i] += wgt * po[lane + 32 * i];
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.out) + (static_cast<long long>(b) * a.Hq + h) * SP_DV;
#pragma unroll
    for (int i = 0; i < SP_DV / 32; ++i) out[lane + 32 * i] = __float2bfloat16_rn(acc[i] * inv);
    if (lane == 0 && a.lse) a.lse[static_cast<long long>(b) * a.Hq + h] = L > 0.f ? (Mu + __log2f(L)) * kLn2 : -INFINITY;
}

}  // namespace

int sparse_chunks(int k) { return (k + SP_CHUNK - 1) / SP_CHUNK; }

size_t sparse_partial_bytes(int B, int Hq, int k)
{
    const int c = sparse_chunks(k);
    if (c <= 1) return 0;
    return static_cast<size_t>(B) * c * Hq * (SP_DV + 2) * sizeof(float);
}

cudaError_t launch_sparse_attn(const SparseLaunch& l, cudaStream_t stream)
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
    a.q = l.q;
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
    e = launch_pdl(sparse_attn_kernel, dim3(a.chunks, l.Hq / SP_HB, l.B), dim3(SP_THREADS), SP_SMEM, stream, a);
    if (e != cudaSuccess || a.chunks == 1) return e;
    const int warps = l.B * l.Hq;
    return launch_pdl(sparse_merge_kernel, dim3((warps * 32 + 255) / 256), dim3(256), 0, stream, a);
}

}  // namespace kvattn
