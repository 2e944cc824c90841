// qsa.cu -- the block-level indexer's key builder: the keys of complete 4-token
// groups ("attention" page, "Qwen Sparse Attention (QSA)" §3 ①).
//
// Block key of group j (tokens 4j .. 4j+3): the mean of the four indexer keys,
// RMS-normalised (x / sqrt(mean(x^2) + eps), no gain), then rotated by RoPE at
// the group's first position 4j.  Keys are built once per completed group and
// stored in bf16 beside the indexer cache, so that a decode step scores L/4
// stored keys instead of L token keys: the scoring and top-k are the lightning
// indexer's kernels run over the block keys (dsa.cu, lengths shifted by 2).
//
// Expand (written by the top-k kernel's compaction in its groups mode): the n_top
// selected groups become 4 n_top token positions in increasing order, and the
// 0..3 tokens of the trailing incomplete group follow unconditionally; the list is
// -1 padded to 4 n_top + 3 entries.
#include "common.cuh"
#include "kernels.h"

namespace kvattn {

namespace {

constexpr int QK_DIM = 128;              // indexer key width
constexpr int QK_LANES = QK_DIM / 8;     // 16 lanes per group, 8 elements (one 16-byte chunk) each
constexpr int QK_THREADS = 256;
constexpr int QK_GROUPS = QK_THREADS / QK_LANES;  // groups per CTA per pass

__device__ __forceinline__ void unpack8(uint4 v, float (&x)[8])
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = bf16_lo(w[i]);
        x[2 * i + 1] = bf16_hi(w[i]);
    }
}

// grid (x: CTAs per row, y: batch row).  A 16-lane group builds one block key.
__global__ void __launch_bounds__(QK_THREADS) qsa_block_keys_kernel(QsaKeysArgs a)
{
    pdl_wait();
    pdl_trigger();
    const int b = blockIdx.y;
    const int nb_max = a.L_max / QSA_BLOCK;
    const int len_raw = a.seq_lens[b];
    const int len = min(max(len_raw, 0), a.L_max);
    if (len != len_raw && blockIdx.x == 0 && threadIdx.x == 0) report_status(a.dev_status, KVATTN_STATUS_BAD_LENGTH);
    const int nb = len / QSA_BLOCK;
    const int from = a.block_from ? min(max(a.block_from[b], 0), nb) : 0;
    const int end = min(nb, from + a.max_new);
    const int grp = threadIdx.x / QK_LANES, c = threadIdx.x % QK_LANES;
    const unsigned gmask = 0xffffu << (threadIdx.x & 16);  // the 16 lanes of this group
    for (int j = from + blockIdx.x * QK_GROUPS + grp; j < end; j += gridDim.x * QK_GROUPS) {
        // the four keys of the group: 16 lanes x 16 bytes per row, rows contiguous
        const uint4* src = reinterpret_cast<const uint4*>(
            a.k_idx + (static_cast<long long>(b) * a.L_max + static_cast<long long>(j) * QSA_BLOCK) * QK_DIM);
        float k0[8], k1[8], k2[8], k3[8];
        unpack8(__ldg(src + c), k0);
        unpack8(__ldg(src + QK_LANES + c), k1);
        unpack8(__ldg(src + 2 * QK_LANES + c), k2);
        unpack8(__ldg(src + 3 * QK_LANES + c), k3);
        float x[8], ss = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            x[i] = ((k0[i] + k1[i]) + (k2[i] + k3[i])) * 0.25f;
            ss = __fmaf_rn(x[i], x[i], ss);
        }
#pragma unroll
        for (int o = QK_LANES / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(gmask, ss, o);
        const float inv = 1.0f / sqrtf(ss / QK_DIM + a.eps);
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] *= inv;
        // RoPE at the group's first token
        const int p = j * QSA_BLOCK;
        float y[8];
        if (p < a.max_pos) {
            const float* cs = a.cos_tab + static_cast<long long>(p) * (QK_DIM / 2);
            const float* sn = a.sin_tab + static_cast<long long>(p) * (QK_DIM / 2);
            if (a.pair_style == 0) {
                // adjacent pairs (2i, 2i+1): this lane's pairs are 4c .. 4c+3
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 r = rope_pair(x[2 * i], x[2 * i + 1], cs[4 * c + i], sn[4 * c + i]);
                    y[2 * i] = r.x;
                    y[2 * i + 1] = r.y;
                }
            } else {
                // halves: element e pairs with e + 64; lanes c and c ^ 8 hold the two partners
                float o8[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) o8[i] = __shfl_xor_sync(gmask, x[i], 8);
                const bool first = c < QK_LANES / 2;
                const int e0 = (first ? c : c - QK_LANES / 2) * 8;  // pair index of element 0
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float2 r = first ? rope_pair(x[i], o8[i], cs[e0 + i], sn[e0 + i])
                                           : rope_pair(o8[i], x[i], cs[e0 + i], sn[e0 + i]);
                    y[i] = first ? r.x : r.y;
                }
            }
        } else {
            if (c == 0) report_status(a.dev_status, KVATTN_STATUS_BAD_POSITION);
#pragma unroll
            for (int i = 0; i < 8; ++i) y[i] = x[i];
        }
        uint4* dst = reinterpret_cast<uint4*>(
            a.block_keys + (static_cast<long long>(b) * nb_max + j) * QK_DIM);
        dst[c] = make_uint4(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]), pack_bf16x2(y[4], y[5]),
                            pack_bf16x2(y[6], y[7]));
    }
}

}  // namespace

cudaError_t launch_qsa_block_keys(const QsaKeysArgs& a, cudaStream_t stream)
{
    const int nb_max = a.L_max / QSA_BLOCK;
    const int per_row = a.max_new < nb_max ? a.max_new : nb_max;
    int gx = (per_row + QK_GROUPS - 1) / QK_GROUPS;
    if (gx > 4096) gx = 4096;  // grid-stride beyond
    if (gx < 1) gx = 1;
    return launch_pdl(qsa_block_keys_kernel, dim3(gx, a.B), dim3(QK_THREADS), 0, stream, a);
}

}  // namespace kvattn
