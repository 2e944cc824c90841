// merge.cu -- decode results over disjoint key sets merged into the decode over
// their union: the last step of a sequence-sharded decode, where each GPU (or
// each call) attends to one slice of a long cache and the slices' (o_j, lse_j)
// are exchanged once.
//
// Softmax over a union of key sets: with LSE = ln sum_j exp(lse_j),
// out = sum_j exp(lse_j - LSE) o_j (o_j normalised within its set), and a set
// with no keys (lse_j = -inf) has weight 0.  One warp per (batch, head): the n
// lse values are read first (the max and the normaliser), then the n output
// rows, each lane holding d/32 dimensions.
#include "common.cuh"
#include "kernels.h"

namespace kvattn {

namespace {

constexpr int MG_WARPS = 8;

template <int D>
__global__ void __launch_bounds__(MG_WARPS * 32) merge_lse_kernel(MergeArgs a)
{
    constexpr int PL = D / 32;  // dimensions per lane
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const long long row = static_cast<long long>(blockIdx.x) * MG_WARPS + (threadIdx.x >> 5);  // b * H + h
    const long long rows = static_cast<long long>(a.B) * a.H;
    if (row >= rows) return;
    // the largest lse, then the sum of exp(lse_j - max); lanes take parts j = lane, lane + 32, ...
    float mx = -INFINITY;
    for (int j = lane; j < a.n; j += 32) mx = fmaxf(mx, a.lse_parts[j * rows + row]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.out) + row * D + lane * PL;
    if (mx == -INFINITY) {  // no part saw a key
#pragma unroll
        for (int i = 0; i < PL; ++i) out[i] = __float2bfloat16_rn(0.f);
        if (lane == 0 && a.lse) a.lse[row] = -INFINITY;
        return;
    }
    float den = 0.f;
    for (int j = lane; j < a.n; j += 32) den += expf(a.lse_parts[j * rows + row] - mx);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    float acc[PL];
#pragma unroll
    for (int i = 0; i < PL; ++i) acc[i] = 0.f;
    for (int j = 0; j < a.n; ++j) {
        const float wj = expf(a.lse_parts[j * rows + row] - mx) / den;
        const __nv_bfloat16* oj = reinterpret_cast<const __nv_bfloat16*>(a.o_parts) + (j * rows + row) * D + lane * PL;
        if (PL == 4) {
            const uint2 v = *reinterpret_cast<const uint2*>(oj);
            acc[0] += wj * bf16_lo(v.x);
            acc[1] += wj * bf16_hi(v.x);
            acc[PL - 2] += wj * bf16_lo(v.y);
            acc[PL - 1] += wj * bf16_hi(v.y);
        } else {
            const uint32_t v = *reinterpret_cast<const uint32_t*>(oj);
            acc[0] += wj * bf16_lo(v);
            acc[PL - 1] += wj * bf16_hi(v);
        }
    }
    if (PL == 4) {
        *reinterpret_cast<uint2*>(out) = make_uint2(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[PL - 2], acc[PL - 1]));
    } else {
        *reinterpret_cast<uint32_t*>(out) = pack_bf16x2(acc[0], acc[PL - 1]);
    }
    if (lane == 0 && a.lse) a.lse[row] = mx + logf(den);
}

}  // namespace

cudaError_t launch_merge_lse(const MergeArgs& a, cudaStream_t stream)
{
    const long long rows = static_cast<long long>(a.B) * a.H;
    const dim3 grid(static_cast<unsigned>((rows + MG_WARPS - 1) / MG_WARPS));
    if (a.d == 128) return launch_pdl(merge_lse_kernel<128>, grid, dim3(MG_WARPS * 32), 0, stream, a);
    return launch_pdl(merge_lse_kernel<64>, grid, dim3(MG_WARPS * 32), 0, stream, a);
}

}  // namespace kvattn
