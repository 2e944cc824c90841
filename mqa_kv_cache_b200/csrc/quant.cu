// quant.cu -- FP8 (E4M3) quantisation of latent rows and indexer keys.
//
// "稀疏注意力：省了什么，没省什么", 改进一: a DeepSeek-V3.2 cache keeps, per token and
// layer, 656 bytes -- the FP8 latent, its scales and the bf16 RoPE part -- and an
// indexer key of about 132 bytes; "Agentic RL 入门3" §2.2 (1): the indexer runs
// stably in fp8.  The pages fix the byte budget, not the rounding rule; the
// reading implemented here: the 512 latent values in 4 groups of 128 (the
// indexer key: one group of 128), each group one fp32 scale s = absmax / 448
// (448 = the largest finite E4M3 value) and codes = E4M3 round-to-nearest-even
// of x / s, saturating; an all-zero group has s = 0 and codes 0.  Both
// divisions are IEEE fp32 divisions (__fdiv_rn), so the codes are a function of
// the inputs alone.  Packed latent row: codes [512], scales fp32 [4], RoPE part
// bf16 [64] = 656 bytes.  Memory-bound: one read of the row, one write.
#include "common.cuh"
#include "kernels.h"

namespace kvattn {

namespace {

__device__ __forceinline__ float absmax8(uint4 x)
{
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
    float a = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) a = fmaxf(a, fmaxf(fabsf(bf16_lo(w[i])), fabsf(bf16_hi(w[i]))));
    return a;
}

// Two fp32 -> two E4M3 codes (lo in the low byte), round to nearest even, saturating.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Eight bf16 values -> eight codes at scale s (0: all codes 0).
__device__ __forceinline__ uint2 quant8(uint4 x, float s)
{
    if (s == 0.f) return make_uint2(0u, 0u);
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
    uint32_t c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) c[i] = e4m3x2(__fdiv_rn(bf16_lo(w[i]), s), __fdiv_rn(bf16_hi(w[i]), s));
    return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

constexpr int LQ_WARPS = 8;

// One warp per latent row: lane l holds 16-byte chunks l and l + 32 of the 512
// latent values (groups l / 16 and 2 + l / 16) and, for l < 8, chunk 64 + l of
// the RoPE part.
__global__ void __launch_bounds__(LQ_WARPS * 32) latent_quant_kernel(const kvattn_bf16* src, long long n_rows,
                                                                     uint8_t* dst)
{
    const long long row = static_cast<long long>(blockIdx.x) * LQ_WARPS + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= n_rows) return;
    const uint4* s = reinterpret_cast<const uint4*>(src + row * 576);
    uint8_t* d = dst + row * 656;
    const uint4 x0 = s[lane], x1 = s[lane + 32];
    float a0 = absmax8(x0), a1 = absmax8(x1);
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) {
        a0 = fmaxf(a0, __shfl_xor_sync(0xffffffffu, a0, o));
        a1 = fmaxf(a1, __shfl_xor_sync(0xffffffffu, a1, o));
    }
    const float s0 = __fdiv_rn(a0, 448.f), s1 = __fdiv_rn(a1, 448.f);
    *reinterpret_cast<uint2*>(d + 8 * lane) = quant8(x0, s0);
    *reinterpret_cast<uint2*>(d + 8 * (lane + 32)) = quant8(x1, s1);
    if ((lane & 15) == 0) {
        reinterpret_cast<float*>(d + 512)[lane >> 4] = s0;
        reinterpret_cast<float*>(d + 512)[2 + (lane >> 4)] = s1;
    }
    if (lane < 8) reinterpret_cast<uint4*>(d + 528)[lane] = s[64 + lane];
}

// Sixteen lanes per 128-wide indexer key (one group), two keys per warp.
__global__ void __launch_bounds__(256) idx_key_quant_kernel(const kvattn_bf16* src, long long n_rows, uint8_t* codes,
                                                            float* scales)
{
    pdl_trigger();  // a following kernel launched with programmatic serialisation may set up early
    const long long row = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 4;
    const int l = threadIdx.x & 15;
    const unsigned half = 0xffffu << (threadIdx.x & 16);
    if (row >= n_rows) return;  // both lanes of a half-warp pair leave together
    const uint4 x = reinterpret_cast<const uint4*>(src + row * 128)[l];
    float a = absmax8(x);
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(half, a, o));
    const float s = __fdiv_rn(a, 448.f);
    reinterpret_cast<uint2*>(codes + row * 128)[l] = quant8(x, s);
    if (l == 0) scales[row] = s;
}

}  // namespace

cudaError_t launch_latent_quant_fp8(const kvattn_bf16* src, long long n_rows, uint8_t* dst, cudaStream_t stream)
{
    if (n_rows == 0) return cudaSuccess;
    const long long blocks = (n_rows + LQ_WARPS - 1) / LQ_WARPS;
    latent_quant_kernel<<<static_cast<unsigned>(blocks), LQ_WARPS * 32, 0, stream>>>(src, n_rows, dst);
    return cudaGetLastError();
}

cudaError_t launch_idx_key_quant_fp8(const kvattn_bf16* src, long long n_rows, uint8_t* codes, float* scales,
                                     cudaStream_t stream)
{
    if (n_rows == 0) return cudaSuccess;
    const long long blocks = (n_rows * 16 + 255) / 256;
    idx_key_quant_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(src, n_rows, codes, scales);
    return cudaGetLastError();
}

}  // namespace kvattn
