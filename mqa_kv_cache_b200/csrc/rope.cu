// rope.cu -- RoPE cos/sin table construction and in-place rotation of q and k.
//
// Table: "Agentic RL 入门3：transformer 架构" §1.1 (theta_i = base^(-2i/d),
// rotation R(m, theta_i)) and §1.2 ① PI, ② NTK-aware base, ③ YaRN ramp and
// attention temperature, ④ dynamic NTK.  Angles are formed and evaluated in
// fp64 (m * theta reaches ~3e4 rad at the 32K configurations, where an fp32
// angle would already be off by ~2e-3 rad) and stored as fp32.
//
// Rotation: memory-bound.  One thread owns one 16-byte chunk (8 bf16) of a
// head vector; for adjacent pairs that is 4 whole pairs, for half-split pairs
// the thread also owns the partner chunk d/2 further on.  Math in fp32,
// bf16 round-to-nearest-even on store.  v is never passed here.
#include "common.cuh"
#include "kernels.h"

namespace kvattn {

namespace {

constexpr double kTwoPi = 6.283185307179586476925286766559;

__global__ void rope_table_kernel(kvattn_rope_params p, int max_pos, float* __restrict__ cos_out,
                                  float* __restrict__ sin_out)
{
    const int half = p.head_dim / 2;
    const long long total = static_cast<long long>(max_pos) * half;
    for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < total;
         idx += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int m = static_cast<int>(idx / half);
        const int i = static_cast<int>(idx - static_cast<long long>(m) * half);
        const double d = static_cast<double>(p.head_dim);

        double base = p.base;
        if (p.scaling == KVATTN_ROPE_NTK) {
            base = p.base * pow(p.s, d / (d - 2.0));
        } else if (p.scaling == KVATTN_ROPE_DYN_NTK) {
            const double s_dyn = fmax(1.0, p.L_cur / p.L_train);
            base = p.base * pow(s_dyn, d / (d - 2.0));
        }
        // theta_i = base^(-2i/d)
        double theta = exp(-(2.0 * i / d) * log(base));
        double pos = static_cast<double>(m);
        double mag = 1.0;
        if (p.scaling == KVATTN_ROPE_PI) {
            pos = pos / p.s;
        } else if (p.scaling == KVATTN_ROPE_YARN) {
            // turns completed inside the training window decide the blend
            const double r = p.L_train * theta / kTwoPi;
            const double gamma =
                r > p.beta ? 1.0 : (r <= p.alpha ? 0.0 : (r - p.alpha) / (p.beta - p.alpha));
            theta = gamma * theta + (1.0 - gamma) * (theta / p.s);
            mag = 1.0 + 0.1 * log(p.s);
        }
        double sv, cv;
        sincos(pos * theta, &sv, &cv);
        cos_out[idx] = static_cast<float>(mag * cv);
        sin_out[idx] = static_cast<float>(mag * sv);
    }
}

struct RopeView {
    __nv_bfloat16* x;
    const int32_t* pos;
    long long n_vec;  // nb * nt * nh
    int nt, nh;
    long long sb, st, sh;
};

// Rotate one 8-element chunk (adjacent pairs) or one pair of 8-element chunks
// (half-split pairs) of vector `src` with table row cos_row / sin_row into `vec`
// (the same vector for an in-place rotation).
template <int PAIR_STYLE>
__device__ __forceinline__ void rotate_chunk(__nv_bfloat16* vec, int chunk, int half, const float* cos_row,
                                             const float* sin_row, const __nv_bfloat16* src = nullptr)
{
    if (!src) src = vec;
    if (PAIR_STYLE == 0) {
        // elements 8c .. 8c+7 = pairs 4c .. 4c+3
        const float4 c = *reinterpret_cast<const float4*>(cos_row + chunk * 4);
        const float4 s = *reinterpret_cast<const float4*>(sin_row + chunk * 4);
        const float cc[4] = {c.x, c.y, c.z, c.w}, ss[4] = {s.x, s.y, s.z, s.w};
        *reinterpret_cast<uint4*>(vec + chunk * 8) =
            rope_chunk_adjacent(*reinterpret_cast<const uint4*>(src + chunk * 8), cc, ss);
    } else {
        // element 8c + j pairs with 8c + j + d/2; pair index 8c + j
        uint4* pa = reinterpret_cast<uint4*>(vec + chunk * 8);
        uint4* pb = reinterpret_cast<uint4*>(vec + half + chunk * 8);
        const float4 c0 = *reinterpret_cast<const float4*>(cos_row + chunk * 8);
        const float4 c1 = *reinterpret_cast<const float4*>(cos_row + chunk * 8 + 4);
        const float4 s0 = *reinterpret_cast<const float4*>(sin_row + chunk * 8);
        const float4 s1 = *reinterpret_cast<const float4*>(sin_row + chunk * 8 + 4);
        const float cc[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        const float ss[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
        uint4 ra = *reinterpret_cast<const uint4*>(src + chunk * 8);
        uint4 rb = *reinterpret_cast<const uint4*>(src + half + chunk * 8);
        rope_chunk_half(ra, rb, cc, ss);
        *pa = ra;
        *pb = rb;
    }
}

// grid (x: blocks over the tensor's chunks, y: 0 = q, 1 = k).  Index arithmetic in
// 32-bit unsigned (the host checks that every view has fewer than 2^31 chunks):
// the three divisions per chunk are the kernel's main ALU cost.
template <int PAIR_STYLE>
__global__ void rope_apply_kernel(RopeView qv, RopeView kv, const float* __restrict__ cos_tab,
                                  const float* __restrict__ sin_tab, int max_pos, int head_dim,
                                  int32_t* dev_status)
{
    pdl_wait();
    pdl_trigger();
    const RopeView v = blockIdx.y == 0 ? qv : kv;
    const int half = head_dim / 2;
    // threads per head vector: one per chunk of 8 elements (adjacent pairs) or
    // per chunk of the first half (half-split pairs)
    const unsigned per_vec = PAIR_STYLE == 0 ? head_dim / 8 : head_dim / 16;
    const unsigned total = static_cast<unsigned>(v.n_vec) * per_vec;
    const unsigned nh = static_cast<unsigned>(v.nh), nt = static_cast<unsigned>(v.nt);
    for (unsigned tid = blockIdx.x * blockDim.x + threadIdx.x; tid < total; tid += gridDim.x * blockDim.x) {
        const unsigned vec = tid / per_vec;
        const int chunk = static_cast<int>(tid - vec * per_vec);
        const unsigned bt = vec / nh;
        const int h = static_cast<int>(vec - bt * nh);
        const unsigned b = bt / nt;
        const int t = static_cast<int>(bt - b * nt);
        const int m = v.pos[bt];
        if (m < 0 || m >= max_pos) {
            if (chunk == 0) report_status(dev_status, KVATTN_STATUS_BAD_POSITION);
            continue;
        }
        __nv_bfloat16* base = v.x + static_cast<long long>(b) * v.sb + static_cast<long long>(t) * v.st +
                              static_cast<long long>(h) * v.sh;
        rotate_chunk<PAIR_STYLE>(base, chunk, half, cos_tab + static_cast<long long>(m) * half,
                                 sin_tab + static_cast<long long>(m) * half);
    }
}

// New token's k rotated at its position into its cache slot (the position, or its
// place in a rolling cache of sinks + window), v copied there.
// One thread per 8-element chunk (adjacent pairs) or per pair of chunks
// (half-split pairs) of every (batch, kv head) vector.
template <int PAIR_STYLE>
__global__ void kv_append_kernel(KvAppendArgs a)
{
    pdl_wait();
    pdl_trigger();
    const int half = a.head_dim / 2;
    const int per_vec = PAIR_STYLE == 0 ? a.head_dim / 8 : a.head_dim / 16;
    const long long total = static_cast<long long>(a.B) * a.Hk * per_vec;
    for (long long tid = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; tid < total;
         tid += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long vec = tid / per_vec;  // b * Hk + h
        const int chunk = static_cast<int>(tid - vec * per_vec);
        const int b = static_cast<int>(vec / a.Hk);
        const int m = a.pos[b];
        const int slot = (a.window > 0 && m >= a.n_sink) ? a.n_sink + (m - a.n_sink) % a.window : m;
        if (m < 0 || slot >= a.T_max || m >= a.max_pos) {
            if (chunk == 0) report_status(a.dev_status, KVATTN_STATUS_BAD_POSITION);
            continue;
        }
        const long long row = (vec * a.T_max + slot) * a.head_dim;
        const __nv_bfloat16* kn = reinterpret_cast<const __nv_bfloat16*>(a.k_new) + vec * a.head_dim;
        const __nv_bfloat16* vn = reinterpret_cast<const __nv_bfloat16*>(a.v_new) + vec * a.head_dim;
        __nv_bfloat16* kc = reinterpret_cast<__nv_bfloat16*>(a.k_cache) + row;
        __nv_bfloat16* vc = reinterpret_cast<__nv_bfloat16*>(a.v_cache) + row;
        rotate_chunk<PAIR_STYLE>(kc, chunk, half, a.cos_tab + static_cast<long long>(m) * half,
                                 a.sin_tab + static_cast<long long>(m) * half, kn);
        *reinterpret_cast<uint4*>(vc + chunk * 8) = *reinterpret_cast<const uint4*>(vn + chunk * 8);
        if (PAIR_STYLE == 1)
            *reinterpret_cast<uint4*>(vc + half + chunk * 8) = *reinterpret_cast<const uint4*>(vn + half + chunk * 8);
    }
}

}  // namespace

cudaError_t launch_rope_table(const kvattn_rope_params& p, int max_pos, float* cos_out, float* sin_out,
                              cudaStream_t stream)
{
    const long long total = static_cast<long long>(max_pos) * (p.head_dim / 2);
    const int threads = 256;
    const long long blocks = (total + threads - 1) / threads;
    const int grid = static_cast<int>(blocks < 65535 ? blocks : 65535);
    rope_table_kernel<<<grid, threads, 0, stream>>>(p, max_pos, cos_out, sin_out);
    return cudaGetLastError();
}

cudaError_t launch_rope_apply(const RopeApplyArgs& a, cudaStream_t stream)
{
    RopeView qv{reinterpret_cast<__nv_bfloat16*>(a.q), a.q_pos,
                a.q ? static_cast<long long>(a.q_nb) * a.q_nt * a.q_nh : 0, a.q_nt > 0 ? a.q_nt : 1,
                a.q_nh > 0 ? a.q_nh : 1, a.q_sb, a.q_st, a.q_sh};
    RopeView kv{reinterpret_cast<__nv_bfloat16*>(a.k), a.k_pos,
                a.k ? static_cast<long long>(a.k_nb) * a.k_nt * a.k_nh : 0, a.k_nt > 0 ? a.k_nt : 1,
                a.k_nh > 0 ? a.k_nh : 1, a.k_sb, a.k_st, a.k_sh};
    const int per_vec = a.pair_style == 0 ? a.head_dim / 8 : a.head_dim / 16;
    const long long most = (qv.n_vec > kv.n_vec ? qv.n_vec : kv.n_vec) * per_vec;
    if (most == 0) return cudaSuccess;
    if (most >= (1ll << 31)) return cudaErrorInvalidValue;  // the kernel indexes chunks in 32 bits
    const int threads = 256;
    long long blocks = (most + threads - 1) / threads;
    const long long cap = static_cast<long long>(a.num_sms) * 8;  // 8 x 256 threads resident per SM
    if (blocks > cap) blocks = cap;
    auto kern = a.pair_style == 0 ? rope_apply_kernel<0> : rope_apply_kernel<1>;
    return launch_pdl(kern, dim3(static_cast<unsigned>(blocks), 2), dim3(threads), 0, stream, qv, kv, a.cos_tab,
                      a.sin_tab, a.max_pos, a.head_dim, a.dev_status);
}

cudaError_t launch_kv_append(const KvAppendArgs& a, cudaStream_t stream)
{
    const int per_vec = a.pair_style == 0 ? a.head_dim / 8 : a.head_dim / 16;
    const long long total = static_cast<long long>(a.B) * a.Hk * per_vec;
    const int threads = 128;
    long long blocks = (total + threads - 1) / threads;
    if (blocks > 65535) blocks = 65535;
    auto kern = a.pair_style == 0 ? kv_append_kernel<0> : kv_append_kernel<1>;
    return launch_pdl(kern, dim3(static_cast<unsigned>(blocks)), dim3(threads), 0, stream, a);
}

}  // namespace kvattn
