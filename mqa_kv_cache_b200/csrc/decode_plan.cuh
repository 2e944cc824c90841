// decode_plan.cuh -- the ragged split-K work plan shared by the decode kernels.
//
// The cache rows of every (batch, kv-head) unit are cut into tiles of
// DEC_TILE rows; the tiles of all units, in unit order, form one list of N
// tiles; CTA c of the G = min(grid, N) participating CTAs owns the tiles x with
// floor(x G / N) == c.  Where a CTA's range crosses units it makes one piece per
// unit; the pieces of a unit get consecutive partial slots.  Everything is
// computed on the device from the lengths, so the host never waits for them.
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace kvattn {

constexpr int DEC_TILE = 64;  // cache rows per tile

namespace {


__device__ __forceinline__ int owner_of(long long x, long long N, int G)
{
    return static_cast<int>((x * G) / N);
}

__device__ __forceinline__ long long range_start(int c, long long N, int G)
{
    return (static_cast<long long>(c) * N + G - 1) / G;
}

// Pieces of the unit whose first tile is U: the CTAs owning any of its n tiles.
__device__ __forceinline__ int unit_count(long long U, int n, long long N, int G)
{
    return n ? owner_of(U + n - 1, N, G) - owner_of(U, N, G) + 1 : 0;
}

// Block-wide.  s_len[b] = clamped length, s_n[b] = tiles per unit of batch b,
// s_Ub[b] = tiles of one kv-head slice before batch b (s_Ub[B] = total).
// Returns N = Hk * s_Ub[B].
// With q_pos non-null, s_qpos[b] = q_pos[b] too (read in the same round trip).
// With len_cap > 0 a length counts as min(len, len_cap) rows (a rolling cache).
// With seq_lens null every row has T_max rows.
__device__ long long plan_prefix(const int32_t* __restrict__ seq_lens, int B, int Hk, int T_max, int* s_len,
                                 int* s_n, int* s_Ub, int32_t* dev_status, bool report,
                                 const int32_t* __restrict__ q_pos = nullptr, int* s_qpos = nullptr,
                                 int len_cap = 0)
{
    for (int b = threadIdx.x; b < B; b += blockDim.x) {
        if (q_pos) s_qpos[b] = q_pos[b];
        const int len_raw = seq_lens ? seq_lens[b] : T_max;
        const int len = (len_cap > 0 && len_raw > len_cap) ? len_cap : len_raw;
        const int lc = min(max(len, 0), T_max);
        if (lc != len && report) report_status(dev_status, KVATTN_STATUS_BAD_LENGTH);
        s_len[b] = lc;
        s_n[b] = (lc + DEC_TILE - 1) / DEC_TILE;
    }
    __syncthreads();
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        const int per = (B + 31) / 32;
        const int beg = min(lane * per, B), end = min(beg + per, B);
        int sum = 0;
        for (int b = beg; b < end; ++b) sum += s_n[b];
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        int run = incl - sum;
        for (int b = beg; b < end; ++b) {
            s_Ub[b] = run;
            run += s_n[b];
        }
        if (lane == 31) s_Ub[B] = incl;
    }
    __syncthreads();
    return static_cast<long long>(Hk) * s_Ub[B];
}

// Block-wide: number of partial slots used by units 0 .. u_end-1.
__device__ int slots_before(int u_end, int Hk, const int* s_n, const int* s_Ub, long long N, int G, int* s_acc)
{
    if (threadIdx.x == 0) *s_acc = 0;
    __syncthreads();
    int local = 0;
    for (int u = threadIdx.x; u < u_end; u += blockDim.x) {
        const int b = u / Hk, kvh = u - b * Hk;
        const int n = s_n[b];
        const long long U = static_cast<long long>(Hk) * s_Ub[b] + static_cast<long long>(kvh) * n;
        local += unit_count(U, n, N, G);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) local += __shfl_xor_sync(0xffffffffu, local, o);
    if ((threadIdx.x & 31) == 0 && local) atomicAdd(s_acc, local);
    __syncthreads();
    const int r = *s_acc;
    __syncthreads();
    return r;
}

// Position in the unit walk of one CTA.
struct Walk {
    int b, kvh;
    long long U;  // first global tile of the unit
    int S;        // first partial slot of the unit
};

// Tiles [tb, te) of the unit at w (n tiles) that lie in the range [lo, hi) of
// global tiles; false when there are none.
__device__ __forceinline__ bool piece_tiles(const Walk& w, int n, long long lo, long long hi, long long& tb,
                                            long long& te)
{
    tb = (lo > w.U ? lo : w.U) - w.U;
    te = (hi < w.U + n ? hi : w.U + n) - w.U;
    return tb < te;
}

// The CTA owning the unit's first tile (its piece takes the unit's first slot).
__device__ __forceinline__ int unit_first_owner(long long U, long long N, int G) { return owner_of(U, N, G); }

// The unit holding global tile lo: b = the last batch entry starting at or before lo.
__device__ __forceinline__ Walk walk_from(long long lo, int B, int Hk, const int* s_n, const int* s_Ub, int S)
{
    int lo_b = 0, hi_b = B - 1;
    while (lo_b < hi_b) {
        const int mid = (lo_b + hi_b + 1) >> 1;
        if (static_cast<long long>(Hk) * s_Ub[mid] <= lo) lo_b = mid;
        else hi_b = mid - 1;
    }
    const long long Ub = static_cast<long long>(Hk) * s_Ub[lo_b];
    const int n = s_n[lo_b];
    const int kvh = static_cast<int>((lo - Ub) / n);
    return Walk{lo_b, kvh, Ub + static_cast<long long>(kvh) * n, S};
}

__device__ __forceinline__ void walk_next(Walk& w, int B, int Hk, const int* s_n, long long N, int G)
{
    const int n = s_n[w.b];
    w.S += unit_count(w.U, n, N, G);
    w.U += n;
    if (++w.kvh == Hk) {
        w.kvh = 0;
        ++w.b;
        while (w.b < B && s_n[w.b] == 0) ++w.b;
    }
}

}  // namespace

}  // namespace kvattn
