// api.cu -- the extern "C" boundary of libkvattn.so.
//
// Every entry point validates its arguments on the host (returning a
// KVATTN_ERR_* code and a thread-local message before anything is launched),
// lays out the caller's workspace, encodes TMA tensor maps where a kernel
// streams through one, and launches on the caller's stream.  Nothing here
// allocates device memory or synchronises the host.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "kernels.h"

namespace {

thread_local char g_err[512] = "";

int fail(int code, const char* fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return code;
}

int ok()
{
    g_err[0] = '\0';
    return KVATTN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr size_t kWsAlign = 256;
size_t align_up(size_t x) { return (x + kWsAlign - 1) / kWsAlign * kWsAlign; }

// Per-device SM count, queried once.
int num_sms_current(int* out)
{
    static std::mutex mu;
    static int cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    std::lock_guard<std::mutex> lk(mu);
    if (dev >= 64) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
        *out = n;
        return 0;
    }
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
        cache[dev] = n;
    }
    *out = cache[dev];
    return 0;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Encoded tensor maps, kept per (device, rank, base address, extents, box): a map
// holds nothing but those, so a cached one is the map a fresh encode would give.
// Decode steps call with the same cache pointers every step; the cache saves the
// host-side encodes on each call.  Replacement is round-robin.
struct MapKey {
    int dev, rank, u8;
    const void* base;
    uint64_t dims[4];
    uint32_t box;
    bool operator==(const MapKey& o) const
    {
        return dev == o.dev && rank == o.rank && u8 == o.u8 && base == o.base && box == o.box &&
               dims[0] == o.dims[0] && dims[1] == o.dims[1] && dims[2] == o.dims[2] && dims[3] == o.dims[3];
    }
};
constexpr int kMapSlots = 64;
struct MapCache {
    std::mutex mu;
    MapKey key[kMapSlots];
    CUtensorMap map[kMapSlots];
    bool used[kMapSlots] = {};
    int next = 0;
};
MapCache& map_cache()
{
    static MapCache c;
    return c;
}

// Tensor map of rank 3 ([z][y][x], box {128 bytes of x, box, 1}) or 4 ([w][z][y][x], box
// {128 bytes of x, 1, box, 1}) over bf16 (or, with u8, bytes), 128-byte swizzle, zero fill
// out of range; from the cache when present.
int make_map(CUtensorMap* map, int rank, const void* base, const uint64_t (&d)[4], uint32_t box_rows,
             bool u8 = false)
{
    MapKey key{};
    if (cudaGetDevice(&key.dev) != cudaSuccess) return fail(KVATTN_ERR_CUDA, "no CUDA device");
    key.rank = rank;
    key.u8 = u8;
    key.base = base;
    for (int i = 0; i < 4; ++i) key.dims[i] = i < rank ? d[i] : 0;
    key.box = box_rows;
    MapCache& c = map_cache();
    {
        std::lock_guard<std::mutex> lk(c.mu);
        for (int i = 0; i < kMapSlots; ++i)
            if (c.used[i] && c.key[i] == key) {
                *map = c.map[i];
                return KVATTN_OK;
            }
    }
    auto fn = encode_fn();
    if (!fn) return fail(KVATTN_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    const uint64_t es = u8 ? 1 : 2;          // element bytes
    const cuuint32_t bx = u8 ? 128 : 64;     // 128 bytes of x per box row
    cuuint64_t dims[4] = {d[0], d[1], d[2], d[3]};
    cuuint64_t strides[3] = {d[0] * es, d[0] * d[1] * es, d[0] * d[1] * d[2] * es};
    cuuint32_t box3[3] = {bx, box_rows, 1};
    cuuint32_t box4[4] = {bx, 1, box_rows, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, u8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank,
                    const_cast<void*>(base), dims, strides,
                    rank == 3 ? box3 : box4, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(KVATTN_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    std::lock_guard<std::mutex> lk(c.mu);
    const int i = c.next;
    c.next = (c.next + 1) % kMapSlots;
    c.key[i] = key;
    c.map[i] = *map;
    c.used[i] = true;
    return KVATTN_OK;
}

// 3-D bf16 tensor map over [z][y][x] (x innermost) with a {64, box_y, 1} box and
// 128-byte swizzle; out-of-range rows read as zero.
int make_map_3d(CUtensorMap* map, const void* base, uint64_t x, uint64_t y, uint64_t z, uint32_t box_y)
{
    const uint64_t d[4] = {x, y, z, 0};
    return make_map(map, 3, base, d, box_y);
}

// 4-D bf16 tensor map over [w][z][y][x] with a {64, 1, box_z, 1} box and
// 128-byte swizzle (one head's rows of a [B][T][H][d] tensor).
int make_map_4d_rows(CUtensorMap* map, const void* base, uint64_t x, uint64_t y, uint64_t z, uint64_t w,
                     uint32_t box_z)
{
    const uint64_t d[4] = {x, y, z, w};
    return make_map(map, 4, base, d, box_z);
}

int cuda_status(cudaError_t e, const char* what)
{
    if (e != cudaSuccess) return fail(KVATTN_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return ok();
}

bool g_supported(int g) { return g == 1 || g == 2 || g == 4 || g == 8 || g == 16 || g == 32 || g == 64; }

// Failure-detection test settings of the calling thread (kvattn_test_decode_stall).
thread_local int g_test_drop_tile = -1;
thread_local unsigned long long g_test_wait_ns = 0;

// Decode workspace layout for a given grid.
// [0, KVATTN_DECODE_WS_ZERO_BYTES): per-unit piece counters (zero between calls, at a
// fixed place so that calls of any shape agree on it); then the partials.
struct DecodeWs {
    size_t off_o, off_ml, off_info, total;
};

DecodeWs decode_ws(int B, int n_head, int n_kv_head, int head_dim, int grid)
{
    const long long slots = kvattn::decode_max_slots(B, n_kv_head, grid);
    const int g = n_head / n_kv_head;
    DecodeWs w;
    w.off_o = KVATTN_DECODE_WS_ZERO_BYTES;
    w.off_ml = w.off_o + align_up(static_cast<size_t>(slots) * g * head_dim * sizeof(float));
    w.off_info = w.off_ml + align_up(static_cast<size_t>(slots) * g * 2 * sizeof(float));
    w.total = w.off_info + align_up(static_cast<size_t>(B) * n_kv_head * sizeof(int2));
    return w;
}

}  // namespace

int kvattn::record_error(int code, const char* fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return code;
}

extern "C" {

const char* kvattn_last_error_string(void) { return g_err; }

const char* kvattn_version(void) { return "kvattn 0.2.0 (sm_100a)"; }

int kvattn_test_decode_stall(int drop_tile, long long wait_limit_ns)
{
    if (drop_tile < -1) return fail(KVATTN_ERR_SHAPE, "kvattn_test_decode_stall: drop_tile %d < -1", drop_tile);
    if (wait_limit_ns < 0 || wait_limit_ns > 10000000000ll)
        return fail(KVATTN_ERR_SHAPE, "kvattn_test_decode_stall: wait limit %lld ns outside 0 .. 10 s",
                    wait_limit_ns);
    g_test_drop_tile = drop_tile;
    g_test_wait_ns = static_cast<unsigned long long>(wait_limit_ns);
    return ok();
}

// ---------------------------------------------------------------------------
int rope_table_build(const kvattn_rope_params* p, int max_pos, float* cos_out, float* sin_out, void* stream)
{
    if (!p || !cos_out || !sin_out) return fail(KVATTN_ERR_NULL, "rope_table_build: NULL argument");
    if (p->reserved != 0) return fail(KVATTN_ERR_SHAPE, "rope_table_build: reserved must be 0");
    if (p->head_dim < 4 || p->head_dim > 256 || (p->head_dim & 1))
        return fail(KVATTN_ERR_SHAPE, "rope_table_build: head_dim %d must be even, 4..256", p->head_dim);
    if (max_pos < 1) return fail(KVATTN_ERR_SHAPE, "rope_table_build: max_pos %d < 1", max_pos);
    if (p->scaling < KVATTN_ROPE_NONE || p->scaling > KVATTN_ROPE_DYN_NTK)
        return fail(KVATTN_ERR_UNSUPPORTED, "rope_table_build: unknown scaling %d", p->scaling);
    if (p->pair_style != 0 && p->pair_style != 1)
        return fail(KVATTN_ERR_UNSUPPORTED, "rope_table_build: pair_style %d", p->pair_style);
    if (!(p->base > 0.0) || !std::isfinite(p->base)) return fail(KVATTN_ERR_SHAPE, "rope_table_build: base must be > 0");
    const bool uses_s = p->scaling == KVATTN_ROPE_PI || p->scaling == KVATTN_ROPE_NTK || p->scaling == KVATTN_ROPE_YARN;
    if (uses_s && !(p->s >= 1.0 && std::isfinite(p->s)))
        return fail(KVATTN_ERR_SHAPE, "rope_table_build: s must be >= 1");
    if ((p->scaling == KVATTN_ROPE_YARN || p->scaling == KVATTN_ROPE_DYN_NTK) && !(p->L_train > 0.0))
        return fail(KVATTN_ERR_SHAPE, "rope_table_build: L_train must be > 0");
    if (p->scaling == KVATTN_ROPE_YARN && !(p->beta > p->alpha))
        return fail(KVATTN_ERR_SHAPE, "rope_table_build: beta must exceed alpha");
    if (p->scaling == KVATTN_ROPE_DYN_NTK && !(p->L_cur >= 0.0))
        return fail(KVATTN_ERR_SHAPE, "rope_table_build: L_cur must be >= 0");
    if (static_cast<long long>(max_pos) * (p->head_dim / 2) > (1ll << 40))
        return fail(KVATTN_ERR_SHAPE, "rope_table_build: table too large");
    return cuda_status(kvattn::launch_rope_table(*p, max_pos, cos_out, sin_out, static_cast<cudaStream_t>(stream)),
                       "rope_table_build launch");
}

// ---------------------------------------------------------------------------
int rope_apply_qk(kvattn_bf16* q, int q_nb, int q_nt, int q_nh, int64_t q_sb, int64_t q_st, int64_t q_sh,
                  const int32_t* q_pos, kvattn_bf16* k, int k_nb, int k_nt, int k_nh, int64_t k_sb, int64_t k_st,
                  int64_t k_sh, const int32_t* k_pos, const float* cos_tab, const float* sin_tab, int max_pos,
                  int head_dim, int pair_style, int32_t* dev_status, void* stream)
{
    if (!cos_tab || !sin_tab) return fail(KVATTN_ERR_NULL, "rope_apply_qk: NULL table");
    if (head_dim < 16 || head_dim > 256 || head_dim % 16)
        return fail(KVATTN_ERR_UNSUPPORTED, "rope_apply_qk: head_dim %d must be a multiple of 16, <= 256", head_dim);
    if (pair_style != 0 && pair_style != 1) return fail(KVATTN_ERR_UNSUPPORTED, "rope_apply_qk: pair_style");
    if (max_pos < 1) return fail(KVATTN_ERR_SHAPE, "rope_apply_qk: max_pos < 1");
    if (!aligned16(cos_tab) || !aligned16(sin_tab)) return fail(KVATTN_ERR_ALIGN, "rope_apply_qk: table alignment");
    struct V {
        kvattn_bf16* x;
        int nb, nt, nh;
        int64_t sb, st, sh;
        const int32_t* pos;
        const char* name;
    } views[2] = {{q, q_nb, q_nt, q_nh, q_sb, q_st, q_sh, q_pos, "q"}, {k, k_nb, k_nt, k_nh, k_sb, k_st, k_sh, k_pos, "k"}};
    for (auto& v : views) {
        if (!v.x) continue;
        if (!v.pos) return fail(KVATTN_ERR_NULL, "rope_apply_qk: %s positions NULL", v.name);
        if (v.nb < 0 || v.nt < 0 || v.nh < 0) return fail(KVATTN_ERR_SHAPE, "rope_apply_qk: negative %s size", v.name);
        if (!aligned16(v.x)) return fail(KVATTN_ERR_ALIGN, "rope_apply_qk: %s not 16-byte aligned", v.name);
        if (v.sb % 8 || v.st % 8 || v.sh % 8 || v.sb < 0 || v.st < 0 || v.sh < 0)
            return fail(KVATTN_ERR_ALIGN, "rope_apply_qk: %s strides must be non-negative multiples of 8", v.name);
        if (static_cast<long long>(v.nb) * v.nt * v.nh * (head_dim / 8) >= (1ll << 31))
            return fail(KVATTN_ERR_SHAPE, "rope_apply_qk: %s has 2^31 or more 16-byte chunks", v.name);
    }
    int sms = 0;
    if (num_sms_current(&sms) != 0) return fail(KVATTN_ERR_CUDA, "rope_apply_qk: no CUDA device");
    kvattn::RopeApplyArgs a{};
    a.q = q;
    a.q_nb = q ? q_nb : 0;
    a.q_nt = q_nt;
    a.q_nh = q_nh;
    a.q_sb = q_sb;
    a.q_st = q_st;
    a.q_sh = q_sh;
    a.q_pos = q_pos;
    a.k = k;
    a.k_nb = k ? k_nb : 0;
    a.k_nt = k_nt;
    a.k_nh = k_nh;
    a.k_sb = k_sb;
    a.k_st = k_st;
    a.k_sh = k_sh;
    a.k_pos = k_pos;
    a.cos_tab = cos_tab;
    a.sin_tab = sin_tab;
    a.max_pos = max_pos;
    a.head_dim = head_dim;
    a.pair_style = pair_style;
    a.dev_status = dev_status;
    a.num_sms = sms;
    return cuda_status(kvattn::launch_rope_apply(a, static_cast<cudaStream_t>(stream)), "rope_apply_qk launch");
}

// ---------------------------------------------------------------------------
size_t attn_decode_gqa_workspace_bytes(int B, int n_head, int n_kv_head, int head_dim, int T_max)
{
    (void)T_max;
    if (B < 1 || n_head < 1 || n_kv_head < 1 || n_head % n_kv_head || head_dim < 1) return 0;
    int sms = 0;
    if (num_sms_current(&sms) != 0) return 0;
    return decode_ws(B, n_head, n_kv_head, head_dim, kvattn::decode_grid(sms)).total;
}

// Shared by attn_decode_gqa (rope == nullptr) and attn_decode_gqa_rope.
struct DecodeRope {
    const int32_t* q_pos;
    const float* cos_tab;
    const float* sin_tab;
    int max_pos, pair_style;
};

struct DecodeGather {
    const int32_t* idx;  // [B][n_idx] cache rows; the row counts come in seq_lens (may be NULL)
    int n_idx;
};

static int decode_call(const char* name, const kvattn_bf16* q, const kvattn_bf16* k_cache,
                       const kvattn_bf16* v_cache, const int32_t* seq_lens, int B, int n_head, int n_kv_head,
                       int head_dim, int T_max, float scale, kvattn_bf16* out, float* lse, void* workspace,
                       size_t workspace_bytes, int32_t* dev_status, void* stream, const DecodeRope* rope,
                       int len_cap = 0, const DecodeGather* gather = nullptr)
{
    if (!q || !k_cache || !v_cache || (!seq_lens && !gather) || !out)
        return fail(KVATTN_ERR_NULL, "%s: NULL argument", name);
    if (gather) {
        if (!gather->idx) return fail(KVATTN_ERR_NULL, "%s: NULL index list", name);
        if (gather->n_idx < 1) return fail(KVATTN_ERR_SHAPE, "%s: n_idx %d", name, gather->n_idx);
        if (head_dim == 128 && n_head > 32 * n_kv_head)
            return fail(KVATTN_ERR_UNSUPPORTED, "%s: group size above 32 at head_dim 128", name);
        if (static_cast<long long>(B) * gather->n_idx > (1ll << 31))
            return fail(KVATTN_ERR_SHAPE, "%s: B * n_idx too large", name);
    }
    if (B < 1 || B > kvattn::DECODE_MAX_B) return fail(KVATTN_ERR_SHAPE, "%s: B %d outside 1..%d", name, B, kvattn::DECODE_MAX_B);
    if (n_head < 1 || n_kv_head < 1 || n_head % n_kv_head)
        return fail(KVATTN_ERR_SHAPE, "%s: n_head %d not a multiple of n_kv_head %d", name, n_head, n_kv_head);
    const int g = n_head / n_kv_head;
    if (!g_supported(g)) return fail(KVATTN_ERR_UNSUPPORTED, "%s: group size %d", name, g);
    if (head_dim != 64 && head_dim != 128) return fail(KVATTN_ERR_UNSUPPORTED, "%s: head_dim %d", name, head_dim);
    if (T_max < 1) return fail(KVATTN_ERR_SHAPE, "%s: T_max %d", name, T_max);
    if (static_cast<long long>(B) * n_kv_head > KVATTN_DECODE_WS_ZERO_BYTES / 4)
        return fail(KVATTN_ERR_UNSUPPORTED, "%s: B * n_kv_head = %lld above %u", name,
                    static_cast<long long>(B) * n_kv_head, KVATTN_DECODE_WS_ZERO_BYTES / 4);
    if (!(scale > 0.0f) || !std::isfinite(scale)) return fail(KVATTN_ERR_SHAPE, "%s: scale must be finite > 0", name);
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
        return fail(KVATTN_ERR_ALIGN, "%s: tensors must be 16-byte aligned", name);
    if (rope) {
        if (!rope->q_pos || !rope->cos_tab || !rope->sin_tab) return fail(KVATTN_ERR_NULL, "%s: NULL RoPE argument", name);
        if (rope->pair_style != 0 && rope->pair_style != 1) return fail(KVATTN_ERR_UNSUPPORTED, "%s: pair_style", name);
        if (rope->max_pos < 1) return fail(KVATTN_ERR_SHAPE, "%s: max_pos < 1", name);
        if (!aligned16(rope->cos_tab) || !aligned16(rope->sin_tab))
            return fail(KVATTN_ERR_ALIGN, "%s: tables must be 16-byte aligned", name);
    }
    int sms = 0;
    if (num_sms_current(&sms) != 0) return fail(KVATTN_ERR_CUDA, "%s: no CUDA device", name);
    const int grid = kvattn::decode_grid(sms);
    const DecodeWs ws = decode_ws(B, n_head, n_kv_head, head_dim, grid);
    if (!workspace || workspace_bytes < ws.total)
        return fail(KVATTN_ERR_WORKSPACE, "%s: workspace needs %zu bytes", name, ws.total);
    if (reinterpret_cast<uintptr_t>(workspace) % kWsAlign)
        return fail(KVATTN_ERR_ALIGN, "%s: workspace must be 256-byte aligned", name);

    CUtensorMap tm_q, tm_k, tm_v;
    const uint64_t units = static_cast<uint64_t>(B) * n_kv_head;
    if (make_map_3d(&tm_k, k_cache, head_dim, T_max, units, 64) != KVATTN_OK) return KVATTN_ERR_CUDA;
    if (make_map_3d(&tm_v, v_cache, head_dim, T_max, units, 64) != KVATTN_OK) return KVATTN_ERR_CUDA;
    // the tensor-core path reads the queries of one KV group as a [B*Hk][g][d] box
    memset(&tm_q, 0, sizeof tm_q);
    if (kvattn::decode_tc_supported(head_dim, g) && make_map_3d(&tm_q, q, head_dim, g, units, 64) != KVATTN_OK)
        return KVATTN_ERR_CUDA;

    uint8_t* w = static_cast<uint8_t*>(workspace);
    kvattn::DecodeArgs a{};
    a.q = q;
    a.seq_lens = seq_lens;
    a.out = out;
    a.lse = lse;
    a.part_o = reinterpret_cast<float*>(w + ws.off_o);
    a.part_ml = reinterpret_cast<float*>(w + ws.off_ml);
    a.unit_info = reinterpret_cast<int2*>(w + ws.off_info);
    a.unit_cnt = reinterpret_cast<int*>(w);
    a.dev_status = dev_status;
    a.len_cap = len_cap;
    if (gather) {
        a.idx = gather->idx;
        a.n_idx = gather->n_idx;
        a.k_cache = k_cache;
        a.v_cache = v_cache;
    }
    if (rope) {
        a.q_pos = rope->q_pos;
        a.cos_tab = rope->cos_tab;
        a.sin_tab = rope->sin_tab;
        a.max_pos = rope->max_pos;
        a.pair_style = rope->pair_style;
    }
    a.B = B;
    a.H = n_head;
    a.Hk = n_kv_head;
    a.g = g;
    a.d = head_dim;
    a.T_max = T_max;
    a.scale = scale;
    a.grid = grid;
    a.wait_ns = g_test_wait_ns;
    a.drop_it = g_test_drop_tile;
    return cuda_status(kvattn::launch_decode(a, tm_q, tm_k, tm_v, static_cast<cudaStream_t>(stream)),
                       name);
}

int attn_decode_gqa(const kvattn_bf16* q, const kvattn_bf16* k_cache, const kvattn_bf16* v_cache,
                    const int32_t* seq_lens, int B, int n_head, int n_kv_head, int head_dim, int T_max, float scale,
                    kvattn_bf16* out, float* lse, void* workspace, size_t workspace_bytes, int32_t* dev_status,
                    void* stream)
{
    return decode_call("attn_decode_gqa", q, k_cache, v_cache, seq_lens, B, n_head, n_kv_head, head_dim, T_max,
                       scale, out, lse, workspace, workspace_bytes, dev_status, stream, nullptr);
}

int attn_decode_gqa_rope(const kvattn_bf16* q, const int32_t* q_pos, const float* cos_tab, const float* sin_tab,
                         int max_pos, int pair_style, const kvattn_bf16* k_cache, const kvattn_bf16* v_cache,
                         const int32_t* seq_lens, int B, int n_head, int n_kv_head, int head_dim, int T_max,
                         float scale, kvattn_bf16* out, float* lse, void* workspace, size_t workspace_bytes,
                         int32_t* dev_status, void* stream)
{
    const DecodeRope r{q_pos, cos_tab, sin_tab, max_pos, pair_style};
    return decode_call("attn_decode_gqa_rope", q, k_cache, v_cache, seq_lens, B, n_head, n_kv_head, head_dim,
                       T_max, scale, out, lse, workspace, workspace_bytes, dev_status, stream, &r);
}

int attn_decode_gqa_rope_window(const kvattn_bf16* q, const int32_t* q_pos, const float* cos_tab,
                                const float* sin_tab, int max_pos, int pair_style, const kvattn_bf16* k_cache,
                                const kvattn_bf16* v_cache, const int32_t* seq_lens, int n_sink, int window, int B,
                                int n_head, int n_kv_head, int head_dim, int T_max, float scale, kvattn_bf16* out,
                                float* lse, void* workspace, size_t workspace_bytes, int32_t* dev_status,
                                void* stream)
{
    if (n_sink < 0 || window < 1 || static_cast<long long>(n_sink) + window > T_max)
        return fail(KVATTN_ERR_SHAPE, "attn_decode_gqa_rope_window: n_sink %d, window %d, capacity %d", n_sink, window,
                    T_max);
    const DecodeRope r{q_pos, cos_tab, sin_tab, max_pos, pair_style};
    return decode_call("attn_decode_gqa_rope_window", q, k_cache, v_cache, seq_lens, B, n_head, n_kv_head, head_dim,
                       T_max, scale, out, lse, workspace, workspace_bytes, dev_status, stream, &r, n_sink + window);
}

int attn_merge_lse(const kvattn_bf16* o_parts, const float* lse_parts, int n_parts, int B, int n_head, int head_dim,
                   kvattn_bf16* out, float* lse, void* stream)
{
    if (!o_parts || !lse_parts || !out) return fail(KVATTN_ERR_NULL, "attn_merge_lse: NULL argument");
    if (head_dim != 64 && head_dim != 128)
        return fail(KVATTN_ERR_UNSUPPORTED, "attn_merge_lse: head_dim %d", head_dim);
    if (n_parts < 1 || B < 1 || n_head < 1)
        return fail(KVATTN_ERR_SHAPE, "attn_merge_lse: n_parts %d, B %d, n_head %d", n_parts, B, n_head);
    if (static_cast<long long>(n_parts) * B * n_head * head_dim > (1ll << 40))
        return fail(KVATTN_ERR_SHAPE, "attn_merge_lse: too large");
    if (!aligned16(o_parts) || !aligned16(out) || (reinterpret_cast<uintptr_t>(lse_parts) & 3) ||
        (lse && (reinterpret_cast<uintptr_t>(lse) & 3)))
        return fail(KVATTN_ERR_ALIGN, "attn_merge_lse: tensors must be aligned (16 bytes; 4 for lse)");
    kvattn::MergeArgs a{o_parts, lse_parts, out, lse, n_parts, B, n_head, head_dim};
    return cuda_status(kvattn::launch_merge_lse(a, static_cast<cudaStream_t>(stream)), "attn_merge_lse launch");
}

size_t attn_decode_gqa_sparse_workspace_bytes(int B, int n_head, int n_kv_head, int head_dim, int n_idx)
{
    return attn_decode_gqa_workspace_bytes(B, n_head, n_kv_head, head_dim, n_idx);
}

int attn_decode_gqa_sparse(const kvattn_bf16* q, const kvattn_bf16* k_cache, const kvattn_bf16* v_cache,
                           const int32_t* tok_idx, const int32_t* tok_count, int n_idx, int B, int n_head,
                           int n_kv_head, int head_dim, int T_max, float scale, kvattn_bf16* out, float* lse,
                           void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream)
{
    const DecodeGather gth{tok_idx, n_idx};
    return decode_call("attn_decode_gqa_sparse", q, k_cache, v_cache, tok_count, B, n_head, n_kv_head, head_dim,
                       T_max, scale, out, lse, workspace, workspace_bytes, dev_status, stream, nullptr, 0, &gth);
}

// ---------------------------------------------------------------------------
static int kv_append_call(const char* name, const kvattn_bf16* k_new, const kvattn_bf16* v_new, const int32_t* pos,
                          int B, int n_kv_head, int head_dim, kvattn_bf16* k_cache, kvattn_bf16* v_cache, int T_max,
                          const float* cos_tab, const float* sin_tab, int max_pos, int pair_style, int n_sink,
                          int window, int32_t* dev_status, void* stream)
{
    if (!k_new || !v_new || !pos || !k_cache || !v_cache || !cos_tab || !sin_tab)
        return fail(KVATTN_ERR_NULL, "%s: NULL argument", name);
    if (B < 1 || n_kv_head < 1 || T_max < 1 || max_pos < 1)
        return fail(KVATTN_ERR_SHAPE, "%s: B %d, n_kv_head %d, T_max %d, max_pos %d", name, B, n_kv_head, T_max,
                    max_pos);
    if (head_dim < 16 || head_dim > 256 || head_dim % 16)
        return fail(KVATTN_ERR_UNSUPPORTED, "%s: head_dim %d must be a multiple of 16, <= 256", name, head_dim);
    if (pair_style != 0 && pair_style != 1) return fail(KVATTN_ERR_UNSUPPORTED, "%s: pair_style", name);
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(cos_tab) ||
        !aligned16(sin_tab))
        return fail(KVATTN_ERR_ALIGN, "%s: tensors must be 16-byte aligned", name);
    kvattn::KvAppendArgs a{k_new, v_new, pos, k_cache, v_cache, cos_tab, sin_tab, B, n_kv_head, head_dim, T_max,
                           max_pos, pair_style, n_sink, window, dev_status};
    return cuda_status(kvattn::launch_kv_append(a, static_cast<cudaStream_t>(stream)), name);
}

int kv_append_rope_ring(const kvattn_bf16* k_new, const kvattn_bf16* v_new, const int32_t* pos, int n_sink,
                        int window, int B, int n_kv_head, int head_dim, kvattn_bf16* k_cache, kvattn_bf16* v_cache,
                        int T_max, const float* cos_tab, const float* sin_tab, int max_pos, int pair_style,
                        int32_t* dev_status, void* stream)
{
    if (n_sink < 0 || window < 1 || static_cast<long long>(n_sink) + window > T_max)
        return fail(KVATTN_ERR_SHAPE, "kv_append_rope_ring: n_sink %d, window %d, capacity %d", n_sink, window, T_max);
    return kv_append_call("kv_append_rope_ring", k_new, v_new, pos, B, n_kv_head, head_dim, k_cache, v_cache, T_max,
                          cos_tab, sin_tab, max_pos, pair_style, n_sink, window, dev_status, stream);
}

// ---------------------------------------------------------------------------
int kv_append_rope(const kvattn_bf16* k_new, const kvattn_bf16* v_new, const int32_t* pos, int B, int n_kv_head,
                   int head_dim, kvattn_bf16* k_cache, kvattn_bf16* v_cache, int T_max, const float* cos_tab,
                   const float* sin_tab, int max_pos, int pair_style, int32_t* dev_status, void* stream)
{
    return kv_append_call("kv_append_rope", k_new, v_new, pos, B, n_kv_head, head_dim, k_cache, v_cache, T_max,
                          cos_tab, sin_tab, max_pos, pair_style, 0, 0, dev_status, stream);
}

// ---------------------------------------------------------------------------
static int prefill_call(const char* name, const kvattn_bf16* q, const kvattn_bf16* k, const kvattn_bf16* v, int B,
                        int T, int n_head, int n_kv_head, int head_dim, float scale, kvattn_bf16* out, float* lse,
                        int n_sink, int window, void* stream)
{
    if (!q || !k || !v || !out) return fail(KVATTN_ERR_NULL, "%s: NULL argument", name);
    if (head_dim != 128) return fail(KVATTN_ERR_UNSUPPORTED, "%s: head_dim %d (needs 128)", name, head_dim);
    if (B < 1 || T < 1 || n_head < 1 || n_kv_head < 1 || n_head % n_kv_head)
        return fail(KVATTN_ERR_SHAPE, "%s: B %d T %d n_head %d n_kv_head %d", name, B, T, n_head, n_kv_head);
    if (!g_supported(n_head / n_kv_head))
        return fail(KVATTN_ERR_UNSUPPORTED, "%s: group size %d", name, n_head / n_kv_head);
    if (static_cast<long long>(B) * n_kv_head > (1ll << 31) - 1 || T > (1 << 30) ||
        static_cast<long long>((T + 255) / 256) * B * n_head > (1ll << 31) - 1)
        return fail(KVATTN_ERR_SHAPE, "%s: problem too large", name);
    if (!(scale > 0.0f) || !std::isfinite(scale))
        return fail(KVATTN_ERR_SHAPE, "%s: scale must be finite > 0", name);
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
        return fail(KVATTN_ERR_ALIGN, "%s: tensors must be 16-byte aligned", name);
    CUtensorMap tm_q, tm_k, tm_v;
    if (make_map_4d_rows(&tm_q, q, head_dim, n_head, T, B, kvattn::PREFILL_Q_ROWS) != KVATTN_OK)
        return KVATTN_ERR_CUDA;
    const uint64_t units = static_cast<uint64_t>(B) * n_kv_head;
    if (make_map_3d(&tm_k, k, head_dim, T, units, kvattn::PREFILL_KV_ROWS) != KVATTN_OK) return KVATTN_ERR_CUDA;
    if (make_map_3d(&tm_v, v, head_dim, T, units, kvattn::PREFILL_KV_ROWS) != KVATTN_OK) return KVATTN_ERR_CUDA;
    kvattn::PrefillLaunch l{out, lse, nullptr, B, T, n_head, n_kv_head, scale, n_sink, window};
    return cuda_status(kvattn::launch_prefill(l, tm_q, tm_k, tm_v, static_cast<cudaStream_t>(stream)),
                       name);
}

int attn_prefill_causal(const kvattn_bf16* q, const kvattn_bf16* k, const kvattn_bf16* v, int B, int T, int n_head,
                        int n_kv_head, int head_dim, float scale, kvattn_bf16* out, float* lse, void* stream)
{
    return prefill_call("attn_prefill_causal", q, k, v, B, T, n_head, n_kv_head, head_dim, scale, out, lse, 0, 0,
                        stream);
}

int attn_prefill_causal_window(const kvattn_bf16* q, const kvattn_bf16* k, const kvattn_bf16* v, int B, int T,
                               int n_head, int n_kv_head, int head_dim, int n_sink, int window, float scale,
                               kvattn_bf16* out, float* lse, void* stream)
{
    if (n_sink < 0 || window < 1)
        return fail(KVATTN_ERR_SHAPE, "attn_prefill_causal_window: n_sink %d, window %d", n_sink, window);
    return prefill_call("attn_prefill_causal_window", q, k, v, B, T, n_head, n_kv_head, head_dim, scale, out, lse,
                        n_sink, window, stream);
}

// DSA / QSA selection workspace: [0, hist) the per-row first-digit counts of the top-k
// (zero between calls), then the scores when the caller keeps none.
// ... then (FP8 calls) the quantised query heads: codes [B][64][128] and scales [B][64].
static size_t dsa_ws_hist(int B) { return align_up(kvattn::dsa_hist_bytes(B)); }
static size_t dsa_ws_q8(int B) { return align_up(static_cast<size_t>(B) * 64 * 128) + align_up(static_cast<size_t>(B) * 64 * 4); }

size_t dsa_index_topk_workspace_bytes(int B, int L_max, int k)
{
    (void)k;
    if (B < 1 || L_max < 1) return 0;
    return dsa_ws_hist(B) + dsa_ws_q8(B) + align_up(kvattn::dsa_scores_bytes(B, L_max));
}

// Checks the selection workspace; on success sets the histogram, the scores buffer and
// (with q8 non-null) the quantised query heads.
static int dsa_ws(const char* name, int B, int L_max, float* scores_out, void* workspace, size_t workspace_bytes,
                  uint32_t** hist, float** scores, uint8_t** q8 = nullptr, float** q8_scale = nullptr)
{
    const size_t q8b = q8 ? dsa_ws_q8(B) : 0;
    const size_t need = dsa_ws_hist(B) + q8b + (scores_out ? 0 : align_up(kvattn::dsa_scores_bytes(B, L_max)));
    if (!workspace || workspace_bytes < need) return fail(KVATTN_ERR_WORKSPACE, "%s: workspace needs %zu bytes", name, need);
    if (reinterpret_cast<uintptr_t>(workspace) % kWsAlign)
        return fail(KVATTN_ERR_ALIGN, "%s: workspace must be 256-byte aligned", name);
    uint8_t* w = static_cast<uint8_t*>(workspace);
    *hist = reinterpret_cast<uint32_t*>(w);
    if (q8) {
        *q8 = w + dsa_ws_hist(B);
        *q8_scale = reinterpret_cast<float*>(w + dsa_ws_hist(B) + align_up(static_cast<size_t>(B) * 64 * 128));
    }
    *scores = scores_out ? scores_out : reinterpret_cast<float*>(w + dsa_ws_hist(B) + q8b);
    return KVATTN_OK;
}

int dsa_index_topk(const kvattn_bf16* q_idx, const float* w, const kvattn_bf16* k_idx, const int32_t* seq_lens, int B,
                   int n_idx_head, int idx_dim, int L_max, int k, int32_t* topk_idx, float* scores_out,
                   void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream)
{
    if (!q_idx || !w || !k_idx || !topk_idx) return fail(KVATTN_ERR_NULL, "dsa_index_topk: NULL argument");
    if (n_idx_head != 64 || idx_dim != 128)
        return fail(KVATTN_ERR_UNSUPPORTED, "dsa_index_topk: needs 64 indexer heads of width 128 (got %d x %d)",
                    n_idx_head, idx_dim);
    if (B < 1 || L_max < 1 || k < 1 || k > 2048)
        return fail(KVATTN_ERR_SHAPE, "dsa_index_topk: B %d, L_max %d, k %d (k must be 1..2048)", B, L_max, k);
    if (L_max > 131072)
        return fail(KVATTN_ERR_UNSUPPORTED, "dsa_index_topk: L_max %d above 131072", L_max);
    if (static_cast<long long>(B) * L_max > (1ll << 31))
        return fail(KVATTN_ERR_SHAPE, "dsa_index_topk: B * L_max too large");
    if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(w) || !aligned16(topk_idx) ||
        (scores_out && !aligned16(scores_out)))
        return fail(KVATTN_ERR_ALIGN, "dsa_index_topk: tensors must be 16-byte aligned");
    float* scores = nullptr;
    uint32_t* hist = nullptr;
    const int ws_rc = dsa_ws("dsa_index_topk", B, L_max, scores_out, workspace, workspace_bytes, &hist, &scores);
    if (ws_rc != KVATTN_OK) return ws_rc;
    int sms = 0;
    if (num_sms_current(&sms) != 0) return fail(KVATTN_ERR_CUDA, "dsa_index_topk: no CUDA device");
    CUtensorMap tm_k, tm_q;
    if (make_map_3d(&tm_k, k_idx, 128, L_max, B, 128) != KVATTN_OK) return KVATTN_ERR_CUDA;
    if (make_map_3d(&tm_q, q_idx, 128, 64, B, 64) != KVATTN_OK) return KVATTN_ERR_CUDA;
    kvattn::DsaIndexArgs a{w, seq_lens, scores, topk_idx, dev_status, B, L_max, k, sms};
    a.hist = hist;
    return cuda_status(kvattn::launch_dsa_index_topk(a, tm_k, tm_q, static_cast<cudaStream_t>(stream)),
                       "dsa_index_topk launch");
}

int dsa_index_topk_fp8(const kvattn_bf16* q_idx, const float* w, const uint8_t* k_codes, const float* k_scales,
                       const int32_t* seq_lens, int B, int n_idx_head, int idx_dim, int L_max, int k, int32_t* topk_idx,
                       float* scores_out, void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream)
{
    if (!q_idx || !w || !k_codes || !k_scales || !topk_idx)
        return fail(KVATTN_ERR_NULL, "dsa_index_topk_fp8: NULL argument");
    if (n_idx_head != 64 || idx_dim != 128)
        return fail(KVATTN_ERR_UNSUPPORTED, "dsa_index_topk_fp8: needs 64 indexer heads of width 128 (got %d x %d)",
                    n_idx_head, idx_dim);
    if (B < 1 || L_max < 1 || k < 1 || k > 2048)
        return fail(KVATTN_ERR_SHAPE, "dsa_index_topk_fp8: B %d, L_max %d, k %d (k must be 1..2048)", B, L_max, k);
    if (L_max > 131072) return fail(KVATTN_ERR_UNSUPPORTED, "dsa_index_topk_fp8: L_max %d above 131072", L_max);
    if (static_cast<long long>(B) * L_max > (1ll << 31))
        return fail(KVATTN_ERR_SHAPE, "dsa_index_topk_fp8: B * L_max too large");
    if (!aligned16(q_idx) || !aligned16(k_codes) || !aligned16(w) || !aligned16(topk_idx) ||
        (reinterpret_cast<uintptr_t>(k_scales) & 3) || (scores_out && !aligned16(scores_out)))
        return fail(KVATTN_ERR_ALIGN, "dsa_index_topk_fp8: tensors must be 16-byte aligned (scales 4)");
    float* scores = nullptr;
    uint32_t* hist = nullptr;
    uint8_t* q8 = nullptr;
    float* q8_scale = nullptr;
    const int ws_rc = dsa_ws("dsa_index_topk_fp8", B, L_max, scores_out, workspace, workspace_bytes, &hist, &scores,
                             &q8, &q8_scale);
    if (ws_rc != KVATTN_OK) return ws_rc;
    int sms = 0;
    if (num_sms_current(&sms) != 0) return fail(KVATTN_ERR_CUDA, "dsa_index_topk_fp8: no CUDA device");
    CUtensorMap tm_k, tm_q;
    const uint64_t dk[4] = {128, static_cast<uint64_t>(L_max), static_cast<uint64_t>(B), 0};
    const uint64_t dq[4] = {128, 64, static_cast<uint64_t>(B), 0};
    if (make_map(&tm_k, 3, k_codes, dk, 128, true) != KVATTN_OK) return KVATTN_ERR_CUDA;
    if (make_map(&tm_q, 3, q8, dq, 64, true) != KVATTN_OK) return KVATTN_ERR_CUDA;
    kvattn::DsaIndexArgs a{w, seq_lens, scores, topk_idx, dev_status, B, L_max, k, sms};
    a.kscale = k_scales;
    a.q_idx = q_idx;
    a.q8 = q8;
    a.q8_scale = q8_scale;
    a.hist = hist;
    return cuda_status(kvattn::launch_dsa_index_topk(a, tm_k, tm_q, static_cast<cudaStream_t>(stream)),
                       "dsa_index_topk_fp8 launch");
}

int dsa_topk_candidates(const float* scores, const int32_t* topk_idx, int B, int L_slice, int k, int idx_offset,
                        float* cand_scores, int32_t* cand_idx, void* stream)
{
    if (!scores || !topk_idx || !cand_scores || !cand_idx) return fail(KVATTN_ERR_NULL, "dsa_topk_candidates: NULL");
    if (B < 1 || L_slice < 1 || k < 1 || k > 2048 || idx_offset < 0 ||
        static_cast<long long>(idx_offset) + L_slice > (1ll << 31) - 1 || static_cast<long long>(B) * L_slice > (1ll << 31))
        return fail(KVATTN_ERR_SHAPE, "dsa_topk_candidates: B %d, L_slice %d, k %d, offset %d", B, L_slice, k,
                    idx_offset);
    if ((reinterpret_cast<uintptr_t>(scores) | reinterpret_cast<uintptr_t>(topk_idx) |
         reinterpret_cast<uintptr_t>(cand_scores) | reinterpret_cast<uintptr_t>(cand_idx)) & 3)
        return fail(KVATTN_ERR_ALIGN, "dsa_topk_candidates: 4-byte alignment");
    return cuda_status(kvattn::launch_topk_candidates(scores, topk_idx, B, L_slice, k, idx_offset, cand_scores,
                                                      cand_idx, static_cast<cudaStream_t>(stream)),
                       "dsa_topk_candidates launch");
}

int dsa_topk_merge(const float* cand_scores, const int32_t* cand_idx, int n_parts, int B, int k, int32_t* topk_idx,
                   int32_t* dev_status, void* stream)
{
    if (!cand_scores || !cand_idx || !topk_idx) return fail(KVATTN_ERR_NULL, "dsa_topk_merge: NULL");
    if (n_parts < 1 || B < 1 || k < 1 || k > 2048 || B > 65535)
        return fail(KVATTN_ERR_SHAPE, "dsa_topk_merge: n_parts %d, B %d, k %d", n_parts, B, k);
    if (static_cast<long long>(n_parts) * k > kvattn::TOPK_MERGE_MAX)
        return fail(KVATTN_ERR_UNSUPPORTED, "dsa_topk_merge: n_parts * k = %lld above %d",
                    static_cast<long long>(n_parts) * k, kvattn::TOPK_MERGE_MAX);
    if ((reinterpret_cast<uintptr_t>(cand_scores) | reinterpret_cast<uintptr_t>(cand_idx) |
         reinterpret_cast<uintptr_t>(topk_idx)) & 3)
        return fail(KVATTN_ERR_ALIGN, "dsa_topk_merge: 4-byte alignment");
    return cuda_status(kvattn::launch_topk_merge(cand_scores, cand_idx, n_parts, B, k, topk_idx, dev_status,
                                                 static_cast<cudaStream_t>(stream)),
                       "dsa_topk_merge launch");
}

// ---------------------------------------------------------------------------
int qsa_block_keys(const kvattn_bf16* k_idx, const int32_t* seq_lens, const int32_t* block_from, int max_new, int B,
                   int idx_dim, int L_max, const float* cos_tab, const float* sin_tab, int max_pos, int pair_style,
                   float eps, kvattn_bf16* block_keys, int32_t* dev_status, void* stream)
{
    if (!k_idx || !seq_lens || !cos_tab || !sin_tab || !block_keys)
        return fail(KVATTN_ERR_NULL, "qsa_block_keys: NULL argument");
    if (idx_dim != 128) return fail(KVATTN_ERR_UNSUPPORTED, "qsa_block_keys: idx_dim %d (needs 128)", idx_dim);
    if (B < 1 || L_max < kvattn::QSA_BLOCK || L_max % kvattn::QSA_BLOCK)
        return fail(KVATTN_ERR_SHAPE, "qsa_block_keys: B %d, L_max %d (a positive multiple of 4)", B, L_max);
    if (B > 65535) return fail(KVATTN_ERR_SHAPE, "qsa_block_keys: B %d above 65535", B);
    if (max_pos < 1) return fail(KVATTN_ERR_SHAPE, "qsa_block_keys: max_pos < 1");
    if (pair_style != 0 && pair_style != 1) return fail(KVATTN_ERR_UNSUPPORTED, "qsa_block_keys: pair_style");
    if (!(eps >= 0.0f) || !std::isfinite(eps)) return fail(KVATTN_ERR_SHAPE, "qsa_block_keys: eps must be finite >= 0");
    if (!aligned16(k_idx) || !aligned16(block_keys) || !aligned16(cos_tab) || !aligned16(sin_tab))
        return fail(KVATTN_ERR_ALIGN, "qsa_block_keys: tensors must be 16-byte aligned");
    kvattn::QsaKeysArgs a{};
    a.k_idx = k_idx;
    a.seq_lens = seq_lens;
    a.block_from = block_from;
    a.cos_tab = cos_tab;
    a.sin_tab = sin_tab;
    a.block_keys = block_keys;
    a.dev_status = dev_status;
    a.B = B;
    a.L_max = L_max;
    a.max_pos = max_pos;
    a.pair_style = pair_style;
    a.max_new = max_new > 0 ? max_new : L_max / kvattn::QSA_BLOCK;
    a.eps = eps;
    return cuda_status(kvattn::launch_qsa_block_keys(a, static_cast<cudaStream_t>(stream)), "qsa_block_keys launch");
}

size_t qsa_select_workspace_bytes(int B, int L_max, int n_top)
{
    if (B < 1 || L_max < kvattn::QSA_BLOCK || n_top < 1) return 0;
    (void)n_top;
    return dsa_ws_hist(B) + align_up(kvattn::dsa_scores_bytes(B, L_max / kvattn::QSA_BLOCK));
}

int qsa_select(const kvattn_bf16* q_idx, const float* w, const kvattn_bf16* block_keys, const int32_t* seq_lens, int B,
               int n_idx_head, int idx_dim, int L_max, int n_top, int32_t* tok_idx, int32_t* tok_count,
               float* scores_out, void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream)
{
    if (!q_idx || !w || !block_keys || !seq_lens || !tok_idx || !tok_count)
        return fail(KVATTN_ERR_NULL, "qsa_select: NULL argument");
    if (n_idx_head != 64 || idx_dim != 128)
        return fail(KVATTN_ERR_UNSUPPORTED, "qsa_select: needs 64 indexer heads of width 128 (got %d x %d)", n_idx_head,
                    idx_dim);
    if (B < 1 || L_max < kvattn::QSA_BLOCK || L_max % kvattn::QSA_BLOCK || n_top < 1 || n_top > 2048)
        return fail(KVATTN_ERR_SHAPE, "qsa_select: B %d, L_max %d (a positive multiple of 4), n_top %d (1..2048)", B,
                    L_max, n_top);
    const int nb_max = L_max / kvattn::QSA_BLOCK;
    if (nb_max > 131072) return fail(KVATTN_ERR_UNSUPPORTED, "qsa_select: L_max %d above 4 * 131072", L_max);
    if (static_cast<long long>(B) * L_max > (1ll << 31)) return fail(KVATTN_ERR_SHAPE, "qsa_select: B * L_max too large");
    if (!aligned16(q_idx) || !aligned16(block_keys) || !aligned16(w) || !aligned16(tok_idx) ||
        (scores_out && !aligned16(scores_out)))
        return fail(KVATTN_ERR_ALIGN, "qsa_select: tensors must be 16-byte aligned");
    float* scores = nullptr;
    uint32_t* hist = nullptr;
    const int ws_rc = dsa_ws("qsa_select", B, nb_max, scores_out, workspace, workspace_bytes, &hist, &scores);
    if (ws_rc != KVATTN_OK) return ws_rc;
    int sms = 0;
    if (num_sms_current(&sms) != 0) return fail(KVATTN_ERR_CUDA, "qsa_select: no CUDA device");
    CUtensorMap tm_k, tm_q;
    if (make_map_3d(&tm_k, block_keys, 128, nb_max, B, 128) != KVATTN_OK) return KVATTN_ERR_CUDA;
    if (make_map_3d(&tm_q, q_idx, 128, 64, B, 64) != KVATTN_OK) return KVATTN_ERR_CUDA;
    kvattn::DsaIndexArgs a{w, seq_lens, scores, nullptr, dev_status, B, nb_max, n_top, sms};
    static_assert(kvattn::QSA_BLOCK == 4, "len_shift below is log2 of the group size");
    a.len_shift = 2;  // a row of L tokens has L / 4 complete groups
    a.hist = hist;
    a.tok_idx = tok_idx;  // the top-k writes the groups' tokens and the tail directly
    a.tok_count = tok_count;
    a.L_tok = L_max;
    return cuda_status(kvattn::launch_dsa_index_topk(a, tm_k, tm_q, static_cast<cudaStream_t>(stream)),
                       "qsa_select");
}

size_t attn_decode_sparse_workspace_bytes(int B, int Hq, int Dv, int k)
{
    if (B < 1 || Hq < 1 || Dv != 512 || k < 1) return 0;
    return align_up(kvattn::sparse_partial_bytes(B, Hq, k));
}

// Shared by attn_decode_sparse (bf16 latent rows) and attn_decode_sparse_fp8 (packed rows).
static int sparse_call(const char* name, const kvattn_bf16* q, const void* latent, bool fp8, const int32_t* topk_idx,
                       int B, int Hq, int Dk, int Dv, int L_max, int k, float scale, kvattn_bf16* out, float* lse,
                       void* workspace, size_t workspace_bytes, int32_t* dev_status, void* stream)
{
    if (!q || !latent || !topk_idx || !out) return fail(KVATTN_ERR_NULL, "%s: NULL argument", name);
    if (Dk != 576 || Dv != 512)
        return fail(KVATTN_ERR_UNSUPPORTED, "%s: needs Dk 576, Dv 512 (got %d, %d)", name, Dk, Dv);
    if (Hq != 64 && Hq != 128) return fail(KVATTN_ERR_UNSUPPORTED, "%s: Hq must be 64 or 128 (got %d)", name, Hq);
    if (B < 1 || L_max < 1 || k < 1 || k > 2048)
        return fail(KVATTN_ERR_SHAPE, "%s: B %d, L_max %d, k %d (k must be 1..2048)", name, B, L_max, k);
    if (B > 65535) return fail(KVATTN_ERR_SHAPE, "%s: B %d above 65535", name, B);
    if (!(scale > 0.0f) || !std::isfinite(scale)) return fail(KVATTN_ERR_SHAPE, "%s: scale must be finite > 0", name);
    if (!aligned16(q) || !aligned16(latent) || !aligned16(out) || !aligned16(topk_idx) ||
        (lse && (reinterpret_cast<uintptr_t>(lse) & 3)))
        return fail(KVATTN_ERR_ALIGN, "%s: tensors must be 16-byte aligned", name);
    const size_t need = align_up(kvattn::sparse_partial_bytes(B, Hq, k));
    if (need > 0 && (!workspace || workspace_bytes < need))
        return fail(KVATTN_ERR_WORKSPACE, "%s: workspace needs %zu bytes", name, need);
    if (need > 0 && reinterpret_cast<uintptr_t>(workspace) % kWsAlign)
        return fail(KVATTN_ERR_ALIGN, "%s: workspace must be 256-byte aligned", name);
    const int chunks = kvattn::sparse_chunks(k);
    int sms = 0;
    if (num_sms_current(&sms) != 0) return fail(KVATTN_ERR_CUDA, "%s: no CUDA device", name);
    CUtensorMap tm_q, tm_o, tm_pm;
    if (make_map_3d(&tm_q, q, Dk, Hq, B, Hq) != KVATTN_OK) return KVATTN_ERR_CUDA;
    if (chunks == 1) {
        if (make_map_3d(&tm_o, out, Dv, Hq, B, Hq) != KVATTN_OK) return KVATTN_ERR_CUDA;
        tm_pm = tm_o;  // no merge
    } else {
        // the chunk parts: stored by their CTAs ({64 columns, Hq heads} boxes), read back by the
        // in-kernel merge in tiles of 64 columns x 64 heads
        const void* parts = static_cast<const uint8_t*>(workspace) + kvattn::sparse_counter_bytes(B);
        if (make_map_3d(&tm_o, parts, Dv, Hq, static_cast<uint64_t>(B) * chunks, Hq) != KVATTN_OK)
            return KVATTN_ERR_CUDA;
        if (make_map_3d(&tm_pm, parts, Dv, Hq, static_cast<uint64_t>(B) * chunks, 64) != KVATTN_OK)
            return KVATTN_ERR_CUDA;
    }
    kvattn::SparseLaunch l{q, latent, topk_idx, out, lse, need > 0 ? workspace : nullptr, dev_status, B, Hq, L_max,
                           k, scale, fp8, sms};
    return cuda_status(kvattn::launch_sparse_attn(l, tm_q, tm_o, tm_pm, static_cast<cudaStream_t>(stream)), name);
}

int attn_decode_sparse(const kvattn_bf16* q, const kvattn_bf16* latent, const int32_t* topk_idx, int B, int Hq, int Dk,
                       int Dv, int L_max, int k, float scale, kvattn_bf16* out, float* lse, void* workspace,
                       size_t workspace_bytes, int32_t* dev_status, void* stream)
{
    return sparse_call("attn_decode_sparse", q, latent, false, topk_idx, B, Hq, Dk, Dv, L_max, k, scale, out, lse,
                       workspace, workspace_bytes, dev_status, stream);
}

int attn_decode_sparse_fp8(const kvattn_bf16* q, const uint8_t* latent_fp8, const int32_t* topk_idx, int B, int Hq,
                           int Dk, int Dv, int L_max, int k, float scale, kvattn_bf16* out, float* lse, void* workspace,
                           size_t workspace_bytes, int32_t* dev_status, void* stream)
{
    return sparse_call("attn_decode_sparse_fp8", q, latent_fp8, true, topk_idx, B, Hq, Dk, Dv, L_max, k, scale, out,
                       lse, workspace, workspace_bytes, dev_status, stream);
}

// ---------------------------------------------------------------------------
int latent_quant_fp8(const kvattn_bf16* latent, long long n_rows, uint8_t* packed, void* stream)
{
    if ((!latent || !packed) && n_rows > 0) return fail(KVATTN_ERR_NULL, "latent_quant_fp8: NULL argument");
    if (n_rows < 0 || n_rows > (1ll << 34)) return fail(KVATTN_ERR_SHAPE, "latent_quant_fp8: n_rows %lld", n_rows);
    if (!aligned16(latent) || !aligned16(packed))
        return fail(KVATTN_ERR_ALIGN, "latent_quant_fp8: tensors must be 16-byte aligned");
    return cuda_status(kvattn::launch_latent_quant_fp8(latent, n_rows, packed, static_cast<cudaStream_t>(stream)),
                       "latent_quant_fp8 launch");
}

int idx_key_quant_fp8(const kvattn_bf16* k_idx, long long n_rows, uint8_t* codes, float* scales, void* stream)
{
    if ((!k_idx || !codes || !scales) && n_rows > 0) return fail(KVATTN_ERR_NULL, "idx_key_quant_fp8: NULL argument");
    if (n_rows < 0 || n_rows > (1ll << 34)) return fail(KVATTN_ERR_SHAPE, "idx_key_quant_fp8: n_rows %lld", n_rows);
    if (!aligned16(k_idx) || !aligned16(codes) || (reinterpret_cast<uintptr_t>(scales) & 3))
        return fail(KVATTN_ERR_ALIGN, "idx_key_quant_fp8: k_idx and codes 16-byte aligned, scales 4-byte aligned");
    return cuda_status(
        kvattn::launch_idx_key_quant_fp8(k_idx, n_rows, codes, scales, static_cast<cudaStream_t>(stream)),
        "idx_key_quant_fp8 launch");
}

}  // extern "C"
