// decode_noalloc.cu -- attn_decode_gqa for callers that cannot allocate.
//
// Some callers have no way to hand this library device scratch memory: code
// that runs inside another runtime's fixed memory pool (which owns the whole
// device and forbids cudaMalloc behind its back), code on a latency-critical
// path where cudaMalloc would implicitly synchronise the device, and C callers
// linked against this library alone, with no allocator of their own.  For
// them this file keeps the decode scratch in a file-scope device array that
// the CUDA module reserves when it is loaded, so a call needs no workspace
// argument and performs no allocation.
//
// Limits and sharing rules (also stated in include/kvattn.h):
//  - the array holds KVATTN_NOALLOC_SCRATCH_BYTES; a call whose scratch need
//    (attn_decode_gqa_workspace_bytes) is larger is rejected with
//    KVATTN_ERR_WORKSPACE;
//  - every call on a device uses the same array: calls that may run at the
//    same time on the GPU (different streams, or graphs replayed
//    concurrently) race and corrupt each other's results;
//  - the array keeps whatever the previous call left.  Its first
//    KVATTN_DECODE_WS_ZERO_BYTES hold the per-(batch, KV head) piece counters
//    that the split-K merge counts on: they start zero because the array is
//    zero-initialised when the module loads, and every call leaves them zero
//    again -- except a call that reports KVATTN_STATUS_TIMEOUT, after which
//    attn_decode_gqa_noalloc_reset must clear them.  The rest of the array
//    (partial outputs and their max/sum) is written before it is read;
//  - the array's device address is looked up once per device and kept, so
//    the entry points may not be used on a device after cudaDeviceReset;
//  - every GPU that loads this library holds the array until the process
//    exits.
#include <mutex>

#include "kernels.h"

// The decode scratch of every call made through attn_decode_gqa_noalloc.
static __device__ __align__(256) unsigned char g_decode_scratch[KVATTN_NOALLOC_SCRATCH_BYTES];

namespace {

// Device address of g_decode_scratch on the current device, looked up once
// per device (the host-side name is only a stand-in, never a device address).
int scratch_address(void** out)
{
    static std::mutex mu;
    static void* cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    std::lock_guard<std::mutex> lk(mu);
    if (dev < 64 && cache[dev]) {
        *out = cache[dev];
        return 0;
    }
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || p == nullptr) return -1;
    if (dev < 64) cache[dev] = p;
    *out = p;
    return 0;
}

}  // namespace

extern "C" {

int attn_decode_gqa_noalloc(const kvattn_bf16* q, const kvattn_bf16* k_cache, const kvattn_bf16* v_cache,
                            const int32_t* seq_lens, int B, int n_head, int n_kv_head, int head_dim, int T_max,
                            float scale, kvattn_bf16* out, float* lse, int32_t* dev_status, void* stream)
{
    const size_t need = attn_decode_gqa_workspace_bytes(B, n_head, n_kv_head, head_dim, T_max);
    if (need > KVATTN_NOALLOC_SCRATCH_BYTES)
        return kvattn::record_error(KVATTN_ERR_WORKSPACE,
                                    "attn_decode_gqa_noalloc: this shape needs %zu bytes of scratch but the static "
                                    "array holds %u; use attn_decode_gqa with a caller-provided workspace",
                                    need, static_cast<unsigned>(KVATTN_NOALLOC_SCRATCH_BYTES));
    void* scratch = nullptr;
    if (need > 0 && scratch_address(&scratch) != 0)
        return kvattn::record_error(KVATTN_ERR_CUDA,
                                    "attn_decode_gqa_noalloc: cudaGetSymbolAddress of the static scratch failed");
    // need == 0 means the shape is invalid: attn_decode_gqa reports why.
    return attn_decode_gqa(q, k_cache, v_cache, seq_lens, B, n_head, n_kv_head, head_dim, T_max, scale, out, lse,
                           scratch, KVATTN_NOALLOC_SCRATCH_BYTES, dev_status, stream);
}

int attn_decode_gqa_noalloc_reset(void* stream)
{
    void* scratch = nullptr;
    if (scratch_address(&scratch) != 0)
        return kvattn::record_error(KVATTN_ERR_CUDA,
                                    "attn_decode_gqa_noalloc_reset: cudaGetSymbolAddress of the static scratch failed");
    const cudaError_t e =
        cudaMemsetAsync(scratch, 0, KVATTN_DECODE_WS_ZERO_BYTES, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
        return kvattn::record_error(KVATTN_ERR_CUDA, "attn_decode_gqa_noalloc_reset: %s", cudaGetErrorString(e));
    return kvattn::record_error(KVATTN_OK, "%s", "");
}

}  // extern "C"
