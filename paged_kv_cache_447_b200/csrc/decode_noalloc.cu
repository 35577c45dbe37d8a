// decode_noalloc.cu -- paged decode attention for callers that cannot allocate device
// memory.
//
// Who needs this: an inference engine usually hands almost all of a GPU's memory to its
// paged KV pool at start-up, so a cudaMalloc issued later from inside the decode step can
// fail, and on a latency-critical step a cudaMalloc/cudaFree pair may also synchronise the
// device.  Plugins hosted by a framework that owns every allocation are in the same
// position.  pkv_paged_decode_attention_noalloc lets such callers run decode attention
// without providing the split-context workspace: the workspace lives in a fixed-size
// array that is part of this library's device image.
//
// The array is file-scope device memory.  Its name in host code is only a host-side
// stand-in for the symbol, not a device address, so host code never passes it to a
// kernel; instead the set-up below asks the runtime for the device address with
// cudaGetSymbolAddress (with the device current) and hands that pointer on.  The set-up
// runs on the first call on each device, and again if that device's context has been
// replaced (after cudaDeviceReset the library's module is loaded again and the array may
// sit at another address).
#include "../../include/pkv.h"
#include "internal.h"

#include <cuda_runtime.h>
#include <mutex>

namespace {

constexpr size_t kScratchBytes = PKV_NOALLOC_SCRATCH_BYTES;

// Held by every GPU that loads this library, until the process exits.
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
pkv::CachedSymbol g_scratch_cache[kMaxDevices];

// Device address of the scratch array in the current device's context.
int scratch_for_current_device(void **out) {
    void *p = pkv::cached_symbol_address(
        g_scratch_cache, kMaxDevices, g_scratch_mu,
        [](void **o) { return cudaGetSymbolAddress(o, g_decode_scratch); });
    if (!p) return PKV_E_CUDA;
    *out = p;
    return PKV_OK;
}

}  // namespace

extern "C" int pkv_paged_decode_attention_noalloc(
    void *out, const void *q, const void *k_cache, const void *v_cache,
    const int32_t *block_tables, int max_blocks_per_seq, const int32_t *context_lens,
    int num_seqs, int n_q_heads, int n_kv_heads, int head_dim, int block_size,
    long long num_blocks, float scale, int cache_dtype, const float *k_scale,
    const float *v_scale, const float *rope_cos_sin, int max_pos, pkv_stream_t stream) {
    const size_t need = pkv_decode_workspace_bytes(num_seqs, n_q_heads, n_kv_heads, head_dim);
    if (need > kScratchBytes) return PKV_E_SCRATCH_LIMIT;
    void *scratch = nullptr;
    const int st = scratch_for_current_device(&scratch);
    if (st != PKV_OK) return st;
    // The workspace needs no initial contents (every value is written before it is read),
    // so nothing is cleared between calls.
    return pkv_paged_decode_attention(out, q, k_cache, v_cache, block_tables,
                                      max_blocks_per_seq, context_lens, num_seqs, n_q_heads,
                                      n_kv_heads, head_dim, block_size, num_blocks, scale,
                                      cache_dtype, k_scale, v_scale, rope_cos_sin, max_pos,
                                      scratch, kScratchBytes, stream);
}
