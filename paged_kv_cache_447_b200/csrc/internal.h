// internal.h -- launcher interface between the C ABI (api.cu) and the kernel files.
// Arguments reaching these launchers have been validated by api.cu.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

namespace pkv {

struct StoreArgs {
    const void *k, *v;
    void *k_cache, *v_cache;
    const int32_t *slot_mapping;
    int num_tokens, n_kv_heads, head_dim;
    long long num_slots;  // num_blocks * block_size
    bool fp8;
    const float *k_scale, *v_scale;
    const float *rope;  // NULL = no K rotation
    int max_pos;
    const int32_t *cu_seqlens, *context_lens;
    int num_seqs;
    int *err;
    // decode step (slot_mapping NULL): token t is sequence t's new token, at position
    // context_lens[t] - 1, its slot read from the block table
    const int32_t *block_tables = nullptr;
    int max_blocks = 0, block_size = 16;
};

struct RopeArgs {
    void *q, *k;
    const float *rope;
    int max_pos;
    const int32_t *cu_seqlens, *context_lens;
    int num_seqs, num_tokens, n_q_heads, n_kv_heads, head_dim;
    int *err;
};

struct DecodeArgs {
    void *out;
    const void *q;
    const void *k_cache, *v_cache;
    const int32_t *block_tables;
    int max_blocks_per_seq;
    const int32_t *context_lens;
    int num_seqs, n_q_heads, n_kv_heads, head_dim;
    long long num_blocks;
    float scale;
    bool fp8;
    const float *k_scale, *v_scale;
    const float *rope;
    int max_pos;
    void *workspace;
    size_t workspace_bytes;
    int *err;
    // pkv_paged_decode_step only: the step's new K and V ([num_seqs, n_kv_heads, head_dim]
    // bf16) and the same caches, writable
    const void *k_new = nullptr, *v_new = nullptr;
    void *k_cache_w = nullptr, *v_cache_w = nullptr;
    int block_size = 16;
};

struct PrefillArgs {
    void *out;
    const void *q;
    const void *k_cache, *v_cache;
    const int32_t *cu_seqlens;
    const int32_t *block_tables;
    int max_blocks_per_seq;
    const int32_t *context_lens;
    int num_seqs, num_tokens, n_q_heads, n_kv_heads, head_dim;
    long long num_blocks;
    float scale;
    bool fp8;
    const float *k_scale, *v_scale;
    const float *rope;
    int max_pos, max_new_tokens;
    int *err;
    int block_size = 16;
};

struct SlotArgs {
    int32_t *slot_mapping;
    const int32_t *block_tables;
    int max_blocks;
    const int32_t *cu_seqlens, *context_lens;
    int num_seqs, num_tokens;
    long long num_blocks;
    int *err;
    int block_size;
};

struct CopyArgs {
    void *k_cache, *v_cache;
    const int32_t *pairs;  // [num_pairs][2] (src, dst)
    int num_pairs;
    long long block_bytes;  // one block of one cache
    long long num_blocks;
    int *err;
};

struct PoolArgs {
    int32_t *pool;  // [4 + 2 * num_blocks]: free count, (3 unused), stack, free flags
    long long num_blocks;
    int32_t *block_tables;
    int max_blocks;
    const int32_t *cu_seqlens, *context_lens;
    int num_seqs;
    int *err;
    int block_size;
};

struct PoolFreeArgs {
    int32_t *pool;
    long long num_blocks;
    const int32_t *ids;
    int num_ids;
    int *err;
};

// 3-D tiled TMA descriptor over a row-major [d2][d1][d0] tensor of `esize`-byte elements
// (bf16 or bytes), box b0 x b1 x b2, optionally 128-byte swizzled.  Each launcher encodes
// the maps its kernel reads, from the same compile-time geometry the kernel uses.
bool encode_tensor_map_3d(CUtensorMap *map, const void *base, int esize, uint64_t d0, uint64_t d1,
                          uint64_t d2, uint32_t b0, uint32_t b1, uint32_t b2, bool swizzle128);
// The same with explicit byte strides of dims 1 and 2 (dims in any order) and L2 promotion.
bool encode_tensor_map_3d_strided(CUtensorMap *map, const void *base, int esize, uint64_t d0,
                                  uint64_t d1, uint64_t d2, uint64_t stride1, uint64_t stride2,
                                  uint32_t b0, uint32_t b1, uint32_t b2, bool swizzle128,
                                  int promo_bytes);

// 4-D tiled map with explicit byte strides of dims 1..3 (dims in any order) and L2 promotion.
bool encode_tensor_map_4d_strided(CUtensorMap *map, const void *base, int esize, const uint64_t (&dim)[4],
                                  const uint64_t (&stride)[3], const uint32_t (&boxdim)[4], bool swizzle128,
                                  int promo_bytes);

cudaError_t launch_kv_store(const StoreArgs &a, cudaStream_t s);
cudaError_t launch_rope_apply(const RopeArgs &a, cudaStream_t s);
// Returns cudaErrorInvalidValue if the workspace is too small.
cudaError_t launch_paged_decode(const DecodeArgs &a, cudaStream_t s);
size_t decode_workspace_bytes(int num_seqs, int n_q_heads, int n_kv_heads, int head_dim,
                              int num_sms);
// The decode step: store each sequence's new token, attend, merge split partials in-kernel.
// Its workspace is decode_workspace_bytes(...) followed by num_seqs * n_kv_heads int
// counters that must be zero before the first call (every call leaves them zero).
cudaError_t launch_paged_decode_step(const DecodeArgs &a, cudaStream_t s);
int set_decode_step_mode(int mode);  // returns the previous mode (PKV_STEP_*)
// Grouped heads over an E4M3 cache at head dim 128 run on the tcgen05 decode kernel.
bool decode_tc_supported(const DecodeArgs &a);
cudaError_t launch_paged_decode_tc(const DecodeArgs &a, cudaStream_t s);
cudaError_t launch_paged_decode_step_tc(const DecodeArgs &a, cudaStream_t s);
size_t decode_step_workspace_bytes(int num_seqs, int n_q_heads, int n_kv_heads, int head_dim,
                                   int num_sms);
cudaError_t launch_paged_prefill(const PrefillArgs &a, cudaStream_t s);
cudaError_t launch_wait_timeout(unsigned long long limit_ns, int *err, cudaStream_t s);
cudaError_t launch_slot_mapping(const SlotArgs &a, cudaStream_t s);
cudaError_t launch_copy_blocks(const CopyArgs &a, cudaStream_t s);
size_t block_pool_bytes(long long num_blocks);
cudaError_t launch_pool_init(int32_t *pool, long long num_blocks, cudaStream_t s);
cudaError_t launch_pool_alloc(const PoolArgs &a, cudaStream_t s);
cudaError_t launch_pool_free(const PoolFreeArgs &a, cudaStream_t s);

// Id of the CUDA context current on this thread (unique for the life of the process,
// unlike a context handle or a device ordinal); false if there is none or the driver
// cannot say.
bool current_context_id(unsigned long long *id);

// Device address of a file-scope __device__ symbol in the current context, looked up with
// `lookup` (a cudaGetSymbolAddress call) the first time on each device and again whenever
// the current context differs from the one the cached address came from.
struct CachedSymbol {
    void *ptr = nullptr;
    bool have_ctx = false;
    unsigned long long ctx_id = 0;
};
void *cached_symbol_address(CachedSymbol *cache, int n, std::mutex &mu,
                            cudaError_t (*lookup)(void **));

// SM count and opt-in maximum of dynamic shared memory per block of device `dev`, read
// once per device (148 and 232448 on a B200 if the query fails).
int device_sm_count(int dev);
int max_optin_smem(int dev);
// The same for the current device.
int current_sm_count();

// Number of persistent decode CTAs the library launches on a device with `num_sms` SMs.
int decode_grid_ctas(int num_sms);

}  // namespace pkv
