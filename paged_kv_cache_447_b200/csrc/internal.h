// internal.h -- launcher interface between the C ABI (api.cu) and the kernel files.
// Arguments reaching these launchers have been validated by api.cu.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

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
};

struct SlotArgs {
    int32_t *slot_mapping;
    const int32_t *block_tables;
    int max_blocks;
    const int32_t *cu_seqlens, *context_lens;
    int num_seqs, num_tokens;
    long long num_blocks;
    int *err;
};

struct CopyArgs {
    void *k_cache, *v_cache;
    const int32_t *pairs;  // [num_pairs][2] (src, dst)
    int num_pairs;
    long long block_bytes;  // one block of one cache
    long long num_blocks;
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

cudaError_t launch_kv_store(const StoreArgs &a, cudaStream_t s);
cudaError_t launch_rope_apply(const RopeArgs &a, cudaStream_t s);
// Returns cudaErrorInvalidValue if the workspace is too small.
cudaError_t launch_paged_decode(const DecodeArgs &a, cudaStream_t s);
size_t decode_workspace_bytes(int num_seqs, int n_q_heads, int n_kv_heads, int head_dim,
                              int num_sms);
cudaError_t launch_paged_prefill(const PrefillArgs &a, cudaStream_t s);
cudaError_t launch_wait_timeout(unsigned long long limit_ns, int *err, cudaStream_t s);
cudaError_t launch_slot_mapping(const SlotArgs &a, cudaStream_t s);
cudaError_t launch_copy_blocks(const CopyArgs &a, cudaStream_t s);

// Number of persistent decode CTAs the library launches on a device with `num_sms` SMs.
int decode_grid_ctas(int num_sms);

}  // namespace pkv
