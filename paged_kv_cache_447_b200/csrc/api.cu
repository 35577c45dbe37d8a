// api.cu -- the extern "C" entry points of libpagedkv.so (declared in include/pkv.h):
// host-side argument checks, TMA descriptor encoding, the per-device error word, and
// dispatch to the kernel launchers.
#include "../../include/pkv.h"
#include "common.cuh"
#include "internal.h"

#include <cudaTypedefs.h>

#include <atomic>
#include <math.h>
#include <mutex>
#include <string.h>

namespace pkv {
namespace {

// Per-device error word.  Kernels receive its device address as an argument; host code
// reaches it only through the address obtained from cudaGetSymbolAddress (the symbol's
// name in host code is a host-side stand-in, not a device address).  The address belongs
// to the context it was looked up in: after cudaDeviceReset the library's module is
// loaded again in a new context and the symbol may move, so the cache is keyed on the
// context's id as well as the device.
__device__ int g_error_word;

constexpr int kMaxDevices = 64;
std::mutex g_mu;
CachedSymbol g_err_cache[kMaxDevices];

int *error_word() {
    void *p = cached_symbol_address(g_err_cache, kMaxDevices, g_mu,
                                    [](void **out) { return cudaGetSymbolAddress(out, g_error_word); });
    return static_cast<int *>(p);
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

bool encoder() {
    static std::once_flag once;
    std::call_once(once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    return g_encode != nullptr;
}

}  // namespace

bool current_context_id(unsigned long long *id) {
    static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
    static PFN_cuCtxGetId_v12000 get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
        fn = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(fn);
    });
    if (!get_current || !get_id) return false;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

namespace {
constexpr int kAttrDevices = 64;
std::atomic<int> g_sm_count[kAttrDevices];
std::atomic<int> g_optin_smem[kAttrDevices];

int device_attr(std::atomic<int> *cache, int dev, cudaDeviceAttr attr, int fallback) {
    if (dev < 0 || dev >= kAttrDevices) return fallback;
    int v = cache[dev].load(std::memory_order_relaxed);
    if (v > 0) return v;
    if (cudaDeviceGetAttribute(&v, attr, dev) != cudaSuccess || v <= 0) return fallback;
    cache[dev].store(v, std::memory_order_relaxed);
    return v;
}
}  // namespace

int device_sm_count(int dev) {
    return device_attr(g_sm_count, dev, cudaDevAttrMultiProcessorCount, 148);
}

int max_optin_smem(int dev) {
    return device_attr(g_optin_smem, dev, cudaDevAttrMaxSharedMemoryPerBlockOptin, 232448);
}

int current_sm_count() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    return device_sm_count(dev);
}

void *cached_symbol_address(CachedSymbol *cache, int n, std::mutex &mu,
                            cudaError_t (*lookup)(void **)) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= n) return nullptr;
    unsigned long long id = 0;
    bool have_id = current_context_id(&id);
    std::lock_guard<std::mutex> lock(mu);
    CachedSymbol &c = cache[dev];
    if (have_id && c.ptr && c.have_ctx && c.ctx_id == id) return c.ptr;
    void *p = nullptr;
    if (lookup(&p) != cudaSuccess || p == nullptr) return nullptr;
    if (!have_id) have_id = current_context_id(&id);  // the lookup created the context
    c.ptr = p;
    c.have_ctx = have_id;
    c.ctx_id = id;
    return p;
}

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int status_of(cudaError_t e) { return e == cudaSuccess ? PKV_OK : PKV_E_CUDA; }

bool block_size_ok(int block_size) { return block_size == 8 || block_size == 16 || block_size == 32; }

int check_cache_shape(int n_kv_heads, int head_dim, int block_size, long long num_blocks,
                      int cache_dtype) {
    if (n_kv_heads <= 0 || num_blocks <= 0) return PKV_E_INVALID;
    if (head_dim != 64 && head_dim != 128 && head_dim != 256) return PKV_E_UNSUPPORTED;
    if (!block_size_ok(block_size)) return PKV_E_UNSUPPORTED;
    if (cache_dtype != PKV_BF16 && cache_dtype != PKV_FP8_E4M3) return PKV_E_UNSUPPORTED;
    if (num_blocks * (long long)block_size >= (1LL << 31)) return PKV_E_UNSUPPORTED;
    return PKV_OK;
}

int check_group(int n_q_heads, int n_kv_heads) {
    if (n_q_heads <= 0 || n_kv_heads <= 0 || n_q_heads % n_kv_heads) return PKV_E_INVALID;
    const int g = n_q_heads / n_kv_heads;
    if (g != 1 && g != 2 && g != 4 && g != 8) return PKV_E_UNSUPPORTED;
    return PKV_OK;
}

__global__ void wait_timeout_kernel(unsigned long long limit_ns, int *err) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        fence_mbar_init();
        // Nothing ever arrives on `bar`: phase 0 never completes, the wait runs out.
        mbar_wait_bounded(smem_u32(&bar), 0, err, limit_ns);
    }
}

}  // namespace

// 3-D tiled map with explicit byte strides for dims 1 and 2 (the dims need not be listed in
// address order) and an L2 promotion of `promo_bytes` (64, 128 or 256).
bool encode_tensor_map_3d_strided(CUtensorMap *map, const void *base, int esize, uint64_t d0,
                                  uint64_t d1, uint64_t d2, uint64_t stride1, uint64_t stride2,
                                  uint32_t b0, uint32_t b1, uint32_t b2, bool swizzle128,
                                  int promo_bytes) {
    // A descriptor is fully determined by these arguments, so a per-thread cache of recent
    // ones saves re-encoding on every call (the caches of an engine's layers stay put).
    struct Key {
        const void *base;
        int esize, promo;
        uint64_t d0, d1, d2, s1, s2;
        uint32_t b0, b1, b2;
        bool swz;
        bool operator==(const Key &o) const {
            return base == o.base && esize == o.esize && promo == o.promo && d0 == o.d0 &&
                   d1 == o.d1 && d2 == o.d2 && s1 == o.s1 && s2 == o.s2 && b0 == o.b0 &&
                   b1 == o.b1 && b2 == o.b2 && swz == o.swz;
        }
    };
    struct Entry {
        Key key;
        CUtensorMap map;
        bool used;
    };
    constexpr int kEntries = 128;
    thread_local Entry cache[kEntries] = {};
    thread_local int next = 0;
    const Key key{base, esize, promo_bytes, d0, d1, d2, stride1, stride2, b0, b1, b2, swizzle128};
    for (int i = 0; i < kEntries; ++i)
        if (cache[i].used && cache[i].key == key) {
            *map = cache[i].map;
            return true;
        }
    if (!encoder()) return false;
    const cuuint64_t dims[3] = {d0, d1, d2};
    const cuuint64_t strides[2] = {stride1, stride2};
    const cuuint32_t box[3] = {b0, b1, b2};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUtensorMapL2promotion promo = promo_bytes >= 256 ? CU_TENSOR_MAP_L2_PROMOTION_L2_256B
                                         : promo_bytes >= 128 ? CU_TENSOR_MAP_L2_PROMOTION_L2_128B
                                                              : CU_TENSOR_MAP_L2_PROMOTION_L2_64B;
    CUresult r = g_encode(map, esize == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8,
                          3, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE,
                          swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                          promo, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
    cache[next] = Entry{key, *map, true};
    next = (next + 1) % kEntries;
    return true;
}

// 4-D tiled map with explicit byte strides for dims 1..3 (in any order), cached like the
// 3-D one.
bool encode_tensor_map_4d_strided(CUtensorMap *map, const void *base, int esize, const uint64_t (&dim)[4],
                                  const uint64_t (&stride)[3], const uint32_t (&boxdim)[4], bool swizzle128,
                                  int promo_bytes) {
    struct Key {
        const void *base;
        int esize, promo;
        uint64_t d[4], s[3];
        uint32_t b[4];
        bool swz;
        bool operator==(const Key &o) const {
            return base == o.base && esize == o.esize && promo == o.promo && swz == o.swz &&
                   memcmp(d, o.d, sizeof d) == 0 && memcmp(s, o.s, sizeof s) == 0 &&
                   memcmp(b, o.b, sizeof b) == 0;
        }
    };
    struct Entry {
        Key key;
        CUtensorMap map;
        bool used;
    };
    constexpr int kEntries = 64;
    thread_local Entry cache[kEntries] = {};
    thread_local int next = 0;
    Key key{base, esize, promo_bytes, {dim[0], dim[1], dim[2], dim[3]}, {stride[0], stride[1], stride[2]},
            {boxdim[0], boxdim[1], boxdim[2], boxdim[3]}, swizzle128};
    for (int i = 0; i < kEntries; ++i)
        if (cache[i].used && cache[i].key == key) {
            *map = cache[i].map;
            return true;
        }
    if (!encoder()) return false;
    const cuuint64_t dims[4] = {dim[0], dim[1], dim[2], dim[3]};
    const cuuint64_t strides[3] = {stride[0], stride[1], stride[2]};
    const cuuint32_t box[4] = {boxdim[0], boxdim[1], boxdim[2], boxdim[3]};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUtensorMapL2promotion promo = promo_bytes >= 256 ? CU_TENSOR_MAP_L2_PROMOTION_L2_256B
                                         : promo_bytes >= 128 ? CU_TENSOR_MAP_L2_PROMOTION_L2_128B
                                                              : CU_TENSOR_MAP_L2_PROMOTION_L2_64B;
    CUresult r = g_encode(map, esize == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8,
                          4, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE, promo,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
    cache[next] = Entry{key, *map, true};
    next = (next + 1) % kEntries;
    return true;
}

// 3-D tiled map over a row-major [d2, d1, d0] tensor of `esize`-byte elements.  L2 fetches
// are promoted to one contiguous row at most: a wider promotion would drag in the next
// head's row of the same slot, which the paged layout does not read next.
bool encode_tensor_map_3d(CUtensorMap *map, const void *base, int esize, uint64_t d0, uint64_t d1,
               uint64_t d2, uint32_t b0, uint32_t b1, uint32_t b2, bool swizzle128) {
    const uint64_t row = d0 * esize;
    return encode_tensor_map_3d_strided(map, base, esize, d0, d1, d2, row, row * d1, b0, b1, b2,
                                        swizzle128, (int)(row >= 256 ? 256 : row));
}

cudaError_t launch_wait_timeout(unsigned long long limit_ns, int *err, cudaStream_t s) {
    wait_timeout_kernel<<<1, 32, 0, s>>>(limit_ns, err);
    return cudaGetLastError();
}

}  // namespace pkv

using namespace pkv;

extern "C" {

int pkv_version(void) { return (1 << 16) | 0; }

const char *pkv_strerror(int code) {
    switch (code) {
        case PKV_OK: return "ok";
        case PKV_E_INVALID: return "invalid argument";
        case PKV_E_UNSUPPORTED: return "unsupported shape or dtype";
        case PKV_E_WORKSPACE: return "workspace missing or too small";
        case PKV_E_CUDA: return "CUDA runtime error";
        case PKV_E_TIMEOUT: return "a bounded wait inside a kernel ran out";
        case PKV_E_BOUNDS: return "slot, block id or position out of range";
        case PKV_E_ALIGN: return "pointer not 16-byte aligned";
        case PKV_E_SCRATCH_LIMIT: return "call needs more than the built-in decode scratch array";
        case PKV_E_POOL: return "block pool cannot cover the allocation";
        default: return "unknown status";
    }
}

int pkv_rope_build_table(float *out, int max_pos, int head_dim, double base) {
    if (!out || max_pos < 1 || head_dim <= 0 || (head_dim & 1) || !(base > 0.0))
        return PKV_E_INVALID;
    const int half = head_dim / 2;
    for (int p = 0; p < max_pos; ++p) {
        float *row = out + (size_t)p * head_dim;
        for (int i = 0; i < half; ++i) {
            // theta_i = base^(-2i/D); angle = p * theta_i; both in fp64, one rounding to fp32
            const double theta = pow(base, -(2.0 * (double)i) / (double)head_dim);
            const double angle = (double)p * theta;
            row[i] = (float)cos(angle);
            row[half + i] = (float)sin(angle);
        }
    }
    return PKV_OK;
}

size_t pkv_cache_bytes(int num_layers, long long num_blocks, int block_size, int n_kv_heads,
                       int head_dim, int cache_dtype) {
    if (num_layers < 0 || num_blocks < 0 || block_size <= 0 || n_kv_heads <= 0 || head_dim <= 0)
        return 0;
    if (cache_dtype != PKV_BF16 && cache_dtype != PKV_FP8_E4M3) return 0;
    const size_t elem = cache_dtype == PKV_BF16 ? 2 : 1;
    return (size_t)2 * num_layers * (size_t)num_blocks * block_size * n_kv_heads * head_dim * elem;
}

int pkv_kv_store(const void *k, const void *v, void *k_cache, void *v_cache,
                 const int32_t *slot_mapping, int num_tokens, int n_kv_heads, int head_dim,
                 int block_size, long long num_blocks, int cache_dtype, const float *k_scale,
                 const float *v_scale, const float *rope_cos_sin, int max_pos,
                 const int32_t *cu_seqlens, const int32_t *context_lens, int num_seqs,
                 pkv_stream_t stream) {
    int st = check_cache_shape(n_kv_heads, head_dim, block_size, num_blocks, cache_dtype);
    if (st) return st;
    if (num_tokens < 0) return PKV_E_INVALID;
    if (num_tokens == 0) return PKV_OK;
    if (!k || !v || !k_cache || !v_cache || !slot_mapping) return PKV_E_INVALID;
    if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache))
        return PKV_E_ALIGN;
    const bool fp8 = cache_dtype == PKV_FP8_E4M3;
    if (fp8 && (!k_scale || !v_scale)) return PKV_E_INVALID;
    if (rope_cos_sin && (!cu_seqlens || !context_lens || num_seqs <= 0 || max_pos < 1))
        return PKV_E_INVALID;
    int *err = error_word();
    if (!err) return PKV_E_CUDA;
    StoreArgs a{k, v, k_cache, v_cache, slot_mapping, num_tokens, n_kv_heads, head_dim,
                num_blocks * block_size, fp8, k_scale, v_scale, rope_cos_sin, max_pos,
                cu_seqlens, context_lens, num_seqs, err};
    return status_of(launch_kv_store(a, reinterpret_cast<cudaStream_t>(stream)));
}

int pkv_slot_mapping(int32_t *slot_mapping, const int32_t *block_tables, int max_blocks_per_seq,
                     const int32_t *cu_seqlens, const int32_t *context_lens, int num_seqs,
                     int num_tokens, int block_size, long long num_blocks, pkv_stream_t stream) {
    if (!block_size_ok(block_size)) return PKV_E_UNSUPPORTED;
    if (num_tokens < 0 || num_seqs < 0 || max_blocks_per_seq < 0 || num_blocks < 0)
        return PKV_E_INVALID;
    if (num_blocks * (long long)block_size >= (1LL << 31)) return PKV_E_UNSUPPORTED;
    if (num_tokens == 0) return PKV_OK;
    if (!slot_mapping || !block_tables || !cu_seqlens || !context_lens || num_seqs == 0 ||
        max_blocks_per_seq == 0)
        return PKV_E_INVALID;
    int *err = error_word();
    if (!err) return PKV_E_CUDA;
    SlotArgs a{slot_mapping, block_tables, max_blocks_per_seq, cu_seqlens, context_lens,
               num_seqs, num_tokens, num_blocks, err, block_size};
    return status_of(launch_slot_mapping(a, reinterpret_cast<cudaStream_t>(stream)));
}

int pkv_copy_blocks(void *k_cache, void *v_cache, const int32_t *block_pairs, int num_pairs,
                    int n_kv_heads, int head_dim, int block_size, long long num_blocks,
                    int cache_dtype, pkv_stream_t stream) {
    int st = check_cache_shape(n_kv_heads, head_dim, block_size, num_blocks, cache_dtype);
    if (st) return st;
    if (num_pairs < 0) return PKV_E_INVALID;
    if (num_pairs == 0) return PKV_OK;
    if (!k_cache || !v_cache || !block_pairs) return PKV_E_INVALID;
    if (!aligned16(k_cache) || !aligned16(v_cache)) return PKV_E_ALIGN;
    int *err = error_word();
    if (!err) return PKV_E_CUDA;
    const long long esize = cache_dtype == PKV_FP8_E4M3 ? 1 : 2;
    CopyArgs a{k_cache, v_cache, block_pairs, num_pairs,
               (long long)block_size * n_kv_heads * head_dim * esize, num_blocks, err};
    return status_of(launch_copy_blocks(a, reinterpret_cast<cudaStream_t>(stream)));
}

size_t pkv_block_pool_bytes(long long num_blocks) {
    if (num_blocks <= 0 || num_blocks >= (1LL << 31) / 32) return 0;
    return block_pool_bytes(num_blocks);
}

int pkv_block_pool_init(void *pool, long long num_blocks, pkv_stream_t stream) {
    if (!pool || num_blocks <= 0) return PKV_E_INVALID;
    if (num_blocks >= (1LL << 31) / 32) return PKV_E_UNSUPPORTED;
    if (!aligned16(pool)) return PKV_E_ALIGN;
    return status_of(launch_pool_init(static_cast<int32_t *>(pool), num_blocks,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

int pkv_block_pool_alloc(void *pool, long long num_blocks, int32_t *block_tables,
                         int max_blocks_per_seq, const int32_t *cu_seqlens,
                         const int32_t *context_lens, int num_seqs, int block_size,
                         pkv_stream_t stream) {
    if (!block_size_ok(block_size)) return PKV_E_UNSUPPORTED;
    if (num_blocks <= 0 || num_seqs < 0 || max_blocks_per_seq < 1) return PKV_E_INVALID;
    if (num_blocks >= (1LL << 31) / 32) return PKV_E_UNSUPPORTED;
    if (num_seqs == 0) return PKV_OK;
    if (!pool || !block_tables || !cu_seqlens || !context_lens) return PKV_E_INVALID;
    if (!aligned16(pool)) return PKV_E_ALIGN;
    int *err = error_word();
    if (!err) return PKV_E_CUDA;
    PoolArgs a{static_cast<int32_t *>(pool), num_blocks, block_tables, max_blocks_per_seq,
               cu_seqlens, context_lens, num_seqs, err, block_size};
    return status_of(launch_pool_alloc(a, reinterpret_cast<cudaStream_t>(stream)));
}

int pkv_block_pool_free(void *pool, long long num_blocks, const int32_t *block_ids, int num_ids,
                        pkv_stream_t stream) {
    if (num_blocks <= 0 || num_ids < 0) return PKV_E_INVALID;
    if (num_blocks >= (1LL << 31) / 32) return PKV_E_UNSUPPORTED;
    if (num_ids == 0) return PKV_OK;
    if (!pool || !block_ids) return PKV_E_INVALID;
    if (!aligned16(pool)) return PKV_E_ALIGN;
    int *err = error_word();
    if (!err) return PKV_E_CUDA;
    PoolFreeArgs a{static_cast<int32_t *>(pool), num_blocks, block_ids, num_ids, err};
    return status_of(launch_pool_free(a, reinterpret_cast<cudaStream_t>(stream)));
}

int pkv_rope_apply(void *q, void *k, const float *rope_cos_sin, int max_pos,
                   const int32_t *cu_seqlens, const int32_t *context_lens, int num_seqs,
                   int num_tokens, int n_q_heads, int n_kv_heads, int head_dim,
                   pkv_stream_t stream) {
    if (num_tokens < 0 || n_q_heads < 0 || n_kv_heads < 0) return PKV_E_INVALID;
    if (head_dim != 64 && head_dim != 128 && head_dim != 256) return PKV_E_UNSUPPORTED;
    if (num_tokens == 0 || (!q && !k)) return PKV_OK;
    if (!rope_cos_sin || !cu_seqlens || !context_lens || num_seqs <= 0 || max_pos < 1)
        return PKV_E_INVALID;
    if ((q && !aligned16(q)) || (k && !aligned16(k))) return PKV_E_ALIGN;
    int *err = error_word();
    if (!err) return PKV_E_CUDA;
    RopeArgs a{q, k, rope_cos_sin, max_pos, cu_seqlens, context_lens, num_seqs, num_tokens,
               q ? n_q_heads : 0, k ? n_kv_heads : 0, head_dim, err};
    if (!q) a.n_q_heads = 0;
    return status_of(launch_rope_apply(a, reinterpret_cast<cudaStream_t>(stream)));
}

size_t pkv_decode_workspace_bytes(int num_seqs, int n_q_heads, int n_kv_heads, int head_dim) {
    if (num_seqs < 0 || check_group(n_q_heads, n_kv_heads) || head_dim <= 0) return 0;
    // (no device visible: sized for a B200's 148 SMs)
    return decode_workspace_bytes(num_seqs, n_q_heads, n_kv_heads, head_dim, current_sm_count());
}

int pkv_paged_decode_attention(void *out, const void *q, const void *k_cache,
                               const void *v_cache, const int32_t *block_tables,
                               int max_blocks_per_seq, const int32_t *context_lens,
                               int num_seqs, int n_q_heads, int n_kv_heads, int head_dim,
                               int block_size, long long num_blocks, float scale,
                               int cache_dtype, const float *k_scale, const float *v_scale,
                               const float *rope_cos_sin, int max_pos, void *workspace,
                               size_t workspace_bytes, pkv_stream_t stream) {
    int st = check_cache_shape(n_kv_heads, head_dim, block_size, num_blocks, cache_dtype);
    if (st) return st;
    if ((st = check_group(n_q_heads, n_kv_heads))) return st;
    if (num_seqs < 0 || max_blocks_per_seq < 1) return PKV_E_INVALID;
    if (num_seqs == 0) return PKV_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens) return PKV_E_INVALID;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
        return PKV_E_ALIGN;
    const bool fp8 = cache_dtype == PKV_FP8_E4M3;
    if (fp8 && (!k_scale || !v_scale)) return PKV_E_INVALID;
    if (rope_cos_sin && max_pos < 1) return PKV_E_INVALID;
    if (!workspace || !aligned16(workspace) ||
        workspace_bytes < pkv_decode_workspace_bytes(num_seqs, n_q_heads, n_kv_heads, head_dim))
        return PKV_E_WORKSPACE;
    int *err = error_word();
    if (!err) return PKV_E_CUDA;
    DecodeArgs a{out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                 num_seqs, n_q_heads, n_kv_heads, head_dim, num_blocks, scale, fp8, k_scale,
                 v_scale, rope_cos_sin, max_pos, workspace, workspace_bytes, err};
    a.block_size = block_size;
    cudaError_t e = launch_paged_decode(a, reinterpret_cast<cudaStream_t>(stream));
    if (e == cudaErrorNotSupported) return PKV_E_UNSUPPORTED;  // batch too large for one launch
    return status_of(e);
}

size_t pkv_decode_step_workspace_bytes(int num_seqs, int n_q_heads, int n_kv_heads,
                                       int head_dim) {
    if (num_seqs < 0 || check_group(n_q_heads, n_kv_heads) || head_dim <= 0) return 0;
    return decode_step_workspace_bytes(num_seqs, n_q_heads, n_kv_heads, head_dim, current_sm_count());
}

int pkv_paged_decode_step(void *out, const void *q, const void *k, const void *v, void *k_cache,
                          void *v_cache, const int32_t *block_tables, int max_blocks_per_seq,
                          const int32_t *context_lens, int num_seqs, int n_q_heads,
                          int n_kv_heads, int head_dim, int block_size, long long num_blocks,
                          float scale, int cache_dtype, const float *k_scale,
                          const float *v_scale, const float *rope_cos_sin, int max_pos,
                          void *workspace, size_t workspace_bytes, pkv_stream_t stream) {
    int st = check_cache_shape(n_kv_heads, head_dim, block_size, num_blocks, cache_dtype);
    if (st) return st;
    if ((st = check_group(n_q_heads, n_kv_heads))) return st;
    if (num_seqs < 0 || max_blocks_per_seq < 1) return PKV_E_INVALID;
    if (num_seqs == 0) return PKV_OK;
    if (!out || !q || !k || !v || !k_cache || !v_cache || !block_tables || !context_lens)
        return PKV_E_INVALID;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(k_cache) ||
        !aligned16(v_cache))
        return PKV_E_ALIGN;
    const bool fp8 = cache_dtype == PKV_FP8_E4M3;
    if (fp8 && (!k_scale || !v_scale)) return PKV_E_INVALID;
    if (rope_cos_sin && max_pos < 1) return PKV_E_INVALID;
    if (!workspace || !aligned16(workspace) ||
        workspace_bytes < pkv_decode_step_workspace_bytes(num_seqs, n_q_heads, n_kv_heads, head_dim))
        return PKV_E_WORKSPACE;
    int *err = error_word();
    if (!err) return PKV_E_CUDA;
    DecodeArgs a{out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                 num_seqs, n_q_heads, n_kv_heads, head_dim, num_blocks, scale, fp8, k_scale,
                 v_scale, rope_cos_sin, max_pos, workspace, workspace_bytes, err};
    a.block_size = block_size;
    a.k_new = k;
    a.v_new = v;
    a.k_cache_w = k_cache;
    a.v_cache_w = v_cache;
    cudaError_t e = launch_paged_decode_step(a, reinterpret_cast<cudaStream_t>(stream));
    if (e == cudaErrorNotSupported) return PKV_E_UNSUPPORTED;
    return status_of(e);
}

int pkv_set_decode_step_mode(int mode) {
    if (mode != PKV_STEP_AUTO && mode != PKV_STEP_FUSED && mode != PKV_STEP_SPLIT) return PKV_E_INVALID;
    return set_decode_step_mode(mode);
}

int pkv_paged_prefill_attention(void *out, const void *q, const void *k_cache,
                                const void *v_cache, const int32_t *cu_seqlens,
                                const int32_t *block_tables, int max_blocks_per_seq,
                                const int32_t *context_lens, int num_seqs, int num_tokens,
                                int n_q_heads, int n_kv_heads, int head_dim, int block_size,
                                long long num_blocks, float scale, int cache_dtype,
                                const float *k_scale, const float *v_scale,
                                const float *rope_cos_sin, int max_pos, int max_new_tokens,
                                pkv_stream_t stream) {
    int st = check_cache_shape(n_kv_heads, head_dim, block_size, num_blocks, cache_dtype);
    if (st) return st;
    if (head_dim == 256) return PKV_E_UNSUPPORTED;  // (the prefill tiles are built for 64 / 128)
    if ((st = check_group(n_q_heads, n_kv_heads))) return st;
    if (num_seqs < 0 || num_tokens < 0 || max_blocks_per_seq < 1 || max_new_tokens < 0)
        return PKV_E_INVALID;
    if (num_seqs == 0 || num_tokens == 0) return PKV_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !cu_seqlens)
        return PKV_E_INVALID;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
        return PKV_E_ALIGN;
    const bool fp8 = cache_dtype == PKV_FP8_E4M3;
    if (fp8 && (!k_scale || !v_scale)) return PKV_E_INVALID;
    if (rope_cos_sin && max_pos < 1) return PKV_E_INVALID;
    int *err = error_word();
    if (!err) return PKV_E_CUDA;
    PrefillArgs a{out, q, k_cache, v_cache, cu_seqlens, block_tables, max_blocks_per_seq,
                  context_lens, num_seqs, num_tokens, n_q_heads, n_kv_heads, head_dim, num_blocks,
                  scale, fp8, k_scale, v_scale, rope_cos_sin, max_pos, max_new_tokens, err};
    a.block_size = block_size;
    cudaError_t e = launch_paged_prefill(a, reinterpret_cast<cudaStream_t>(stream));
    if (e == cudaErrorNotSupported) return PKV_E_UNSUPPORTED;
    return status_of(e);
}

int pkv_get_error(pkv_stream_t stream) {
    int *err = error_word();
    if (!err) return PKV_E_CUDA;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int host = 0;
    if (cudaStreamSynchronize(s) != cudaSuccess) return PKV_E_CUDA;
    if (cudaMemcpyAsync(&host, err, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return PKV_E_CUDA;
    if (cudaMemsetAsync(err, 0, sizeof(int), s) != cudaSuccess) return PKV_E_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return PKV_E_CUDA;
    if (host & kErrTimeout) return PKV_E_TIMEOUT;
    if (host & kErrBounds) return PKV_E_BOUNDS;
    if (host & kErrPool) return PKV_E_POOL;
    return PKV_OK;
}

int pkv_debug_wait_timeout(long long timeout_ns, pkv_stream_t stream) {
    if (timeout_ns < 1000) timeout_ns = 1000;
    if (timeout_ns > 2000000000LL) timeout_ns = 2000000000LL;
    int *err = error_word();
    if (!err) return PKV_E_CUDA;
    return status_of(launch_wait_timeout((unsigned long long)timeout_ns, err,
                                         reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
