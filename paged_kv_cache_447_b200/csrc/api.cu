// api.cu -- the extern "C" entry points of libpagedkv.so (declared in include/pkv.h):
// host-side argument checks, TMA descriptor encoding, the per-device error word, and
// dispatch to the kernel launchers.
#include "../../include/pkv.h"
#include "common.cuh"
#include "internal.h"

#include <cudaTypedefs.h>

#include <math.h>
#include <mutex>
#include <string.h>

namespace pkv {
namespace {

// Per-device error word.  Kernels receive its device address as an argument; host code
// reaches it only through the address obtained from cudaGetSymbolAddress (the symbol's
// name in host code is a host-side stand-in, not a device address).
__device__ int g_error_word;

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int *g_err_ptr[kMaxDevices] = {};

int *error_word() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_err_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return nullptr;
        g_err_ptr[dev] = static_cast<int *>(p);
    }
    return g_err_ptr[dev];
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

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int status_of(cudaError_t e) { return e == cudaSuccess ? PKV_OK : PKV_E_CUDA; }

int check_cache_shape(int n_kv_heads, int head_dim, int block_size, long long num_blocks,
                      int cache_dtype) {
    if (n_kv_heads <= 0 || num_blocks <= 0) return PKV_E_INVALID;
    if (head_dim != 64 && head_dim != 128) return PKV_E_UNSUPPORTED;
    if (block_size != kBlockSize) return PKV_E_UNSUPPORTED;
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
    return r == CUDA_SUCCESS;
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
    if (block_size != kBlockSize) return PKV_E_UNSUPPORTED;
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
               num_seqs, num_tokens, num_blocks, err};
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

int pkv_rope_apply(void *q, void *k, const float *rope_cos_sin, int max_pos,
                   const int32_t *cu_seqlens, const int32_t *context_lens, int num_seqs,
                   int num_tokens, int n_q_heads, int n_kv_heads, int head_dim,
                   pkv_stream_t stream) {
    if (num_tokens < 0 || n_q_heads < 0 || n_kv_heads < 0) return PKV_E_INVALID;
    if (head_dim != 64 && head_dim != 128) return PKV_E_UNSUPPORTED;
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
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        sms = 148;  // no device visible: size for a B200
    return decode_workspace_bytes(num_seqs, n_q_heads, n_kv_heads, head_dim, sms);
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
    cudaError_t e = launch_paged_decode(a, reinterpret_cast<cudaStream_t>(stream));
    if (e == cudaErrorInvalidValue) return PKV_E_WORKSPACE;
    return status_of(e);
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
