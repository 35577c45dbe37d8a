// kv_store.cu -- slot-mapped scatter of new K/V into the paged cache, and standalone RoPE.
//
// "Nano-vLLM Part 2: model internals, KV cache and tensor parallelism", §5.1-5.3: the K
// and V vectors of every token are cached so they are not recomputed, and a dedicated
// kernel writes them into the block-structured cache.  "Inside the Nano-vLLM engine",
// §2.1 (append on every decode step) and §2.2 (fixed-size blocks addressed through slots).
//
// Both kernels are HBM-bound streams: every thread owns one pair of 16-byte chunks of a
// (token, head) row -- dims [8c, 8c+8) and [8c + D/2, 8c + D/2 + 8), the two halves that
// rotate together -- so a row is read once, rotated in registers and written once, with
// 16-byte vector accesses.  A token's heads are contiguous in both the source and the
// cache slot, so consecutive threads touch consecutive 16-byte chunks.
#include "common.cuh"
#include "internal.h"

namespace pkv {
namespace {

struct Chunk {
    uint4 lo, hi;  // dims [8c, 8c+8) and [8c+D/2, 8c+D/2+8)
};

__device__ __forceinline__ void rotate_chunk(Chunk &x, const float *cos_row, const float *sin_row,
                                             int c) {
    const uint16_t *a = reinterpret_cast<const uint16_t *>(&x.lo);
    const uint16_t *b = reinterpret_cast<const uint16_t *>(&x.hi);
    uint16_t ra[8], rb[8];
    float4 c0 = __ldg(reinterpret_cast<const float4 *>(cos_row + 8 * c));
    float4 c1 = __ldg(reinterpret_cast<const float4 *>(cos_row + 8 * c + 4));
    float4 s0 = __ldg(reinterpret_cast<const float4 *>(sin_row + 8 * c));
    float4 s1 = __ldg(reinterpret_cast<const float4 *>(sin_row + 8 * c + 4));
    const float cs[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
    const float sn[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) rope_pair_fast(a[e], b[e], cs[e], sn[e], ra[e], rb[e]);
    x.lo = *reinterpret_cast<uint4 *>(ra);
    x.hi = *reinterpret_cast<uint4 *>(rb);
}

// Quantise 8 bf16 values (one 16-byte chunk) to 8 E4M3 codes with scale s: each the code of
// the exact quotient (e4m3_of_quotient).
__device__ __forceinline__ uint2 quantize_chunk(uint4 v, float s) {
    const uint16_t *e = reinterpret_cast<const uint16_t *>(&v);
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) lo |= e4m3_of_quotient(__uint_as_float((uint32_t)e[i] << 16), s) << (8 * i);
#pragma unroll
    for (int i = 0; i < 4; ++i) hi |= e4m3_of_quotient(__uint_as_float((uint32_t)e[4 + i] << 16), s) << (8 * i);
    return make_uint2(lo, hi);
}

template <bool FP8, bool ROPE>
__global__ void __launch_bounds__(256) kv_store_kernel(StoreArgs a) {
    pdl_wait();
    pdl_trigger();
    const int D = a.head_dim, H = a.n_kv_heads;
    const int cpr = D / 16;                      // chunk pairs per head row
    const long long items = (long long)a.num_tokens * H * cpr;
    for (long long it = blockIdx.x * (long long)blockDim.x + threadIdx.x; it < items;
         it += (long long)gridDim.x * blockDim.x) {
        const int c = (int)(it % cpr);
        const long long th = it / cpr;
        const int h = (int)(th % H);
        const int t = (int)(th / H);
        int slot;
        long long step_pos = -1;
        if (a.slot_mapping) {
            slot = __ldg(a.slot_mapping + t);
            if (slot < 0) continue;                  // padding token
        } else {
            // decode step: sequence t's new token at L - 1 (none for an empty sequence, and
            // none when the context exceeds the block table: attention flags that one)
            const int L = __ldg(a.context_lens + t);
            if (L < 1 || (long long)L > (long long)a.max_blocks * a.block_size) continue;
            step_pos = L - 1;
            const int e = __ldg(a.block_tables + (size_t)t * a.max_blocks + (int)(step_pos / a.block_size));
            if (e < 0 || (long long)e * a.block_size >= a.num_slots) {
                atomicOr(a.err, kErrBounds);
                continue;
            }
            slot = e * a.block_size + (int)(step_pos % a.block_size);
        }
        if ((long long)slot >= a.num_slots) {        // never write outside the cache
            atomicOr(a.err, kErrBounds);
            continue;
        }
        const size_t src = ((size_t)t * H + h) * D;
        const uint4 *ks = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(a.k) + src);
        const uint4 *vs = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(a.v) + src);
        Chunk kx{__ldg(ks + c), __ldg(ks + c + cpr)};
        Chunk vx{__ldg(vs + c), __ldg(vs + c + cpr)};
        if (ROPE) {
            long long pos = step_pos;
            if (a.slot_mapping) {
                const int b = owner_seq(a.cu_seqlens, a.num_seqs, t);
                const int n = __ldg(a.cu_seqlens + b + 1) - __ldg(a.cu_seqlens + b);
                pos = (long long)__ldg(a.context_lens + b) - n + (t - __ldg(a.cu_seqlens + b));
            }
            if (pos < 0 || pos >= a.max_pos) {
                atomicOr(a.err, kErrBounds);
                continue;
            }
            const float *row = a.rope + (size_t)pos * D;
            rotate_chunk(kx, row, row + D / 2, c);
        }
        const size_t dst = ((size_t)slot * H + h) * D;
        if (FP8) {
            const float ksc = __ldg(a.k_scale + h), vsc = __ldg(a.v_scale + h);
            uint2 *kd = reinterpret_cast<uint2 *>(static_cast<uint8_t *>(a.k_cache) + dst);
            uint2 *vd = reinterpret_cast<uint2 *>(static_cast<uint8_t *>(a.v_cache) + dst);
            kd[c] = quantize_chunk(kx.lo, ksc);
            kd[c + cpr] = quantize_chunk(kx.hi, ksc);
            vd[c] = quantize_chunk(vx.lo, vsc);
            vd[c + cpr] = quantize_chunk(vx.hi, vsc);
        } else {
            uint4 *kd = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(a.k_cache) + dst);
            uint4 *vd = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(a.v_cache) + dst);
            kd[c] = kx.lo;
            kd[c + cpr] = kx.hi;
            vd[c] = vx.lo;
            vd[c + cpr] = vx.hi;
        }
    }
}

__global__ void __launch_bounds__(256) rope_apply_kernel(RopeArgs a) {
    pdl_wait();
    pdl_trigger();
    const int D = a.head_dim, H = a.n_q_heads + a.n_kv_heads;
    const int cpr = D / 16;
    const long long items = (long long)a.num_tokens * H * cpr;
    for (long long it = blockIdx.x * (long long)blockDim.x + threadIdx.x; it < items;
         it += (long long)gridDim.x * blockDim.x) {
        const int c = (int)(it % cpr);
        const long long th = it / cpr;
        const int h = (int)(th % H);
        const int t = (int)(th / H);
        uint16_t *base;
        if (h < a.n_q_heads) {
            if (!a.q) continue;
            base = static_cast<uint16_t *>(a.q) + ((size_t)t * a.n_q_heads + h) * D;
        } else {
            if (!a.k) continue;
            base = static_cast<uint16_t *>(a.k) + ((size_t)t * a.n_kv_heads + (h - a.n_q_heads)) * D;
        }
        const int b = owner_seq(a.cu_seqlens, a.num_seqs, t);
        const int n = __ldg(a.cu_seqlens + b + 1) - __ldg(a.cu_seqlens + b);
        const long long pos = (long long)__ldg(a.context_lens + b) - n + (t - __ldg(a.cu_seqlens + b));
        if (pos < 0 || pos >= a.max_pos) {
            atomicOr(a.err, kErrBounds);
            continue;
        }
        uint4 *p = reinterpret_cast<uint4 *>(base);
        Chunk x{p[c], p[c + cpr]};
        const float *row = a.rope + (size_t)pos * D;
        rotate_chunk(x, row, row + D / 2, c);
        p[c] = x.lo;
        p[c + cpr] = x.hi;
    }
}

int grid_for(long long items, int threads) {
    const int sms = current_sm_count();
    long long blocks = (items + threads - 1) / threads;
    long long cap = (long long)sms * 8;  // 8 x 256 threads resident per SM
    if (blocks > cap) blocks = cap;
    return (int)(blocks < 1 ? 1 : blocks);
}

}  // namespace

cudaError_t launch_kv_store(const StoreArgs &a, cudaStream_t s) {
    const long long items = (long long)a.num_tokens * a.n_kv_heads * (a.head_dim / 16);
    if (items == 0) return cudaSuccess;
    const int grid = grid_for(items, 256);
    auto k = a.fp8 ? (a.rope ? kv_store_kernel<true, true> : kv_store_kernel<true, false>)
                   : (a.rope ? kv_store_kernel<false, true> : kv_store_kernel<false, false>);
    return launch_pdl(k, dim3(grid), dim3(256), 0, s, a);
}

cudaError_t launch_rope_apply(const RopeArgs &a, cudaStream_t s) {
    const long long items =
        (long long)a.num_tokens * (a.n_q_heads + a.n_kv_heads) * (a.head_dim / 16);
    if (items == 0) return cudaSuccess;
    return launch_pdl(rope_apply_kernel, dim3(grid_for(items, 256)), dim3(256), 0, s, a);
}

}  // namespace pkv
