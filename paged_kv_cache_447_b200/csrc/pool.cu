// pool.cu -- the physical-block pool on the device: allocation of the blocks a batch's new
// tokens need, and their return when a request finishes.
//
// "Inside the Nano-vLLM engine: KV cache, attention and tensor parallelism", §2.2: physical
// blocks come from a pool; a sequence receives a new block only when its tokens outgrow the
// blocks it holds, and a finished request gives its blocks back ("LLM primer", §17.7: the
// block table works like an operating system's page table).
//
// Pool state (int32, caller-allocated, pkv_block_pool_bytes): [0] free count, [1..3] unused,
// [4 .. 4+N) the stack of free ids (bottom first), [4+N .. 4+2N) one free flag per block.
// Both kernels run as ONE CTA, so the whole request sees one consistent pool and the ids
// come out in a fixed order: sequence by sequence, each sequence's new blocks in table
// order, popped from the top of the stack; frees push in argument order.
#include "common.cuh"
#include "internal.h"

namespace pkv {
namespace {

constexpr int kPoolThreads = 1024;
constexpr int kHeader = 4;

// Exclusive prefix over the block of `v` (one value per thread); the block's total in *tot.
__device__ int block_exclusive_scan(int v, int *tot) {
    __shared__ int warp_sum[kPoolThreads / 32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) warp_sum[warp] = incl;
    __syncthreads();
    int before = 0, all = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
        const int ws = warp_sum[w];
        if (w < warp) before += ws;
        all += ws;
    }
    __syncthreads();  // warp_sum is reused by the next call
    *tot = all;
    return before + incl - v;
}

__global__ void __launch_bounds__(256) pool_init_kernel(int32_t *pool, int32_t n) {
    pdl_wait();
    pdl_trigger();
    int32_t *stack = pool + kHeader, *flags = pool + kHeader + n;
    for (int32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        stack[i] = n - 1 - i;  // top of the stack = block 0
        flags[i] = 1;
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) pool[0] = n;
}

// New blocks of sequence b: ceil(L / bs) - ceil((L - n) / bs), or -1 if the table is too short.
__device__ __forceinline__ int new_blocks(const PoolArgs &a, int b, int *have) {
    const int L = __ldg(a.context_lens + b);
    const int n = __ldg(a.cu_seqlens + b + 1) - __ldg(a.cu_seqlens + b);
    const int bs = a.block_size;
    const int h = (L - n + bs - 1) / bs;
    const int need = (L + bs - 1) / bs;
    *have = h;
    if (L < 0 || n < 0 || n > L || need > a.max_blocks) return -1;
    return need - h;
}

__global__ void __launch_bounds__(kPoolThreads) pool_alloc_kernel(PoolArgs a) {
    pdl_wait();
    pdl_trigger();
    __shared__ int bad_s;
    if (threadIdx.x == 0) bad_s = 0;
    __syncthreads();
    // pass 1: the request's size (and whether every table can take its blocks)
    long long total = 0;
    for (int base = 0; base < a.num_seqs; base += blockDim.x) {
        const int b = base + threadIdx.x;
        int have = 0, k = 0;
        if (b < a.num_seqs) {
            k = new_blocks(a, b, &have);
            if (k < 0) {
                atomicOr(&bad_s, 1);
                k = 0;
            }
        }
        int tot = 0;
        block_exclusive_scan(k, &tot);
        total += tot;
    }
    __syncthreads();
    const int32_t free_n = a.pool[0];
    if (bad_s || total > free_n) {
        if (threadIdx.x == 0) atomicOr(a.err, bad_s ? kErrBounds : kErrPool);
        return;  // all or nothing
    }
    // pass 2: sequence b takes the ids at stack positions free_n - 1 - (offset_b + i)
    const int32_t *stack = a.pool + kHeader;
    int32_t *flags = a.pool + kHeader + a.num_blocks;
    long long carry = 0;
    for (int base = 0; base < a.num_seqs; base += blockDim.x) {
        const int b = base + threadIdx.x;
        int have = 0, k = 0;
        if (b < a.num_seqs) k = new_blocks(a, b, &have);
        int tot = 0;
        const int off = block_exclusive_scan(k, &tot);
        for (int i = 0; i < k; ++i) {
            const int32_t id = stack[free_n - 1 - (int)(carry + off + i)];
            flags[id] = 0;
            a.block_tables[(size_t)b * a.max_blocks + have + i] = id;
        }
        carry += tot;
    }
    __syncthreads();
    if (threadIdx.x == 0) a.pool[0] = free_n - (int32_t)total;
}

// Frees in argument order.  An id outside the pool, not currently allocated, or repeated
// within the call (after its first valid occurrence) is rejected.  The first valid
// occurrence of each id claims it by writing -(num_ids - i) into its flag (atomicMin: the
// smallest i wins), so acceptance does not depend on thread timing.
__global__ void __launch_bounds__(kPoolThreads) pool_free_kernel(PoolFreeArgs a) {
    pdl_wait();
    pdl_trigger();
    int32_t *stack = a.pool + kHeader, *flags = a.pool + kHeader + a.num_blocks;
    for (int i = threadIdx.x; i < a.num_ids; i += blockDim.x) {
        const int32_t id = __ldg(a.ids + i);
        if (id >= 0 && (long long)id < a.num_blocks && flags[id] <= 0)
            atomicMin(flags + id, -(a.num_ids - i));
    }
    __syncthreads();
    const int32_t free_n = a.pool[0];
    __shared__ int rejected_s;
    if (threadIdx.x == 0) rejected_s = 0;
    __syncthreads();
    long long carry = 0;
    for (int base = 0; base < a.num_ids; base += blockDim.x) {
        const int i = base + threadIdx.x;
        int32_t id = -1;
        int ok = 0;
        if (i < a.num_ids) {
            id = __ldg(a.ids + i);
            ok = (id >= 0 && (long long)id < a.num_blocks && flags[id] == -(a.num_ids - i)) ? 1 : 0;
            if (!ok) atomicAdd(&rejected_s, 1);
        }
        int tot = 0;
        const int pos = block_exclusive_scan(ok, &tot);
        if (ok) stack[free_n + carry + pos] = id;
        carry += tot;
    }
    __syncthreads();  // every claim was read before any flag is set back to free
    for (int i = threadIdx.x; i < a.num_ids; i += blockDim.x) {
        const int32_t id = __ldg(a.ids + i);
        if (id >= 0 && (long long)id < a.num_blocks && flags[id] == -(a.num_ids - i)) flags[id] = 1;
    }
    if (threadIdx.x == 0) {
        a.pool[0] = free_n + (int32_t)carry;
        if (rejected_s) atomicOr(a.err, kErrBounds);
    }
}

}  // namespace

size_t block_pool_bytes(long long num_blocks) {
    return (size_t)(kHeader + 2 * num_blocks) * sizeof(int32_t);
}

cudaError_t launch_pool_init(int32_t *pool, long long num_blocks, cudaStream_t s) {
    long long grid = (num_blocks + 255) / 256;
    const long long cap = (long long)current_sm_count() * 8;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    return launch_pdl(pool_init_kernel, dim3((unsigned)grid), dim3(256), 0, s, pool, (int32_t)num_blocks);
}

cudaError_t launch_pool_alloc(const PoolArgs &a, cudaStream_t s) {
    return launch_pdl(pool_alloc_kernel, dim3(1), dim3(kPoolThreads), 0, s, a);
}

cudaError_t launch_pool_free(const PoolFreeArgs &a, cudaStream_t s) {
    return launch_pdl(pool_free_kernel, dim3(1), dim3(kPoolThreads), 0, s, a);
}

}  // namespace pkv
