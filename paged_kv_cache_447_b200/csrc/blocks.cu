// blocks.cu -- block bookkeeping on the device: the cache slot of every new token, and
// copy-on-write copies of whole physical blocks.
//
// "Inside the Nano-vLLM engine: KV cache, attention and tensor parallelism", §2.2: a
// sequence's block table lists the physical blocks that hold its tokens, in order, 16
// tokens per block (block_size here), so position p lives at offset p % block_size of block
// table[p / block_size]; requests
// that share a prefix point at the same physical blocks, and a shared block is copied when
// one of them writes into it (copy on write; "LLM primer", §17.7 lists the same idea).
// Both kernels are small: the slot kernel is latency-bound (one int per token), the copy
// kernel an HBM stream of 16-byte vectors.
#include "common.cuh"
#include "internal.h"

namespace pkv {
namespace {

__global__ void __launch_bounds__(256) slot_mapping_kernel(SlotArgs a) {
    pdl_wait();
    pdl_trigger();
    for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < a.num_tokens;
         t += gridDim.x * blockDim.x) {
        const int b = owner_seq(a.cu_seqlens, a.num_seqs, t);
        const int c0 = __ldg(a.cu_seqlens + b);
        const int n = __ldg(a.cu_seqlens + b + 1) - c0;
        const long long p = (long long)__ldg(a.context_lens + b) - n + (t - c0);
        int slot = -1;
        const int bs = a.block_size;
        if (p < 0 || p >= (long long)a.max_blocks * bs) {
            atomicOr(a.err, kErrBounds);
        } else {
            const int blk = __ldg(a.block_tables + (size_t)b * a.max_blocks + (size_t)(p / bs));
            if (blk < 0 || (long long)blk >= a.num_blocks)
                atomicOr(a.err, kErrBounds);
            else
                slot = blk * bs + (int)(p % bs);
        }
        a.slot_mapping[t] = slot;
    }
}

// One thread per 16-byte chunk of a block (K and V), over all pairs.
__global__ void __launch_bounds__(256) copy_blocks_kernel(CopyArgs a) {
    pdl_wait();
    pdl_trigger();
    const long long chunks = a.block_bytes / 16;
    const long long total = (long long)a.num_pairs * chunks;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const int pr = (int)(i / chunks);
        const long long c = i % chunks;
        const int src = __ldg(a.pairs + 2 * pr), dst = __ldg(a.pairs + 2 * pr + 1);
        if (src < 0 || (long long)src >= a.num_blocks || dst < 0 || (long long)dst >= a.num_blocks) {
            if (c == 0) atomicOr(a.err, kErrBounds);
            continue;
        }
        if (src == dst) continue;
        const size_t so = (size_t)src * (size_t)a.block_bytes, d_o = (size_t)dst * (size_t)a.block_bytes;
        const uint4 *ks = reinterpret_cast<const uint4 *>(static_cast<const uint8_t *>(a.k_cache) + so);
        const uint4 *vs = reinterpret_cast<const uint4 *>(static_cast<const uint8_t *>(a.v_cache) + so);
        uint4 *kd = reinterpret_cast<uint4 *>(static_cast<uint8_t *>(a.k_cache) + d_o);
        uint4 *vd = reinterpret_cast<uint4 *>(static_cast<uint8_t *>(a.v_cache) + d_o);
        const uint4 kx = ks[c], vx = vs[c];
        kd[c] = kx;
        vd[c] = vx;
    }
}

int grid_cap(long long items) {
    const int sms = current_sm_count();
    long long blocks = (items + 255) / 256;
    const long long cap = (long long)sms * 8;
    if (blocks > cap) blocks = cap;
    return (int)(blocks < 1 ? 1 : blocks);
}

}  // namespace

cudaError_t launch_slot_mapping(const SlotArgs &a, cudaStream_t s) {
    if (a.num_tokens == 0) return cudaSuccess;
    return launch_pdl(slot_mapping_kernel, dim3(grid_cap(a.num_tokens)), dim3(256), 0, s, a);
}

cudaError_t launch_copy_blocks(const CopyArgs &a, cudaStream_t s) {
    if (a.num_pairs == 0) return cudaSuccess;
    return launch_pdl(copy_blocks_kernel, dim3(grid_cap((long long)a.num_pairs * (a.block_bytes / 16))),
                      dim3(256), 0, s, a);
}

}  // namespace pkv
