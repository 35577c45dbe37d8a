// decode_step.cu -- pkv_paged_decode_step: one whole decode step of a batch in one launch.
//
// "LLM primer: from text to tokens, embeddings, QKV and Transformer", §17.1: decode runs one
// token per sequence per step, bound by memory bandwidth, and its latency per step is the
// time per output token.  "Inside the Nano-vLLM engine: KV cache, attention and tensor
// parallelism", §2.1 (each step appends the new token's K/V to the cache and attends over
// all of it) and §6.3 (fusing kernels to cut launches).  The decode attention kernel
// (decode_kernel.cuh) runs with STEP set: the warp that streams a sequence's last block
// also stores the step's new token into the cache and into its shared-memory tile, and the
// CTAs that split a sequence merge their partials themselves (the last to arrive, counted
// with an atomic) -- so the store, the attention and the merge are one kernel.
#include "decode_kernel.cuh"

namespace pkv {

size_t decode_step_workspace_bytes(int num_seqs, int n_q_heads, int n_kv_heads, int head_dim,
                                   int num_sms) {
    return decode_workspace_bytes(num_seqs, n_q_heads, n_kv_heads, head_dim, num_sms) +
           align16((size_t)num_seqs * n_kv_heads * sizeof(int));
}

cudaError_t launch_paged_decode_step(const DecodeArgs &a, cudaStream_t s) {
    if (decode_tc_supported(a)) return launch_paged_decode_step_tc(a, s);
    return dispatch_decode<true>(a, s);
}

}  // namespace pkv
