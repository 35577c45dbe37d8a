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
// with an atomic) -- so the store, the attention and the merge are one kernel.  (Which of
// that and three launches runs is chosen per call, below.)
#include <atomic>

#include "decode_kernel.cuh"
#include "pkv.h"

namespace pkv {

size_t decode_step_workspace_bytes(int num_seqs, int n_q_heads, int n_kv_heads, int head_dim,
                                   int num_sms) {
    return decode_workspace_bytes(num_seqs, n_q_heads, n_kv_heads, head_dim, num_sms) +
           align16((size_t)num_seqs * n_kv_heads * sizeof(int));
}

namespace {
std::atomic<int> g_step_mode{PKV_STEP_AUTO};
}

int set_decode_step_mode(int mode) { return g_step_mode.exchange(mode); }

// Auto: one launch when the batch has at most one (sequence, kv head) segment per SM -- the
// latency-bound case the fused step is for.  A larger batch runs the store as its own launch
// and the attention with its merge kernel: measured faster there, because the fused kernel's
// extra code (the new token's store, the in-kernel merge) slows every tile of the
// tensor-core path through instruction fetch (ncu: no_instruction stalls 2.2 vs 0.9 per
// issue), while two extra launches cost a few microseconds.
cudaError_t launch_paged_decode_step(const DecodeArgs &a, cudaStream_t s) {
    const int mode = g_step_mode.load(std::memory_order_relaxed);
    const bool fused = mode == PKV_STEP_FUSED ||
                       (mode == PKV_STEP_AUTO && (long long)a.num_seqs * a.n_kv_heads <= current_sm_count());
    if (fused) {
        if (decode_tc_supported(a)) return launch_paged_decode_step_tc(a, s);
        return dispatch_decode<true>(a, s);
    }
    StoreArgs st{};
    st.k = a.k_new;
    st.v = a.v_new;
    st.k_cache = a.k_cache_w;
    st.v_cache = a.v_cache_w;
    st.slot_mapping = nullptr;
    st.num_tokens = a.num_seqs;
    st.n_kv_heads = a.n_kv_heads;
    st.head_dim = a.head_dim;
    st.num_slots = a.num_blocks * a.block_size;
    st.fp8 = a.fp8;
    st.k_scale = a.k_scale;
    st.v_scale = a.v_scale;
    st.rope = a.rope;
    st.max_pos = a.max_pos;
    st.cu_seqlens = nullptr;
    st.context_lens = a.context_lens;
    st.num_seqs = a.num_seqs;
    st.err = a.err;
    st.block_tables = a.block_tables;
    st.max_blocks = a.max_blocks_per_seq;
    st.block_size = a.block_size;
    cudaError_t e = launch_kv_store(st, s);
    if (e != cudaSuccess) return e;
    return launch_paged_decode(a, s);
}

}  // namespace pkv
