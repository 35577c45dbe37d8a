// decode.cu -- pkv_paged_decode_attention: one query token per sequence over its whole
// paged cache (the kernel and its design notes are in decode_kernel.cuh).
#include "decode_kernel.cuh"

namespace pkv {

int decode_grid_ctas(int num_sms) { return num_sms * kMaxCtasPerSm; }

size_t decode_workspace_bytes(int num_seqs, int n_q_heads, int n_kv_heads, int head_dim,
                              int num_sms) {
    const int G = n_q_heads / n_kv_heads;
    // one slot per (sequence, kv head), plus up to two per CTA (a CTA's range splits at most
    // two segments, and a segment may carry two kv heads)
    const size_t slots = (size_t)num_seqs * n_kv_heads + 2 * (size_t)decode_grid_ctas(num_sms);
    return align16((size_t)(num_seqs + 1) * sizeof(int)) +
           slots * (size_t)G * (head_dim + 2) * sizeof(float);
}

cudaError_t launch_paged_decode(const DecodeArgs &a, cudaStream_t s) {
    if (decode_tc_supported(a)) return launch_paged_decode_tc(a, s);
    return dispatch_decode<false>(a, s);
}

}  // namespace pkv
