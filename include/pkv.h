/*
 * pkv.h -- C ABI of libpagedkv.so, a paged KV-cache data plane for NVIDIA B200 (sm_100a).
 *
 * The operations follow three explainer pages on KV caching in vLLM/Nano-vLLM-style
 * inference engines; each entry point cites the passage that defines it:
 *   "Nano-vLLM Part 2: model internals, KV cache and tensor parallelism"          (NV2)
 *   "Inside the Nano-vLLM engine: KV cache, attention and tensor parallelism"     (ENG)
 *   "LLM primer: from text to tokens, embeddings, QKV and Transformer"            (PRM)
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Memory.   Every tensor argument is a DEVICE pointer owned by the caller, contiguous,
 *           row-major in the shape given.  The library never allocates, frees or
 *           synchronises on these calls (pkv_get_error is the one exception: it
 *           synchronises the stream it is given).  Work is enqueued on `stream`
 *           (a cudaStream_t; NULL = the legacy default stream) and runs asynchronously.
 * Cache.    k_cache / v_cache are [num_blocks, block_size, n_kv_heads, head_dim]:
 *           a physical block holds block_size consecutive tokens of one sequence, all kv
 *           heads of a token are adjacent (ENG §2.2: fixed-size blocks; NV2 §5.2: block,
 *           K/V and token dimensions).  Element type: bf16 (PKV_BF16) or OCP FP8 E4M3-FN
 *           codes with one fp32 scale per kv head for K and for V (PKV_FP8_E4M3; value =
 *           code_value * scale).  block_size 8, 16 or 32 (ENG §2.2 uses 16 as an example);
 *           head_dim 64 or 128 everywhere, and 256 for the store, RoPE and decode entry
 *           points (pkv_paged_prefill_attention returns PKV_E_UNSUPPORTED for 256).
 * Slots.    slot = physical_block * block_size + offset_in_block; slot -1 = padding token.
 * Tables.   block_tables [num_seqs, max_blocks_per_seq] int32: logical block i of sequence
 *           b lives in physical block block_tables[b][i] (ENG §2.2, PRM §17.7).  Entries
 *           past ceil(context_lens[b] / block_size) are never read.
 * Batches.  A call carries num_seqs sequences.  cu_seqlens [num_seqs+1] int32 (cu[0]=0)
 *           splits the call's num_tokens new tokens by sequence; context_lens [num_seqs]
 *           int32 is L_b, the number of cached tokens of sequence b INCLUDING this call's
 *           new ones.  New token r of sequence b (0-based) sits at position
 *           L_b - n_b + r, n_b = cu[b+1]-cu[b] (the new tokens are the last n_b).
 * RoPE.     rope_cos_sin is a [max_pos, head_dim] fp32 table made by pkv_rope_build_table:
 *           row p holds cos(p*theta_i) for i < head_dim/2, then sin(p*theta_i), with
 *           theta_i = base^(-2i/head_dim) (rotate-half pairing (i, i+head_dim/2)).
 *           A rotated value is computed in fp64 from the bf16 input and the fp32 table and
 *           rounded once to bf16 (round to nearest even), so every entry point that
 *           rotates produces the same bits (PRM §21.2; ENG §3.2).  NULL = no rotation.
 * Errors.   Entry points return PKV_OK (0) or a negative PKV_E_* code; host-detected
 *           problems (bad sizes, unsupported shapes, misalignment, a too-small workspace)
 *           are reported before anything is enqueued.  Conditions only the device sees (a
 *           slot, block id or position out of range; a bounded wait that ran out) never
 *           trap: the kernel skips the access, records a flag in a per-device error word
 *           and finishes; pkv_get_error() returns and clears it.
 */
#ifndef PKV_H_
#define PKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *pkv_stream_t; /* same type as cudaStream_t */

enum pkv_dtype { PKV_BF16 = 0, PKV_FP8_E4M3 = 1 };

enum pkv_status {
    PKV_OK = 0,
    PKV_E_INVALID = -1,     /* null pointer, negative size, inconsistent arguments       */
    PKV_E_UNSUPPORTED = -2, /* shape/dtype outside the compiled set                      */
    PKV_E_WORKSPACE = -3,   /* workspace missing or smaller than pkv_decode_workspace_bytes */
    PKV_E_CUDA = -4,        /* a CUDA runtime call or launch failed                      */
    PKV_E_TIMEOUT = -5,     /* (device) a bounded wait inside a kernel ran out            */
    PKV_E_BOUNDS = -6,      /* (device) slot / block id / position outside its array      */
    PKV_E_ALIGN = -7,       /* a pointer is not 16-byte aligned                           */
    PKV_E_SCRATCH_LIMIT = -8, /* the call needs more than PKV_NOALLOC_SCRATCH_BYTES of scratch */
    PKV_E_POOL = -9          /* (device) a block-pool allocation the pool could not cover    */
};

/* Size of the built-in decode scratch array used by pkv_paged_decode_attention_noalloc. */
#define PKV_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)

/* Library version, (major << 16) | minor. */
int pkv_version(void);

/* Text for a status code (static storage). */
const char *pkv_strerror(int code);

/*
 * pkv_rope_build_table -- fill a HOST array out[max_pos * head_dim] (fp32) with the RoPE
 * table described above, evaluated in fp64 (cos/sin/pow of the C library) and rounded
 * once to fp32.  Copy it to the device once and pass it as rope_cos_sin.
 * (PRM §21.2: RoPE rotates Q/K inside attention; ENG §3.2: apply_rotary_pos_emb.)
 * Returns PKV_E_INVALID for max_pos < 1, odd or non-positive head_dim, base <= 0.
 */
int pkv_rope_build_table(float *out, int max_pos, int head_dim, double base);

/*
 * pkv_cache_bytes -- bytes of ONE cache tensor pair (K and V) for num_layers layers of
 * num_blocks blocks: 2 * num_layers * num_blocks * block_size * n_kv_heads * head_dim *
 * element_bytes.  With cached_tokens = num_blocks * block_size this is the sizing formula
 * of PRM §17.3 and §17.6.  Returns 0 for invalid arguments.
 */
size_t pkv_cache_bytes(int num_layers, long long num_blocks, int block_size, int n_kv_heads,
                       int head_dim, int cache_dtype);

/*
 * pkv_kv_store -- slot-mapped scatter of new K/V into the paged cache
 * (NV2 §5.1-5.3: the K and V of every token are cached, a kernel writes them into the
 * block-structured cache; ENG §2.1: appended on every decode step; ENG §2.2: slots).
 *   k, v          [num_tokens, n_kv_heads, head_dim] bf16
 *   k_cache,
 *   v_cache       cache tensors (see Cache); written only at the mapped slots
 *   slot_mapping  [num_tokens] int32; -1 = skip the token
 *   k_scale,
 *   v_scale       [n_kv_heads] fp32, required for PKV_FP8_E4M3 (ignored for bf16):
 *                 code = E4M3(value / scale): the exact quotient rounded to nearest even
 *                 (the same code as rounding its fp64 value), saturated to +-448
 *   rope_cos_sin  RoPE table or NULL; when given, K is rotated at its position before it
 *                 is stored (V never is), and cu_seqlens/context_lens/num_seqs/max_pos
 *                 must describe the batch; otherwise they are ignored and may be NULL/0
 * Bit-exact: the stored bf16 (or E4M3) patterns are fully determined by the inputs.
 * Device errors: slot >= num_blocks*block_size, position >= max_pos -> PKV_E_BOUNDS flag,
 * that token is skipped.
 */
int pkv_kv_store(const void *k, const void *v, void *k_cache, void *v_cache,
                 const int32_t *slot_mapping, int num_tokens, int n_kv_heads, int head_dim,
                 int block_size, long long num_blocks, int cache_dtype, const float *k_scale,
                 const float *v_scale, const float *rope_cos_sin, int max_pos,
                 const int32_t *cu_seqlens, const int32_t *context_lens, int num_seqs,
                 pkv_stream_t stream);

/*
 * pkv_slot_mapping -- the cache slot of every new token of a batch, from the block tables
 * (ENG §2.2: a sequence's block table lists the physical blocks holding its tokens, in
 * order, block_size tokens each).  New token r of sequence b sits at position
 * p = L_b - n_b + r (see Batches), i.e. at offset p % block_size of physical block
 * block_tables[b][p / block_size]:
 *     slot_mapping[t] = block_tables[b][p / block_size] * block_size + p % block_size
 * This is the slot_mapping that pkv_kv_store takes.
 *   slot_mapping  [num_tokens] int32, written; num_tokens = cu_seqlens[num_seqs]
 *   block_tables, max_blocks_per_seq, cu_seqlens, context_lens, num_seqs: see Tables and
 *                 Batches; num_blocks: physical blocks of the cache (bounds check only)
 * Bit-exact (integer arithmetic).  Device errors: a position outside
 * [0, max_blocks_per_seq * block_size) or a table entry outside [0, num_blocks) ->
 * PKV_E_BOUNDS flag, that token's slot is -1 (so a following store skips it).
 */
int pkv_slot_mapping(int32_t *slot_mapping, const int32_t *block_tables, int max_blocks_per_seq,
                     const int32_t *cu_seqlens, const int32_t *context_lens, int num_seqs,
                     int num_tokens, int block_size, long long num_blocks, pkv_stream_t stream);

/*
 * pkv_copy_blocks -- copy whole physical blocks of the K and V caches, src -> dst, for
 * every pair: the copy-on-write step when sequences that share the blocks of a common
 * prefix diverge (ENG §2.2: requests with a common prefix point at the same physical
 * blocks, copied on write; PRM §17.7).
 *   k_cache,
 *   v_cache       cache tensors (see Cache); blocks dst are overwritten
 *   block_pairs   [num_pairs, 2] int32: (src, dst) physical block ids
 * Every slot and head of the block is copied byte for byte (bf16 values or E4M3 codes; the
 * per-head scales are shared, so codes stay valid).  No dst may appear as a src or dst of
 * another pair of the same call (the copies run concurrently); src == dst is a no-op.
 * Device errors: an id outside [0, num_blocks) -> PKV_E_BOUNDS flag, that pair is skipped.
 */
int pkv_copy_blocks(void *k_cache, void *v_cache, const int32_t *block_pairs, int num_pairs,
                    int n_kv_heads, int head_dim, int block_size, long long num_blocks,
                    int cache_dtype, pkv_stream_t stream);

/*
 * Block pool on the device (ENG §2.2: physical blocks come from a pool, a sequence receives
 * a new block only when its tokens outgrow the blocks it holds, and a finished request
 * returns its blocks; PRM §17.7: the block table works like a page table).
 * The pool is a caller-allocated device buffer of pkv_block_pool_bytes(num_blocks) bytes:
 * int32 [0] = number of free blocks (readable by the caller), then the stack of free ids and
 * one free flag per block.  Calls on one pool must not overlap in time; each runs as one
 * small kernel on `stream`, so the results are in stream order with the other entry points.
 *
 * pkv_block_pool_init -- every block free; the first allocations hand out 0, 1, 2, ...
 *
 * pkv_block_pool_alloc -- for every sequence b (cu_seqlens / context_lens as in Batches:
 * n_b new tokens, L_b cached tokens including them) the blocks its new tokens need beyond
 * the ceil((L_b - n_b) / block_size) it holds: ceil(L_b / block_size) - that many, taken in
 * sequence order from the top of the free stack and written to block_tables[b] right after
 * its held entries.  All or nothing: if the pool cannot cover the whole request the call
 * takes nothing and sets the PKV_E_POOL flag; a table too short for L_b (or a negative
 * count) takes nothing and sets PKV_E_BOUNDS.  Follow it with pkv_slot_mapping and
 * pkv_kv_store.
 *
 * pkv_block_pool_free -- push block_ids[0 .. num_ids) back in that order (last freed, first
 * reused).  An id outside the pool, not allocated, or repeated within the call is skipped and
 * sets the PKV_E_BOUNDS flag.  (Reference counts for blocks shared by several sequences are
 * the caller's: free a shared block once, when its last user finishes.)
 */
size_t pkv_block_pool_bytes(long long num_blocks);
int pkv_block_pool_init(void *pool, long long num_blocks, pkv_stream_t stream);
int pkv_block_pool_alloc(void *pool, long long num_blocks, int32_t *block_tables,
                         int max_blocks_per_seq, const int32_t *cu_seqlens,
                         const int32_t *context_lens, int num_seqs, int block_size,
                         pkv_stream_t stream);
int pkv_block_pool_free(void *pool, long long num_blocks, const int32_t *block_ids, int num_ids,
                        pkv_stream_t stream);

/*
 * pkv_rope_apply -- rotate q [num_tokens, n_q_heads, head_dim] and k [num_tokens,
 * n_kv_heads, head_dim] (bf16) IN PLACE at each token's position (PRM §21.2, ENG §3.2).
 * Either q or k may be NULL.  Device errors: position outside [0, max_pos) ->
 * PKV_E_BOUNDS flag, that token is left unchanged.
 */
int pkv_rope_apply(void *q, void *k, const float *rope_cos_sin, int max_pos,
                   const int32_t *cu_seqlens, const int32_t *context_lens, int num_seqs,
                   int num_tokens, int n_q_heads, int n_kv_heads, int head_dim,
                   pkv_stream_t stream);

/*
 * pkv_decode_workspace_bytes -- size of the device scratch buffer that
 * pkv_paged_decode_attention needs for its split-context partial results, for the
 * CURRENT device.  Depends only on the arguments and the device's SM count.
 */
size_t pkv_decode_workspace_bytes(int num_seqs, int n_q_heads, int n_kv_heads, int head_dim);

/*
 * pkv_paged_decode_attention -- one query token per sequence against its whole paged
 * cache (ENG §3: Q [batch, heads, 1, d] against cached K/V [batch, heads, seq_len, d];
 * ENG §3.1 incremental decoding; ENG §3.2 max subtraction; PRM §17.1: decode is bound
 * by memory bandwidth).  For sequence b and query head h (kv head g = h / (n_q_heads /
 * n_kv_heads)):
 *     s_j = scale * <q[b,h], K_b[j]>,  j < L_b = context_lens[b]
 *     out[b,h] = sum_j exp(s_j - max s) V_b[j] / sum_j exp(s_j - max s)
 * The query is the sequence's newest token, so every cached token is visible.
 *   out           [num_seqs, n_q_heads, head_dim] bf16 (a row with L_b = 0 is zero)
 *   q             [num_seqs, n_q_heads, head_dim] bf16
 *   rope_cos_sin  NULL, or the RoPE table: q is then rotated at position L_b - 1 first
 *   k_scale,
 *   v_scale       [n_kv_heads] fp32 for PKV_FP8_E4M3, else ignored
 *   workspace     device scratch of at least pkv_decode_workspace_bytes(...) bytes,
 *                 16-byte aligned; its contents need no initialisation and are
 *                 overwritten.  Calls that share a workspace must not overlap in time.
 * Sizes: num_seqs up to about 39,000 per call (each CTA keeps the prefix of the sequences'
 * block counts in shared memory); a larger call returns PKV_E_UNSUPPORTED and enqueues
 * nothing.
 * Device errors: block id outside [0, num_blocks) or L_b > max_blocks_per_seq*block_size
 * -> PKV_E_BOUNDS flag (the block reads as zeros / the context is clipped).
 */
int pkv_paged_decode_attention(void *out, const void *q, const void *k_cache,
                               const void *v_cache, const int32_t *block_tables,
                               int max_blocks_per_seq, const int32_t *context_lens,
                               int num_seqs, int n_q_heads, int n_kv_heads, int head_dim,
                               int block_size, long long num_blocks, float scale,
                               int cache_dtype, const float *k_scale, const float *v_scale,
                               const float *rope_cos_sin, int max_pos, void *workspace,
                               size_t workspace_bytes, pkv_stream_t stream);

/*
 * pkv_decode_step_workspace_bytes -- size of the device buffer pkv_paged_decode_step needs,
 * for the CURRENT device: the decode attention workspace followed by one int counter per
 * (sequence, kv head).
 */
size_t pkv_decode_step_workspace_bytes(int num_seqs, int n_q_heads, int n_kv_heads,
                                       int head_dim);

/*
 * pkv_paged_decode_step -- one whole decode step: store each sequence's new token into the
 * paged cache and run decode attention over the cache including it.  In one launch when
 * the batch is latency-bound (see pkv_set_decode_step_mode); otherwise the store runs as
 * its own launch before the attention and its merge, chained on the stream
 * (ENG §2.1: every decode step appends the new token's K/V to the cache and attends over
 * all of it; PRM §17.1: decode is one token per sequence per step and its latency is the
 * time per output token; ENG §6.3: fusing kernels).  The result is that of
 *     pkv_kv_store(k, v, ..., slot of position L_b - 1, K rotated at L_b - 1)
 *     pkv_paged_decode_attention(out, q, ...)
 * with the same cache bytes and bit-identical outputs.
 *   k, v          [num_seqs, n_kv_heads, head_dim] bf16: the new token of each sequence.
 *                 Its slot follows from the block table: position p = L_b - 1 is offset
 *                 p % block_size of block block_tables[b][p / block_size] (ENG §2.2), so
 *                 no slot mapping is taken; a sequence with L_b = 0 has no new token.
 *   k_cache,
 *   v_cache       written at those slots (E4M3 codes for PKV_FP8_E4M3, of the quotient by
 *                 the head's scale, as in pkv_kv_store)
 *   other arguments as pkv_paged_decode_attention (rope_cos_sin rotates both the new K and q
 *   at L_b - 1)
 *   workspace     at least pkv_decode_step_workspace_bytes(...) bytes, 16-byte aligned,
 *                 FILLED WITH ZEROS before its first use (cudaMemset); every call that
 *                 completes leaves its counters at zero again.  A call that ran into a
 *                 PKV_E_TIMEOUT may not: zero the workspace again after one.  Calls that share
 *                 a workspace must not overlap in time.
 * Device errors: as pkv_paged_decode_attention and pkv_kv_store (a table entry outside the
 * pool or a position past the RoPE table stores nothing and sets PKV_E_BOUNDS).
 */
int pkv_paged_decode_step(void *out, const void *q, const void *k, const void *v, void *k_cache,
                          void *v_cache, const int32_t *block_tables, int max_blocks_per_seq,
                          const int32_t *context_lens, int num_seqs, int n_q_heads,
                          int n_kv_heads, int head_dim, int block_size, long long num_blocks,
                          float scale, int cache_dtype, const float *k_scale,
                          const float *v_scale, const float *rope_cos_sin, int max_pos,
                          void *workspace, size_t workspace_bytes, pkv_stream_t stream);

/*
 * pkv_set_decode_step_mode -- how pkv_paged_decode_step runs, for the whole process:
 *   PKV_STEP_AUTO   one launch when num_seqs * n_kv_heads <= the device's SM count (the
 *                   latency-bound case), else store + attention + merge (measured faster
 *                   for large batches); the default
 *   PKV_STEP_FUSED  always one launch
 *   PKV_STEP_SPLIT  always store, then attention and merge
 * The outputs and cache bytes are the same in every mode.  Returns the previous mode, or
 * PKV_E_INVALID for an unknown one (nothing changes).  Host-side only; not thread-safe
 * against concurrent decode-step calls that should see a change.
 */
enum pkv_step_mode { PKV_STEP_AUTO = 0, PKV_STEP_FUSED = 1, PKV_STEP_SPLIT = 2 };
int pkv_set_decode_step_mode(int mode);

/*
 * pkv_paged_prefill_attention -- causal attention of a chunk of new tokens per sequence
 * over the paged cache, which must already hold those tokens' K/V (PRM §17.1 and ENG §2.1:
 * prefill processes all prompt tokens in parallel and is compute-bound; ENG §3.2 causal
 * mask; PRM §22 steps 6-8).  Row r of sequence b (position p = L_b - n_b + r) attends
 * to the cached tokens j <= p (bottom-right alignment: a chunk appended to a cached
 * prefix sees all of the prefix).
 *   out           [num_tokens, n_q_heads, head_dim] bf16
 *   q             [num_tokens, n_q_heads, head_dim] bf16, rows grouped by cu_seqlens
 *   max_new_tokens host upper bound on every n_b (sizes the grid; no device read-back)
 *   rope_cos_sin  NULL, or the RoPE table: q is rotated at its position on load
 *   k_scale,
 *   v_scale       [n_kv_heads] fp32 for PKV_FP8_E4M3, else ignored
 * Device errors: as pkv_paged_decode_attention.
 */
int pkv_paged_prefill_attention(void *out, const void *q, const void *k_cache,
                                const void *v_cache, const int32_t *cu_seqlens,
                                const int32_t *block_tables, int max_blocks_per_seq,
                                const int32_t *context_lens, int num_seqs, int num_tokens,
                                int n_q_heads, int n_kv_heads, int head_dim, int block_size,
                                long long num_blocks, float scale, int cache_dtype,
                                const float *k_scale, const float *v_scale,
                                const float *rope_cos_sin, int max_pos, int max_new_tokens,
                                pkv_stream_t stream);

/*
 * pkv_paged_decode_attention_noalloc -- pkv_paged_decode_attention for callers that cannot
 * allocate device memory.  (Not an operation of the pages: they have no counterpart.)
 * Engines typically give nearly all HBM to the KV-block pool when they start, so a
 * cudaMalloc from inside a decode step may fail, and on a latency-critical step a
 * cudaMalloc/cudaFree pair can synchronise the device; framework plugins that must not
 * allocate outside their host's allocator are in the same position.  This entry point
 * takes the same arguments minus the workspace, allocates nothing, and uses instead a
 * fixed array of PKV_NOALLOC_SCRATCH_BYTES (8 MiB) of device memory that is part of the
 * library image: every GPU that loads the library holds it until the process exits.
 *   - Calls needing more than PKV_NOALLOC_SCRATCH_BYTES (see pkv_decode_workspace_bytes)
 *     return PKV_E_SCRATCH_LIMIT and enqueue nothing.
 *   - All calls on a device share the one array: calls that overlap on the GPU (other
 *     streams, other host threads) race on it and must be serialised by the caller.  The
 *     array keeps the last call's contents; none of them needs to start at zero, so
 *     nothing is cleared.
 *   - The first call on each device (with that device current) looks up the array's
 *     device address with cudaGetSymbolAddress, and so does the first call after that
 *     device's context was replaced (cudaDeviceReset); make such a call before any stream
 *     capture begins.
 * Results equal pkv_paged_decode_attention's for the same inputs.
 */
int pkv_paged_decode_attention_noalloc(void *out, const void *q, const void *k_cache,
                                       const void *v_cache, const int32_t *block_tables,
                                       int max_blocks_per_seq, const int32_t *context_lens,
                                       int num_seqs, int n_q_heads, int n_kv_heads,
                                       int head_dim, int block_size, long long num_blocks,
                                       float scale, int cache_dtype, const float *k_scale,
                                       const float *v_scale, const float *rope_cos_sin,
                                       int max_pos, pkv_stream_t stream);

/*
 * pkv_get_error -- synchronise `stream`, then return and clear the current device's error
 * word: PKV_OK, PKV_E_TIMEOUT, PKV_E_BOUNDS or PKV_E_POOL (in that order of precedence), or
 * PKV_E_CUDA if the synchronisation itself failed.
 */
int pkv_get_error(pkv_stream_t stream);

/*
 * pkv_debug_wait_timeout -- failure-detection self test.  Launches one kernel whose
 * mbarrier wait can never complete (nothing arrives on it); the wait gives up after
 * timeout_ns nanoseconds (clamped to [1e3, 2e9]), sets the PKV_E_TIMEOUT flag and the
 * kernel returns normally, so the context stays usable.  Read the result with
 * pkv_get_error().
 */
int pkv_debug_wait_timeout(long long timeout_ns, pkv_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* PKV_H_ */
