/*
 * pkv_oracle.c -- plain, slow, obviously-correct CPU oracle for the paged KV-cache
 * data plane.  TEST INFRASTRUCTURE ONLY: the product path never links, loads or calls
 * this file.  Only the tests, the package's smoke check and the benchmark's CPU-baseline
 * leg use it.  It shares no code, header, table or constant with the CUDA library.
 *
 * Arithmetic is IEEE fp64 throughout (built with -ffp-contract=off so that no multiply-add
 * is fused behind our back).  Values enter as bf16 bit patterns or E4M3 codes and are
 * widened exactly; the only roundings are the ones the definitions below state.
 *
 * Sources (three web pages on KV caching in Nano-vLLM/vLLM-style engines):
 *   [NV2]  "Nano-vLLM Part 2: model internals, KV cache and tensor parallelism"
 *   [ENG]  "Inside the Nano-vLLM engine: KV cache, attention and tensor parallelism"
 *   [PRM]  "LLM primer: from text to tokens, embeddings, QKV and Transformer"
 *
 * Parity pins (what ties each function to something other than itself) are listed in
 * the docstrings of oracle/__init__.py and exercised by tests/test_oracle_pins.py.
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------------------ */
/* Number formats                                                                       */
/* ------------------------------------------------------------------------------------ */

/* bf16 -> fp64: a bf16 value is the top half of an IEEE binary32 pattern; widening to
 * binary32 and then to binary64 is exact. */
double orc_bf16_to_f64(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* fp64 -> bf16, round to nearest, ties to even, computed directly on the real value
 * (no intermediate binary32 rounding).  bf16 keeps 8 significant bits and the binary32
 * exponent range: normal numbers in [2^-126, 2^128), subnormals spaced 2^-133. */
uint16_t orc_f64_to_bf16(double x)
{
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    if (isnan(x)) return (uint16_t)(sign | 0x7FC0u);
    double a = fabs(x);
    if (isinf(a)) return (uint16_t)(sign | 0x7F80u);
    if (a == 0.0) return sign;
    int e;
    (void)frexp(a, &e);             /* a = m * 2^e with m in [0.5, 1): a in [2^(e-1), 2^e) */
    int q_exp = (e - 1) - 7;        /* spacing of 8-significant-bit numbers in that binade */
    if (q_exp < -133) q_exp = -133; /* subnormal range spacing */
    double n = nearbyint(ldexp(a, -q_exp)); /* exact scaling; ties-to-even in default mode */
    double r = ldexp(n, q_exp);
    if (r >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7F80u); /* overflow -> inf */
    float f = (float)r;             /* exact: r has <= 8 significant bits, in range */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | ((u >> 16) & 0x7FFFu));
}

/* OCP FP8 E4M3 ("FN": no infinities).  Code layout s.eeee.mmm, bias 7.
 * E = 0      : subnormal, value = (m/8) * 2^-6
 * E = 1..15  : normal,    value = (1 + m/8) * 2^(E-7), except E=15,m=7 which is NaN.
 * Largest finite magnitude: 1.75 * 2^8 = 448.
 * Only "FP8 = 1 byte per element" is on the pages ([PRM] §17.6); the E4M3 format and
 * per-head scale are the workload's choice. */
double orc_e4m3_decode(uint8_t c)
{
    int s = (c >> 7) & 1, E = (c >> 3) & 15, m = c & 7;
    double v;
    if (E == 15 && m == 7) return NAN;
    if (E == 0) v = ldexp((double)m / 8.0, -6);
    else v = ldexp(1.0 + (double)m / 8.0, E - 7);
    return s ? -v : v;
}

/* fp64 -> E4M3, round to nearest even, saturating to +-448 (finite inputs only; NaN in
 * gives the NaN code).  The rounded magnitude is located by searching the table of the
 * 127 non-negative finite codes, which keeps the encoder a literal reading of the format. */
uint8_t orc_e4m3_encode(double x)
{
    uint8_t sign = signbit(x) ? 0x80u : 0u;
    if (isnan(x)) return (uint8_t)(sign | 0x7Fu);
    double a = fabs(x);
    if (a == 0.0) return sign;
    int q_exp;
    if (a < ldexp(1.0, -6)) {
        q_exp = -9;                 /* subnormal spacing 2^-9 */
    } else {
        int e;
        (void)frexp(a, &e);         /* a in [2^(e-1), 2^e) */
        q_exp = (e - 1) - 3;        /* 4 significant bits */
    }
    double r = ldexp(nearbyint(ldexp(a, -q_exp)), q_exp);
    if (r > 448.0) r = 448.0;       /* satfinite */
    for (int c = 0; c <= 126; ++c)
        if (orc_e4m3_decode((uint8_t)c) == r) return (uint8_t)(sign | c);
    return (uint8_t)(sign | 0x7Fu); /* unreachable for finite input */
}

/* ------------------------------------------------------------------------------------ */
/* Rotary position embedding                                                            */
/* ------------------------------------------------------------------------------------ */

/* Angle table.  [PRM] §21.2 (RoPE rotates Q/K inside attention) and [ENG] §3.2
 * (apply_rotary_pos_emb) name the operation; the pairing and frequencies are the
 * rotate-half convention with theta_i = base^(-2i/D).
 * table[p][0][i] = fp32(cos(p * theta_i)), table[p][1][i] = fp32(sin(p * theta_i)),
 * evaluated in fp64 and rounded once to binary32. */
void orc_rope_table(float *table, int max_pos, int head_dim, double base)
{
    int half = head_dim / 2;
    for (int p = 0; p < max_pos; ++p)
        for (int i = 0; i < half; ++i) {
            double theta = pow(base, -(2.0 * (double)i) / (double)head_dim);
            double ang = (double)p * theta;
            table[(size_t)p * head_dim + i] = (float)cos(ang);
            table[(size_t)p * head_dim + half + i] = (float)sin(ang);
        }
}

/* Rotate one head vector x[0..D) (bf16) at position pos into y (bf16):
 *   y_i       = x_i cos - x_{i+D/2} sin
 *   y_{i+D/2} = x_{i+D/2} cos + x_i sin
 * in fp64 with the table's fp32 cos/sin, rounded once to bf16 (RNE). */
static void rope_vec(const uint16_t *x, uint16_t *y, const float *table, int pos, int head_dim)
{
    int half = head_dim / 2;
    const float *c = table + (size_t)pos * head_dim;
    const float *s = c + half;
    for (int i = 0; i < half; ++i) {
        double x1 = orc_bf16_to_f64(x[i]), x2 = orc_bf16_to_f64(x[i + half]);
        double ci = (double)c[i], si = (double)s[i];
        double y1 = x1 * ci - x2 * si;
        double y2 = x2 * ci + x1 * si;
        y[i] = orc_f64_to_bf16(y1);
        y[i + half] = orc_f64_to_bf16(y2);
    }
}

/* Position of every new token: sequence b owns rows [cu[b], cu[b+1]) of the call; its
 * n_b = cu[b+1]-cu[b] new tokens are the last n_b of its L_b = context_lens[b] cached
 * tokens, so row t sits at position L_b - n_b + (t - cu[b]). */
void orc_positions(const int32_t *cu_seqlens, const int32_t *context_lens, int num_seqs,
                   int64_t *pos_out)
{
    for (int b = 0; b < num_seqs; ++b) {
        int n = cu_seqlens[b + 1] - cu_seqlens[b];
        for (int t = cu_seqlens[b]; t < cu_seqlens[b + 1]; ++t)
            pos_out[t] = (int64_t)context_lens[b] - n + (t - cu_seqlens[b]);
    }
}

/* Rotate rows of x [num_tokens, n_heads, head_dim] in place, row t at positions[t]. */
void orc_rope(uint16_t *x, int num_tokens, int n_heads, int head_dim, const int64_t *positions,
              const float *table)
{
    uint16_t tmp[1024];
    for (int t = 0; t < num_tokens; ++t)
        for (int h = 0; h < n_heads; ++h) {
            uint16_t *row = x + ((size_t)t * n_heads + h) * head_dim;
            rope_vec(row, tmp, table, (int)positions[t], head_dim);
            memcpy(row, tmp, (size_t)head_dim * sizeof(uint16_t));
        }
}

/* ------------------------------------------------------------------------------------ */
/* KV store: slot-mapped scatter into the paged cache                                   */
/* ------------------------------------------------------------------------------------ */

/* [NV2] §5.1-5.3 (K/V of every token are cached; a kernel writes them into the cache),
 * [ENG] §2.1 (append on every decode step) and §2.2 (fixed-size blocks, slots/offsets).
 * For token t with s = slot_mapping[t] >= 0, for every kv head h:
 *   cache[s / block_size][s % block_size][h][:] = k[t][h][:]   (and likewise v)
 * slot -1 marks a padding token and writes nothing.
 * rope_table != NULL: K is first rotated at positions[t].
 * fp8 != 0: the cache holds E4M3 codes, code = e4m3(value / scale[h]), the quotient
 * taken in fp64 on the bf16 value.  Caches are byte arrays (2 B or 1 B per element). */
void orc_kv_store(const uint16_t *k, const uint16_t *v, void *k_cache, void *v_cache,
                  const int32_t *slot_mapping, int num_tokens, int n_kv_heads, int head_dim,
                  int block_size, int fp8, const float *k_scale, const float *v_scale,
                  const float *rope_table, const int64_t *positions)
{
    uint16_t krot[1024];
    for (int t = 0; t < num_tokens; ++t) {
        int s = slot_mapping[t];
        if (s < 0) continue;
        size_t blk = (size_t)(s / block_size), off = (size_t)(s % block_size);
        for (int h = 0; h < n_kv_heads; ++h) {
            const uint16_t *kr = k + ((size_t)t * n_kv_heads + h) * head_dim;
            const uint16_t *vr = v + ((size_t)t * n_kv_heads + h) * head_dim;
            if (rope_table) {
                rope_vec(kr, krot, rope_table, (int)positions[t], head_dim);
                kr = krot;
            }
            size_t dst = ((blk * block_size + off) * n_kv_heads + h) * head_dim;
            for (int d = 0; d < head_dim; ++d) {
                if (fp8) {
                    ((uint8_t *)k_cache)[dst + d] =
                        orc_e4m3_encode(orc_bf16_to_f64(kr[d]) / (double)k_scale[h]);
                    ((uint8_t *)v_cache)[dst + d] =
                        orc_e4m3_encode(orc_bf16_to_f64(vr[d]) / (double)v_scale[h]);
                } else {
                    ((uint16_t *)k_cache)[dst + d] = kr[d];
                    ((uint16_t *)v_cache)[dst + d] = vr[d];
                }
            }
        }
    }
}

/* ------------------------------------------------------------------------------------ */
/* Block bookkeeping: slots of new tokens, copy-on-write block copies                   */
/* ------------------------------------------------------------------------------------ */

/* [ENG] §2.2: a sequence's block table lists the physical blocks that hold its tokens,
 * in order, block_size tokens per block.  The token at position p of sequence b is
 * therefore the (p mod block_size)-th slot of the (p div block_size)-th block of its
 * table, i.e. slot = table[p / block_size] * block_size + p % block_size.  New token r of
 * sequence b is at p = L_b - n_b + r.  A position past the table or a table entry outside
 * [0, num_blocks) gives slot -1 (and no store). */
void orc_slot_mapping(int32_t *slot_mapping, const int32_t *block_tables, int max_blocks,
                      const int32_t *cu_seqlens, const int32_t *context_lens, int num_seqs,
                      int block_size, int64_t num_blocks)
{
    for (int b = 0; b < num_seqs; ++b) {
        int n = cu_seqlens[b + 1] - cu_seqlens[b];
        for (int r = 0; r < n; ++r) {
            int64_t p = (int64_t)context_lens[b] - n + r;
            int32_t slot = -1;
            if (p >= 0 && p < (int64_t)max_blocks * block_size) {
                int32_t blk = block_tables[(size_t)b * max_blocks + (size_t)(p / block_size)];
                if (blk >= 0 && blk < num_blocks)
                    slot = (int32_t)((int64_t)blk * block_size + p % block_size);
            }
            slot_mapping[cu_seqlens[b] + r] = slot;
        }
    }
}

/* [ENG] §2.2 (requests that share a prefix point at the same physical blocks; a shared
 * block is copied when one of them writes to it: copy on write) and [PRM] §17.7.  For each
 * pair (src, dst): block dst of both caches becomes a byte copy of block src.  Pairs are
 * applied in order; ids outside [0, num_blocks) skip the pair.  block_bytes is the size of
 * one block of one cache (block_size * n_kv_heads * head_dim * element size). */
void orc_copy_blocks(uint8_t *k_cache, uint8_t *v_cache, const int32_t *pairs, int num_pairs,
                     int64_t block_bytes, int64_t num_blocks)
{
    for (int i = 0; i < num_pairs; ++i) {
        int32_t src = pairs[2 * i], dst = pairs[2 * i + 1];
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks || src == dst)
            continue;
        for (int64_t j = 0; j < block_bytes; ++j) {
            k_cache[(int64_t)dst * block_bytes + j] = k_cache[(int64_t)src * block_bytes + j];
            v_cache[(int64_t)dst * block_bytes + j] = v_cache[(int64_t)src * block_bytes + j];
        }
    }
}

/* [ENG] §2.2: physical blocks come from a pool; a sequence gets a new block when its
 * tokens outgrow the blocks it has, and a finished request returns its blocks to the pool
 * ([PRM] §17.7 likens the block table to an operating system's page table).  The pool here
 * is a stack of free ids plus a free flag per block:
 *   init   : every block free, stacked so that the first allocations hand out 0, 1, 2, ...
 *   alloc  : sequence by sequence, the blocks its new tokens need beyond those its cached
 *            tokens already fill, taken one by one from the top of the stack and written to
 *            the sequence's table after its existing entries.  If the pool cannot cover the
 *            whole request, nothing is taken and -1 is returned.
 *   free   : ids pushed back one by one; an id outside the pool or already free is skipped
 *            and counted.
 * State layout (int32): [0] = number of free ids, [1 .. num_blocks] = the stack (bottom first),
 * then num_blocks free flags. */
void orc_pool_init(int32_t *pool, int32_t num_blocks)
{
    pool[0] = num_blocks;
    for (int32_t i = 0; i < num_blocks; ++i) {
        pool[1 + i] = num_blocks - 1 - i;          /* top of the stack = block 0 */
        pool[1 + num_blocks + i] = 1;
    }
}

int orc_pool_alloc(int32_t *pool, int32_t num_blocks, int32_t *block_tables, int max_blocks,
                   const int32_t *cu_seqlens, const int32_t *context_lens, int num_seqs,
                   int block_size)
{
    int64_t total = 0;
    for (int b = 0; b < num_seqs; ++b) {
        int n = cu_seqlens[b + 1] - cu_seqlens[b];
        int have = (context_lens[b] - n + block_size - 1) / block_size;
        int need = (context_lens[b] + block_size - 1) / block_size;
        if (need > max_blocks) return -1;
        total += need - have;
    }
    if (total > pool[0]) return -1;
    for (int b = 0; b < num_seqs; ++b) {
        int n = cu_seqlens[b + 1] - cu_seqlens[b];
        int have = (context_lens[b] - n + block_size - 1) / block_size;
        int need = (context_lens[b] + block_size - 1) / block_size;
        for (int j = have; j < need; ++j) {
            int32_t id = pool[pool[0]];              /* top of the stack */
            pool[0] -= 1;
            pool[1 + num_blocks + id] = 0;
            block_tables[(size_t)b * max_blocks + j] = id;
        }
    }
    return 0;
}

int orc_pool_free(int32_t *pool, int32_t num_blocks, const int32_t *ids, int num_ids)
{
    int rejected = 0;
    for (int i = 0; i < num_ids; ++i) {
        int32_t id = ids[i];
        if (id < 0 || id >= num_blocks || pool[1 + num_blocks + id]) {
            ++rejected;
            continue;
        }
        pool[0] += 1;
        pool[pool[0]] = id;
        pool[1 + num_blocks + id] = 1;
    }
    return rejected;
}

/* ------------------------------------------------------------------------------------ */
/* Attention over the paged cache                                                       */
/* ------------------------------------------------------------------------------------ */

static double cache_value(const void *cache, size_t idx, int fp8, double scale)
{
    if (fp8) return orc_e4m3_decode(((const uint8_t *)cache)[idx]) * scale;
    return orc_bf16_to_f64(((const uint16_t *)cache)[idx]);
}

/* Scaled dot-product attention, [ENG] §3 (softmax(Q K^T / sqrt(d_k)) V) with the causal
 * mask of [ENG] §3.2 / [PRM] §22 step 6 and the max subtraction of [ENG] §3.2, read
 * through the block table of [ENG] §2.2.  For each requested output row (t, h):
 *   b      = the sequence owning row t,  n_b its new tokens, L_b = context_lens[b]
 *   pos    = L_b - n_b + (t - cu[b])     (bottom-right causal alignment)
 *   g      = h / (n_q_heads / n_kv_heads)           (consecutive q heads share a kv head)
 *   step 1 gather: K_b[j] = cache[block_tables[b][j / bs]][j % bs][g][:] for j < L_b,
 *          into a contiguous [L_b, D] array (likewise V_b); fp8 codes are dequantised
 *          as code_value * scale[g]
 *   step 2 s_j = scale * <q_{t,h}, K_b[j]>                    for j <= pos (mask)
 *   step 3 m = max_j s_j,  p_j = exp(s_j - m),  l = sum_j p_j
 *   step 4 o = (sum_j p_j V_b[j]) / l            (a row with no visible key is zero)
 * q holds bf16 patterns [num_tokens, n_q_heads, D]; if rope_table is given, q is first
 * rotated at pos and rounded to bf16 (the same result as rotating it beforehand).
 * rows == NULL computes every (t, h) into out[num_tokens, n_q_heads, D];
 * otherwise rows[2r] = t, rows[2r+1] = h and out is [num_rows, D].  fp64 output. */
void orc_attention(const uint16_t *q, const void *k_cache, const void *v_cache,
                   const int32_t *cu_seqlens, const int32_t *block_tables,
                   int max_blocks_per_seq, const int32_t *context_lens, int num_seqs,
                   int num_tokens, int n_q_heads, int n_kv_heads, int head_dim, int block_size,
                   double scale, int fp8, const float *k_scale, const float *v_scale,
                   const float *rope_table, const int32_t *rows, int num_rows, double *out)
{
    int group = n_q_heads / n_kv_heads;
    int64_t n_out = rows ? (int64_t)num_rows : (int64_t)num_tokens * n_q_heads;
    /* Owner sequence of each row (a plain scan over cu_seqlens). */
    int32_t *owner = (int32_t *)malloc(sizeof(int32_t) * (size_t)(num_tokens > 0 ? num_tokens : 1));
    for (int b = 0; b < num_seqs; ++b)
        for (int t = cu_seqlens[b]; t < cu_seqlens[b + 1]; ++t) owner[t] = b;

#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_out; ++r) {
        int t = rows ? rows[2 * r] : (int)(r / n_q_heads);
        int h = rows ? rows[2 * r + 1] : (int)(r % n_q_heads);
        double *o = out + (size_t)r * head_dim;
        int b = owner[t];
        int n_new = cu_seqlens[b + 1] - cu_seqlens[b];
        int L = context_lens[b];
        int64_t pos = (int64_t)L - n_new + (t - cu_seqlens[b]);
        int g = h / group;

        /* q row (optionally rotated), widened to fp64 */
        uint16_t qb[1024];
        memcpy(qb, q + ((size_t)t * n_q_heads + h) * head_dim, sizeof(uint16_t) * head_dim);
        if (rope_table) {
            uint16_t tmp[1024];
            rope_vec(qb, tmp, rope_table, (int)pos, head_dim);
            memcpy(qb, tmp, sizeof(uint16_t) * head_dim);
        }
        double qd[1024];
        for (int d = 0; d < head_dim; ++d) qd[d] = orc_bf16_to_f64(qb[d]);

        int nvis = (int)(pos + 1 < L ? pos + 1 : L); /* keys j <= pos that exist */
        for (int d = 0; d < head_dim; ++d) o[d] = 0.0;
        if (nvis <= 0) continue;

        /* step 1: gather this sequence's K and V for kv head g into contiguous arrays */
        double *Kb = (double *)malloc(sizeof(double) * (size_t)L * head_dim);
        double *Vb = (double *)malloc(sizeof(double) * (size_t)L * head_dim);
        double ks = fp8 ? (double)k_scale[g] : 1.0, vs = fp8 ? (double)v_scale[g] : 1.0;
        for (int j = 0; j < L; ++j) {
            size_t blk = (size_t)block_tables[(size_t)b * max_blocks_per_seq + j / block_size];
            size_t base = ((blk * block_size + (size_t)(j % block_size)) * n_kv_heads + g) *
                          (size_t)head_dim;
            for (int d = 0; d < head_dim; ++d) {
                Kb[(size_t)j * head_dim + d] = cache_value(k_cache, base + d, fp8, ks);
                Vb[(size_t)j * head_dim + d] = cache_value(v_cache, base + d, fp8, vs);
            }
        }
        /* step 2: masked scores */
        double *s = (double *)malloc(sizeof(double) * (size_t)nvis);
        for (int j = 0; j < nvis; ++j) {
            double acc = 0.0;
            for (int d = 0; d < head_dim; ++d) acc += qd[d] * Kb[(size_t)j * head_dim + d];
            s[j] = scale * acc;
        }
        /* step 3: max-subtracted softmax */
        double m = s[0];
        for (int j = 1; j < nvis; ++j) if (s[j] > m) m = s[j];
        double l = 0.0;
        for (int j = 0; j < nvis; ++j) { s[j] = exp(s[j] - m); l += s[j]; }
        /* step 4: weighted sum of values */
        for (int j = 0; j < nvis; ++j) {
            double p = s[j] / l;
            for (int d = 0; d < head_dim; ++d) o[d] += p * Vb[(size_t)j * head_dim + d];
        }
        free(s);
        free(Kb);
        free(Vb);
    }
    free(owner);
}

/* Probability rows of the same definition (steps 1-3 only), for pins on the weights:
 * out[r][j] = p_j for j < L_b (0 where masked).  rows as above, out is [num_rows, Lmax]. */
void orc_attention_weights(const uint16_t *q, const void *k_cache, const int32_t *cu_seqlens,
                           const int32_t *block_tables, int max_blocks_per_seq,
                           const int32_t *context_lens, int num_seqs, int num_tokens,
                           int n_q_heads, int n_kv_heads, int head_dim, int block_size,
                           double scale, const int32_t *rows, int num_rows, int lmax,
                           double *out)
{
    int group = n_q_heads / n_kv_heads;
    for (int r = 0; r < num_rows; ++r) {
        int t = rows[2 * r], h = rows[2 * r + 1];
        int b = 0;
        while (b < num_seqs && !(t >= cu_seqlens[b] && t < cu_seqlens[b + 1])) ++b;
        int n_new = cu_seqlens[b + 1] - cu_seqlens[b];
        int L = context_lens[b];
        int64_t pos = (int64_t)L - n_new + (t - cu_seqlens[b]);
        int g = h / group;
        double *w = out + (size_t)r * lmax;
        for (int j = 0; j < lmax; ++j) w[j] = 0.0;
        int nvis = (int)(pos + 1 < L ? pos + 1 : L);
        if (nvis <= 0) continue;
        double *s = (double *)malloc(sizeof(double) * (size_t)nvis);
        for (int j = 0; j < nvis; ++j) {
            size_t blk = (size_t)block_tables[(size_t)b * max_blocks_per_seq + j / block_size];
            size_t base = ((blk * block_size + (size_t)(j % block_size)) * n_kv_heads + g) *
                          (size_t)head_dim;
            double acc = 0.0;
            for (int d = 0; d < head_dim; ++d)
                acc += orc_bf16_to_f64(q[((size_t)t * n_q_heads + h) * head_dim + d]) *
                       orc_bf16_to_f64(((const uint16_t *)k_cache)[base + d]);
            s[j] = scale * acc;
        }
        double m = s[0];
        for (int j = 1; j < nvis; ++j) if (s[j] > m) m = s[j];
        double l = 0.0;
        for (int j = 0; j < nvis; ++j) { s[j] = exp(s[j] - m); l += s[j]; }
        for (int j = 0; j < nvis && j < lmax; ++j) w[j] = s[j] / l;
        free(s);
    }
}

/* ------------------------------------------------------------------------------------ */
/* Sizing                                                                               */
/* ------------------------------------------------------------------------------------ */

/* [PRM] §17.3 / §17.6: KV bytes = 2 (K and V) x layers x kv_heads x head_dim
 *                                 x cached_tokens x bytes_per_element. */
int64_t orc_kv_cache_bytes(int64_t num_layers, int64_t n_kv_heads, int64_t head_dim,
                           int64_t cached_tokens, int64_t bytes_per_element)
{
    return 2 * num_layers * n_kv_heads * head_dim * cached_tokens * bytes_per_element;
}

/* Threads the OpenMP loops above use (reported beside CPU timings). */
int orc_num_threads(void) { return omp_get_max_threads(); }
