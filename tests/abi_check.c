/*
 * abi_check.c -- a plain C caller of libpagedkv.so, compiled against include/pkv.h alone
 * (with -Wall -Wextra -Werror), so the header's prototypes are what the compiler checks
 * every call against.
 *
 *   abi_check host
 *       every host-side entry point (version, status text, RoPE table, cache sizing,
 *       workspace sizing) and the argument checks that return before touching a device
 *   abi_check device DIR Hq Hkv D NB MAXPOS  B_pre T_pre MB_pre MAXNEW  B_dec T_dec MB_dec
 *       reads a tiny two-step batch (a prefill of whole prompts, then one decode token per
 *       sequence) from raw files in DIR, allocates its own device buffers, runs kv_store
 *       (K rotated), paged prefill attention and paged decode attention through the
 *       header's prototypes, and writes out_pre, out_dec and k_cache_out back to DIR
 *
 * Exit status 0 = every check passed.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime.h>

#include "pkv.h"

static int failures = 0;

#define EXPECT(cond)                                                   \
    do {                                                               \
        if (!(cond)) {                                                 \
            fprintf(stderr, "%s:%d: check failed: %s\n", __FILE__, __LINE__, #cond); \
            ++failures;                                                \
        }                                                              \
    } while (0)

static int host_checks(void) {
    EXPECT((pkv_version() >> 16) == 1);
    for (int c = 0; c >= -8; --c) EXPECT(pkv_strerror(c) != NULL && strlen(pkv_strerror(c)) > 0);
    EXPECT(strcmp(pkv_strerror(PKV_E_UNSUPPORTED), "unsupported shape or dtype") == 0);

    /* RoPE table: row 0 is cos 1 / sin 0; pair 0 of row p is (cos p, sin p) */
    float tab[8 * 64];
    EXPECT(pkv_rope_build_table(tab, 8, 64, 10000.0) == PKV_OK);
    EXPECT(tab[0] == 1.0f && tab[32] == 0.0f);
    EXPECT(tab[5 * 64 + 0] == (float)cos(5.0) && tab[5 * 64 + 32] == (float)sin(5.0));
    EXPECT(pkv_rope_build_table(NULL, 8, 64, 10000.0) == PKV_E_INVALID);
    EXPECT(pkv_rope_build_table(tab, 8, 63, 10000.0) == PKV_E_INVALID);

    /* sizing: 32 layers x 8 kv heads x 128 dims x 4096 tokens x 2 bytes x (K, V) = 0.5 GiB */
    EXPECT(pkv_cache_bytes(32, 4096 / 16, 16, 8, 128, PKV_BF16) == (size_t)536870912);
    EXPECT(pkv_cache_bytes(32, 1, 16, 32, 128, PKV_FP8_E4M3) == (size_t)32 * 2 * 16 * 32 * 128);
    EXPECT(pkv_cache_bytes(1, 1, 16, 1, 64, 7) == 0);

    /* the workspace grows with the batch; an uncompiled group has none */
    const size_t w64 = pkv_decode_workspace_bytes(64, 32, 32, 128);
    EXPECT(w64 > 0 && w64 < pkv_decode_workspace_bytes(128, 32, 32, 128));
    EXPECT(pkv_decode_workspace_bytes(64, 32, 5, 128) == 0);

    /* argument checks that need no device */
    EXPECT(pkv_kv_store(NULL, NULL, NULL, NULL, NULL, 4, 2, 96, 16, 32, PKV_BF16, NULL, NULL,
                        NULL, 0, NULL, NULL, 0, NULL) == PKV_E_UNSUPPORTED);
    EXPECT(pkv_kv_store(NULL, NULL, NULL, NULL, NULL, 4, 2, 64, 16, 32, PKV_BF16, NULL, NULL,
                        NULL, 0, NULL, NULL, 0, NULL) == PKV_E_INVALID);
    EXPECT(pkv_kv_store(NULL, NULL, NULL, NULL, NULL, 0, 2, 64, 16, 32, PKV_BF16, NULL, NULL,
                        NULL, 0, NULL, NULL, 0, NULL) == PKV_OK);
    EXPECT(pkv_paged_decode_attention(NULL, NULL, NULL, NULL, NULL, 4, NULL, 2, 6, 4, 64, 16, 32,
                                      1.0f, PKV_BF16, NULL, NULL, NULL, 0, NULL, 0,
                                      NULL) == PKV_E_INVALID);
    EXPECT(pkv_paged_decode_attention(NULL, NULL, NULL, NULL, NULL, 4, NULL, 2, 6, 2, 64, 16, 32,
                                      1.0f, PKV_BF16, NULL, NULL, NULL, 0, NULL, 0,
                                      NULL) == PKV_E_UNSUPPORTED);
    EXPECT(pkv_paged_prefill_attention(NULL, NULL, NULL, NULL, NULL, NULL, 4, NULL, 2, 10, 8, 2,
                                       64, 16, 32, 1.0f, PKV_BF16, NULL, NULL, NULL, 0, 5,
                                       NULL) == PKV_E_INVALID);
    EXPECT(pkv_rope_apply(NULL, NULL, NULL, 8, NULL, NULL, 1, 4, 8, 2, 96, NULL) ==
           PKV_E_UNSUPPORTED);
    EXPECT(pkv_slot_mapping(NULL, NULL, 4, NULL, NULL, 2, 0, 16, 32, NULL) == PKV_OK);
    EXPECT(pkv_copy_blocks(NULL, NULL, NULL, 0, 2, 64, 16, 32, PKV_BF16, NULL) == PKV_OK);
    EXPECT(pkv_copy_blocks(NULL, NULL, NULL, 1, 2, 64, 16, 32, PKV_BF16, NULL) == PKV_E_INVALID);
    if (failures == 0) printf("host checks passed\n");
    return failures == 0 ? 0 : 1;
}

/* ---------------------------------------------------------------- device pipeline */

static void *read_file(const char *dir, const char *name, size_t *bytes) {
    char path[4096];
    snprintf(path, sizeof path, "%s/%s", dir, name);
    FILE *f = fopen(path, "rb");
    if (!f) {
        fprintf(stderr, "cannot open %s\n", path);
        exit(2);
    }
    fseek(f, 0, SEEK_END);
    long n = ftell(f);
    fseek(f, 0, SEEK_SET);
    void *buf = malloc(n > 0 ? (size_t)n : 1);
    if (n > 0 && fread(buf, 1, (size_t)n, f) != (size_t)n) exit(2);
    fclose(f);
    *bytes = (size_t)n;
    return buf;
}

static void write_file(const char *dir, const char *name, const void *buf, size_t bytes) {
    char path[4096];
    snprintf(path, sizeof path, "%s/%s", dir, name);
    FILE *f = fopen(path, "wb");
    if (!f || fwrite(buf, 1, bytes, f) != bytes) exit(2);
    fclose(f);
}

#define CUDA_OK(call)                                                              \
    do {                                                                           \
        cudaError_t e_ = (call);                                                   \
        if (e_ != cudaSuccess) {                                                   \
            fprintf(stderr, "%s:%d: %s\n", __FILE__, __LINE__, cudaGetErrorString(e_)); \
            exit(3);                                                               \
        }                                                                          \
    } while (0)

static void *to_device(const char *dir, const char *name) {
    size_t n = 0;
    void *h = read_file(dir, name, &n);
    void *d = NULL;
    CUDA_OK(cudaMalloc(&d, n > 0 ? n : 16));
    if (n) CUDA_OK(cudaMemcpy(d, h, n, cudaMemcpyHostToDevice));
    free(h);
    return d;
}

struct step {
    void *q, *k, *v, *slots, *cu, *ctx, *tables;
    int B, T, max_blocks;
};

static struct step load_step(const char *dir, const char *tag, int B, int T, int max_blocks) {
    struct step s;
    char name[64];
#define LOAD(field, what)                                  \
    snprintf(name, sizeof name, "%s_%s", tag, what);       \
    s.field = to_device(dir, name);
    LOAD(q, "q") LOAD(k, "k") LOAD(v, "v") LOAD(slots, "slot_mapping") LOAD(cu, "cu_seqlens")
    LOAD(ctx, "context_lens") LOAD(tables, "block_tables")
#undef LOAD
    s.B = B;
    s.T = T;
    s.max_blocks = max_blocks;
    return s;
}

static int device_run(int argc, char **argv) {
    if (argc != 15) {
        fprintf(stderr, "usage: abi_check device DIR Hq Hkv D NB MAXPOS B_pre T_pre MB_pre MAXNEW "
                        "B_dec T_dec MB_dec\n");
        return 2;
    }
    const char *dir = argv[2];
    const int hq = atoi(argv[3]), hkv = atoi(argv[4]), d = atoi(argv[5]), nb = atoi(argv[6]);
    const int max_pos = atoi(argv[7]);
    struct step pre = load_step(dir, "pre", atoi(argv[8]), atoi(argv[9]), atoi(argv[10]));
    const int max_new = atoi(argv[11]);
    struct step dec = load_step(dir, "dec", atoi(argv[12]), atoi(argv[13]), atoi(argv[14]));
    void *kc = to_device(dir, "k_cache"), *vc = to_device(dir, "v_cache");
    const float scale = 1.0f / sqrtf((float)d);
    cudaStream_t stream;
    CUDA_OK(cudaStreamCreate(&stream));
    pkv_stream_t s = (pkv_stream_t)stream;

    float *tab_h = (float *)malloc(sizeof(float) * (size_t)max_pos * d);
    EXPECT(pkv_rope_build_table(tab_h, max_pos, d, 10000.0) == PKV_OK);
    float *tab = NULL;
    CUDA_OK(cudaMalloc((void **)&tab, sizeof(float) * (size_t)max_pos * d));
    CUDA_OK(cudaMemcpy(tab, tab_h, sizeof(float) * (size_t)max_pos * d, cudaMemcpyHostToDevice));

    /* step 1: store every prompt token (K rotated), prefill attention over the prompts */
    void *out_pre = NULL, *out_dec = NULL;
    CUDA_OK(cudaMalloc(&out_pre, (size_t)pre.T * hq * d * 2));
    CUDA_OK(cudaMalloc(&out_dec, (size_t)dec.T * hq * d * 2));
    EXPECT(pkv_kv_store(pre.k, pre.v, kc, vc, (const int32_t *)pre.slots, pre.T, hkv, d, 16, nb,
                        PKV_BF16, NULL, NULL, tab, max_pos, (const int32_t *)pre.cu,
                        (const int32_t *)pre.ctx, pre.B, s) == PKV_OK);
    EXPECT(pkv_paged_prefill_attention(out_pre, pre.q, kc, vc, (const int32_t *)pre.cu,
                                       (const int32_t *)pre.tables, pre.max_blocks,
                                       (const int32_t *)pre.ctx, pre.B, pre.T, hq, hkv, d, 16, nb,
                                       scale, PKV_BF16, NULL, NULL, tab, max_pos, max_new,
                                       s) == PKV_OK);
    /* step 2: one new token per sequence, decode attention over the whole cache */
    EXPECT(pkv_kv_store(dec.k, dec.v, kc, vc, (const int32_t *)dec.slots, dec.T, hkv, d, 16, nb,
                        PKV_BF16, NULL, NULL, tab, max_pos, (const int32_t *)dec.cu,
                        (const int32_t *)dec.ctx, dec.B, s) == PKV_OK);
    const size_t ws_bytes = pkv_decode_workspace_bytes(dec.B, hq, hkv, d);
    void *ws = NULL;
    CUDA_OK(cudaMalloc(&ws, ws_bytes));
    EXPECT(pkv_paged_decode_attention(out_dec, dec.q, kc, vc, (const int32_t *)dec.tables,
                                      dec.max_blocks, (const int32_t *)dec.ctx, dec.B, hq, hkv, d,
                                      16, nb, scale, PKV_BF16, NULL, NULL, tab, max_pos, ws,
                                      ws_bytes, s) == PKV_OK);
    /* a workspace one byte short is refused before anything is enqueued */
    EXPECT(pkv_paged_decode_attention(out_dec, dec.q, kc, vc, (const int32_t *)dec.tables,
                                      dec.max_blocks, (const int32_t *)dec.ctx, dec.B, hq, hkv, d,
                                      16, nb, scale, PKV_BF16, NULL, NULL, tab, max_pos, ws,
                                      ws_bytes - 1, s) == PKV_E_WORKSPACE);
    EXPECT(pkv_get_error(s) == PKV_OK);

    const size_t cache_bytes = (size_t)nb * 16 * hkv * d * 2;
    void *h = malloc(cache_bytes);
    CUDA_OK(cudaMemcpy(h, kc, cache_bytes, cudaMemcpyDeviceToHost));
    write_file(dir, "k_cache_out", h, cache_bytes);
    free(h);
    h = malloc((size_t)pre.T * hq * d * 2);
    CUDA_OK(cudaMemcpy(h, out_pre, (size_t)pre.T * hq * d * 2, cudaMemcpyDeviceToHost));
    write_file(dir, "out_pre", h, (size_t)pre.T * hq * d * 2);
    free(h);
    h = malloc((size_t)dec.T * hq * d * 2);
    CUDA_OK(cudaMemcpy(h, out_dec, (size_t)dec.T * hq * d * 2, cudaMemcpyDeviceToHost));
    write_file(dir, "out_dec", h, (size_t)dec.T * hq * d * 2);
    free(h);
    free(tab_h);
    CUDA_OK(cudaStreamDestroy(stream));
    if (failures == 0) printf("device pipeline ran\n");
    return failures == 0 ? 0 : 1;
}

int main(int argc, char **argv) {
    if (argc >= 2 && strcmp(argv[1], "host") == 0) return host_checks();
    if (argc >= 2 && strcmp(argv[1], "device") == 0) return device_run(argc, argv);
    fprintf(stderr, "usage: abi_check host | device DIR ...\n");
    return 2;
}
