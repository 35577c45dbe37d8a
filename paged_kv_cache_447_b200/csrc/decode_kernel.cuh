// decode_kernel.cuh -- the paged decode attention kernel template and its launchers, shared
// by decode.cu (pkv_paged_decode_attention: attention over the cache, split-context
// partials merged by a second small kernel) and decode_step.cu (pkv_paged_decode_step: the
// same pass that also stores the step's new token and merges the partials in-kernel).
//
//
// "Inside the Nano-vLLM engine: KV cache, attention and tensor parallelism", §3 (Q of the
// new token, [batch, heads, 1, d], against the cached K/V, [batch, heads, seq_len, d]),
// §3.1 (incremental decoding; FlashAttention-style tiling with the softmax kept on chip),
// §3.2 (subtract the maximum before the exponential).  "LLM primer", §17.1: decode is
// bound by memory bandwidth, the cache keeps growing.
//
// Design (HBM-bound: every cached K/V byte is streamed from HBM exactly once):
//  * Work unit = one 16-token block of one (sequence, kv-head group) -- the group is two
//    adjacent kv heads when the kv-head count is even (else one; and one for bf16 grouped
//    heads at D 128, whose two-slab tiles would halve the ring), so that each cache slot
//    row fetched is 2 x D x esize contiguous bytes: short rows measured far below the DRAM
//    bandwidth long ones reach (E4M3 at D 128, idle consumers: 3.8 TB/s with 128-byte rows,
//    5.0-5.2 TB/s with 256-byte rows).  Units are numbered sequence-major; the whole unit space
//    is cut into equal contiguous ranges, one per persistent CTA, so every CTA streams the
//    same number of bytes whatever the length mix.  A CTA's range crosses sequence
//    boundaries; each piece of a (sequence, kv-head group) it covers becomes one partial
//    softmax state per kv head.
//  * Warp 0 is the producer: it reads block-table entries 32 at a time and issues TMA loads
//    of K and V into a ring of shared-memory stages (mbarrier full/empty pairs).  Warps 1-4
//    consume stages round robin; with two kv heads per unit they form two pairs, one warp
//    per head, each pair taking every other unit.
//  * A consumer warp handles all G = Hq/Hkv query heads of the kv head, so each K/V tile
//    is read from shared memory once for the whole group.  Online softmax (running max m,
//    sum l) per warp in exp2 space.
//      - one q head per kv head, and E4M3 grouped heads at D 64: CUDA cores.  q.k: two
//        lanes per token (each half the head dim, chunk order rotated per token so
//        shared-memory reads are conflict-free), packed fp32x2 FMAs.  p.v: each lane owns
//        D/32 output dims.
//      - grouped heads (G = 2, 4, 8), bf16, and E4M3 at D 128: tensor cores, mma.sync
//        m16n8k16.  S = Q K^T with the G heads as rows of A (q held in registers for the
//        whole piece; K fragments by ldmatrix, or E4M3 bytes widened to f16); P stays in
//        registers and feeds O^T = V^T P^T as the B operand (V^T fragments by
//        ldmatrix.trans, or E4M3 bytes regrouped by byte permutes and widened), so O needs
//        D/16 accumulator tiles and no shuffles.
//  * At the end of a piece the consumer warps of each head merge (m, l, acc) through shared
//    memory.  A piece that covers its whole sequence writes the normalised bf16 output;
//    otherwise its partial goes to the workspace and a small combine kernel merges the
//    partials of that sequence:  M = max m_k,  o = sum e^(m_k-M) acc_k / sum e^(m_k-M) l_k.
#pragma once

#include "common.cuh"
#include "internal.h"

#include <algorithm>
#include <atomic>
#include <mutex>

namespace pkv {
namespace {

// Launch geometry per instantiation (measured on B200): several small CTAs per SM beat
// one large one -- each CTA brings its own TMA producer, and the SM overlaps their rings.
//   bf16 MHA:     4 consumer warps, 3 CTAs per SM, ~72 KB each (8-stage ring)
//   bf16 grouped: 4 consumer warps, 3 CTAs per SM, ~60 KB each (q, merge scratch grow with G)
//   E4M3 MHA:     4 consumer warps, 4 CTAs per SM, ~48 KB each (4 KB stages)
//   E4M3 grouped: 4 consumer warps, 3 CTAs per SM, ~64 KB each (tensor-core consumers need
//                 the registers of 3 CTAs per SM)
//   head dim 256: 4 consumer warps, 2 CTAs per SM, ~100 KB each (16-32 KB stages)
struct DecodeCfg {
    int consumers, ctas_per_sm, smem_budget;
};
__host__ __device__ constexpr DecodeCfg decode_cfg(int G, bool fp8, int D = 128) {
    return D == 256 ? DecodeCfg{4, 2, 100 * 1024}
           : fp8    ? (G > 1 ? DecodeCfg{4, 3, 64 * 1024} : DecodeCfg{4, 4, 48 * 1024})
                    : (G > 1 ? DecodeCfg{4, 3, 60 * 1024} : DecodeCfg{4, 3, 72 * 1024});
}
constexpr int kMaxThreads = 32 * (1 + 8);
constexpr int kMaxCtasPerSm = 4;  // sizes the workspace for any instantiation
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.0f;  // tensor-core path: lazy max update threshold (log2)
constexpr int kMergeBar = 1;

struct DecodeParams {
    __nv_bfloat16 *out;
    const uint16_t *q;
    const int32_t *block_tables;
    int max_blocks;
    const int32_t *context_lens;
    int B, Hq, Hkv;
    long long num_blocks;
    int bs;          // tokens per physical block (8, 16 or 32)
    int max_tokens;  // max_blocks * bs: the most tokens a table can describe
    float scale_log2;
    const float *k_scale, *v_scale;
    const float *rope;
    int max_pos;
    int *prefix;      // [B+1] block prefix, written by CTA 0 for the combine kernel
    float *partials;  // [(B*Hkv + 2*nctas)][G][D+2]
    int nctas;
    int *err;
    // decode step only: new K/V [B][Hkv][D] bf16, the writable caches, and one arrival
    // counter per split (sequence, kv-head group) segment (zero between calls)
    const uint16_t *k_new, *v_new;
    void *k_cache_w, *v_cache_w;
    int *counters;
    // tensor-core decode without the step: one arrival counter per CTA (the segment whose
    // first piece is that CTA's last), its high 48 bits naming the call (`epoch`), so the
    // workspace needs no zeroing
    unsigned long long *ectr = nullptr;
    unsigned long long epoch = 0;
};

template <int D, bool FP8, int G, int HPU>
struct Geometry {
    static constexpr DecodeCfg kCfg = decode_cfg(G, FP8, D);
    static constexpr int kConsumers = kCfg.consumers;
    static constexpr int kThreads = 32 * (1 + kConsumers);
    static constexpr int kCtasPerSm = kCfg.ctas_per_sm;
    // register budget hint for ptxas (the E4M3 tensor-core consumers need more than 3 CTAs
    // per SM would leave them at 128; the launch checks the occupancy it really gets)
    static constexpr int kMinCtasPerSm = kCtasPerSm;
    static constexpr int kElem = FP8 ? 1 : 2;
    static constexpr int kRowBytes = D * kElem;
    static constexpr int kTileBytes = kPiece * kRowBytes;          // one K (or V) block, one head
    static constexpr int kStageBytes = 2 * HPU * kTileBytes;           // K + V of the unit's heads
    static constexpr int kGroups = kConsumers / HPU;                   // consumer groups (warp per head)
    // q, probabilities and merge scratch, plus room for 1024 sequences' prefix
    // grouped heads on the tensor cores (bf16 caches, and E4M3 at head dim 128) keep q as bf16
    // (head dim 256 stays on the CUDA cores: the fragments would not fit the registers)
    static constexpr bool kMma = G >= 2 && (FP8 ? D == 128 : D <= 128);
    static constexpr int kQFloats = kMma ? HPU * G * D / 2 : HPU * G * D;  // q scratch
    static constexpr int kExtraBytes = kQFloats * 4 + kConsumers * G * 16 * 4 +
                                       kConsumers * G * (D + 2) * 4 + 4 * 1025;
    // the ring takes what the instantiation's shared-memory budget leaves
    // The stage count is a multiple of the consumer-group count, so that every fill of a
    // given stage is consumed by the same warp(s): a warp then never waits on a barrier more
    // than one phase ahead (a parity wait cannot tell phase n from phase n+2).
    static constexpr int kStagesRaw = (kCfg.smem_budget - kExtraBytes) / kStageBytes;
    static constexpr int kStagesQ = (kStagesRaw / kGroups) * kGroups;
    static constexpr int kStages = kStagesQ < kGroups ? kGroups : (kStagesQ > 64 ? 64 : kStagesQ);
    static_assert(kStages % kGroups == 0, "stage count must be a multiple of the consumer groups");
    static_assert(kConsumers % HPU == 0, "one consumer warp per head of a unit");
    static_assert(HPU * 2 * D * kElem <= kConsumers * G * (D + 2) * 4, "new-token rows fit the merge scratch");
    static constexpr int kChunkElems = 16 / kElem;                     // elements per 16 B
    static constexpr int kChunks = kRowBytes / 16;                     // 16-B chunks per row
    static constexpr int kQuads = kChunkElems / 4;                     // float4 per chunk
    static constexpr int kDimsPerLane = D / 32;                        // p.v ownership
};

// Units of sequence b: ceil(min(L_b, max_tokens) / 16) (16-token tiles).
__device__ __forceinline__ int seq_blocks(int L, int max_tokens, int *err) {
    if (L < 0) L = 0;
    if (L > max_tokens) {
        atomicOr(err, kErrBounds);
        L = max_tokens;
    }
    return (L + kPiece - 1) / kPiece;
}

// Cache row of offset `off` in block table entry `e` (physical block), or the first row past
// the cache (read as zeros by TMA) if the entry is outside the pool.
__device__ __forceinline__ int cache_row(const DecodeParams &p, int e, int off) {
    if (e < 0 || (long long)e >= p.num_blocks) {
        atomicOr(p.err, kErrBounds);
        return (int)(p.num_blocks * p.bs < 0x7fffffffLL ? p.num_blocks * p.bs : 0x7fffffff);
    }
    return e * p.bs + off;
}

// Exclusive prefix over sequences of their block counts, into pfx[0..B] (shared memory).
template <int kThreads>
__device__ void block_prefix(const DecodeParams &p, int *pfx) {
    __shared__ int warp_tot[kMaxThreads / 32];
    __shared__ int carry_s;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) carry_s = 0;
    __syncthreads();
    for (int base = 0; base < p.B; base += kThreads) {
        const int b = base + threadIdx.x;
        int v = (b < p.B) ? seq_blocks(__ldg(p.context_lens + b), p.max_tokens, p.err) : 0;
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) warp_tot[warp] = incl;
        __syncthreads();
        int before = carry_s;
        for (int w = 0; w < warp; ++w) before += warp_tot[w];
        if (b < p.B) pfx[b] = before + incl - v;
        __syncthreads();
        if (threadIdx.x == kThreads - 1) carry_s = before + incl;
        __syncthreads();
    }
    if (threadIdx.x == 0) pfx[p.B] = carry_s;
    __syncthreads();
}

// Last sequence b with Hkv*pfx[b] <= u (skips empty sequences).
__device__ __forceinline__ int find_seq(const int *pfx, int B, int Hkv, long long u) {
    int lo = 0, hi = B - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if ((long long)Hkv * pfx[mid] <= u) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

struct UnitPos {
    int b, kvh, blk, nb;
};

__device__ __forceinline__ UnitPos locate(const int *pfx, int B, int Hkv, long long u) {
    UnitPos r;
    r.b = find_seq(pfx, B, Hkv, u);
    r.nb = pfx[r.b + 1] - pfx[r.b];
    long long rel = u - (long long)Hkv * pfx[r.b];
    r.kvh = (int)(rel / r.nb);
    r.blk = (int)(rel % r.nb);
    return r;
}

// ---- grouped heads on the tensor cores (mma.sync m16n8k16, bf16 in, fp32 accumulate)
// The G query heads of a kv head are the rows of the A operand (rows G..15 are zero), a
// 16-token block is the N (q.k) or K (p.v) extent.  K and V tiles arrive 128-byte swizzled
// (16-byte chunk index XOR row & 7), so the eight 16-byte rows one ldmatrix phase reads
// fall in eight different bank groups.

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}

// c += A * B for one 16x8 tile; A rows 8..15 are zero (a2a3 = a6a7 = 0), so c[2], c[3]
// stay zero.
__device__ __forceinline__ void mma_rows8(float (&c)[4], uint32_t a01, uint32_t a45, uint32_t b01,
                                          uint32_t b23) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a01), "r"(0u), "r"(a45), "r"(0u), "r"(b01), "r"(b23));
}

// c += A * B for one 16x8 tile with a full 16x16 A fragment.
__device__ __forceinline__ void mma_full(float (&c)[4], const uint32_t (&a)[4], uint32_t b01,
                                         uint32_t b23) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b01), "r"(b23));
}

// The same two tiles in f16 (E4M3 caches: K/V widened exactly to f16, q and P rounded).
__device__ __forceinline__ void mma_rows8_f16(float (&c)[4], uint32_t a01, uint32_t a45,
                                              uint32_t b01, uint32_t b23) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a01), "r"(0u), "r"(a45), "r"(0u), "r"(b01), "r"(b23));
}

__device__ __forceinline__ void mma_full_f16(float (&c)[4], const uint32_t (&a)[4], uint32_t b01,
                                             uint32_t b23) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b01), "r"(b23));
}

// Two E4M3 codes (bits 0-7 and 8-15 of `two`) -> f16x2, low code in the low half (exact).
__device__ __forceinline__ uint32_t e4m3x2_f16x2(uint32_t two) {
    uint32_t r;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"((uint16_t)two));
    return r;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Offset of the 16-byte chunk c of row t (0..15) in a swizzled tile: slabs of 16 rows x
// 128 bytes (64 bf16 columns, or a whole 128-byte E4M3 row), kSlabStride bytes apart (the
// heads of a unit interleave by slab: 2 KB x heads per unit).
template <int kSlabStride>
__device__ __forceinline__ uint32_t swz(int t, int c) {
    return (uint32_t)((c >> 3) * kSlabStride + t * 128 + (((c & 7) ^ (t & 7)) << 4));
}

// Output element (head hd of the unit's group, q head g of that kv head, dim d) of split
// segment segu, merged from the partial states of CTAs c0..c1:
//   M = max m_k,  o = sum e^(m_k - M) acc_k / sum e^(m_k - M) l_k  (times the V scale).
template <int D, int G, int HPU>
__device__ __forceinline__ float merge_partials(const DecodeParams &p, int segu, int hd, int g, int d,
                                                int c0, int c1, float vsc) {
    float M = -INFINITY;
    for (int cc = c0; cc <= c1; ++cc) {
        const float *slot = p.partials + (size_t)(HPU * (segu + cc) + hd) * (G * (D + 2));
        M = fmaxf(M, __ldcg(slot + G * D + g));
    }
    float o = 0.f, lsum = 0.f;
    for (int cc = c0; cc <= c1; ++cc) {
        const float *slot = p.partials + (size_t)(HPU * (segu + cc) + hd) * (G * (D + 2));
        const float mk = __ldcg(slot + G * D + g);
        const float f = (mk == -INFINITY) ? 0.f : ex2(mk - M);
        o += f * __ldcg(slot + g * D + d);
        lsum += f * __ldcg(slot + G * D + G + g);
    }
    return lsum > 0.f ? o / lsum * vsc : 0.f;
}

template <int D, bool FP8, int G, int HPU, bool STEP>
__global__ void __launch_bounds__(Geometry<D, FP8, G, HPU>::kThreads,
                                  Geometry<D, FP8, G, HPU>::kMinCtasPerSm)
    decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const DecodeParams p) {
    using Geo = Geometry<D, FP8, G, HPU>;
    constexpr int NS = Geo::kStages;
    constexpr int kConsumers = Geo::kConsumers;
    constexpr int kThreads = Geo::kThreads;
    constexpr bool kMma = Geo::kMma;  // grouped heads on the tensor cores
    constexpr int kSlabs = Geo::kRowBytes / 128;  // swizzled boxes per tile (kMma)
    constexpr int kSlabStride = HPU * 2048;       // swizzled slabs of a unit's heads interleave
    // a head's tile inside a stage (K tiles, then V tiles): swizzled tiles interleave by slab
    constexpr int kHeadStride = kMma ? 2048 : Geo::kTileBytes;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *stages = smem;                                                  // NS x stage
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + NS * Geo::kStageBytes);
    uint64_t *empty = full + NS;
    float *qs = reinterpret_cast<float *>(empty + NS);                      // [HPU][G][quads][chunks][4]
    float *pbuf = qs + Geo::kQFloats;                                        // [consumers][G][16]
    float *mrg = pbuf + kConsumers * G * 16;                                 // [consumers][G][D+2]
    int *pfx = reinterpret_cast<int *>(mrg + kConsumers * G * (D + 2));      // [B+1]
    __shared__ volatile int abort_s;
    __shared__ int last_s;  // decode step: this CTA merges the segment's partials

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    pdl_wait();
    pdl_trigger();
    block_prefix<kThreads>(p, pfx);
    const int Hu = p.Hkv / HPU;  // kv-head groups (units per block of a sequence)
    const long long total = (long long)Hu * pfx[p.B];
    if (!STEP && blockIdx.x == 0)
        for (int i = threadIdx.x; i <= p.B; i += kThreads) p.prefix[i] = pfx[i];
    // sequences with an empty context get zero rows (strided over the CTAs)
    for (int b = blockIdx.x; b < p.B; b += gridDim.x)
        if (pfx[b + 1] == pfx[b])
            for (int e = threadIdx.x; e < p.Hq * D; e += kThreads)
                p.out[(size_t)b * p.Hq * D + e] = __float2bfloat16_rn(0.f);
    const long long U = total > 0 ? (total + p.nctas - 1) / p.nctas : 1;
    const long long u0 = (long long)blockIdx.x * U;
    const long long u1 = (u0 + U < total) ? u0 + U : total;
    if (u0 >= u1) return;  // uniform across the CTA
    const int nunits = (int)(u1 - u0);

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(smem_u32(full + s), 1);
            mbar_init(smem_u32(empty + s), HPU);  // one arrival per head's warp
        }
        abort_s = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == 0) {
        // ------------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
        }
        uint64_t issued_mask = 0, issued_phase = 0;  // stage ever filled / parity of last fill
        bool ok = true;
        for (int k0 = 0; k0 < nunits; k0 += 32) {
            const int k = k0 + lane;
            // the unit's 16 cache rows: one run from row0 (16- and 32-token blocks), or two
            // runs of 8 from row0 and row1 (8-token blocks)
            int row0 = 0, row1 = 0, kvh = 0;
            if (k < nunits) {
                UnitPos up = locate(pfx, p.B, Hu, u0 + k);
                kvh = up.kvh;
                const int32_t *tab = p.block_tables + (size_t)up.b * p.max_blocks;
                if (p.bs == 16) {
                    row0 = cache_row(p, __ldg(tab + up.blk), 0);
                } else if (p.bs == 32) {
                    row0 = cache_row(p, __ldg(tab + (up.blk >> 1)), (up.blk & 1) * 16);
                } else {
                    row0 = cache_row(p, __ldg(tab + 2 * up.blk), 0);
                    const bool second = up.blk + 1 < up.nb ||
                                        (2 * up.blk + 1) * 8 < min(__ldg(p.context_lens + up.b), p.max_tokens);
                    row1 = second ? cache_row(p, __ldg(tab + 2 * up.blk + 1), 0)
                                  : (int)(p.num_blocks * 8 < 0x7fffffffLL ? p.num_blocks * 8 : 0x7fffffff);
                }
            }
            const int n = min(32, nunits - k0);
            for (int j = 0; j < n; ++j) {
                const int ph = __shfl_sync(0xffffffffu, row0, j);
                const int ph1 = __shfl_sync(0xffffffffu, row1, j);
                const int hh = __shfl_sync(0xffffffffu, kvh, j);
                if (lane == 0 && ok) {
                    const int kk = k0 + j, s = kk % NS;
                    const uint32_t parity = ((kk / NS) & 1) ^ 1;
                    if (!mbar_wait_bounded(smem_u32(empty + s), parity, p.err) || abort_s) {
                        ok = false;
                        abort_s = 1;
                    } else {
                        const uint32_t fb = smem_u32(full + s);
                        const uint32_t dst = smem_u32(stages + s * Geo::kStageBytes);
                        mbar_arrive_expect_tx(fb, Geo::kStageBytes);
                        if constexpr (HPU == 2) {
                            // one box per tensor (per slab when swizzled): 16 slots x 2 adjacent
                            // heads, landing as the two heads' tiles (slab-interleaved); never
                            // used with 8-token blocks
#pragma unroll
                            for (int h = 0; h < (kMma ? kSlabs : 1); ++h) {
                                const int x = kMma ? h * (128 / Geo::kElem) : 0;
                                tma_load_3d(dst + h * kSlabStride, &tm_k, fb, x, ph, 2 * hh);
                                tma_load_3d(dst + 2 * Geo::kTileBytes + h * kSlabStride, &tm_v, fb, x, ph, 2 * hh);
                            }
                        } else {
                            // one box per 64-column slab (tensor-core tiles, swizzled) or per row
                            // run; with 8-token blocks each box is 8 rows and a second one fills
                            // rows 8-15 from the next block
                            constexpr int kBoxes = kMma ? kSlabs : 1;
                            constexpr int kBoxStride = kMma ? 2048 : 0;
                            const int pitch = kMma ? 128 : Geo::kRowBytes;  // bytes per row of a box
#pragma unroll
                            for (int h = 0; h < kBoxes; ++h) {
                                const int x = kMma ? h * (128 / Geo::kElem) : 0;
                                const uint32_t dk = dst + h * kBoxStride, dv = dk + Geo::kTileBytes;
                                tma_load_3d(dk, &tm_k, fb, x, hh, ph);
                                tma_load_3d(dv, &tm_v, fb, x, hh, ph);
                                if (p.bs == 8) {
                                    tma_load_3d(dk + 8 * pitch, &tm_k, fb, x, hh, ph1);
                                    tma_load_3d(dv + 8 * pitch, &tm_v, fb, x, hh, ph1);
                                }
                            }
                        }
                        issued_mask |= 1ull << s;
                        issued_phase = (issued_phase & ~(1ull << s)) | ((uint64_t)((kk / NS) & 1) << s);
                    }
                }
                __syncwarp();
            }
        }
        // Drain: never leave the CTA with a TMA copy still landing in its shared memory.
        if (lane == 0) {
            for (int s = 0; s < NS; ++s)
                if ((issued_mask >> s) & 1)
                    mbar_wait_bounded(smem_u32(full + s), (uint32_t)((issued_phase >> s) & 1), p.err);
        }
        return;
    }

    // ---------------------------------------------------------------------- consumers
    const int cw = warp - 1;          // consumer index 0..3
    const int ct = threadIdx.x - 32;  // consumer thread 0..127
    const int cgrp = cw / HPU, hsel = cw % HPU;  // consumer group; head of the unit it serves
    // q.k lane mapping (see the q.k loop): kTPL tokens per lane group of kLPG lanes
    constexpr int kTPL = (G == 2 || G == 4) ? 2 : 1;
    constexpr int kLPG = 2 * kTPL;
    constexpr int kCPL = Geo::kChunks / kLPG;  // 16-byte chunks per lane per row
    static_assert(kCPL >= 1 && (kCPL & (kCPL - 1)) == 0, "chunks per lane: a power of two");
    const int grp = lane / kLPG, sub = lane % kLPG;

    float m[G], l[G], acc[G][Geo::kDimsPerLane];
    // tensor-core path: lane = 4 * row + q4.  The lane's S fragment holds head `row` (valid
    // when row < G) against tokens 2*q4, 2*q4+1, 8+2*q4, 9+2*q4 of the block; its O^T
    // fragment of tile mt holds, for heads 2*q4 and 2*q4+1, dims odim(mt, row) and
    // odim(mt, row + 8):  bf16: 16*mt + r;  E4M3: 16*row + 8*(r >= 8) + mt, so that a lane's
    // V bytes are one contiguous 16-byte chunk of each token row.  (Any permutation of the
    // contracted dims, applied to q and K alike, and of the output dims, undone at the merge,
    // leaves the result unchanged.)
    constexpr int kMT = kMma ? D / 16 : 1;
    const int row = lane >> 2, q4 = lane & 3;
    float mr = -INFINITY, lr = 0.f;
    float o[kMT][4];
    uint32_t qa[kMT][2];

    const uint32_t qs_a = smem_u32(qs);
    const uint32_t pbuf_a = smem_u32(pbuf + cw * G * 16);

    int k = 0;
    UnitPos cur = locate(pfx, p.B, Hu, u0);
    bool dead = false;
    while (k < nunits) {
        // fresh softmax state for this piece
            if constexpr (kMma) {
                mr = -INFINITY;
                lr = 0.f;
    #pragma unroll
                for (int mt = 0; mt < kMT; ++mt)
    #pragma unroll
                    for (int i = 0; i < 4; ++i) o[mt][i] = 0.f;
            } else {
    #pragma unroll
                for (int g = 0; g < G; ++g) {
                    m[g] = -INFINITY;
                    l[g] = 0.f;
    #pragma unroll
                    for (int d = 0; d < Geo::kDimsPerLane; ++d) acc[g][d] = 0.f;
                }
            }
        // piece = the rest of the current (sequence, kv-head group) segment inside this range
        const int piece_len = min(cur.nb - cur.blk, nunits - k);
        const int b = cur.b, kvg = cur.kvh;
        const int kvh = kvg * HPU + hsel;  // this warp's kv head
        // score scale in exp2 units (E4M3: with the head's K scale folded in)
        const float sc_piece = p.scale_log2 * (FP8 ? __ldg(p.k_scale + kvh) : 1.f);
        const int L = min(__ldg(p.context_lens + b), p.max_tokens);
        const bool whole = (cur.blk == 0) && (piece_len == cur.nb);

        // decode step: issue the loads of the new token (if this piece stores it) ahead of q's
        constexpr int kNt = STEP ? (HPU * D / 2 + kConsumers * 32 - 1) / (kConsumers * 32) : 1;
        uint16_t nt_k[kNt][2], nt_v[kNt][2];
        float nt_c[kNt], nt_s[kNt];
        bool nt_has = false;
        int nt_e = -1, nt_lraw = -1;
        if constexpr (STEP) {
            nt_has = cur.blk + piece_len == cur.nb;
            if (nt_has) {
                const int pos = L - 1;
                nt_lraw = __ldg(p.context_lens + b);
                nt_e = __ldg(p.block_tables + (size_t)b * p.max_blocks + pos / p.bs);
                const bool rope_ok = p.rope && pos < p.max_pos;
#pragma unroll
                for (int j = 0; j < kNt; ++j) {
                    const int e2 = ct + j * kConsumers * 32;
                    if (e2 >= HPU * D / 2) break;
                    const int hh = e2 / (D / 2), i = e2 % (D / 2), kvo = kvg * HPU + hh;
                    const uint16_t *kin = p.k_new + ((size_t)b * p.Hkv + kvo) * D;
                    const uint16_t *vin = p.v_new + ((size_t)b * p.Hkv + kvo) * D;
                    nt_k[j][0] = __ldg(kin + i);
                    nt_k[j][1] = __ldg(kin + i + D / 2);
                    nt_v[j][0] = __ldg(vin + i);
                    nt_v[j][1] = __ldg(vin + i + D / 2);
                    if (rope_ok) {
                        nt_c[j] = __ldg(p.rope + (size_t)pos * D + i);
                        nt_s[j] = __ldg(p.rope + (size_t)pos * D + D / 2 + i);
                    }
                }
            }
        }
        // ---- stage q for this (b, kv-head group): rotate (optional), scale, split layout
        for (int e = ct; e < HPU * G * D / 2; e += kConsumers * 32) {
            const int hh = e / (G * D / 2), g = (e / (D / 2)) % G, i = e % (D / 2);
            const int h = (kvg * HPU + hh) * G + g;
            const uint16_t *qr = p.q + ((size_t)b * p.Hq + h) * D;
            uint16_t x1 = __ldg(qr + i), x2 = __ldg(qr + i + D / 2);
            if (p.rope) {
                const int pos = L - 1;
                if (pos >= 0 && pos < p.max_pos) {
                    const float *row = p.rope + (size_t)pos * D;
                    rope_pair_fast(x1, x2, __ldg(row + i), __ldg(row + D / 2 + i), x1, x2);
                } else {
                    atomicOr(p.err, kErrBounds);
                }
            }
            if constexpr (kMma) {
                // rotated bf16 q, [HPU][G][D]; the scale is applied to the fp32 scores
                uint16_t *qh = reinterpret_cast<uint16_t *>(qs) + (hh * G + g) * D;
                qh[i] = x1;
                qh[i + D / 2] = x2;
                continue;
            }
            const float sc = p.scale_log2 * (FP8 ? __ldg(p.k_scale + kvg * HPU + hh) : 1.f);
            const int idx[2] = {i, i + D / 2};
            const float val[2] = {__uint_as_float((uint32_t)x1 << 16) * sc,
                                  __uint_as_float((uint32_t)x2 << 16) * sc};
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int dim = idx[r];
                const int c = dim / Geo::kChunkElems, w = dim % Geo::kChunkElems;
                const int quad = w / 4, comp = w % 4;
                qs[hh * G * D + ((g * Geo::kQuads + quad) * Geo::kChunks + c) * 4 + comp] = val[r];
            }
        }
        bool nt_ok = false;
        if constexpr (STEP) {
            // The step's new token of this group's heads, when this piece holds its sequence's
            // last block (and the context was not clipped to the block table): K rotated at
            // L - 1 and V, converted as the cache stores them (E4M3 codes of the exact quotient
            // by the head's scale, as pkv_kv_store does), go into the cache and into
            // mrg, which is free until the piece's merge.  The warp that takes the last block
            // copies its head's rows from there into its tile, so no global load sits on that
            // warp's path.  (The loads were issued before q's, in nt_*.)
            if (nt_has) {
                const int pos = L - 1;
                const bool rope_ok = !p.rope || pos < p.max_pos;
                if (!rope_ok && ct == 0) atomicOr(p.err, kErrBounds);
                nt_ok = L == nt_lraw && rope_ok && nt_e >= 0 && (long long)nt_e < p.num_blocks;
                if (nt_ok) {
                    const int slot = nt_e * p.bs + pos % p.bs;
                    uint8_t *nt = reinterpret_cast<uint8_t *>(mrg);
#pragma unroll
                    for (int j = 0; j < kNt; ++j) {
                        const int e2 = ct + j * kConsumers * 32;
                        if (e2 >= HPU * D / 2) break;
                        const int hh = e2 / (D / 2), i = e2 % (D / 2), kvo = kvg * HPU + hh;
                        uint16_t kb[2] = {nt_k[j][0], nt_k[j][1]};
                        if (p.rope) rope_pair_fast(kb[0], kb[1], nt_c[j], nt_s[j], kb[0], kb[1]);
                        const size_t dst = ((size_t)slot * p.Hkv + kvo) * D;  // element index
                        uint8_t *krow = nt + 2 * hh * Geo::kRowBytes, *vrow = krow + Geo::kRowBytes;
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int el = i + h * (D / 2);
                            if constexpr (FP8) {
                                const uint32_t kc =
                                    e4m3_of_quotient(__uint_as_float((uint32_t)kb[h] << 16), __ldg(p.k_scale + kvo));
                                const uint32_t vc =
                                    e4m3_of_quotient(__uint_as_float((uint32_t)nt_v[j][h] << 16), __ldg(p.v_scale + kvo));
                                static_cast<uint8_t *>(p.k_cache_w)[dst + el] = (uint8_t)kc;
                                static_cast<uint8_t *>(p.v_cache_w)[dst + el] = (uint8_t)vc;
                                krow[el] = (uint8_t)kc;
                                vrow[el] = (uint8_t)vc;
                            } else {
                                static_cast<uint16_t *>(p.k_cache_w)[dst + el] = kb[h];
                                static_cast<uint16_t *>(p.v_cache_w)[dst + el] = nt_v[j][h];
                                reinterpret_cast<uint16_t *>(krow)[el] = kb[h];
                                reinterpret_cast<uint16_t *>(vrow)[el] = nt_v[j][h];
                            }
                        }
                    }
                }
            }
        }
        named_bar(kMergeBar, kConsumers * 32);
        if constexpr (kMma) {
            // A fragments of Q for every 16-dim k step (zero for rows past the group)
#pragma unroll
            for (int ks = 0; ks < kMT; ++ks) {
                if constexpr (FP8) {
                    // k step ks, quad lane q4: dims 32*q4 + 4*ks + {0,1 | 2,3}, in f16
                    const uint32_t a = qs_a + (uint32_t)(((hsel * G + row) * D + 32 * q4 + 4 * ks) * 2);
                    const uint2 w = row < G ? lds64(a) : make_uint2(0u, 0u);
                    qa[ks][0] = pack_f16x2(bf16lo(w.x), bf16hi(w.x));
                    qa[ks][1] = pack_f16x2(bf16lo(w.y), bf16hi(w.y));
                } else {
                    // k step ks, quad lane q4: dims 16*ks + 2*q4 + {0,1 | 8,9}
                    const uint32_t a = qs_a + (uint32_t)(((hsel * G + row) * D + 16 * ks + 2 * q4) * 2);
                    qa[ks][0] = row < G ? lds32(a) : 0u;
                    qa[ks][1] = row < G ? lds32(a + 16) : 0u;
                }
            }
        }

        // ---- stream this piece's blocks
        for (int j = 0; j < piece_len; ++j, ++k) {
            if ((k % Geo::kGroups) != cgrp) continue;
            const int s = k % NS;
            const uint32_t parity = (k / NS) & 1;
            if (!dead) {
                if (abort_s || !mbar_wait_bounded(smem_u32(full + s), parity, p.err)) {
                    dead = true;
                    abort_s = 1;
                }
            }
            if (dead) continue;
            const int blk = cur.blk + j;
            const int valid = min(kPiece, L - blk * kPiece);
            // this warp's head: K tile hsel, then V tile hsel after the HPU K tiles
            const uint32_t ks_a = smem_u32(stages + s * Geo::kStageBytes) + hsel * kHeadStride;
            const uint32_t vs_a = ks_a + HPU * Geo::kTileBytes;
            if constexpr (STEP) {
                // the sequence's last block holds the step's new token: its rows, staged in
                // mrg with the piece's q, replace the slot's previous contents in the tile
                if (blk == cur.nb - 1 && nt_ok) {
                    const int r = (L - 1) % kPiece;
                    const uint8_t *krow = reinterpret_cast<const uint8_t *>(mrg) + 2 * hsel * Geo::kRowBytes;
                    for (int c = lane; c < Geo::kChunks; c += 32) {  // 16-byte chunks of the row
                        const uint4 kx = *reinterpret_cast<const uint4 *>(krow + 16 * c);
                        const uint4 vx = *reinterpret_cast<const uint4 *>(krow + Geo::kRowBytes + 16 * c);
                        const uint32_t off = kMma ? swz<kSlabStride>(r, c) : (uint32_t)(r * Geo::kRowBytes + 16 * c);
                        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(ks_a + off), "r"(kx.x),
                                     "r"(kx.y), "r"(kx.z), "r"(kx.w) : "memory");
                        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(vs_a + off), "r"(vx.x),
                                     "r"(vx.y), "r"(vx.z), "r"(vx.w) : "memory");
                    }
                    fence_proxy_async_smem();  // before the stage is refilled by TMA
                    __syncwarp();
                }
            }
            if constexpr (kMma) {
                // S = Q K^T: n tile 0 = tokens 0-7, n tile 1 = tokens 8-15.  ldmatrix x4
                // matrices: (tokens 0-7 | 8-15) x (first | second 8 dims of the k step).
                float sa[2][4];
#pragma unroll
                for (int i = 0; i < 4; ++i) sa[0][i] = sa[1][i] = 0.f;
                if constexpr (FP8) {
                    // B fragment of n tile nt: token 8*nt + row, bytes [32*q4, 32*q4 + 32) of
                    // its row (two swizzled chunks), widened to f16 per k step
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        const int t = 8 * nt + row;
                        const uint4 k0 = lds128(ks_a + swz<kSlabStride>(t, 2 * q4));
                        const uint4 k1 = lds128(ks_a + swz<kSlabStride>(t, 2 * q4 + 1));
                        const uint32_t kw[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
#pragma unroll
                        for (int ks = 0; ks < kMT; ++ks)
                            mma_rows8_f16(sa[nt], qa[ks][0], qa[ks][1], e4m3x2_f16x2(kw[ks]),
                                          e4m3x2_f16x2(kw[ks] >> 16));
                    }
                } else {
                    const int tk = ((lane >> 4) << 3) | (lane & 7), hk = (lane >> 3) & 1;
#pragma unroll
                    for (int ks = 0; ks < kMT; ++ks) {
                        uint32_t b[4];
                        ldsm_x4(ks_a + swz<kSlabStride>(tk, 2 * ks + hk), b);
                        mma_rows8(sa[0], qa[ks][0], qa[ks][1], b[0], b[1]);
                        mma_rows8(sa[1], qa[ks][0], qa[ks][1], b[2], b[3]);
                    }
                }
                // online softmax of row `row` over this block (the quad holds its 16 tokens)
                const float sc = sc_piece;
                const int t0 = 2 * q4;
                float sv[4] = {sa[0][0] * sc, sa[0][1] * sc, sa[1][0] * sc, sa[1][1] * sc};
                if (valid < kPiece) {
                    if (t0 >= valid) sv[0] = -INFINITY;
                    if (t0 + 1 >= valid) sv[1] = -INFINITY;
                    if (t0 + 8 >= valid) sv[2] = -INFINITY;
                    if (t0 + 9 >= valid) sv[3] = -INFINITY;
                    // V rows past the sequence are zeroed (0 * NaN would poison O)
                    constexpr int kRowChunks = Geo::kRowBytes / 16;
                    for (int e = lane; e < (kPiece - valid) * kRowChunks; e += 32) {
                        const int t = valid + e / kRowChunks, c = e % kRowChunks;
                        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(vs_a + swz<kSlabStride>(t, c)),
                                     "r"(0u) : "memory");
                    }
                    fence_proxy_async_smem();  // before the stage is refilled by TMA
                    __syncwarp();
                }
                float mt = fmaxf(fmaxf(sv[0], sv[1]), fmaxf(sv[2], sv[3]));
                mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
                mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
                // Lazy rescale: the reference max mr moves only when the block's max exceeds
                // it by more than 2^8 (mt is finite: token 0 of a block is always valid), so
                // P <= 2^8 and O is rescaled only on the rare blocks that move it.
                float alpha = 1.f;
                if (mt > mr + kRescaleLog2) {
                    alpha = ex2(mr - mt);  // 0 on the first block (mr = -inf; O, l are 0)
                    mr = mt;
                }
                float pr[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) pr[i] = ex2(sv[i] - mr);
                lr = lr * alpha + ((pr[0] + pr[1]) + (pr[2] + pr[3]));
                if (__any_sync(0xffffffffu, alpha != 1.f)) {
                    // O^T columns are heads 2*q4, 2*q4+1: their alphas live in lanes 8*q4, 8*q4+4
                    const float al0 = __shfl_sync(0xffffffffu, alpha, 8 * q4);
                    const float al1 = __shfl_sync(0xffffffffu, alpha, 8 * q4 + 4);
#pragma unroll
                    for (int mt2 = 0; mt2 < kMT; ++mt2) {
                        o[mt2][0] *= al0;
                        o[mt2][1] *= al1;
                        o[mt2][2] *= al0;
                        o[mt2][3] *= al1;
                    }
                }
                if constexpr (FP8) {
                    // O^T += V^T P^T in f16.  The A fragment of tile mt needs, at dims
                    // 16*row + mt and 16*row + 8 + mt, tokens 2q4, 2q4+1 (a0a1, a2a3) and
                    // 8+2q4, 9+2q4 (a4a5, a6a7): one 16-byte chunk of each of the four token
                    // rows, regrouped into token pairs by byte permutes, then widened.
                    const uint32_t pb01 = pack_f16x2(pr[0], pr[1]), pb23 = pack_f16x2(pr[2], pr[3]);
                    const int tA = 2 * q4;
                    const uint4 vA = lds128(vs_a + swz<kSlabStride>(tA, row)), vB = lds128(vs_a + swz<kSlabStride>(tA + 1, row));
                    const uint4 vC = lds128(vs_a + swz<kSlabStride>(tA + 8, row)), vD = lds128(vs_a + swz<kSlabStride>(tA + 9, row));
                    const uint32_t wA[4] = {vA.x, vA.y, vA.z, vA.w}, wB[4] = {vB.x, vB.y, vB.z, vB.w};
                    const uint32_t wC[4] = {vC.x, vC.y, vC.z, vC.w}, wD[4] = {vD.x, vD.y, vD.z, vD.w};
#pragma unroll
                    for (int mp = 0; mp < 4; ++mp) {  // m tiles 2mp, 2mp+1 = bytes 2mp, 2mp+1
                        const uint32_t sel = (mp & 1) ? 0x7362u : 0x5140u;  // [x_b, y_b, x_b+1, y_b+1]
                        const uint32_t lo01 = prmt(wA[mp >> 1], wB[mp >> 1], sel);
                        const uint32_t hi01 = prmt(wA[2 + (mp >> 1)], wB[2 + (mp >> 1)], sel);
                        const uint32_t lo23 = prmt(wC[mp >> 1], wD[mp >> 1], sel);
                        const uint32_t hi23 = prmt(wC[2 + (mp >> 1)], wD[2 + (mp >> 1)], sel);
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const uint32_t af[4] = {e4m3x2_f16x2(lo01 >> (16 * e)), e4m3x2_f16x2(hi01 >> (16 * e)),
                                                    e4m3x2_f16x2(lo23 >> (16 * e)), e4m3x2_f16x2(hi23 >> (16 * e))};
                            mma_full_f16(o[2 * mp + e], af, pb01, pb23);
                        }
                    }
                } else {
                    const uint32_t pb01 = pack_bf16x2(pr[0], pr[1]), pb23 = pack_bf16x2(pr[2], pr[3]);
                    // O^T += V^T P^T: ldmatrix.trans matrices (tokens 0-7 | 8-15) x (dims
                    // 16mt..+7 | 16mt+8..+15) give the A fragment; P^T is the S fragment.
                    const int tv = ((lane >> 4) << 3) | (lane & 7), hv = (lane >> 3) & 1;
#pragma unroll
                    for (int mt2 = 0; mt2 < kMT; ++mt2) {
                        uint32_t a[4];
                        ldsm_x4_trans(vs_a + swz<kSlabStride>(tv, 2 * mt2 + hv), a);
                        const uint32_t af[4] = {a[0], a[1], a[2], a[3]};
                        mma_full(o[mt2], af, pb01, pb23);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(empty + s));
                continue;
            }

            // q.k: the 16 tokens form groups of kTPL, each served by kLPG = 2*kTPL lanes; lane
            // `sub` of a group owns chunks sub, sub + kLPG, ... of the row, so one q load
            // feeds kTPL tokens.  Groups start at different chunks (rotation by group), which
            // keeps every 8-lane phase of the shared-memory loads conflict-free.
            float2 sacc[G][kTPL];
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int u = 0; u < kTPL; ++u) sacc[g][u] = make_float2(0.f, 0.f);
#pragma unroll
            for (int mi = 0; mi < kCPL; ++mi) {
                const int mm = (mi + grp) & (kCPL - 1);
                const int c = sub + kLPG * mm;
                float kf[kTPL][Geo::kChunkElems];
#pragma unroll
                for (int u = 0; u < kTPL; ++u) {
                    const uint4 kr = lds128(ks_a + (grp * kTPL + u) * Geo::kRowBytes + c * 16);
                    const uint32_t w4[4] = {kr.x, kr.y, kr.z, kr.w};
                    if constexpr (FP8) {
#pragma unroll
                        for (int wi = 0; wi < 4; ++wi) {
#pragma unroll
                            for (int hb = 0; hb < 2; ++hb) {
                                uint32_t h2;
                                const uint16_t pair = (uint16_t)(w4[wi] >> (16 * hb));
                                asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(pair));
                                const float2 f = __half22float2(*reinterpret_cast<__half2 *>(&h2));
                                kf[u][wi * 4 + hb * 2 + 0] = f.x;
                                kf[u][wi * 4 + hb * 2 + 1] = f.y;
                            }
                        }
                    } else {
#pragma unroll
                        for (int wi = 0; wi < 4; ++wi) {
                            kf[u][2 * wi] = bf16lo(w4[wi]);
                            kf[u][2 * wi + 1] = bf16hi(w4[wi]);
                        }
                    }
                }
#pragma unroll
                for (int g = 0; g < G; ++g) {
#pragma unroll
                    for (int qd = 0; qd < Geo::kQuads; ++qd) {
                        const float4 qv = lds128f(qs_a + hsel * G * D * 4 +
                                                  (((g * Geo::kQuads + qd) * Geo::kChunks + c) * 16));
#pragma unroll
                        for (int u = 0; u < kTPL; ++u) {
                            sacc[g][u] = __ffma2_rn(make_float2(kf[u][4 * qd + 0], kf[u][4 * qd + 1]),
                                                    make_float2(qv.x, qv.y), sacc[g][u]);
                            sacc[g][u] = __ffma2_rn(make_float2(kf[u][4 * qd + 2], kf[u][4 * qd + 3]),
                                                    make_float2(qv.z, qv.w), sacc[g][u]);
                        }
                    }
                }
            }
            // softmax update for this block: after the group reduction every lane of a group
            // holds its kTPL tokens' scores
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float sc[kTPL];
                float mt = -INFINITY;
#pragma unroll
                for (int u = 0; u < kTPL; ++u) {
                    float v = sacc[g][u].x + sacc[g][u].y;
#pragma unroll
                    for (int o = 1; o < kLPG; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                    sc[u] = (grp * kTPL + u < valid) ? v : -INFINITY;
                    mt = fmaxf(mt, sc[u]);
                }
#pragma unroll
                for (int o = kLPG; o < 32; o <<= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o));
                const float mn = fmaxf(m[g], mt);
                const float alpha = ex2(m[g] - mn);
                float ls = 0.f;
#pragma unroll
                for (int u = 0; u < kTPL; ++u) {
                    const float pj = ex2(sc[u] - mn);
                    if (sub == 0) {
                        pbuf[cw * G * 16 + g * 16 + grp * kTPL + u] = pj;
                        ls += pj;
                    }
                }
                l[g] = l[g] * alpha + ls;
                m[g] = mn;
#pragma unroll
                for (int d = 0; d < Geo::kDimsPerLane; ++d) acc[g][d] *= alpha;
            }
            __syncwarp();
            // p.v: lane owns dims [lane*DPL, (lane+1)*DPL)
            constexpr int DPL = Geo::kDimsPerLane;
            static_assert(DPL == 2 || DPL == 4 || DPL == 8, "head dim 64, 128 or 256");
            auto pv_row = [&](int jj, const float *pw) {
                float vf[DPL];
                const uint32_t va = vs_a + jj * Geo::kRowBytes + lane * DPL * Geo::kElem;
                if constexpr (FP8) {
                    if constexpr (DPL == 8) {
                        const uint2 w2 = lds64(va);
                        const uint32_t ww[2] = {w2.x, w2.y};
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            uint32_t h2;
                            const uint16_t pair = (uint16_t)(ww[q >> 1] >> (16 * (q & 1)));
                            asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(pair));
                            float2 f = __half22float2(*reinterpret_cast<__half2 *>(&h2));
                            vf[2 * q] = f.x;
                            vf[2 * q + 1] = f.y;
                        }
                    } else if constexpr (DPL == 4) {
                        const uint32_t w = lds32(va);
#pragma unroll
                        for (int hb = 0; hb < 2; ++hb) {
                            uint32_t h2;
                            const uint16_t pair = (uint16_t)(w >> (16 * hb));
                            asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(pair));
                            float2 f = __half22float2(*reinterpret_cast<__half2 *>(&h2));
                            vf[2 * hb] = f.x;
                            vf[2 * hb + 1] = f.y;
                        }
                    } else {
                        uint16_t pair;
                        asm volatile("ld.shared.u16 %0, [%1];" : "=h"(pair) : "r"(va));
                        uint32_t h2;
                        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(pair));
                        float2 f = __half22float2(*reinterpret_cast<__half2 *>(&h2));
                        vf[0] = f.x;
                        vf[1] = f.y;
                    }
                } else {
                    if constexpr (DPL == 8) {
                        const uint4 w = lds128(va);
                        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            vf[2 * q] = bf16lo(ww[q]);
                            vf[2 * q + 1] = bf16hi(ww[q]);
                        }
                    } else if constexpr (DPL == 4) {
                        const uint2 w = lds64(va);
                        vf[0] = bf16lo(w.x);
                        vf[1] = bf16hi(w.x);
                        vf[2] = bf16lo(w.y);
                        vf[3] = bf16hi(w.y);
                    } else {
                        const uint32_t w = lds32(va);
                        vf[0] = bf16lo(w);
                        vf[1] = bf16hi(w);
                    }
                }
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float pg = pw[g];
#pragma unroll
                    for (int d = 0; d < DPL; d += 2) {
                        float2 r = __ffma2_rn(make_float2(pg, pg), make_float2(vf[d], vf[d + 1]),
                                              make_float2(acc[g][d], acc[g][d + 1]));
                        acc[g][d] = r.x;
                        acc[g][d + 1] = r.y;
                    }
                }
            };
            if (valid == kPiece) {
#pragma unroll
                for (int j4 = 0; j4 < kPiece; j4 += 4) {
                    float4 pq[G];
#pragma unroll
                    for (int g = 0; g < G; ++g) pq[g] = lds128f(pbuf_a + (g * 16 + j4) * 4);
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        float pw[G];
#pragma unroll
                        for (int g = 0; g < G; ++g)
                            pw[g] = jj == 0 ? pq[g].x : jj == 1 ? pq[g].y : jj == 2 ? pq[g].z : pq[g].w;
                        pv_row(j4 + jj, pw);
                    }
                }
            } else {
                for (int jj = 0; jj < valid; ++jj) {
                    float pw[G];
#pragma unroll
                    for (int g = 0; g < G; ++g) pw[g] = pbuf[cw * G * 16 + g * 16 + jj];
                    pv_row(jj, pw);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(empty + s));
        }

        // ---- merge the four consumer warps' states for this piece
        if constexpr (STEP) {
            // mrg still holds the staged new-token rows until every warp is past its blocks
            if (nt_ok) named_bar(kMergeBar, kConsumers * 32);
        }
        if constexpr (kMma) {
            float lw = lr;
            lw += __shfl_xor_sync(0xffffffffu, lw, 1);
            lw += __shfl_xor_sync(0xffffffffu, lw, 2);
            if (row < G && q4 == 0) {
                float *mw = mrg + (cw * G + row) * (D + 2);
                mw[D] = mr;
                mw[D + 1] = lw;
            }
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int g = 2 * q4 + hh;
                if (g < G) {
                    float *mw = mrg + (cw * G + g) * (D + 2);
#pragma unroll
                    for (int mt = 0; mt < kMT; ++mt) {
                        const int d0 = FP8 ? 16 * row + mt : 16 * mt + row;
                        mw[d0] = o[mt][hh];
                        mw[d0 + 8] = o[mt][2 + hh];
                    }
                }
            }
        }
        if constexpr (!kMma) {
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float lw = l[g];
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) lw += __shfl_xor_sync(0xffffffffu, lw, o);
                float *mw = mrg + (cw * G + g) * (D + 2);
                if (lane == 0) {
                    mw[D] = m[g];
                    mw[D + 1] = lw;
                }
#pragma unroll
                for (int d = 0; d < Geo::kDimsPerLane; ++d) mw[lane * Geo::kDimsPerLane + d] = acc[g][d];
            }
        }
        named_bar(kMergeBar, kConsumers * 32);
        // warps w with w % HPU == hd hold head hd of the group; partial slots are
        // HPU * (segment + CTA) + hd, distinct for every (segment, CTA, head)
        const int segu = b * Hu + kvg;
        for (int e = ct; e < HPU * G * D; e += kConsumers * 32) {
            const int hd = e / (G * D), g = (e / D) % G, d = e % D;
            const int kvo = kvg * HPU + hd;
            float M = -INFINITY;
#pragma unroll
            for (int w = hd; w < kConsumers; w += HPU) M = fmaxf(M, mrg[(w * G + g) * (D + 2) + D]);
            float o = 0.f, lsum = 0.f;
#pragma unroll
            for (int w = hd; w < kConsumers; w += HPU) {
                const float *mw = mrg + (w * G + g) * (D + 2);
                const float f = (mw[D] == -INFINITY) ? 0.f : ex2(mw[D] - M);
                o += f * mw[d];
                lsum += f * mw[D + 1];
            }
            if (whole) {
                const float vs = FP8 ? __ldg(p.v_scale + kvo) : 1.f;
                const float r = (lsum > 0.f) ? o / lsum * vs : 0.f;
                p.out[((size_t)b * p.Hq + kvo * G + g) * D + d] = __float2bfloat16_rn(r);
            } else {
                float *slot = p.partials + (size_t)(HPU * (segu + blockIdx.x) + hd) * (G * (D + 2));
                slot[g * D + d] = o;
                if (d == 0) {
                    slot[G * D + g] = M;
                    slot[G * D + G + g] = lsum;
                }
            }
        }
        if (STEP && !whole) __threadfence();  // partials visible before this CTA's arrival
        named_bar(kMergeBar, kConsumers * 32);
        if constexpr (STEP) {
            if (!whole) {
                // The CTAs c0..c1 whose ranges cut this segment each add one arrival; the last
                // to arrive merges their partials (as the combine kernel does) and clears
                // the counter for the next call.
                const long long start = (long long)Hu * pfx[b] + (long long)kvg * cur.nb;
                const int c0 = (int)(start / U), c1 = (int)((start + cur.nb - 1) / U);
                if (ct == 0) last_s = (atomicAdd(p.counters + segu, 1) == c1 - c0) ? 1 : 0;
                named_bar(kMergeBar, kConsumers * 32);
                if (last_s) {
                    __threadfence();
                    for (int e = ct; e < HPU * G * D; e += kConsumers * 32) {
                        const int hd = e / (G * D), g = (e / D) % G, d = e % D;
                        const int kvo = kvg * HPU + hd;
                        const float vsc = FP8 ? __ldg(p.v_scale + kvo) : 1.f;
                        p.out[((size_t)b * p.Hq + kvo * G + g) * D + d] =
                            __float2bfloat16_rn(merge_partials<D, G, HPU>(p, segu, hd, g, d, c0, c1, vsc));
                    }
                    if (ct == 0) p.counters[segu] = 0;
                }
                named_bar(kMergeBar, kConsumers * 32);
            }
        }
        // advance to the next segment
        cur.blk += piece_len;
        if (cur.blk >= cur.nb && k < nunits) cur = locate(pfx, p.B, Hu, u0 + k);
    }
}

// Merge the partial states of every (sequence, kv head) that was split across CTAs.
// A segment is split iff some CTA boundary c*U falls strictly inside it; the CTA of the
// first such boundary merges it (one CTA per decode CTA, most have nothing to do).
__device__ __forceinline__ int find_seq_global(const int *pfx, int B, int Hkv, long long u) {
    int lo = 0, hi = B - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if ((long long)Hkv * __ldg(pfx + mid) <= u) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

template <int D, int G, int HPU>
__global__ void __launch_bounds__(128) combine_kernel(const DecodeParams p) {
    constexpr int kSmemPfx = 4096;  // sequences whose prefix is searched in shared memory
    __shared__ int spfx[kSmemPfx];
    pdl_wait();
    pdl_trigger();
    const int c = blockIdx.x;
    const int Hu = p.Hkv / HPU;
    const long long total = (long long)Hu * __ldg(p.prefix + p.B);
    if (c == 0 || total == 0) return;
    const long long U = (total + p.nctas - 1) / p.nctas;
    const long long x = (long long)c * U;
    if (x >= total) return;
    // the segment holding boundary x: one coalesced copy of the prefix, then a search in
    // shared memory (the search in global memory would chain a load per step)
    int b;
    if (p.B + 1 <= kSmemPfx) {
        for (int i = threadIdx.x; i <= p.B; i += blockDim.x) spfx[i] = __ldg(p.prefix + i);
        __syncthreads();
        b = find_seq(spfx, p.B, Hu, x);
    } else {
        b = find_seq_global(p.prefix, p.B, Hu, x);
    }
    const int pb = __ldg(p.prefix + b), nb = __ldg(p.prefix + b + 1) - pb;
    const int kvg = (int)((x - (long long)Hu * pb) / nb);
    const long long start = (long long)Hu * pb + (long long)kvg * nb;
    if (start == x) return;                          // boundary at a segment start: no split
    const int c0 = (int)(start / U), c1 = (int)((start + nb - 1) / U);
    if (c0 != c - 1) return;                         // an earlier boundary's CTA merges it
    const int segu = b * Hu + kvg;
    // four dims per thread, every load of a thread issued before it is used; the arithmetic
    // is merge_partials' for each dim (the same order, so the same rounding).  A slot holds
    // G * (D + 2) floats, so slots start on 16 bytes only when that is a multiple of 4.
    for (int e4 = threadIdx.x; e4 < HPU * G * D / 4; e4 += blockDim.x) {
        const int e = 4 * e4;
        const int hd = e / (G * D), g = (e / D) % G, d = e % D;
        const int kvo = kvg * HPU + hd;
        float M = -INFINITY;
        for (int cc = c0; cc <= c1; ++cc)
            M = fmaxf(M, __ldcg(p.partials + (size_t)(HPU * (segu + cc) + hd) * (G * (D + 2)) + G * D + g));
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
        float lsum = 0.f;
        for (int cc = c0; cc <= c1; ++cc) {
            const float *slot = p.partials + (size_t)(HPU * (segu + cc) + hd) * (G * (D + 2));
            const float mk = __ldcg(slot + G * D + g);
            const float f = (mk == -INFINITY) ? 0.f : ex2(mk - M);
            float4 a;
            if constexpr ((G * (D + 2)) % 4 == 0) {  // slots 16-byte aligned: one vector load
                a = __ldcg(reinterpret_cast<const float4 *>(slot + g * D + d));
            } else {
                a = make_float4(__ldcg(slot + g * D + d), __ldcg(slot + g * D + d + 1), __ldcg(slot + g * D + d + 2),
                                __ldcg(slot + g * D + d + 3));
            }
            o.x += f * a.x;
            o.y += f * a.y;
            o.z += f * a.z;
            o.w += f * a.w;
            lsum += f * __ldcg(slot + G * D + G + g);
        }
        const float vsc = p.v_scale ? __ldg(p.v_scale + kvo) : 1.f;
        const bool any = lsum > 0.f;
        uint2 w;
        w.x = pack_bf16x2(any ? o.x / lsum * vsc : 0.f, any ? o.y / lsum * vsc : 0.f);
        w.y = pack_bf16x2(any ? o.z / lsum * vsc : 0.f, any ? o.w / lsum * vsc : 0.f);
        *reinterpret_cast<uint2 *>(p.out + ((size_t)b * p.Hq + kvo * G + g) * D + d) = w;
    }
}

template <int D, bool FP8, int G, int HPU>
size_t smem_bytes(int B) {
    using Geo = Geometry<D, FP8, G, HPU>;
    constexpr int kConsumers = Geo::kConsumers;
    size_t s = (size_t)Geo::kStages * Geo::kStageBytes + 2 * Geo::kStages * sizeof(uint64_t);
    s += (size_t)Geo::kQFloats * 4 + (size_t)kConsumers * G * 16 * 4 + (size_t)kConsumers * G * (D + 2) * 4;
    s += (size_t)(B + 1) * 4;
    return s + 1024;  // alignment slack for the swizzled stages
}

// Per device, per instantiation: the dynamic shared-memory limit is raised once to the
// device's opt-in maximum, and the occupancy is computed once per 4 KB step of the
// sequence-prefix size (the only part of the shared memory that depends on the call).
constexpr int kMaxDev = 64;
constexpr int kPrefixBuckets = 64;  // 1024 sequences per bucket

template <int D, bool FP8, int G, int HPU, bool STEP>
cudaError_t launch_t(const DecodeParams &prm, const DecodeArgs &a, int dev, cudaStream_t s) {
    using Geo = Geometry<D, FP8, G, HPU>;
    auto kern = decode_kernel<D, FP8, G, HPU, STEP>;
    constexpr int kThreads = Geo::kThreads;
    // largest dynamic shared-memory size allowed so far (the limit only ever grows)
    static std::atomic<int> attr_smem[kMaxDev];
    static std::mutex attr_mu;
    static std::atomic<int> occ_cache[kMaxDev][kPrefixBuckets];  // occupancy + 1; 0 = unknown
    const int bucket = (a.num_seqs + 1 + 1023) / 1024;           // prefix ints, rounded up
    const size_t smem = smem_bytes<D, FP8, G, HPU>(bucket * 1024 - 1);
    // (static shared memory counts against the same per-block limit)
    if (smem + 2048 > (size_t)max_optin_smem(dev)) return cudaErrorNotSupported;  // too many sequences
    if ((size_t)attr_smem[dev].load(std::memory_order_acquire) < smem) {
        std::lock_guard<std::mutex> lock(attr_mu);
        if ((size_t)attr_smem[dev].load(std::memory_order_relaxed) < smem) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
            attr_smem[dev].store((int)smem, std::memory_order_release);
        }
    }
    int occ = bucket < kPrefixBuckets ? occ_cache[dev][bucket].load(std::memory_order_relaxed) - 1 : -1;
    if (occ < 0) {
        cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kThreads, smem);
        if (e != cudaSuccess) return e;
        if (bucket < kPrefixBuckets) occ_cache[dev][bucket].store(occ + 1, std::memory_order_relaxed);
    }
    if (occ < 1) return cudaErrorNotSupported;
    DecodeParams lp = prm;
    lp.nctas = std::min(prm.nctas / kMaxCtasPerSm * Geo::kCtasPerSm, occ * (prm.nctas / kMaxCtasPerSm));
    // K/V maps with exactly the boxes the kernel's producer issues.
    //   CUDA-core consumers: one box per tile, a whole 16-token block of one kv head.
    //   Tensor-core consumers: one 128-byte-swizzled box per 64-column slab.
    //   Two heads per unit: dims listed (column, slot, head) so that one box of 16 slots x 2
    //   heads lands as the two heads' tiles back to back, fetched 256 bytes at a time.
    CUtensorMap tk, tv;
    const uint64_t slots = (uint64_t)a.num_blocks * a.block_size;
    const uint32_t box_rows = a.block_size == 8 ? 8u : (uint32_t)kPiece;
    constexpr bool kMma = Geo::kMma;
    bool ok;
    if constexpr (HPU == 2) {
        const uint64_t row = (uint64_t)a.n_kv_heads * D * Geo::kElem, head = (uint64_t)D * Geo::kElem;
        const uint32_t box0 = kMma ? 128u / Geo::kElem : (uint32_t)D;
        ok = encode_tensor_map_3d_strided(&tk, a.k_cache, Geo::kElem, D, slots, a.n_kv_heads, row, head,
                                          box0, box_rows, 2, kMma, 256) &&
             encode_tensor_map_3d_strided(&tv, a.v_cache, Geo::kElem, D, slots, a.n_kv_heads, row, head,
                                          box0, box_rows, 2, kMma, 256);
    } else {
        const uint32_t box0 = kMma ? 128u / Geo::kElem : (uint32_t)D;
        ok = encode_tensor_map_3d(&tk, a.k_cache, Geo::kElem, D, a.n_kv_heads, slots, box0, 1, box_rows, kMma) &&
             encode_tensor_map_3d(&tv, a.v_cache, Geo::kElem, D, a.n_kv_heads, slots, box0, 1, box_rows, kMma);
    }
    if (!ok) return cudaErrorUnknown;
    static_assert(kPiece * D * Geo::kElem == Geo::kTileBytes, "one head's box fills one tile");
    const size_t smem_call = smem_bytes<D, FP8, G, HPU>(a.num_seqs);
    cudaError_t e = launch_pdl(kern, dim3(lp.nctas), dim3(kThreads), smem_call, s, tk, tv, lp);
    if (e != cudaSuccess || STEP) return e;
    DecodeParams cp = lp;
    cp.v_scale = FP8 ? a.v_scale : nullptr;
    return launch_pdl(combine_kernel<D, G, HPU>, dim3(lp.nctas), dim3(128), 0, s, cp);
}

template <int D, bool FP8, int G, bool STEP>
cudaError_t launch_h(const DecodeParams &prm, const DecodeArgs &a, int dev, cudaStream_t s) {
    // Two adjacent kv heads per unit (longer contiguous rows) when the kv-head count is even,
    // for the CUDA-core consumers and for tensor-core tiles of one 128-byte slab.  Measured:
    // MHA bf16 D 128 5.90 -> 6.12 TB/s, E4M3 grouped 3.8 -> 4.1 TB/s; bf16 grouped D 128
    // (two slabs per row) loses ring depth and ran 15 % slower, so it keeps one head.
    constexpr bool kTwo = !Geometry<D, FP8, G, 1>::kMma || D * (FP8 ? 1 : 2) <= 128;
    if constexpr (kTwo)
        if (a.n_kv_heads % 2 == 0 && a.block_size != 8) return launch_t<D, FP8, G, 2, STEP>(prm, a, dev, s);
    return launch_t<D, FP8, G, 1, STEP>(prm, a, dev, s);
}

template <int D, bool FP8, bool STEP>
cudaError_t launch_g(const DecodeParams &prm, const DecodeArgs &a, int dev, cudaStream_t s) {
    switch (a.n_q_heads / a.n_kv_heads) {
        case 1: return launch_h<D, FP8, 1, STEP>(prm, a, dev, s);
        case 2: return launch_h<D, FP8, 2, STEP>(prm, a, dev, s);
        case 4: return launch_h<D, FP8, 4, STEP>(prm, a, dev, s);
        case 8: return launch_h<D, FP8, 8, STEP>(prm, a, dev, s);
        default: return cudaErrorInvalidValue;
    }
}

size_t align16(size_t x) { return (x + 15) & ~size_t(15); }

// Kernel parameters from the checked arguments, and dispatch on head dim, cache type and
// group size.  STEP: the decode step (new token stored, partials merged in-kernel).
template <bool STEP>
cudaError_t dispatch_decode(const DecodeArgs &a, cudaStream_t s) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
    const int sms = device_sm_count(dev);
    if (a.num_seqs == 0) return cudaSuccess;
    DecodeParams prm;
    prm.out = static_cast<__nv_bfloat16 *>(a.out);
    prm.q = static_cast<const uint16_t *>(a.q);
    prm.block_tables = a.block_tables;
    prm.max_blocks = a.max_blocks_per_seq;
    prm.context_lens = a.context_lens;
    prm.B = a.num_seqs;
    prm.Hq = a.n_q_heads;
    prm.Hkv = a.n_kv_heads;
    prm.num_blocks = a.num_blocks;
    prm.bs = a.block_size;
    prm.max_tokens = (int)std::min<long long>((long long)a.max_blocks_per_seq * a.block_size, 0x7fffffffLL);
    prm.scale_log2 = a.scale * kLog2e;
    prm.k_scale = a.k_scale;
    prm.v_scale = a.v_scale;
    prm.rope = a.rope;
    prm.max_pos = a.max_pos;
    prm.prefix = static_cast<int *>(a.workspace);
    const size_t prefix_bytes = align16((size_t)(a.num_seqs + 1) * sizeof(int));
    prm.partials = reinterpret_cast<float *>(static_cast<uint8_t *>(a.workspace) + prefix_bytes);
    prm.nctas = sms * kMaxCtasPerSm;
    prm.err = a.err;
    prm.k_new = static_cast<const uint16_t *>(a.k_new);
    prm.v_new = static_cast<const uint16_t *>(a.v_new);
    prm.k_cache_w = a.k_cache_w;
    prm.v_cache_w = a.v_cache_w;
    prm.counters = nullptr;
    if (STEP) {
        // counters follow the attention workspace
        const int G = a.n_q_heads / a.n_kv_heads;
        const size_t slots = (size_t)a.num_seqs * a.n_kv_heads + 2 * (size_t)prm.nctas;
        prm.counters = reinterpret_cast<int *>(static_cast<uint8_t *>(a.workspace) + prefix_bytes +
                                               slots * (size_t)G * (a.head_dim + 2) * sizeof(float));
    }
    if (a.head_dim == 128)
        return a.fp8 ? launch_g<128, true, STEP>(prm, a, dev, s) : launch_g<128, false, STEP>(prm, a, dev, s);
    if (a.head_dim == 256)
        return a.fp8 ? launch_g<256, true, STEP>(prm, a, dev, s) : launch_g<256, false, STEP>(prm, a, dev, s);
    if (a.head_dim == 64)
        return a.fp8 ? launch_g<64, true, STEP>(prm, a, dev, s) : launch_g<64, false, STEP>(prm, a, dev, s);
    return cudaErrorInvalidValue;
}

}  // namespace
}  // namespace pkv
