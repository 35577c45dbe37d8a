// decode_tc.cu -- paged decode attention of grouped query heads over an E4M3 cache on the
// 5th-generation tensor cores (tcgen05.mma kind::f8f6f4).
//
// "Inside the Nano-vLLM engine: KV cache, attention and tensor parallelism", §3 (one query
// token per sequence against the cached K/V), §3.1 (tiles, softmax kept on chip), §3.2
// (subtract the maximum); "LLM primer", §17.1 (decode is bound by memory bandwidth) and
// §17.6 (an FP8 cache halves the bytes per token).  The result is that of decode_kernel;
// what differs is how the arithmetic reaches the hardware.
//
// Work: persistent CTAs (one per SM) split the units -- 128-token tiles of one (sequence,
// pair of adjacent kv heads), numbered sequence-major -- into contiguous ranges of equal cost
// (stream-K, a segment's first tile costing a little more); a range's run of tiles of one
// segment is a piece with one softmax state per head.  A segment cut by several CTAs is
// merged, in the combine kernel's arithmetic, by whichever of them finishes its piece last.
//
// Why pairs of heads: a TMA box costs the copy engine about the same up to several KB, and
// one box of 16 tokens of two adjacent heads (their rows sit side by side in the cache) is
// 4 KB where one head's is 2 KB, so the producer issues half as many boxes per byte.  The
// cache is read through a 4-D map (dim, slot % 8, head, slot / 8): a box lands as
// [slot / 8][head][slot % 8][128 bytes], so each head's rows form 8-row, 1024-byte swizzle
// atoms 2048 bytes apart -- a canonical K-major operand (K) and MN-major operand (V).
//   warp 0      TMA producer of K: a tile's K boxes (one lane per box) into a 2-slot ring of
//               32 KB slots, each freed when its S^T MMAs complete
//   warp 15     TMA producer of V: the same for V (3 slots), each freed when its PV completes
//               (K's slots turn over long before V's, so neither waits for the other)
//   warp 1      TMEM owner; lane 0 issues the S^T MMAs
//   warps 2-5   128 softmax threads, thread t = token t of the tile = TMEM lane t
//   warp 6      lane 0 issues the PV MMAs
//   warps 7, 12-14  q stagers (piece i to stager i % 4): each piece's q (rotated, scaled,
//               split), its context length and scales, and (decode step) its new token
//   warps 8-11  epilogue, thread = dim: O of a finished piece -> output rows or partial slots
// Per tile, for each head h of the pair:
//   S^T = K Q^T   M = 128 tokens, N = 16, K = 128 dims (4 MMAs of 32): A = head h's K rows
//                 as the cache stores them (K-major), B = q as E4M3 rows -- the G heads'
//                 high parts in rows 0..G-1, their low parts (the E4M3 remainder) in rows
//                 G..2G-1, zeros after -- so one MMA yields both partial scores of every head.
//   softmax       thread t adds its two parts, masks past the context, updates the lazy
//                 running max (O is rescaled only when a max grows by more than 2^8) and
//                 writes p as high and low E4M3 parts into a shared-memory P tile: row g /
//                 8+g, byte t.
//   O^T += V^T P^T  M = 128 dims, N = 16, K = 128 tokens: A = head h's V rows read MN-major,
//                 B = the P tile's 16 rows (K-major), so column g of O^T gathers the high
//                 parts and column 8+g the low parts; the epilogue adds the two.
// S^T and PV are issued by two threads, each waiting only for its own inputs, so a K slot goes
// back to its producer as soon as its S^T completes, a V slot as soon as its PV does, and S^T
// of later tiles runs ahead.  TMEM:
// S^T buffers of 32 columns (16 per head) at 0..127, O^T buffers of 32 columns at 128..223.
#include <random>

#include "decode_kernel.cuh"
#include "tcgen05.cuh"

namespace pkv {
namespace {

constexpr int kTcThreads = 512;
constexpr int kTcVWarp = 15;    // the V producer
constexpr int kTcPvWarp = 6;    // the PV issuer
constexpr int kTcStagers = 4;   // q stagers (warps 7, 12, 13, 14): stager i takes pieces i, i+4, ...
__device__ __forceinline__ int tc_stager_index(int warp) { return warp == 7 ? 0 : (warp >= 12 && warp <= 14 ? warp - 11 : -1); }
constexpr int kTcEpiWarp = 8;   // the epilogue: warps 8-11, one per TMEM lane quarter (O^T rows = dims)
constexpr int kTcEpiBar = 2;    // named barrier of the 128 epilogue threads
constexpr int kTcHP = 2;        // kv heads per unit
constexpr int kTcTile = 128;    // tokens per unit
constexpr int kTcKSlots = 2;    // K ring slots (32 KB each): a K slot is free once its S^T completes
constexpr int kTcVSlots = 3;    // V ring slots (32 KB each): a V slot is held until its PV completes
constexpr int kTcQBufs = 8;     // q buffers: the stagers run up to this many pieces ahead
constexpr int kTcSBufs = 4;     // S^T buffers in TMEM
constexpr int kTcPBufs = 4;     // P tiles in shared memory
constexpr int kTcSoftmax0 = 2;  // first softmax warp
constexpr int kTcBar = 1;       // named barrier of the 128 softmax threads
constexpr int kTcOBufs = 3;     // O buffers (and stats slots): the epilogue may lag two pieces
constexpr uint32_t kTcSCols = 16 * kTcHP;             // TMEM columns of one S^T (or O^T) buffer
constexpr uint32_t kTcO = kTcSCols * kTcSBufs;        // TMEM column of O^T buffer 0
constexpr uint32_t kTcCols = 256;                     // TMEM columns allocated (a power of two)
static_assert(kTcO + kTcSCols * kTcOBufs <= kTcCols, "TMEM plan");

// What the q stager knows of a piece, for the softmax warps.
struct TcMeta {
    int b, hp, tile, ntiles, piece_len, L;
    float sc[kTcHP];  // score scale in exp2 units, over the q scale: scale * log2(e) * k_scale / sq
    float vs[kTcHP];  // the heads' V scales
    int nt_row;       // decode step: tile row of the new token staged in the slot's codes, or -1
    int pad;
};

// What the softmax hands the epilogue per piece: the piece and its per-head (m, l).
struct TcStats {
    float m[kTcHP][8], l[kTcHP][8];
    int b, hp, ntiles, whole, piece_len;
    float vs[kTcHP];
    int pad;
};

template <int G>
struct TcGeo {
    static constexpr int D = 128;
    static constexpr int kHead = kTcTile * D;       // one head's E4M3 K (or V) tile: 16 KB
    static constexpr int kKV = kTcHP * kHead;       // the pair's K (or V): 32 KB, one ring slot
    static constexpr int kOffV = kTcKSlots * kKV;   // the V ring follows the K ring
    static constexpr int kQ1 = 16 * 128;            // B operand of one head's S^T: 16 rows x 128 codes
    static constexpr int kQ = kTcHP * kQ1;
    // B operand of one head's PV: p's high parts in rows 0..G-1, its low parts in rows
    // 8..8+G-1, zeros in the other rows; 16 rows x 128 tokens
    static constexpr int kP1 = 16 * 128;
    static constexpr int kP = kTcHP * kP1;
    static constexpr int kOffQ = (kTcKSlots + kTcVSlots) * kKV;
    static constexpr int kOffP = kOffQ + kTcQBufs * kQ;
    static constexpr int kOffRed = kOffP + kTcPBufs * kP;          // [4 warps][16] maxima, then sums
    static constexpr int kOffStats = kOffRed + 2 * 4 * 16 * 4;     // [kTcOBufs] TcStats
    static constexpr int kOffMeta = kOffStats + kTcOBufs * (int)sizeof(TcStats);  // [kTcQBufs] TcMeta
    static constexpr int kOffNew = kOffMeta + kTcQBufs * (int)sizeof(TcMeta);     // [q buffer][head][256] new-token codes
    // per P buffer: the tile's valid token count and (decode step) the new token's row, then
    // its V codes for both heads, handed from the softmax to the PV warp with the P tile
    static constexpr int kOffPvInfo = kOffNew + kTcQBufs * kTcHP * 256;            // [kTcPBufs] int2
    static constexpr int kOffPvCodes = kOffPvInfo + kTcPBufs * 8;                   // [kTcPBufs][head][128]
    static constexpr int kOffBar = kOffPvCodes + kTcPBufs * kTcHP * 128;
    static constexpr int kBars = 2 * kTcKSlots + 2 * kTcVSlots + 2 * kTcSBufs + 2 * kTcPBufs + 2 * kTcQBufs + 3 * kTcOBufs + 1;
    static constexpr int kOffPfx = kOffBar + 8 * kBars + 16;
    static_assert(kOffQ % 1024 == 0 && kOffP % 1024 == 0, "swizzled operands on 1024-byte boundaries");
    static_assert(kOffBar % 8 == 0 && kOffNew % 16 == 0 && kOffPvCodes % 16 == 0, "mbarriers and code rows aligned");
    static_assert(2 * G <= 16, "q high and low rows fit the 16 rows of the B operand");
};

// Shared-memory bytes of the [B + 1] tile prefix (the CTAs' first units follow, 8-byte aligned).
__host__ __device__ constexpr int tc_pfx_bytes(int B) { return ((B + 1) * 4 + 7) & ~7; }

// Barrier indices (8 bytes each after kOffBar)
constexpr int kBKFull = 0;                       // [kTcKSlots]  K landed (TMA bytes)
constexpr int kBKEmpty = kTcKSlots;              // [kTcKSlots]  K consumed (S^T commit)
constexpr int kBVFull = 2 * kTcKSlots;           // [kTcVSlots]  V landed (TMA bytes)
constexpr int kBVEmpty = kBVFull + kTcVSlots;    // [kTcVSlots]  V consumed (PV commit)
constexpr int kBSFull = kBVEmpty + kTcVSlots;    // [kTcSBufs] S^T in TMEM (commit)
constexpr int kBSFree = kBSFull + kTcSBufs;      // [kTcSBufs] softmax has read S^T (128 arrivals)
constexpr int kBPFull = kBSFree + kTcSBufs;      // [kTcPBufs] P tile written (128 arrivals)
constexpr int kBPvDone = kBPFull + kTcPBufs;     // [kTcPBufs] PV done reading P buffer (commit)
constexpr int kBQFull = kBPvDone + kTcPBufs;     // [kTcQBufs] q staged (stager)
constexpr int kBQEmpty = kBQFull + kTcQBufs;     // [kTcQBufs] q buffer read by its S^T MMAs (softmax)
constexpr int kBOReady = kBQEmpty + kTcQBufs;    // [kTcOBufs] the piece's last PV has completed (commit)
constexpr int kBStats = kBOReady + kTcOBufs;     // [kTcOBufs] the piece's (m, l) written (softmax)
constexpr int kBOFree = kBStats + kTcOBufs;      // [kTcOBufs] O buffer and stats read by the epilogue (128 arrivals)
constexpr int kBDrain = kBOFree + kTcOBufs;      // every MMA of the CTA has completed (2 commits)
static_assert(kBDrain + 1 == TcGeo<8>::kBars, "barrier count");

__device__ __forceinline__ uint32_t bar_at(uint32_t base, int i) { return base + 8u * (uint32_t)i; }

// Row r, byte c of a 128-byte-row swizzled tile (16-byte chunk index XOR row % 8).
__device__ __forceinline__ uint32_t sw_off(int r, int c) {
    return (uint32_t)(r * 128 + ((((c >> 4) ^ (r & 7)) << 4) | (c & 15)));
}

// Byte c of token t of head h in a stage's K (or V) tile, as the 4-D boxes land it.
__device__ __forceinline__ uint32_t kv_off(int t, int h, int c) {
    return (uint32_t)((t >> 3) * 2048 + h * 1024) + sw_off(t & 7, c);
}

// Position of a unit in the walk over (sequence, head pair, tile): the issuers and the
// producer's lanes step through their units one by one instead of searching each time.
struct TcCursor {
    int b, hp, tile, nt;
};

__device__ __forceinline__ TcCursor tc_cursor(const int *pfx, int B, int Hu, long long u) {
    const UnitPos up = locate(pfx, B, Hu, u);
    return TcCursor{up.b, up.kvh, up.blk, up.nb};
}

__device__ __forceinline__ void tc_next(TcCursor &c, const int *pfx, int B, int Hu) {
    if (++c.tile < c.nt) return;
    c.tile = 0;
    if (++c.hp < Hu) return;
    c.hp = 0;
    do {
        ++c.b;
        c.nt = c.b < B ? pfx[c.b + 1] - pfx[c.b] : 1;
    } while (c.b < B && c.nt == 0);
}

// Cost-balanced split.  A tile costs kTcUnitCost and a segment's first tile kTcPieceCost more
// (the piece's q, its first tile's full maximum, its epilogue: measured at about three tiles),
// so a CTA with many short sequences takes fewer tiles.  key(u) = kTcUnitCost * u
// + kTcPieceCost * (segments starting at or before u) rises by at most kTcUnitCost +
// kTcPieceCost per unit; CTA c starts at the first unit with key(u) * n >= c * Ctot (Ctot =
// key past the last unit), so with Ctot >= (kTcUnitCost + kTcPieceCost) * n every CTA gets
// at least one unit.
constexpr int kTcUnitCost = 1, kTcPieceCost = 3;

// The first unit whose key reaches thr (0 < thr, thr + kTcUnitCost <= Ctot); ne[b] counts the
// sequences before b that hold at least one tile.
__device__ __forceinline__ long long tc_unit_at_key(const int *pfx, const int *ne, int B, int Hu, long long thr) {
    auto base = [&](int b) {
        return (long long)Hu * ((long long)kTcUnitCost * pfx[b] + (long long)kTcPieceCost * ne[b]);
    };
    int lo = 0, hi = B - 1;  // the first sequence whose last key reaches thr
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (base(mid + 1) >= thr + kTcUnitCost) hi = mid;
        else lo = mid + 1;
    }
    const long long nt = pfx[lo + 1] - pfx[lo];
    long long u = (long long)Hu * pfx[lo];
    const long long r = thr - (base(lo) + kTcPieceCost);  // past the sequence's first key
    if (r > 0) {
        const long long seg = kTcUnitCost * nt + kTcPieceCost;  // key span of one segment
        long long sg = r / seg, tile = 0;
        const long long rem = r - sg * seg;
        if (rem > 0) {
            if (rem <= kTcUnitCost * (nt - 1)) tile = (rem + kTcUnitCost - 1) / kTcUnitCost;
            else ++sg;  // past this segment's last tile: the next segment's first
        }
        u += sg * nt + tile;
    }
    return u;
}

// The CTA whose range holds unit u: the last c < n with start[c] <= u.
__device__ __forceinline__ int tc_owner(const long long *start, int n, long long u) {
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (start[mid] <= u) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// Decode step, run by a q stager when a piece ends its sequence: the new token's K (rotated
// at L - 1 by the RoPE factors rc/rs, when a table is given) and V, quantised to the E4M3
// code of the exact quotient by the head's scale (as pkv_kv_store does), into cache slot
// `slot` and into `codes` (128 K codes, then 128 V codes), from where the S^T issuer patches
// the tile.  Lane i holds the pairs (i, i + 64) and (i + 32, i + 96).  Out of line: it runs
// once per sequence, and inlined it would crowd the stager's loop in the instruction cache.
// (It takes plain values, not the kernel's parameter block: a reference to that would move
// the block into local memory for the whole kernel.)
__device__ __noinline__ void tc_store_new_token(uint8_t *k_cache, uint8_t *v_cache, int Hkv, float ksc, float vsc,
                                                bool rope, int kvh, int slot, const uint16_t (&nk)[2][2],
                                                const uint16_t (&nv)[2][2], const float (&rc)[2],
                                                const float (&rs)[2], uint8_t *codes, int lane) {
    constexpr int D = 128, D2 = 64;
    const size_t dst = ((size_t)slot * Hkv + kvh) * D;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        uint16_t k1 = nk[j][0], k2 = nk[j][1];
        if (rope) rope_pair_fast(k1, k2, rc[j], rs[j], k1, k2);
        const uint16_t kb[2] = {k1, k2};
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            const int d = lane + 32 * j + hf * D2;
            const uint8_t kc = (uint8_t)e4m3_of_quotient(__uint_as_float((uint32_t)kb[hf] << 16), ksc);
            const uint8_t vc = (uint8_t)e4m3_of_quotient(__uint_as_float((uint32_t)nv[j][hf] << 16), vsc);
            k_cache[dst + d] = kc;
            v_cache[dst + d] = vc;
            codes[d] = kc;
            codes[D + d] = vc;
        }
    }
}

// One arrival on a counter whose high 48 bits name the call and whose low 16 bits count: a
// count another call left (or whatever the workspace held) gives way to this call's first
// arrival.  Returns the arrivals so far, this one included (0, with the timeout flag, after
// a bounded number of lost races).
__device__ __forceinline__ unsigned tc_arrive_epoch(unsigned long long *ctr, unsigned long long epoch, int *err) {
    unsigned long long cur = atomicAdd(ctr, 0ull);
    for (int i = 0; i < (1 << 16); ++i) {
        const unsigned long long nv = (cur >> 16) == epoch ? cur + 1 : (epoch << 16) | 1ull;
        const unsigned long long prev = atomicCAS(ctr, cur, nv);
        if (prev == cur) return (unsigned)(nv & 0xFFFFu);
        cur = prev;
    }
    atomicOr(err, kErrTimeout);
    return 0;
}


// Run by the first epilogue warp after the partial slots of a piece that is not a whole
// segment are written: the CTAs c0..c1 that cut the segment each add one arrival; the last to
// arrive merges their partials, head by head (as the combine kernel does, rounded alike:
// o / l * v_scale), and clears the counter for the next call.  The decode step counts on a
// per-segment counter the caller zeroed once; the plain decode on call-tagged counters, one
// per CTA (c0's: a CTA's last piece is the first piece of at most one split segment).  A
// segment's partials sit in slots kTcHP * (segment + c) + head.  Out of line: it runs at most
// twice per CTA (and takes plain values, not the kernel's parameter block, for the reason
// given above).
template <int G, bool EPOCH>
__device__ __noinline__ void tc_merge_if_last(int *counters, unsigned long long *ectr, unsigned long long epoch,
                                              int *err, const float *partials, __nv_bfloat16 *out, int Hq,
                                              const int *pfx, int Hu, const long long *start_of, int n, int b,
                                              int hp, int ntiles, int segu, float vs0, float vs1, int lane) {
    constexpr int D = 128;
    __threadfence();
    __syncwarp();
    const long long start = (long long)Hu * pfx[b] + (long long)hp * ntiles;
    const int c0 = tc_owner(start_of, n, start), c1 = tc_owner(start_of, n, start + ntiles - 1);
    int last = 0;
    if (lane == 0) {
        if constexpr (EPOCH) last = tc_arrive_epoch(ectr + c0, epoch, err) == (unsigned)(c1 - c0 + 1);
        else last = atomicAdd(counters + segu, 1) == c1 - c0;
    }
    last = __shfl_sync(0xffffffffu, last, 0);
    if (!last) return;
    __threadfence();
    // lane: dims 4*lane .. 4*lane+3 of every head g.  M_g = max m_c, o = sum e^(m_c - M) acc_c
    // / sum e^(m_c - M) l_c, accumulated over c in order (as the combine kernel does); the
    // loads of one CTA slot go out together, for both kv heads at once where the registers
    // allow (G <= 4).
    const int d = 4 * lane;
    constexpr int NH = G <= 4 ? kTcHP : 1;  // kv heads per pass
#pragma unroll 1
    for (int h0 = 0; h0 < kTcHP; h0 += NH) {
        float M[NH][G];
#pragma unroll
        for (int h = 0; h < NH; ++h)
#pragma unroll
            for (int g = 0; g < G; ++g) M[h][g] = -INFINITY;
        for (int cc = c0; cc <= c1; ++cc) {
            float mk[NH][G];
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                const float *sl = partials + (size_t)(kTcHP * (segu + cc) + h0 + h) * (G * (D + 2)) + G * D;
#pragma unroll
                for (int g = 0; g < G; ++g) mk[h][g] = __ldcg(sl + g);
            }
#pragma unroll
            for (int h = 0; h < NH; ++h)
#pragma unroll
                for (int g = 0; g < G; ++g) M[h][g] = fmaxf(M[h][g], mk[h][g]);
        }
        float4 acc[NH][G];
        float ls[NH][G];
#pragma unroll
        for (int h = 0; h < NH; ++h)
#pragma unroll
            for (int g = 0; g < G; ++g) {
                acc[h][g] = make_float4(0.f, 0.f, 0.f, 0.f);
                ls[h][g] = 0.f;
            }
        for (int cc = c0; cc <= c1; ++cc) {
            float mk[NH][G], lk[NH][G];
            float4 x[NH][G];
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                const float *sl = partials + (size_t)(kTcHP * (segu + cc) + h0 + h) * (G * (D + 2));
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    mk[h][g] = __ldcg(sl + G * D + g);
                    lk[h][g] = __ldcg(sl + G * D + G + g);
                    x[h][g] = __ldcg(reinterpret_cast<const float4 *>(sl + g * D + d));  // (G >= 2: aligned)
                }
            }
#pragma unroll
            for (int h = 0; h < NH; ++h)
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float f = (mk[h][g] == -INFINITY) ? 0.f : ex2(mk[h][g] - M[h][g]);
                    acc[h][g].x += f * x[h][g].x;
                    acc[h][g].y += f * x[h][g].y;
                    acc[h][g].z += f * x[h][g].z;
                    acc[h][g].w += f * x[h][g].w;
                    ls[h][g] += f * lk[h][g];
                }
        }
#pragma unroll
        for (int h = 0; h < NH; ++h) {
            const float vs = h0 + h == 0 ? vs0 : vs1;
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const bool any = ls[h][g] > 0.f;
                uint2 w;
                w.x = tc::pack_bf16x2(any ? acc[h][g].x / ls[h][g] * vs : 0.f, any ? acc[h][g].y / ls[h][g] * vs : 0.f);
                w.y = tc::pack_bf16x2(any ? acc[h][g].z / ls[h][g] * vs : 0.f, any ? acc[h][g].w / ls[h][g] * vs : 0.f);
                *reinterpret_cast<uint2 *>(out + ((size_t)b * Hq + (hp * kTcHP + h0 + h) * G + g) * D + d) = w;
            }
        }
    }
    if (lane == 0) {
        if constexpr (EPOCH) atomicExch(ectr + c0, 0ull);
        else counters[segu] = 0;
    }
}

template <int G, bool STEP>
__global__ void __launch_bounds__(kTcThreads, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                     const DecodeParams p) {
    using Geo = TcGeo<G>;
    constexpr int D = Geo::D;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (sbase - smem_u32(smem_raw));
    const uint32_t sStages = sbase, sQ = sbase + Geo::kOffQ, sP = sbase + Geo::kOffP;
    float *red = reinterpret_cast<float *>(smem + Geo::kOffRed);
    TcStats *stats = reinterpret_cast<TcStats *>(smem + Geo::kOffStats);  // [O buffer]
    TcMeta *meta = reinterpret_cast<TcMeta *>(smem + Geo::kOffMeta);      // [q buffer]
    uint8_t *newcodes = smem + Geo::kOffNew;                               // [q buffer][head][256]
    const uint32_t bars = sbase + Geo::kOffBar;
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(smem + Geo::kOffBar + 8 * Geo::kBars);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Geo::kOffBar + 8 * Geo::kBars + 4);
    int *pfx = reinterpret_cast<int *>(smem + Geo::kOffPfx);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    pdl_wait();
    pdl_trigger();
    // prefix of the sequences' tile counts (units per sequence and kv head), and of the
    // sequences that hold any tile (in the stage ring, free until the producer starts)
    int *ne = reinterpret_cast<int *>(smem);
    {
        __shared__ int wsum[kTcThreads / 32][2];
        __shared__ int carry_s[2];
        if (threadIdx.x == 0) carry_s[0] = carry_s[1] = 0;
        __syncthreads();
        for (int base = 0; base < p.B; base += kTcThreads) {
            const int b = base + threadIdx.x;
            int v = 0;
            if (b < p.B) {
                int L = __ldg(p.context_lens + b);
                if (L < 0) L = 0;
                if (L > p.max_tokens) {
                    atomicOr(p.err, kErrBounds);
                    L = p.max_tokens;
                }
                v = (L + kTcTile - 1) / kTcTile;
            }
            const int e = v > 0 ? 1 : 0;
            int incl = v, incl_e = e;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                const int ye = __shfl_up_sync(0xffffffffu, incl_e, o);
                if (lane >= o) {
                    incl += y;
                    incl_e += ye;
                }
            }
            if (lane == 31) {
                wsum[warp][0] = incl;
                wsum[warp][1] = incl_e;
            }
            __syncthreads();
            int before = carry_s[0], before_e = carry_s[1];
            for (int w = 0; w < warp; ++w) {
                before += wsum[w][0];
                before_e += wsum[w][1];
            }
            if (b < p.B) {
                pfx[b] = before + incl - v;
                ne[b] = before_e + incl_e - e;
            }
            __syncthreads();
            if (threadIdx.x == kTcThreads - 1) {
                carry_s[0] = before + incl;
                carry_s[1] = before_e + incl_e;
            }
            __syncthreads();
        }
        if (threadIdx.x == 0) {
            pfx[p.B] = carry_s[0];
            ne[p.B] = carry_s[1];
        }
        __syncthreads();
    }
    const int Hu = p.Hkv / kTcHP;  // head pairs
    const long long total = (long long)Hu * pfx[p.B];
    // every CTA's first unit (start_of[n] = total): cost-balanced where every CTA then gets a
    // unit, else equal counts (a problem of a few tiles: the last CTAs may get none)
    long long *start_of = reinterpret_cast<long long *>(smem + Geo::kOffPfx + tc_pfx_bytes(p.B));
    {
        const int n = p.nctas;
        const long long ctot = kTcUnitCost * total + (long long)kTcPieceCost * Hu * ne[p.B];
        const bool by_cost = ctot >= (long long)(kTcUnitCost + kTcPieceCost) * n;
        const long long U = total > 0 ? (total + n - 1) / n : 1;
        for (int c = threadIdx.x; c <= n; c += kTcThreads) {
            long long u;
            if (c == 0) u = 0;
            else if (c == n) u = total;
            else if (by_cost) u = tc_unit_at_key(pfx, ne, p.B, Hu, ((long long)c * ctot + n - 1) / n);
            else u = min((long long)c * U, total);
            start_of[c] = u;
        }
        __syncthreads();  // (ne's space is the stage ring's from here on)
    }
    for (int b = blockIdx.x; b < p.B; b += gridDim.x)
        if (pfx[b + 1] == pfx[b])
            for (int e = threadIdx.x; e < p.Hq * D; e += kTcThreads)
                p.out[(size_t)b * p.Hq * D + e] = __float2bfloat16_rn(0.f);
    const long long u0 = start_of[blockIdx.x];
    const long long u1 = start_of[blockIdx.x + 1];
    if (u0 >= u1) return;  // uniform across the CTA
    const int nunits = (int)(u1 - u0);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kTcKSlots; ++s) {
            mbar_init(bar_at(bars, kBKFull + s), 1);
            mbar_init(bar_at(bars, kBKEmpty + s), 1);
        }
        for (int s = 0; s < kTcVSlots; ++s) {
            mbar_init(bar_at(bars, kBVFull + s), 1);
            mbar_init(bar_at(bars, kBVEmpty + s), 1);
        }
        for (int i = 0; i < kTcSBufs; ++i) {
            mbar_init(bar_at(bars, kBSFull + i), 1);
            mbar_init(bar_at(bars, kBSFree + i), 128);
        }
        for (int i = 0; i < kTcPBufs; ++i) {
            mbar_init(bar_at(bars, kBPFull + i), 128);
            mbar_init(bar_at(bars, kBPvDone + i), 1);
        }
        for (int i = 0; i < kTcOBufs; ++i) {
            mbar_init(bar_at(bars, kBOReady + i), 1);
            mbar_init(bar_at(bars, kBStats + i), 1);
            mbar_init(bar_at(bars, kBOFree + i), 128);
        }
        for (int i = 0; i < kTcQBufs; ++i) {
            mbar_init(bar_at(bars, kBQFull + i), 1);
            mbar_init(bar_at(bars, kBQEmpty + i), 1);
        }
        mbar_init(bar_at(bars, kBDrain), 2);
        *abort_flag = 0;
        fence_mbar_init();
    }
    // zero the q and P operands: the rows no head uses (2G.. of q, G..7 and 8+G.. of P) stay zero
    for (int i = threadIdx.x; i < (kTcQBufs * Geo::kQ + kTcPBufs * Geo::kP) / 16; i += kTcThreads)
        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(sQ + 16 * i), "r"(0u) : "memory");
    fence_proxy_async_smem();
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32((const void *)tmem_slot)), "n"(kTcCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // TMEM: S^T buffers at columns 0..127, O^T buffers at 128..223 (128 lanes x 32 each: 16 per head)

    // a bounded wait by lane 0 of the calling warp, its outcome broadcast to the warp (the
    // __syncwarp orders the other lanes' accesses after lane 0's acquire)
    auto wait0 = [&](int bi, uint32_t parity) -> bool {
        bool r = true;
        if (lane == 0) r = !*abort_flag && mbar_wait_bounded(bar_at(bars, bi), parity, p.err);
        __syncwarp();
        return __shfl_sync(0xffffffffu, r ? 1 : 0, 0) != 0;
    };

    if (warp == 0 || warp == kTcVWarp) {
        // ---------------------------------------------------------------- TMA producers
        // warp 0 fills the K ring, warp 15 the V ring, each walking every unit
        const bool is_v = warp == kTcVWarp;
        const CUtensorMap *tm = is_v ? &tm_v : &tm_k;
        const uint32_t ring = sStages + (is_v ? Geo::kOffV : 0);
        const int bfull = is_v ? kBVFull : kBKFull, bempty = is_v ? kBVEmpty : kBKEmpty;
        const int nslots = is_v ? kTcVSlots : kTcKSlots;
        if (lane == 0) prefetch_tmap(tm);
        // A box is one block's bs tokens (8, 16 or 32) of the pair's two heads; lanes cover a
        // batch of tiles: lane = tile of the batch * boxes + box.  One pass of block-table
        // loads serves the whole batch, and each box is issued by its own lane.
        const int n_box = kTcTile / p.bs, tpb = 32 / n_box;
        const int bt = lane / n_box, bx = lane % n_box;
        const uint32_t box_off = (uint32_t)(bx * p.bs * 256);
        // the slot / 8 coordinate just past the cache: the copy engine fills such a box with zeros
        const int oob = (int)(p.num_blocks * p.bs / 8 < 0x7fffffffLL ? p.num_blocks * p.bs / 8 : 0x7fffffff);
        TcCursor cur = tc_cursor(pfx, p.B, Hu, u0 + min(bt, nunits - 1));  // this lane's tile
        // Loads of this lane's block-table entry and context length for the tile k0 + bt;
        // they are issued one batch ahead, so their latency hides behind the waits and
        // copies of the batch before.  (The entry is read only where it lies inside the
        // table row; whether the box holds tokens is decided once L is known.)
        auto fetch = [&](int k0, int &e, int &L) {
            e = -1;
            L = 0;
            if (k0 + bt < nunits) {
                const int idx = cur.tile * n_box + bx;
                if (idx < p.max_blocks) e = __ldg(p.block_tables + (size_t)cur.b * p.max_blocks + idx);
                L = __ldg(p.context_lens + cur.b);
            }
        };
        auto coord_of = [&](int e, int L) -> int {
            L = min(L, p.max_tokens);
            if ((cur.tile * n_box + bx) * p.bs >= L) return oob;  // no token of the context
            if (e < 0 || (long long)e >= p.num_blocks) {
                atomicOr(p.err, kErrBounds);
                return oob;
            }
            return e * (p.bs / 8);
        };
        int e_cur, L_cur;
        fetch(0, e_cur, L_cur);
        uint32_t issued = 0, phases = 0;
        bool ok = true;
        for (int k0 = 0; k0 < nunits && ok; k0 += tpb) {
            const int co = k0 + bt < nunits ? coord_of(e_cur, L_cur) : oob;
            const int hp = cur.hp;
            // this lane's tile of the next batch, and its loads
            for (int t = 0; t < tpb; ++t) tc_next(cur, pfx, p.B, Hu);
            fetch(k0 + tpb, e_cur, L_cur);
            for (int t = 0; t < tpb && k0 + t < nunits; ++t) {
                const int k = k0 + t, s = k % nslots;
                const uint32_t fb = bar_at(bars, bfull + s);
                if (lane == 0) {
                    if (*abort_flag ||
                        !mbar_wait_bounded(bar_at(bars, bempty + s), ((k / nslots) & 1) ^ 1, p.err)) {
                        ok = false;
                        *abort_flag = 1;
                    } else {
                        mbar_arrive_expect_tx(fb, Geo::kKV);
                        issued |= 1u << s;
                        phases = (phases & ~(1u << s)) | ((uint32_t)((k / nslots) & 1) << s);
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                if (!ok) break;
                if (bt == t) tma_load_4d(ring + s * Geo::kKV + box_off, tm, fb, 0, 0, kTcHP * hp, co);
            }
        }
        if (lane == 0)  // never leave with a TMA copy landing in shared memory
            for (int s = 0; s < nslots; ++s)
                if ((issued >> s) & 1) mbar_wait_bounded(bar_at(bars, bfull + s), (phases >> s) & 1, p.err);
    } else if (warp == 1) {
        // ---------------------------------------------------------------- S^T issuer
        // Lane 0 alone walks the units and issues (with STEP it first stores the step's new
        // token into the tile that holds it); the other lanes wait for the TMEM release.
        if (lane == 0) {
            constexpr uint32_t idS = tc::mma_idesc(128, 16, false, true);  // E4M3 x E4M3 -> f32
            bool ok = true;
            int piece = -1;
            TcCursor cur = tc_cursor(pfx, p.B, Hu, u0);
            for (int k = 0; k < nunits && ok; ++k, tc_next(cur, pfx, p.B, Hu)) {
                const int tile = cur.tile, ntiles = cur.nt;
                if (k == 0 || tile == 0) {
                    ++piece;
                    ok = !*abort_flag &&
                         mbar_wait_bounded(bar_at(bars, kBQFull + piece % kTcQBufs), (piece / kTcQBufs) & 1, p.err);
                }
                ok = ok && !*abort_flag &&
                     mbar_wait_bounded(bar_at(bars, kBKFull + k % kTcKSlots), (k / kTcKSlots) & 1, p.err) &&
                     (k < kTcSBufs ||
                      mbar_wait_bounded(bar_at(bars, kBSFree + k % kTcSBufs), ((k - kTcSBufs) / kTcSBufs) & 1, p.err));
                if (!ok) break;
                const uint32_t kd = sStages + (k % kTcKSlots) * Geo::kKV;
                if constexpr (STEP) {
                    const int qs = piece % kTcQBufs, r = meta[qs].nt_row;
                    if (tile == ntiles - 1 && r >= 0) {
                        // the sequence's last tile holds its new token: the stager's codes
                        // replace the slot's previous contents in both heads' K rows (the
                        // softmax patches V once it has landed)
#pragma unroll 1
                        for (int i = 0; i < kTcHP * 8; ++i) {
                            const int h = i >> 3, c = 16 * (i & 7);
                            const uint4 x = *reinterpret_cast<const uint4 *>(newcodes + (qs * kTcHP + h) * 256 + c);
                            const uint32_t dst = kd + kv_off(r, h, c);
                            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(x.x), "r"(x.y),
                                         "r"(x.z), "r"(x.w) : "memory");
                        }
                        fence_proxy_async_smem();  // the tensor cores read these rows next
                    }
                }
                tc::tc_fence_after();
                const uint32_t qd = sQ + (piece % kTcQBufs) * Geo::kQ;
#pragma unroll
                for (int h = 0; h < kTcHP; ++h)
#pragma unroll
                    for (int kk = 0; kk < D / 32; ++kk)
                        tc::mma_ss_f8(tmem + kTcSCols * (k % kTcSBufs) + 16 * h,
                                      tc::sw128_desc(kd + 1024 * h + 32 * kk, 16, 2048),
                                      tc::sw128_desc(qd + Geo::kQ1 * h + 32 * kk, 16, 1024), idS, kk > 0);
                tc::mma_commit(bar_at(bars, kBSFull + k % kTcSBufs));
                tc::mma_commit(bar_at(bars, kBKEmpty + k % kTcKSlots));
            }
            if (!ok) *abort_flag = 1;
            tc::mma_commit(bar_at(bars, kBDrain));  // (with the PV issuer's commit)
        }
        __syncwarp();
    } else if (warp == kTcPvWarp) {
        // ---------------------------------------------------------------- PV issuer
        constexpr uint32_t idO = tc::mma_idesc(128, 16, false, true) | tc::kIdescAMnMajor;  // A (V^T) MN-major
        // The warp walks the tiles; lane 0 waits and issues, and for a tile that ends its
        // context the whole warp first fixes its V rows: the rows of the last block past the
        // context (those past that block were filled with zeros by the copy engine) and
        // (decode step) the new token's row.
        bool ok = true;
        int piece = -1;
        TcCursor cur = tc_cursor(pfx, p.B, Hu, u0);
        for (int k = 0; k < nunits && ok; ++k, tc_next(cur, pfx, p.B, Hu)) {
            const bool first = k == 0 || cur.tile == 0;
            const bool last = k == nunits - 1 || cur.tile == cur.nt - 1;
            if (first) ++piece;
            // a piece's first PV overwrites its O buffer: the epilogue of piece - kTcOBufs
            // must have read it
            if (lane == 0)
                ok = !*abort_flag &&
                     mbar_wait_bounded(bar_at(bars, kBPFull + k % kTcPBufs), (k / kTcPBufs) & 1, p.err) &&
                     mbar_wait_bounded(bar_at(bars, kBVFull + k % kTcVSlots), (k / kTcVSlots) & 1, p.err) &&
                     (!first || piece < kTcOBufs ||
                      mbar_wait_bounded(bar_at(bars, kBOFree + piece % kTcOBufs), (piece / kTcOBufs - 1) & 1, p.err));
            __syncwarp();
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) break;
            const uint32_t vd = sStages + Geo::kOffV + (k % kTcVSlots) * Geo::kKV;
            const int2 info = *reinterpret_cast<const int2 *>(smem + Geo::kOffPvInfo + 8 * (k % kTcPBufs));
            if (info.x < kTcTile || info.y >= 0) {
                const int zend = min(kTcTile, (info.x + p.bs - 1) / p.bs * p.bs);
                for (int i = lane; i < (zend - info.x) * kTcHP * 8; i += 32) {  // 16 bytes per lane and step
                    const int r = info.x + i / (kTcHP * 8), h = (i >> 3) % kTcHP, q = i & 7;
                    asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(vd + (r >> 3) * 2048 + h * 1024 +
                                                                                   (r & 7) * 128 + 16 * q),
                                 "r"(0u) : "memory");
                }
                if (info.y >= 0 && lane < kTcHP * 8) {
                    const int h = lane >> 3, cc = 16 * (lane & 7);
                    const uint4 x = *reinterpret_cast<const uint4 *>(smem + Geo::kOffPvCodes +
                                                                     (k % kTcPBufs) * (kTcHP * 128) + h * 128 + cc);
                    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(vd + kv_off(info.y, h, cc)), "r"(x.x),
                                 "r"(x.y), "r"(x.z), "r"(x.w) : "memory");
                }
                fence_proxy_async_smem();  // the tensor cores read these rows next
                __syncwarp();
            }
            if (lane == 0) {
                tc::tc_fence_after();
                const uint32_t pd = sP + (k % kTcPBufs) * Geo::kP;
                const uint32_t tO = tmem + kTcO + kTcSCols * (uint32_t)(piece % kTcOBufs);
#pragma unroll
                for (int h = 0; h < kTcHP; ++h)
#pragma unroll
                    for (int kk = 0; kk < kTcTile / 32; ++kk)  // 32 tokens per MMA
                        tc::mma_ss_f8(tO + 16 * h, tc::sw128_desc(vd + 1024 * h + 8192 * kk, 16384, 2048),
                                      tc::sw128_desc(pd + Geo::kP1 * h + 32 * kk, 16, 1024), idO,
                                      (first && kk == 0) ? 0u : 1u);
                tc::mma_commit(bar_at(bars, kBVEmpty + k % kTcVSlots));
                tc::mma_commit(bar_at(bars, kBPvDone + k % kTcPBufs));
                if (last) tc::mma_commit(bar_at(bars, kBOReady + piece % kTcOBufs));
            }
            __syncwarp();
        }
        if (lane == 0) {
            if (!ok) *abort_flag = 1;
            // drain: no MMA of either issuer may still write TMEM when it is released
            tc::mma_commit(bar_at(bars, kBDrain));
            mbar_wait_bounded(bar_at(bars, kBDrain), 0, p.err);
        }
        __syncwarp();
    } else if (tc_stager_index(warp) >= 0) {
        // ---------------------------------------------------------------- q stagers
        // Four warps take the pieces in turn (piece i to stager i % 4), each into q buffer
        // piece % kTcQBufs: per head of the pair its G q heads rotated at L - 1, scaled by one
        // power of two and split into high parts (rows 0..G-1) and low parts (rows G..2G-1)
        // as E4M3 codes, plus the piece's description, and (decode step) the new token of a
        // piece that ends its sequence.  Lane i holds dims i, i + 32, i + 64, i + 96 of every
        // q head (the RoPE pairs (i, i + 64) and (i + 32, i + 96)).  All loads of a piece go
        // out in one round; the next piece's context length is fetched while this one is
        // staged.
        constexpr int D2 = D / 2;
        const int par = tc_stager_index(warp);
        TcCursor cur = tc_cursor(pfx, p.B, Hu, u0);
        int k = 0;
        // context length of the next piece this warp stages
        auto next_own = [&](TcCursor c, int kk, int pc) -> int {  // (by value: a look-ahead)
            while (kk < nunits && pc % kTcStagers != par) {
                const int pl = min(c.nt - c.tile, nunits - kk);
                kk += pl;
                for (int t = 0; t < pl; ++t) tc_next(c, pfx, p.B, Hu);
                ++pc;
            }
            return kk < nunits ? __ldg(p.context_lens + c.b) : 0;
        };
        int Lraw = next_own(cur, 0, 0);
        for (int pc = 0; k < nunits; ++pc) {
            const int b = cur.b, hp = cur.hp;
            const int piece_len = min(cur.nt - cur.tile, nunits - k);
            const bool ends = piece_len == cur.nt - cur.tile;  // the piece ends its sequence
            if (pc % kTcStagers == par) {
                const int slot = pc % kTcQBufs;
                const int L = min(Lraw, p.max_tokens), pos = L - 1;
                const bool rope_ok = p.rope && pos >= 0 && pos < p.max_pos;
                if (p.rope && !rope_ok && lane == 0) atomicOr(p.err, kErrBounds);
                // ---- one round of loads: every q head's four dims, their RoPE factors, the
                // new token's K and V and its block entry
                uint16_t qx[kTcHP][G][4];
#pragma unroll
                for (int h = 0; h < kTcHP; ++h)
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        const uint16_t *qr = p.q + ((size_t)b * p.Hq + (hp * kTcHP + h) * G + g) * D + lane;
#pragma unroll
                        for (int j = 0; j < 4; ++j) qx[h][g][j] = __ldg(qr + 32 * j);
                    }
                float rc[2] = {1.f, 1.f}, rs[2] = {0.f, 0.f};
                if (rope_ok)
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        rc[j] = __ldg(p.rope + (size_t)pos * D + lane + 32 * j);
                        rs[j] = __ldg(p.rope + (size_t)pos * D + D2 + lane + 32 * j);
                    }
                bool nt_go = false;
                int nt_e = -1;
                uint16_t nk[kTcHP][2][2], nv[kTcHP][2][2];
                if constexpr (STEP) {
                    // (nothing is stored when the context was clipped to the block table or the
                    // position is outside the RoPE table; a bad block entry is the producer's to flag)
                    nt_go = ends && L == Lraw && L >= 1 && (!p.rope || rope_ok);
                    if (nt_go) {
                        nt_e = __ldg(p.block_tables + (size_t)b * p.max_blocks + pos / p.bs);
#pragma unroll
                        for (int h = 0; h < kTcHP; ++h) {
                            const uint16_t *kin = p.k_new + ((size_t)b * p.Hkv + hp * kTcHP + h) * D;
                            const uint16_t *vin = p.v_new + ((size_t)b * p.Hkv + hp * kTcHP + h) * D;
#pragma unroll
                            for (int j = 0; j < 2; ++j) {
                                nk[h][j][0] = __ldg(kin + lane + 32 * j);
                                nk[h][j][1] = __ldg(kin + lane + 32 * j + D2);
                                nv[h][j][0] = __ldg(vin + lane + 32 * j);
                                nv[h][j][1] = __ldg(vin + lane + 32 * j + D2);
                            }
                        }
                    }
                }
                float ksc[kTcHP], vsc[kTcHP];
#pragma unroll
                for (int h = 0; h < kTcHP; ++h) {
                    ksc[h] = __ldg(p.k_scale + hp * kTcHP + h);
                    vsc[h] = __ldg(p.v_scale + hp * kTcHP + h);
                }
                // the following piece's context length, while this one is computed
                TcCursor nc = cur;
                for (int t = 0; t < piece_len; ++t) tc_next(nc, pfx, p.B, Hu);
                const int Lnext = next_own(nc, k + piece_len, pc + 1);
                // ---- the slot must be free before it is written
                if (!wait0(kBQEmpty + slot, ((pc / kTcQBufs) & 1) ^ 1)) {
                    if (lane == 0) *abort_flag = 1;
                    break;
                }
                const uint32_t qd = sQ + slot * Geo::kQ;
                float sqh[kTcHP];
#pragma unroll
                for (int h = 0; h < kTcHP; ++h) {
                    float x[G][4];
                    float amax = 0.f;
#pragma unroll
                    for (int g = 0; g < G; ++g) {
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            uint16_t x1 = qx[h][g][j], x2 = qx[h][g][j + 2];
                            if (rope_ok) rope_pair_fast(x1, x2, rc[j], rs[j], x1, x2);
                            x[g][j] = __uint_as_float((uint32_t)x1 << 16);
                            x[g][j + 2] = __uint_as_float((uint32_t)x2 << 16);
                        }
#pragma unroll
                        for (int j = 0; j < 4; ++j) amax = fmaxf(amax, fabsf(x[g][j]));
                    }
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                    const float sq = amax > 0.f
                                         ? __int_as_float(__float_as_int(fminf(448.f / amax, 0x1p100f)) & 0x7F800000)
                                         : 1.f;
                    sqh[h] = sq;
                    const uint32_t qh = qd + Geo::kQ1 * h;
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        uint32_t hi, lo;
                        tc::split_e4m3x4(x[g][0] * sq, x[g][1] * sq, x[g][2] * sq, x[g][3] * sq, hi, lo);
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int c = lane + 32 * j;
                            asm volatile("st.shared.u8 [%0], %1;" ::"r"(qh + sw_off(g, c)), "r"((hi >> (8 * j)) & 0xFFu)
                                         : "memory");
                            asm volatile("st.shared.u8 [%0], %1;" ::"r"(qh + sw_off(G + g, c)),
                                         "r"((lo >> (8 * j)) & 0xFFu) : "memory");
                        }
                    }
                }
                int nt_row = -1;
                if constexpr (STEP) {
                    if (nt_go && nt_e >= 0 && (long long)nt_e < p.num_blocks) {
#pragma unroll 1
                        for (int h = 0; h < kTcHP; ++h)
                            tc_store_new_token(static_cast<uint8_t *>(p.k_cache_w), static_cast<uint8_t *>(p.v_cache_w),
                                               p.Hkv, ksc[h], vsc[h], p.rope != nullptr, hp * kTcHP + h,
                                               nt_e * p.bs + pos % p.bs, nk[h], nv[h], rc, rs,
                                               newcodes + (slot * kTcHP + h) * 256, lane);
                        nt_row = pos % kTcTile;
                    }
                }
                if (lane == 0) {
                    TcMeta &mt = meta[slot];
                    mt.nt_row = nt_row;
                    mt.b = b;
                    mt.hp = hp;
                    mt.tile = cur.tile;
                    mt.ntiles = cur.nt;
                    mt.piece_len = piece_len;
                    mt.L = L;
#pragma unroll
                    for (int h = 0; h < kTcHP; ++h) {
                        mt.sc[h] = p.scale_log2 * ksc[h] / sqh[h];
                        mt.vs[h] = vsc[h];
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_at(bars, kBQFull + slot));
                Lraw = Lnext;
            }
            k += piece_len;
            for (int t = 0; t < piece_len; ++t) tc_next(cur, pfx, p.B, Hu);
        }
    } else if (warp >= kTcEpiWarp && warp < kTcEpiWarp + 4) {
        // ---------------------------------------------------------------- epilogue
        // For each piece in turn, once its last PV has completed and the softmax has left the
        // piece's description and (m, l): thread = dim d (TMEM lane d of O^T), each head's
        // columns g + 8+g -> the output rows (a whole segment) or the piece's partial slots,
        // then O buffer free.
        const int quad = warp & 3;
        const int d = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        int k = 0;
        for (int piece = 0; k < nunits; ++piece) {
            const int ob = piece % kTcOBufs, ph = (piece / kTcOBufs) & 1;
            const bool fin = wait0(kBStats + ob, ph) && wait0(kBOReady + ob, ph);
            // the four warps leave together (the decode step's merge has them meet again)
            if (named_bar_any(kTcEpiBar, 128, !fin)) {
                if (lane == 0) *abort_flag = 1;
                break;
            }
            tc::tc_fence_after();
            const TcStats &st = stats[ob];
            const int b = st.b, hp = st.hp, ntiles = st.ntiles, piece_len = st.piece_len;
            const bool whole = st.whole != 0;
            float vs[kTcHP], m[kTcHP][G], l[kTcHP][G];
#pragma unroll
            for (int h = 0; h < kTcHP; ++h) {
                vs[h] = st.vs[h];
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    m[h][g] = st.m[h][g];
                    l[h][g] = st.l[h][g];
                }
            }
            uint32_t rr[32];
            tc::tmem_ld32(tmem + lane_off + kTcO + kTcSCols * (uint32_t)ob, rr);
            tc::tc_wait_ld();
            tc::tc_fence_before();
            mbar_arrive(bar_at(bars, kBOFree + ob));  // O buffer and stats slot read
            const int segu = b * Hu + hp;
#pragma unroll
            for (int h = 0; h < kTcHP; ++h) {
                float o[G];
#pragma unroll
                for (int g = 0; g < G; ++g) o[g] = __uint_as_float(rr[16 * h + g]) + __uint_as_float(rr[16 * h + 8 + g]);
                if (whole) {
#pragma unroll
                    for (int g = 0; g < G; ++g)
                        p.out[((size_t)b * p.Hq + (hp * kTcHP + h) * G + g) * D + d] =
                            __float2bfloat16_rn(l[h][g] > 0.f ? o[g] * (vs[h] / l[h][g]) : 0.f);
                } else {
                    float *slot = p.partials + (size_t)(kTcHP * (segu + blockIdx.x) + h) * (G * (D + 2));
#pragma unroll
                    for (int g = 0; g < G; ++g) slot[g * D + d] = o[g];
                    if (quad == 0 && lane < G) {
                        float mh = 0.f, lh = 0.f;
#pragma unroll
                        for (int g = 0; g < G; ++g)
                            if (lane == g) {
                                mh = m[h][g];
                                lh = l[h][g];
                            }
                        slot[G * D + lane] = mh;
                        slot[G * D + G + lane] = lh;
                    }
                }
            }
            if (!whole) {
                // every epilogue thread's part of the slots is written (and fenced) before the
                // first epilogue warp counts the CTA in
                __threadfence();
                named_bar(kTcEpiBar, 128);
                if (quad == 0)
                    tc_merge_if_last<G, !STEP>(p.counters, p.ectr, p.epoch, p.err, p.partials, p.out, p.Hq, pfx, Hu,
                                               start_of, p.nctas, b, hp, ntiles, segu, vs[0], vs[1], lane);
            }
            k += piece_len;
        }
    } else {
        // ---------------------------------------------------------------- softmax (warps 2-5)
        const int sw = warp - kTcSoftmax0;               // 0..3
        const int quad = warp & 3;                        // TMEM lanes 32*quad .. +31
        const int t = quad * 32 + lane;                   // token of the tile = TMEM lane
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const int ct = threadIdx.x - 32 * kTcSoftmax0;    // 0..127
        bool alive = true;
        int k = 0;
        TcCursor cur = tc_cursor(pfx, p.B, Hu, u0);
        for (int piece = 0; k < nunits; ++piece) {
            const int b = cur.b, hp = cur.hp, tile = cur.tile, ntiles = cur.nt;
            const int piece_len = min(ntiles - tile, nunits - k);
            const int qslot = piece % kTcQBufs;
            const uint32_t tO = tmem + lane_off + kTcO + kTcSCols * (uint32_t)(piece % kTcOBufs);  // this lane's dim
            // the piece's context length and scales (and q) from the stager
            const bool qok = alive && !*abort_flag &&
                             mbar_wait_bounded(bar_at(bars, kBQFull + qslot), (piece / kTcQBufs) & 1, p.err);
            if (!__all_sync(0xffffffffu, qok)) {
                alive = false;
                *abort_flag = 1;
            }
            const int L = alive ? meta[qslot].L : 1;
            const int nt_row = alive ? meta[qslot].nt_row : -1;  // (decode step) the new token's tile row
            float sc[kTcHP], vsc[kTcHP];
#pragma unroll
            for (int h = 0; h < kTcHP; ++h) {
                sc[h] = alive ? meta[qslot].sc[h] : 0.f;
                vsc[h] = alive ? meta[qslot].vs[h] : 0.f;
            }
            float mref[kTcHP][G], lsum[kTcHP][G];
#pragma unroll
            for (int h = 0; h < kTcHP; ++h)
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    mref[h][g] = -INFINITY;
                    lsum[h][g] = 0.f;
                }
            for (int j = 0; j < piece_len; ++j, ++k) {
                const int sb = k % kTcSBufs, s = k % kTcVSlots;  // (s: the tile's V slot)
                bool got = alive && !*abort_flag &&
                           mbar_wait_bounded(bar_at(bars, kBSFull + sb), (k / kTcSBufs) & 1, p.err);
                if (!__all_sync(0xffffffffu, got)) {
                    alive = false;
                    *abort_flag = 1;
                }
                float sv[kTcHP][G];
                int pv_valid = kTcTile, pv_row = -1;  // what the PV warp must fix in this tile's V
                if (alive) {
                    tc::tc_fence_after();
                    uint32_t c[32];
                    tc::tmem_ld32(tmem + lane_off + kTcSCols * sb, c);
                    tc::tc_wait_ld();
                    const int valid = min(kTcTile, L - (tile + j) * kTcTile);
#pragma unroll
                    for (int h = 0; h < kTcHP; ++h)
#pragma unroll
                        for (int g = 0; g < G; ++g)
                            sv[h][g] = t < valid
                                           ? (__uint_as_float(c[16 * h + g]) + __uint_as_float(c[16 * h + G + g])) * sc[h]
                                           : -INFINITY;
                    pv_valid = valid;
                    pv_row = STEP && nt_row >= 0 && tile + j == ntiles - 1 ? nt_row : -1;
                } else {
#pragma unroll
                    for (int h = 0; h < kTcHP; ++h)
#pragma unroll
                        for (int g = 0; g < G; ++g) sv[h][g] = -INFINITY;
                }
                tc::tc_fence_before();
                mbar_arrive(bar_at(bars, kBSFree + sb));
                // The running max of a head moves only when the tile's maximum exceeds it by
                // more than 2^8.  One barrier-vote asks whether any token's score does; only then
                // are the tile maxima reduced (always on a piece's first tile, whose running max
                // is -inf).  (No second barrier guards `red`: the next write to it follows the
                // next tile's vote, which every thread reaches after its reads.)
                bool grow = false;
#pragma unroll
                for (int h = 0; h < kTcHP; ++h)
#pragma unroll
                    for (int g = 0; g < G; ++g) grow = grow || sv[h][g] > mref[h][g] + 8.0f;
                float alpha[kTcHP][G];
#pragma unroll
                for (int h = 0; h < kTcHP; ++h)
#pragma unroll
                    for (int g = 0; g < G; ++g) alpha[h][g] = 1.f;
                bool rescale = false;
                if (named_bar_any(kTcBar, 128, grow)) {
#pragma unroll
                    for (int h = 0; h < kTcHP; ++h)
#pragma unroll
                        for (int g = 0; g < G; ++g) {
                            float m = sv[h][g];
#pragma unroll
                            for (int o = 1; o < 32; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                            if (lane == 0) red[16 * sw + 8 * h + g] = m;
                        }
                    named_bar(kTcBar, 128);
#pragma unroll
                    for (int h = 0; h < kTcHP; ++h)
#pragma unroll
                        for (int g = 0; g < G; ++g) {
                            const int i = 8 * h + g;
                            const float m = fmaxf(fmaxf(red[i], red[16 + i]), fmaxf(red[32 + i], red[48 + i]));
                            if (m > mref[h][g] + 8.0f) {  // (token 0 of a tile is always valid: m is finite)
                                alpha[h][g] = ex2(mref[h][g] - m);
                                mref[h][g] = m;
                                rescale = rescale || j > 0;
                            }
                        }
                }
                float pr[kTcHP][G];
#pragma unroll
                for (int h = 0; h < kTcHP; ++h)
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        pr[h][g] = ex2(sv[h][g] - mref[h][g]);
                        lsum[h][g] = lsum[h][g] * alpha[h][g] + pr[h][g];
                    }
                // P buffer pb was last read by the PV of tile k - kTcPBufs
                const int pb = k % kTcPBufs;
                if (alive && k >= kTcPBufs &&
                    !mbar_wait_bounded(bar_at(bars, kBPvDone + pb), ((k - kTcPBufs) / kTcPBufs) & 1, p.err)) {
                    alive = false;
                    *abort_flag = 1;
                }
                const uint32_t pd = sP + pb * Geo::kP;
                // The PV warp fixes this tile's V once it has landed: rows past the context (which
                // would multiply P = 0 by whatever they hold) and the decode step's new token.
                // It learns what to fix here, with the P tile (buffer pb, free like the P tile).
                if (ct == 0)
                    *reinterpret_cast<int2 *>(smem + Geo::kOffPvInfo + 8 * pb) = make_int2(pv_valid, pv_row);
                if (pv_row >= 0 && t == pv_row) {
                    uint8_t *dst = smem + Geo::kOffPvCodes + pb * (kTcHP * 128);
#pragma unroll
                    for (int i = 0; i < kTcHP * 8; ++i) {
                        const int h = i >> 3, cc = 16 * (i & 7);
                        *reinterpret_cast<uint4 *>(dst + h * 128 + cc) =
                            *reinterpret_cast<const uint4 *>(newcodes + (qslot * kTcHP + h) * 256 + D + cc);
                    }
                }
#pragma unroll
                for (int h = 0; h < kTcHP; ++h)
#pragma unroll
                    for (int g0 = 0; g0 < G; g0 += 4) {  // four heads per conversion (G = 2: two)
                        uint32_t hi, lo;
                        tc::split_e4m3x4(pr[h][g0], g0 + 1 < G ? pr[h][g0 + 1] : 0.f, g0 + 2 < G ? pr[h][g0 + 2] : 0.f,
                                         g0 + 3 < G ? pr[h][g0 + 3] : 0.f, hi, lo);
#pragma unroll
                        for (int i = 0; i < 4 && g0 + i < G; ++i) {
                            const uint32_t ph = pd + Geo::kP1 * h;
                            asm volatile("st.shared.u8 [%0], %1;" ::"r"(ph + sw_off(g0 + i, t)),
                                         "r"((hi >> (8 * i)) & 0xFFu) : "memory");
                            asm volatile("st.shared.u8 [%0], %1;" ::"r"(ph + sw_off(8 + g0 + i, t)),
                                         "r"((lo >> (8 * i)) & 0xFFu) : "memory");
                        }
                    }
                if (rescale && alive) {
                    // O^T columns g and 8+g of each head times alpha (each thread its dim's
                    // lane), once the PV of the previous tile has finished
                    const int pj = (k - 1) % kTcPBufs;
                    if (!mbar_wait_bounded(bar_at(bars, kBPvDone + pj), ((k - 1) / kTcPBufs) & 1, p.err)) {
                        alive = false;
                        *abort_flag = 1;
                    }
                    if (__all_sync(0xffffffffu, alive)) {
                        tc::tc_fence_after();
                        uint32_t rr[32];
                        tc::tmem_ld32(tO, rr);
                        tc::tc_wait_ld();
#pragma unroll
                        for (int h = 0; h < kTcHP; ++h)
#pragma unroll
                            for (int g = 0; g < G; ++g) {
                                rr[16 * h + g] = __float_as_uint(__uint_as_float(rr[16 * h + g]) * alpha[h][g]);
                                rr[16 * h + 8 + g] = __float_as_uint(__uint_as_float(rr[16 * h + 8 + g]) * alpha[h][g]);
                            }
                        tc::tmem_st32(tO, rr);
                        tc::tc_wait_st();
                    }
                }
                fence_proxy_async_smem();
                tc::tc_fence_before();
                mbar_arrive(bar_at(bars, kBPFull + pb));
            }
            // q buffer qslot is free: every S^T of the piece has completed (each SFull was waited)
            if (ct == 0) mbar_arrive(bar_at(bars, kBQEmpty + qslot));
            // ---- end of the piece: its (m, l) per head for the epilogue
#pragma unroll
            for (int h = 0; h < kTcHP; ++h)
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    float l = lsum[h][g];
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
                    if (lane == 0) red[64 + 16 * sw + 8 * h + g] = l;
                }
            named_bar(kTcBar, 128);
            if (quad == 0) {
                // the stats slot was last read by the epilogue of piece - kTcOBufs
                bool ok = alive && (piece < kTcOBufs ||
                                    wait0(kBOFree + piece % kTcOBufs, (piece / kTcOBufs - 1) & 1));
                if (!__all_sync(0xffffffffu, ok)) {
                    alive = false;
                    *abort_flag = 1;
                }
                TcStats &st = stats[piece % kTcOBufs];
                if (lane < kTcHP * 8) {
                    const int h = lane >> 3, g = lane & 7;
                    float m = -INFINITY;
#pragma unroll
                    for (int hh = 0; hh < kTcHP; ++hh)
#pragma unroll
                        for (int gg = 0; gg < G; ++gg)
                            if (hh == h && gg == g) m = mref[hh][gg];
                    const int i = 8 * h + g;
                    st.m[h][g] = m;
                    st.l[h][g] = red[64 + i] + red[80 + i] + red[96 + i] + red[112 + i];
                }
                if (lane == 0) {
                    st.b = b;
                    st.hp = hp;
                    st.ntiles = ntiles;
                    st.whole = tile == 0 && piece_len == ntiles;
                    st.piece_len = piece_len;
#pragma unroll
                    for (int h = 0; h < kTcHP; ++h) st.vs[h] = vsc[h];
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_at(bars, kBStats + piece % kTcOBufs));
            }
            for (int j = 0; j < piece_len; ++j) tc_next(cur, pfx, p.B, Hu);
        }
    }

    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "n"(kTcCols));
    }
}

// Dynamic shared memory of a launch over B sequences on n CTAs, and whether it fits the
// device (the prologue's second prefix borrows the stage ring, so B + 1 ints must fit there).
size_t tc_smem_bytes(int B, int n) {
    return (size_t)TcGeo<8>::kOffPfx + (size_t)tc_pfx_bytes(B) + (size_t)(n + 1) * 8 + 1024;
}

bool tc_fits(int B, int dev) {
    return (size_t)(B + 1) * 4 <= (size_t)TcGeo<8>::kOffQ &&
           tc_smem_bytes(B, device_sm_count(dev)) <= (size_t)max_optin_smem(dev) - 2048;
}

// A 48-bit tag per launch, never 0, starting from a per-process random point so that a
// workspace's leftover contents (another call's or another process's) do not match it.
unsigned long long next_call_tag() {
    static std::atomic<unsigned long long> next{[] {
        std::random_device rd;
        return ((unsigned long long)rd() << 32 | rd()) & ((1ull << 47) - 1);
    }()};
    for (;;) {
        const unsigned long long t = next.fetch_add(1, std::memory_order_relaxed) & ((1ull << 48) - 1);
        if (t != 0) return t;
    }
}

template <int G, bool STEP>
cudaError_t launch_tc_g(DecodeParams prm, const DecodeArgs &a, int dev, cudaStream_t s) {
    using Geo = TcGeo<G>;
    auto kern = decode_tc_kernel<G, STEP>;
    const int nctas = device_sm_count(dev);  // one CTA per SM
    const size_t smem = tc_smem_bytes(a.num_seqs, nctas);
    if (!tc_fits(a.num_seqs, dev)) return cudaErrorNotSupported;
    static std::atomic<int> attr_smem[kMaxDev];
    static std::mutex attr_mu;
    if ((size_t)attr_smem[dev].load(std::memory_order_acquire) < smem) {
        std::lock_guard<std::mutex> lock(attr_mu);
        if ((size_t)attr_smem[dev].load(std::memory_order_relaxed) < smem) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
            attr_smem[dev].store((int)smem, std::memory_order_release);
        }
    }
    prm.nctas = nctas;
    if (!STEP) {
        // the call-tagged merge counters, past the partial slots the split can use (one per
        // (sequence, kv head) plus kTcHP per CTA; the workspace holds at least as many more)
        const size_t used = (size_t)a.num_seqs * a.n_kv_heads + (size_t)kTcHP * nctas;
        const size_t have = (size_t)a.num_seqs * a.n_kv_heads + 2 * (size_t)decode_grid_ctas(nctas);
        if ((have - used) * (size_t)(G * (128 + 2)) * sizeof(float) < (size_t)nctas * sizeof(unsigned long long))
            return cudaErrorNotSupported;
        prm.ectr = reinterpret_cast<unsigned long long *>(prm.partials + used * (size_t)(G * (128 + 2)));
        prm.epoch = next_call_tag();
    }
    // (dim, slot % 8, head, slot / 8); a box is one block's tokens of two adjacent heads
    CUtensorMap tk, tv;
    const uint64_t hk = (uint64_t)a.n_kv_heads;
    const uint64_t dims[4] = {128, 8, hk, (uint64_t)a.num_blocks * a.block_size / 8};
    const uint64_t strides[3] = {hk * 128, 128, 8 * hk * 128};
    const uint32_t box[4] = {128, 8, (uint32_t)kTcHP, (uint32_t)a.block_size / 8};
    if (!encode_tensor_map_4d_strided(&tk, a.k_cache, 1, dims, strides, box, true, 256) ||
        !encode_tensor_map_4d_strided(&tv, a.v_cache, 1, dims, strides, box, true, 256))
        return cudaErrorUnknown;
    return launch_pdl(kern, dim3(prm.nctas), dim3(kTcThreads), smem, s, tk, tv, prm);
}

template <bool STEP>
cudaError_t dispatch_tc(const DecodeArgs &a, cudaStream_t s) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
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
    prm.partials = reinterpret_cast<float *>(static_cast<uint8_t *>(a.workspace) +
                                             align16((size_t)(a.num_seqs + 1) * sizeof(int)));
    prm.err = a.err;
    prm.k_new = static_cast<const uint16_t *>(a.k_new);
    prm.v_new = static_cast<const uint16_t *>(a.v_new);
    prm.k_cache_w = a.k_cache_w;
    prm.v_cache_w = a.v_cache_w;
    prm.counters = nullptr;
    if (STEP)  // counters follow the attention workspace (see decode_step_workspace_bytes)
        prm.counters = reinterpret_cast<int *>(static_cast<uint8_t *>(a.workspace) +
                                               decode_workspace_bytes(a.num_seqs, a.n_q_heads, a.n_kv_heads,
                                                                      a.head_dim, device_sm_count(dev)));
    switch (a.n_q_heads / a.n_kv_heads) {
        case 2: return launch_tc_g<2, STEP>(prm, a, dev, s);
        case 4: return launch_tc_g<4, STEP>(prm, a, dev, s);
        case 8: return launch_tc_g<8, STEP>(prm, a, dev, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool decode_tc_supported(const DecodeArgs &a) {
    const int G = a.n_q_heads / a.n_kv_heads;
    if (!(a.fp8 && a.head_dim == 128 && (G == 2 || G == 4 || G == 8) && a.n_kv_heads % kTcHP == 0 &&
          (a.block_size == 8 || a.block_size == 16 || a.block_size == 32)))
        return false;
    int dev = 0;
    return cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < kMaxDev && tc_fits(a.num_seqs, dev);
}

cudaError_t launch_paged_decode_tc(const DecodeArgs &a, cudaStream_t s) { return dispatch_tc<false>(a, s); }
cudaError_t launch_paged_decode_step_tc(const DecodeArgs &a, cudaStream_t s) { return dispatch_tc<true>(a, s); }

}  // namespace pkv
