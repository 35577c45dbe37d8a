// prefill.cu -- paged causal prefill attention on the 5th-generation tensor cores.
//
// "LLM primer: from text to tokens, embeddings, QKV and Transformer", §17.1: prefill
// processes all prompt tokens at once and is compute-bound.  "Inside the Nano-vLLM engine:
// KV cache, attention and tensor parallelism", §3 (softmax(QK^T/sqrt(d))V), §3.1 (tile the
// computation on chip instead of materialising QK^T -- the FlashAttention idea), §3.2 (causal
// mask, RoPE fused into the attention kernel, max subtraction), §2.2 (K/V read through the
// block table).  The pages give no kernel design; this one is written for sm_100a.
//
// Persistent: one CTA per SM (384 threads; shared memory allows one) takes work items round
// robin.  An item is two 128-row query tiles that share every K/V tile: two heads of one GQA
// group on the same rows, or (group 1) two consecutive row tiles of one head.  The K/V rings
// and the per-tile barriers run on across items; the next item's Q tiles load as soon as the
// current item's last S MMAs have read the buffer and are rotated before the current
// item's epilogue, whose O columns the next item's first PV MMAs wait for.
//   warp 0       TMA producer: Q tiles, then K and V tiles of 128 keys = 8 paged blocks, each
//                block one 128-byte-swizzled box per 64 columns, addressed via the block table,
//                into separate K and V rings
//   warp 1       TMEM owner and MMA issuer (one thread): S_i = Q_i K^T and O_i += P_i V with
//                tcgen05.mma kind::f16 (bf16 in, fp32 accumulate in tensor memory)
//   warps 2-3    E4M3 caches only: widen each raw E4M3 tile (staged by plain TMA boxes) into
//                the swizzled f16 operand layout; the MMAs then run on f16 (Q converted too)
//   warps 4-7    softmax for tile 0, warps 8-11 for tile 1: thread r owns row r; reads its S
//                row from TMEM, masks (bottom-right causal), exp2 with the running max, writes
//                P (bf16) back into the S columns, which the next MMA reads as its A operand
// TMEM: S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [256+D,256+2D).  The running max is
// lazily updated: P is computed against a stale max unless the new one is more than 2^8
// larger, so O needs a rescale (TMEM read-modify-write by the softmax thread) only rarely.
// Keys past the sequence are masked; the one V tile holding the sequence's partial last
// block has its tail rows zeroed in shared memory before use (0 * NaN would poison O).
#include "common.cuh"
#include "internal.h"
#include "tcgen05.cuh"

namespace pkv {
namespace {

constexpr int kThreads = 384;
constexpr int kRows = 128;       // query rows per tile
constexpr int kKeys = 128;       // keys per K/V tile (8 blocks)
constexpr int kSoftmax0 = 4;     // first warp of softmax warpgroup 0
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.0f;  // rescale O only when the max grows by > 2^8

template <int D, bool FP8>
struct PGeo {
    // E4M3 caches at head dim 128: the cache bytes are the operands of kind::f8f6f4 MMAs
    // (one 128-byte swizzled row per key); at head dim 64 they are widened to f16 first.
    static constexpr bool kF8 = FP8 && D == 128;
    static constexpr bool kConv = FP8 && D != 128;
    static constexpr int kSlabs = D / 64;                    // 128-byte column slabs of bf16 Q
    static constexpr int kSlabBytes = kRows * 128;           // 16 KB (128 rows x 128 B)
    static constexpr int kQBytes = kSlabs * kSlabBytes;      // one Q tile
    static constexpr int kKVSlabs = kF8 ? 1 : kSlabs;        // 128-byte slabs of a K/V row
    static constexpr int kKVBytes = kKVSlabs * kSlabBytes;   // one K (or V) tile of 128 keys
    // Separate K and V rings: K(j) is released as soon as S1(j) completes, V(j) after PV1(j),
    // so the K load that gates S(j+2) gets five MMAs of slack instead of two.  (A third K
    // stage fits at D 128 in bf16 but measured 1-2 % slower than two.)  E4M3 tiles are half
    // the size, so their rings are twice as deep.
    static constexpr int kKStages = kF8 ? 4 : (D == 128 ? 2 : 4);
    static constexpr int kVStages = kF8 ? 4 : (D == 128 ? 2 : 4);
    static constexpr int kStgBytes = kConv ? kKeys * D : 0;  // raw E4M3 tile (K or V)
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = 2 * kQBytes;
    static constexpr int kOffV = kOffK + kKStages * kKVBytes;
    static constexpr int kOffStg = kOffV + kVStages * kKVBytes;
    static constexpr int kOffBar = kOffStg + 2 * kStgBytes;
    static constexpr int kBarBytes = 8 * (16 + 2 * kKStages + 2 * kVStages) + 16;
    static constexpr int kSmem = kOffBar + kBarBytes + 1024;  // + alignment slack
    static_assert(kSmem <= 232448, "shared memory budget");
};

struct PrefillParams {
    __nv_bfloat16 *out;
    const int32_t *cu_seqlens, *block_tables, *context_lens;
    int max_blocks, B, Hq, Hkv, n_qt;
    int bs;          // tokens per physical block (8, 16 or 32)
    int max_tokens;  // max_blocks * bs
    int n_items;  // work items (see decode_item); CTAs take them round robin
    long long num_blocks;
    float scale_log2;
    const float *k_scale, *v_scale;
    const float *rope;
    int max_pos;
    int *err;
};

using namespace tc;

// ------------------------------------------------------------------ work item

struct Item {
    int b, kvh, head[2], row0[2], n, L, t_base;
    bool valid[2];
    int n_kv;  // K/V tiles to visit
};

// Item order: (sequence, kv head) major, so the 2 x 16 items that read one (sequence, kv head)
// K/V run on neighbouring SMs at the same time and share its tiles in L2 (row-tile-major
// order spread them over waves, and the concurrent working set overflowed L2); inside a
// group the heaviest (last) row tiles come first, so the light ones fill the tail.
__device__ __forceinline__ Item decode_item(const PrefillParams &p, int idx) {
    Item it;
    const int G = p.Hq / p.Hkv;
    int qt, h0, h1;
    if (G >= 2) {
        const int pairs = G / 2;
        const int pair = idx % pairs;
        int r = idx / pairs;
        qt = p.n_qt - 1 - r % p.n_qt;
        r /= p.n_qt;
        it.kvh = r % p.Hkv;
        it.b = r / p.Hkv;
        h0 = it.kvh * G + 2 * pair;
        h1 = h0 + 1;
        it.row0[0] = it.row0[1] = qt * kRows;
    } else {
        const int nqt2 = (p.n_qt + 1) / 2;
        int r = idx;
        qt = nqt2 - 1 - r % nqt2;
        r /= nqt2;
        const int h = r % p.Hq;
        it.b = r / p.Hq;
        it.kvh = h;
        h0 = h1 = h;
        it.row0[0] = 2 * qt * kRows;
        it.row0[1] = it.row0[0] + kRows;
    }
    it.head[0] = h0;
    it.head[1] = h1;
    it.t_base = __ldg(p.cu_seqlens + it.b);
    it.n = __ldg(p.cu_seqlens + it.b + 1) - it.t_base;
    it.L = __ldg(p.context_lens + it.b);
    int ext = 0;
    for (int i = 0; i < 2; ++i) {
        it.valid[i] = it.row0[i] < it.n;
        if (it.valid[i]) {
            const int e = it.L - it.n + min(it.row0[i] + kRows, it.n);
            ext = max(ext, e);
        }
    }
    ext = min(ext, it.L);
    it.n_kv = ext > 0 ? (ext + kKeys - 1) / kKeys : 0;
    return it;
}

// ------------------------------------------------------------------ the kernel

template <int D, bool FP8>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const PrefillParams p) {
    using Geo = PGeo<D, FP8>;
    constexpr int KS = Geo::kKStages, VS = Geo::kVStages;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t *smem = smem_raw + (sbase - smem_u32(smem_raw));

    const uint32_t sQ = sbase + Geo::kOffQ;
    const uint32_t sK = sbase + Geo::kOffK;
    const uint32_t sV = sbase + Geo::kOffV;
    const uint32_t sStg = sbase + Geo::kOffStg;  // FP8: raw K tile, then raw V tile
    const uint32_t bar0 = sbase + Geo::kOffBar;
    // barrier addresses
    const uint32_t b_qfull = bar0 + 0, b_qready = bar0 + 8, b_vraw = bar0 + 16, b_ofinal = bar0 + 24;
    const uint32_t b_sfull = bar0 + 32;   // [2]
    const uint32_t b_pfull = bar0 + 48;   // [2]
    const uint32_t b_drain = bar0 + 64;
    const uint32_t b_stgfull = bar0 + 80, b_stgempty = bar0 + 88;  // FP8 staging
    const uint32_t b_qfree = bar0 + 96;   // the item's last S MMAs have read the Q tiles
    const uint32_t b_ofree = bar0 + 104;  // [2] the epilogue has read O_i
    const uint32_t b_kfull = bar0 + 128;  // [KS]
    const uint32_t b_kempty = b_kfull + 8 * KS;
    const uint32_t b_vfull = b_kempty + 8 * KS;  // [VS]
    const uint32_t b_vempty = b_vfull + 8 * VS;
    volatile uint32_t *tmem_slot = reinterpret_cast<volatile uint32_t *>(smem + Geo::kOffBar + 72);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Geo::kOffBar + 76);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_wait();
    pdl_trigger();

    if (threadIdx.x == 0) {
        mbar_init(b_qfull, 1);
        mbar_init(b_qready, 256);
        mbar_init(b_vraw, 1);
        mbar_init(b_ofinal, 1);
        mbar_init(b_drain, 1);
        mbar_init(b_qfree, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(b_sfull + 8 * i, 1);
            mbar_init(b_pfull + 8 * i, 128);
            mbar_init(b_ofree + 8 * i, 128);
        }
        // one arrival with the TMA byte count; widened E4M3: the 64 converter threads
        for (int s = 0; s < KS; ++s) {
            mbar_init(b_kfull + 8 * s, Geo::kConv ? 64 : 1);
            mbar_init(b_kempty + 8 * s, 1);
        }
        for (int s = 0; s < VS; ++s) {
            mbar_init(b_vfull + 8 * s, Geo::kConv ? 64 : 1);
            mbar_init(b_vempty + 8 * s, 1);
        }
        mbar_init(b_stgfull, 1);
        mbar_init(b_stgempty, 64);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;"
                     ::"r"(smem_u32((const void *)tmem_slot)));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // Persistent: this CTA takes items blockIdx.x, blockIdx.x + gridDim.x, ...  Every role
    // walks the same list, so the counters below agree: li = active items so far (phases of
    // the per-item barriers), g = key tiles so far (ring stages and per-tile phases).  An
    // item is active when it has rows and keys; an item with rows but no keys only gets
    // zero rows (written by the softmax warps).
    auto active = [&](const Item &it) { return it.valid[0] && it.n_kv > 0; };

    if (warp < kSoftmax0) {
    if (warp == 0) {
        // ---------------------------------------------------------------- producer
        // outstanding fills: bit s = K stage s, bit 8+s = V stage s, bit 16 = E4M3 staging,
        // bit 17 = a partial-last-block V fill (on b_vraw), bit 18 = Q tiles
        uint32_t issued = 0;
        uint32_t phase_bits = 0;
        bool ok = true;
        int li = 0, g = 0, nfix = 0;
        if (lane == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_k);
            prefetch_tmap(&tm_v);
        }
        // first row past the cache: TMA reads it as zeros
        const int oob = (int)min(p.num_blocks * p.bs, (long long)0x7fffffff);
        // The box of every K/V tile this lane loads: 16-key piece box_piece, half box_half
        // (8-token blocks: two boxes of 8 rows per piece) and 64-column slab box_slab.  The
        // boxes of a tile are issued by their lanes at once, so a freed stage refills with
        // one warp instruction instead of a serial run of copies.
        const bool two = p.bs == 8;
        const int n_box = (two ? 16 : 8) * (Geo::kConv ? 1 : Geo::kKVSlabs);
        const int box_half = two ? (lane & 1) : 0;
        const int box_piece = two ? ((lane >> 1) & 7) : (lane & 7);
        const int box_slab = two ? (lane >> 4) : (lane >> 3);
        const uint32_t box_off = (uint32_t)(box_slab * Geo::kSlabBytes + box_piece * 2048 + box_half * 1024);
        for (int idx = blockIdx.x; idx < p.n_items && ok; idx += gridDim.x) {
            const Item it = decode_item(p, idx);
            if (!active(it)) continue;
            const int n_kv = it.n_kv;
            const int Lc = min(it.L, p.max_tokens);
            const int npiece = (Lc + kPiece - 1) / kPiece;  // 16-token pieces holding the sequence
            // Q tiles: the previous item's S MMAs must have finished reading the buffer
            if (lane == 0) {
                if (*abort_flag || (li > 0 && !mbar_wait_bounded(b_qfree, (li - 1) & 1, p.err))) {
                    ok = false;
                    *abort_flag = 1;
                } else {
                    mbar_arrive_expect_tx(b_qfull, 2 * Geo::kQBytes);
                    for (int i = 0; i < 2; ++i)
                        for (int s = 0; s < Geo::kSlabs; ++s)
                            tma_load_3d(sQ + i * Geo::kQBytes + s * Geo::kSlabBytes, &tm_q, b_qfull, 64 * s,
                                        it.head[i], it.t_base + it.row0[i]);
                    issued |= 1u << 18;
                    phase_bits = (phase_bits & ~(1u << 18)) | ((uint32_t)(li & 1) << 18);
                }
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) break;
            for (int j = 0; j < n_kv && ok; ++j) {
                const int gg = g + j;
                const int ks = gg % KS, vs = gg % VS;
                const uint32_t kpar = ((gg / KS) & 1) ^ 1, vpar = ((gg / VS) & 1) ^ 1;
                // This lane's box of the tile (see box_* above): its cache row, from its own
                // block-table entry, or the first row past the cache (read as zeros).
                int row = oob;
                if (lane < n_box) {
                    const int lb = j * 8 + box_piece;  // 16-token piece of the sequence
                    int entry = lb, off = 0;
                    bool valid = lb < npiece;
                    if (p.bs == 32) {
                        entry = lb >> 1;
                        off = (lb & 1) * 16;
                    } else if (p.bs == 8) {
                        entry = 2 * lb + box_half;
                        valid = entry * 8 < Lc;
                    }
                    if (valid) {
                        const int e = __ldg(p.block_tables + (size_t)it.b * p.max_blocks + entry);
                        if (e < 0 || (long long)e >= p.num_blocks) atomicOr(p.err, kErrBounds);
                        else row = e * p.bs + off;
                    }
                }
                if constexpr (Geo::kConv) {
                    // raw E4M3 tiles go to the single staging buffer; the converter warps
                    // widen them into the MMA operand stage
                    if (lane == 0) {
                        if (*abort_flag || !mbar_wait_bounded(b_stgempty, (gg & 1) ^ 1, p.err)) {
                            ok = false;
                            *abort_flag = 1;
                        } else {
                            mbar_arrive_expect_tx(b_stgfull, 2 * Geo::kStgBytes);
                            issued |= 1u << 16;
                            phase_bits = (phase_bits & ~(1u << 16)) | ((uint32_t)(gg & 1) << 16);
                        }
                    }
                    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                    if (!ok) break;
                    if (lane < n_box) {  // (one slab: the boxes are whole D-byte rows)
                        const uint32_t off = (uint32_t)((box_piece * kPiece + box_half * 8) * D);
                        tma_load_3d(sStg + off, &tm_k, b_stgfull, 0, it.kvh, row);
                        tma_load_3d(sStg + Geo::kStgBytes + off, &tm_v, b_stgfull, 0, it.kvh, row);
                    }
                    continue;
                }
                // the tile holding the sequence's partial last block: its rows past Lc hold
                // whatever the block held before and are zeroed before use
                const bool fix = (Lc % p.bs) != 0 && j == (Lc - 1) / kKeys;
                if (lane == 0) {
                    if (*abort_flag || !mbar_wait_bounded(b_kempty + 8 * ks, kpar, p.err)) {
                        ok = false;
                        *abort_flag = 1;
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                if (!ok) break;
                // lane 0 arms the barrier, then every box lane issues its own load
                if (lane == 0) {
                    const uint32_t kb = b_kfull + 8 * ks;
                    mbar_arrive_expect_tx(kb, Geo::kKVBytes);
                    issued |= 1u << ks;
                    phase_bits = (phase_bits & ~(1u << ks)) | ((uint32_t)((gg / KS) & 1) << ks);
                }
                __syncwarp();
                if (lane < n_box)
                    tma_load_3d(sK + ks * Geo::kKVBytes + box_off, &tm_k, b_kfull + 8 * ks, 64 * box_slab, it.kvh, row);
                // V of the same tile: its stage frees later (after PV1 of tile gg - VS)
                const uint32_t vb = fix ? b_vraw : b_vfull + 8 * vs;
                if (lane == 0) {
                    if (*abort_flag || !mbar_wait_bounded(b_vempty + 8 * vs, vpar, p.err)) {
                        ok = false;
                        *abort_flag = 1;
                    } else {
                        mbar_arrive_expect_tx(vb, Geo::kKVBytes);
                        if (!fix) {
                            issued |= 1u << (8 + vs);
                            phase_bits = (phase_bits & ~(1u << (8 + vs))) | ((uint32_t)((gg / VS) & 1) << (8 + vs));
                        } else {
                            // this fill completes on b_vraw; the stage's earlier fill has
                            // landed (its PV1 freed the stage), so its bit is retired
                            issued = (issued & ~(1u << (8 + vs))) | (1u << 17);
                            phase_bits = (phase_bits & ~(1u << 17)) | ((uint32_t)(nfix & 1) << 17);
                        }
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                if (!ok) break;
                if (lane < n_box) tma_load_3d(sV + vs * Geo::kKVBytes + box_off, &tm_v, vb, 64 * box_slab, it.kvh, row);
                ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                if (!ok) break;
                if (fix) {
                    // zero the rows past the sequence in the tile's partial block, then publish
                    bool landed = true;
                    if (lane == 0) landed = mbar_wait_bounded(b_vraw, nfix & 1, p.err);
                    landed = __shfl_sync(0xffffffffu, landed ? 1 : 0, 0) != 0;
                    ++nfix;
                    if (landed) {
                        if (lane == 0) issued &= ~(1u << 17);
                        // tile rows [Lc, end of that block) (the block lies inside the tile)
                        const int first = Lc % kKeys;
                        const int rows = ((Lc + p.bs - 1) / p.bs) * p.bs - Lc;
                        for (int s = 0; s < Geo::kKVSlabs; ++s) {
                            const uint32_t row0 = sV + vs * Geo::kKVBytes + s * Geo::kSlabBytes + first * 128;
                            for (int e = lane; e < rows * 8; e += 32)
                                asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(row0 + e * 16),
                                             "r"(0)
                                             : "memory");
                        }
                        fence_proxy_async_smem();
                    }
                    __syncwarp();
                    if (lane == 0) {
                        if (landed) mbar_arrive(b_vfull + 8 * vs);
                        else *abort_flag = 1;
                    }
                    if (!landed) ok = false;
                }
            }
            g += n_kv;
            ++li;
        }
        // drain outstanding TMA copies before the CTA can exit
        if (lane == 0) {
            if ((issued >> 18) & 1) mbar_wait_bounded(b_qfull, (phase_bits >> 18) & 1, p.err);
            if ((issued >> 16) & 1) mbar_wait_bounded(b_stgfull, (phase_bits >> 16) & 1, p.err);
            if ((issued >> 17) & 1) mbar_wait_bounded(b_vraw, (phase_bits >> 17) & 1, p.err);
            for (int s = 0; s < KS; ++s)
                if ((issued >> s) & 1) mbar_wait_bounded(b_kfull + 8 * s, (phase_bits >> s) & 1, p.err);
            for (int s = 0; s < VS; ++s)
                if ((issued >> (8 + s)) & 1)
                    mbar_wait_bounded(b_vfull + 8 * s, (phase_bits >> (8 + s)) & 1, p.err);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idS = mma_idesc(kRows, kKeys, false, FP8);  // (E4M3: type code 0, as f16)
            constexpr uint32_t idO = mma_idesc(kRows, D, true, FP8);
            const uint32_t tS[2] = {tmem + 0, tmem + 128};
            const uint32_t tO[2] = {tmem + 256, tmem + 256 + D};
            auto issue_s = [&](int i, int kst) {
                if constexpr (Geo::kF8) {
                    // S_i = (Q_hi + Q_lo) K^T: the Q tile holds its rows as E4M3 codes, the high
                    // parts in slab 0 and the low parts in slab 1; 32 codes per k step
#pragma unroll
                    for (int kk = 0; kk < D / 32; ++kk) {
                        const uint64_t kd = sw128_desc(sK + kst * Geo::kKVBytes + kk * 32, 16, 1024);
                        mma_ss_f8(tS[i], sw128_desc(sQ + i * Geo::kQBytes + kk * 32, 16, 1024), kd, idS, kk > 0);
                        mma_ss_f8(tS[i], sw128_desc(sQ + i * Geo::kQBytes + Geo::kSlabBytes + kk * 32, 16, 1024),
                                  kd, idS, 1u);
                    }
                } else {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk / 4) * Geo::kSlabBytes + (kk % 4) * 32;
                        mma_ss(tS[i], sw128_desc(sQ + i * Geo::kQBytes + off, 16, 1024),
                               sw128_desc(sK + kst * Geo::kKVBytes + off, 16, 1024), idS, kk > 0);
                    }
                }
                mma_commit(b_sfull + 8 * i);
                if (i == 1) mma_commit(b_kempty + 8 * kst);  // both S MMAs of this K tile issued
            };
            auto issue_pv = [&](int i, int vst, int j) {
                if constexpr (Geo::kF8) {
                    // O_i += (P_hi + P_lo) V: P as E4M3 codes in TMEM (4 keys per column; the high
                    // parts in columns 0-31, the low in 32-63), V MN-major straight from the cache
#pragma unroll
                    for (int kk = 0; kk < kKeys / 32; ++kk) {
                        const uint64_t vd = sw128_desc(sV + vst * Geo::kKVBytes + kk * 4096, Geo::kSlabBytes, 1024);
                        mma_ts_f8(tO[i], tS[i] + 8 * kk, vd, idO, (j > 0 || kk > 0) ? 1u : 0u);
                        mma_ts_f8(tO[i], tS[i] + 32 + 8 * kk, vd, idO, 1u);
                    }
                } else {
#pragma unroll
                    for (int kk = 0; kk < kKeys / 16; ++kk)
                        mma_ts(tO[i], tS[i] + 8 * kk,
                               sw128_desc(sV + vst * Geo::kKVBytes + kk * 2048, Geo::kSlabBytes, 1024), idO,
                               (j > 0 || kk > 0) ? 1u : 0u);
                }
            };
            bool ok = true;
            int li = 0, g = 0;
            for (int idx = blockIdx.x; idx < p.n_items && ok; idx += gridDim.x) {
                const Item it = decode_item(p, idx);
                if (!active(it)) continue;
                const int n_kv = it.n_kv;
                ok = !*abort_flag && mbar_wait_bounded(b_qready, li & 1, p.err) &&
                     mbar_wait_bounded(b_kfull + 8 * (g % KS), (g / KS) & 1, p.err);
                if (!ok) break;
                tc_fence_after();
                // S MMAs write the S columns in issue order after the previous item's PV
                // MMAs that read them as P
                issue_s(0, g % KS);
                issue_s(1, g % KS);
                if (n_kv == 1) mma_commit(b_qfree);
                for (int j = 0; j < n_kv && ok; ++j) {
                    const int gg = g + j;
                    const int vst = gg % VS;
                    const uint32_t vpar = (gg / VS) & 1;
                    const int kst1 = (gg + 1) % KS;
                    const uint32_t kpar1 = ((gg + 1) / KS) & 1;
                    // the first PV of an item overwrites O_i: the previous item's epilogue
                    // must have read it
                    ok = mbar_wait_bounded(b_vfull + 8 * vst, vpar, p.err) &&
                         mbar_wait_bounded(b_pfull + 0, gg & 1, p.err) &&
                         (j > 0 || li == 0 || mbar_wait_bounded(b_ofree + 0, (li - 1) & 1, p.err));
                    if (!ok) break;
                    tc_fence_after();
                    issue_pv(0, vst, j);
                    if (j + 1 < n_kv) {
                        ok = mbar_wait_bounded(b_kfull + 8 * kst1, kpar1, p.err);
                        if (!ok) break;
                        tc_fence_after();
                        issue_s(0, kst1);
                    }
                    ok = mbar_wait_bounded(b_pfull + 8, gg & 1, p.err) &&
                         (j > 0 || li == 0 || mbar_wait_bounded(b_ofree + 8, (li - 1) & 1, p.err));
                    if (!ok) break;
                    tc_fence_after();
                    issue_pv(1, vst, j);
                    mma_commit(b_vempty + 8 * vst);
                    if (j + 1 < n_kv) {
                        issue_s(1, kst1);
                        if (j + 2 == n_kv) mma_commit(b_qfree);  // the item's last S MMAs
                    }
                }
                mma_commit(b_ofinal);
                g += n_kv;
                ++li;
            }
            if (!ok) *abort_flag = 1;
            // every MMA issued above has finished before TMEM can be released
            mma_commit(b_drain);
            mbar_wait_bounded(b_drain, 0, p.err);
        }
    } else if (Geo::kConv && warp >= 2) {
        // ---------------------------------------------------------------- E4M3 -> f16
        // Warps 2-3 widen each raw tile into the swizzled operand layout (the same
        // 128-byte-swizzled K-major layout TMA produces for 16-bit caches).  V rows of keys
        // past the sequence are written as zeros (0 * NaN would poison O).
        const int ct = threadIdx.x - 64;
        constexpr int CPR = D / 16;  // 16-byte E4M3 chunks per row
        bool run = true;
        int g = 0;
        for (int idx = blockIdx.x; idx < p.n_items && run; idx += gridDim.x) {
            const Item it = decode_item(p, idx);
            if (!active(it)) continue;
            const int Lc = min(it.L, p.max_tokens);
            for (int j = 0; j < it.n_kv; ++j) {
                const int gg = g + j;
                const int ks = gg % KS, vs = gg % VS;
                if (*abort_flag || !mbar_wait_bounded(b_stgfull, gg & 1, p.err)) {
                    *abort_flag = 1;
                    run = false;
                    break;
                }
                const int key0 = j * kKeys;
                bool got = true;
#pragma unroll
                for (int t = 0; t < 2; ++t) {  // K, then V (each into its own ring)
                    const uint32_t empty_b = t == 0 ? b_kempty + 8 * ks : b_vempty + 8 * vs;
                    const uint32_t par = t == 0 ? (((gg / KS) & 1) ^ 1) : (((gg / VS) & 1) ^ 1);
                    if (*abort_flag || !mbar_wait_bounded(empty_b, par, p.err)) {
                        got = false;
                        break;
                    }
                    const uint32_t src = sStg + t * Geo::kStgBytes;
                    const uint32_t dst = t == 0 ? sK + ks * Geo::kKVBytes : sV + vs * Geo::kKVBytes;
#pragma unroll 2
                    for (int idx2 = ct; idx2 < kKeys * CPR; idx2 += 64) {
                        const int row = idx2 / CPR, c = idx2 % CPR;
                        uint4 raw = lds128(src + row * D + c * 16);
                        if (t == 1 && key0 + row >= Lc) raw = make_uint4(0u, 0u, 0u, 0u);
                        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
                        uint32_t h[8];
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            h[2 * q] = e4m3x2_to_f16x2(w[q] & 0xFFFFu);
                            h[2 * q + 1] = e4m3x2_to_f16x2(w[q] >> 16);
                        }
#pragma unroll
                        for (int hf = 0; hf < 2; ++hf) {
                            const int lc = 2 * c + hf;  // 8-element chunk of the 16-bit row
                            const uint32_t a =
                                dst + (lc / 8) * Geo::kSlabBytes + row * 128 + (((lc % 8) ^ (row & 7)) << 4);
                            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(h[4 * hf]),
                                         "r"(h[4 * hf + 1]), "r"(h[4 * hf + 2]), "r"(h[4 * hf + 3])
                                         : "memory");
                        }
                    }
                    fence_proxy_async_smem();
                    mbar_arrive(t == 0 ? b_kfull + 8 * ks : b_vfull + 8 * vs);
                }
                if (!got) {
                    *abort_flag = 1;
                    run = false;
                    break;
                }
                mbar_arrive(b_stgempty);
            }
            g += it.n_kv;
        }
    }
    } else {
        // ---------------------------------------------------------------- softmax
        const int wg = (warp - kSoftmax0) / 4;       // tile index
        const int r = (warp & 3) * 32 + lane;         // row within the tile == TMEM lane
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_off + (uint32_t)(wg * 128);
        const uint32_t tO = tmem + lane_off + (uint32_t)(256 + wg * D);
        bool alive = true;  // false after a wait gave up: later waits are skipped
        int idx = blockIdx.x;
        // The next active item of this CTA; an item with rows but no keys gets zero rows.
        auto next_item = [&](Item &out) -> bool {
            for (; idx < p.n_items; idx += gridDim.x) {
                const Item it = decode_item(p, idx);
                if (!it.valid[0]) continue;
                if (it.n_kv == 0) {
                    const int row = it.row0[wg] + r;
                    if (it.valid[wg] && row < it.n) {
                        uint4 *dst = reinterpret_cast<uint4 *>(p.out + ((size_t)(it.t_base + row) * p.Hq + it.head[wg]) * D);
                        for (int v = 0; v < D / 8; ++v) dst[v] = make_uint4(0u, 0u, 0u, 0u);
                    }
                    continue;
                }
                out = it;
                idx += gridDim.x;
                return true;
            }
            return false;
        };
        // returns the reciprocal of the power-of-two scale applied to this thread's Q row
        // before its E4M3 split (1 on the other paths)
        auto prologue = [&](const Item &it, int li) -> float {
            const int row = it.row0[wg] + r;  // row within the sequence's new tokens
            const bool row_valid = row < it.n;
            const int pos = it.L - it.n + row;
            // Q-RoPE on load: this thread rotates its row in shared memory.  In fp32: one
            // product, one FMA and one rounding to bf16 per value, i.e. within one bf16 ulp of
            // the exact rotation (which pkv_rope_apply and the K rotation of pkv_kv_store
            // produce bit for bit); the difference stays far inside the attention tolerance and
            // keeps this prologue off the critical path of the tensor pipe.
            const bool rope_row = p.rope && row_valid && it.valid[wg];
            const bool pos_ok = pos >= 0 && pos < p.max_pos;
            const bool same_rows = it.row0[0] == it.row0[1];
            constexpr int NP = D / 32;  // chunk pairs per warpgroup (same-rows split)
            const int lc0 = wg * NP;
            bool ok = alive && mbar_wait_bounded(b_qfull, li & 1, p.err);
            if (!ok) alive = false;
            if (ok && rope_row) {
                if (!pos_ok) {
                    atomicOr(p.err, kErrBounds);
                } else if (same_rows) {
                    // Both tiles hold the same rows (two heads of a group): warpgroup wg rotates
                    // its half of the pairs of row r in both tiles, so each thread fetches half
                    // a table row, in one round.
                    const float4 *cs4 = reinterpret_cast<const float4 *>(p.rope + (size_t)pos * D);
                    float4 cv[2 * NP], sv[2 * NP];
#pragma unroll
                    for (int k = 0; k < 2 * NP; ++k) {
                        cv[k] = __ldg(cs4 + lc0 * 2 + k);
                        sv[k] = __ldg(cs4 + D / 8 + lc0 * 2 + k);
                    }
                    const uint32_t sw = (uint32_t)(r & 7);
#pragma unroll
                    for (int tile = 0; tile < 2; ++tile) {
                        const uint32_t qrow = sQ + tile * Geo::kQBytes + r * 128;
#pragma unroll
                        for (int k4 = 0; k4 < NP; ++k4) {
                            const int lc = lc0 + k4, lc2 = lc + D / 16;
                            const uint32_t a1 = qrow + (lc / 8) * Geo::kSlabBytes + (((lc % 8) ^ sw) << 4);
                            const uint32_t a2 = qrow + (lc2 / 8) * Geo::kSlabBytes + (((lc2 % 8) ^ sw) << 4);
                            const uint4 x1 = lds128(a1), x2 = lds128(a2);
                            const uint32_t w1[4] = {x1.x, x1.y, x1.z, x1.w};
                            const uint32_t w2[4] = {x2.x, x2.y, x2.z, x2.w};
                            const float cc[8] = {cv[2 * k4].x, cv[2 * k4].y, cv[2 * k4].z, cv[2 * k4].w,
                                                 cv[2 * k4 + 1].x, cv[2 * k4 + 1].y, cv[2 * k4 + 1].z,
                                                 cv[2 * k4 + 1].w};
                            const float ss[8] = {sv[2 * k4].x, sv[2 * k4].y, sv[2 * k4].z, sv[2 * k4].w,
                                                 sv[2 * k4 + 1].x, sv[2 * k4 + 1].y, sv[2 * k4 + 1].z,
                                                 sv[2 * k4 + 1].w};
                            uint32_t o1[4], o2[4];
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const float a0 = bf16lo(w1[q]), a1v = bf16hi(w1[q]);
                                const float b0 = bf16lo(w2[q]), b1v = bf16hi(w2[q]);
                                const float c0 = cc[2 * q], c1 = cc[2 * q + 1], s0 = ss[2 * q], s1 = ss[2 * q + 1];
                                o1[q] = pack_bf16x2(__fmaf_rn(a0, c0, -__fmul_rn(b0, s0)),
                                                    __fmaf_rn(a1v, c1, -__fmul_rn(b1v, s1)));
                                o2[q] = pack_bf16x2(__fmaf_rn(b0, c0, __fmul_rn(a0, s0)),
                                                    __fmaf_rn(b1v, c1, __fmul_rn(a1v, s1)));
                            }
                            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a1), "r"(o1[0]),
                                         "r"(o1[1]), "r"(o1[2]), "r"(o1[3]) : "memory");
                            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a2), "r"(o2[0]),
                                         "r"(o2[1]), "r"(o2[2]), "r"(o2[3]) : "memory");
                        }
                    }
                } else {
                    const float4 *cs4 = reinterpret_cast<const float4 *>(p.rope + (size_t)pos * D);
                    const uint32_t qrow = sQ + wg * Geo::kQBytes + r * 128;
                    const uint32_t sw = (uint32_t)(r & 7);
#pragma unroll 1
                    for (int g4 = 0; g4 < D / 16; g4 += 4) {
                        float4 cv[8], sv[8];
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            cv[k] = __ldg(cs4 + g4 * 2 + k);
                            sv[k] = __ldg(cs4 + D / 8 + g4 * 2 + k);
                        }
#pragma unroll
                        for (int k4 = 0; k4 < 4; ++k4) {
                            const int lc = g4 + k4, lc2 = lc + D / 16;  // chunk pair (lc, lc + D/16)
                            const uint32_t a1 = qrow + (lc / 8) * Geo::kSlabBytes + (((lc % 8) ^ sw) << 4);
                            const uint32_t a2 = qrow + (lc2 / 8) * Geo::kSlabBytes + (((lc2 % 8) ^ sw) << 4);
                            uint4 x1 = lds128(a1), x2 = lds128(a2);
                            const uint32_t w1[4] = {x1.x, x1.y, x1.z, x1.w};
                            const uint32_t w2[4] = {x2.x, x2.y, x2.z, x2.w};
                            const float cc[8] = {cv[2 * k4].x, cv[2 * k4].y, cv[2 * k4].z, cv[2 * k4].w,
                                                 cv[2 * k4 + 1].x, cv[2 * k4 + 1].y, cv[2 * k4 + 1].z,
                                                 cv[2 * k4 + 1].w};
                            const float ss[8] = {sv[2 * k4].x, sv[2 * k4].y, sv[2 * k4].z, sv[2 * k4].w,
                                                 sv[2 * k4 + 1].x, sv[2 * k4 + 1].y, sv[2 * k4 + 1].z,
                                                 sv[2 * k4 + 1].w};
                            uint32_t o1[4], o2[4];
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const float a0 = bf16lo(w1[q]), a1v = bf16hi(w1[q]);
                                const float b0 = bf16lo(w2[q]), b1v = bf16hi(w2[q]);
                                const float c0 = cc[2 * q], c1 = cc[2 * q + 1], s0 = ss[2 * q], s1 = ss[2 * q + 1];
                                o1[q] = pack_bf16x2(__fmaf_rn(a0, c0, -__fmul_rn(b0, s0)),
                                                    __fmaf_rn(a1v, c1, -__fmul_rn(b1v, s1)));
                                o2[q] = pack_bf16x2(__fmaf_rn(b0, c0, __fmul_rn(a0, s0)),
                                                    __fmaf_rn(b1v, c1, __fmul_rn(a1v, s1)));
                            }
                            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a1), "r"(o1[0]),
                                         "r"(o1[1]), "r"(o1[2]), "r"(o1[3]) : "memory");
                            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a2), "r"(o2[0]),
                                         "r"(o2[1]), "r"(o2[2]), "r"(o2[3]) : "memory");
                        }
                    }
                }
            }
            float qinv = 1.f;
            if constexpr (Geo::kConv) {
                // the widened-E4M3 path multiplies in f16: convert this row of Q (swizzle
                // untouched), after both warpgroups finished rotating (they may share rows)
                named_bar(2, 256);
                if (ok) {
                    const uint32_t qrow = sQ + wg * Geo::kQBytes + r * 128;
#pragma unroll 1
                    for (int ch = 0; ch < D / 8; ++ch) {
                        const uint32_t a = qrow + (ch / 8) * Geo::kSlabBytes + (ch % 8) * 16;
                        uint4 x = lds128(a);
                        uint16_t *e = reinterpret_cast<uint16_t *>(&x);
#pragma unroll
                        for (int k = 0; k < 8; ++k) e[k] = bf16_to_f16_bits(e[k]);
                        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(x.x), "r"(x.y),
                                     "r"(x.z), "r"(x.w) : "memory");
                    }
                }
            }
            if constexpr (Geo::kF8) {
                // E4M3 operands: after both warpgroups finished rotating, this thread turns its
                // row of tile wg into 128 high and 128 low E4M3 codes, in place -- the high
                // ones as slab 0's row, the low ones as slab 1's (each a 128-byte K-major
                // swizzled row, the layout of an E4M3 A tile).  The row is first scaled by the
                // power of two that puts its largest |q| in [224, 448]; the score scale takes
                // the reciprocal.
                named_bar(2, 256);
                if (ok) {
                    const uint32_t qrow = sQ + wg * Geo::kQBytes + r * 128;
                    const uint32_t sw = (uint32_t)(r & 7);
                    uint32_t w[64];
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        const uint4 x = lds128(qrow + (c >> 3) * Geo::kSlabBytes + (((c & 7) ^ sw) << 4));
                        w[4 * c] = x.x;
                        w[4 * c + 1] = x.y;
                        w[4 * c + 2] = x.z;
                        w[4 * c + 3] = x.w;
                    }
                    float amax = 0.f;
#pragma unroll
                    for (int i = 0; i < 64; ++i) amax = fmaxf(amax, fmaxf(fabsf(bf16lo(w[i])), fabsf(bf16hi(w[i]))));
                    const float sq = amax > 0.f
                                         ? __int_as_float(__float_as_int(fminf(448.f / amax, 0x1p100f)) & 0x7F800000)
                                         : 1.f;
                    qinv = 1.f / sq;  // exact: sq is a power of two
#pragma unroll
                    for (int k = 0; k < 8; ++k) {  // codes 16k .. 16k+15 = bf16 words 8k .. 8k+7
                        uint32_t hw[4], lw[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const uint32_t w0 = w[8 * k + 2 * j], w1 = w[8 * k + 2 * j + 1];
                            split_e4m3x4(bf16lo(w0) * sq, bf16hi(w0) * sq, bf16lo(w1) * sq, bf16hi(w1) * sq, hw[j],
                                         lw[j]);
                        }
                        const uint32_t off = (uint32_t)((k ^ sw) << 4);
                        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(qrow + off), "r"(hw[0]),
                                     "r"(hw[1]), "r"(hw[2]), "r"(hw[3]) : "memory");
                        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(qrow + Geo::kSlabBytes + off),
                                     "r"(lw[0]), "r"(lw[1]), "r"(lw[2]), "r"(lw[3]) : "memory");
                    }
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(b_qready);
            return qinv;
        };

        // Q of item li+1 is rotated before the epilogue of item li, so the tensor pipe can
        // start the next item's S MMAs while this item's O is written out.
        Item it;
        bool have = next_item(it);
        float qinv = 1.f;
        if (have) qinv = prologue(it, 0);
        int li = 0, g = 0;
        while (have) {
            if (*abort_flag) alive = false;
            const int n_kv = it.n_kv;
            const int Lc = min(it.L, p.max_tokens);
            if (Lc < it.L && r == 0 && wg == 0) atomicOr(p.err, kErrBounds);
            const int row = it.row0[wg] + r;              // row within the sequence's new tokens
            const bool row_valid = row < it.n;
            const int pos = it.L - it.n + row;
            const int limit = min(pos, Lc - 1);           // last visible key
            const float c = p.scale_log2 * (p.k_scale ? __ldg(p.k_scale + it.kvh) : 1.f) * qinv;
            // Every tcgen05.ld/st below is executed by all 32 lanes of the warp together (the
            // instructions are warp-aligned); per-row differences are data, not control flow.
            float m_used = -INFINITY, l_sum = 0.f;
            for (int j = 0; j < n_kv; ++j) {
                bool got = alive && !*abort_flag && mbar_wait_bounded(b_sfull + 8 * wg, (g + j) & 1, p.err);
                if (!__all_sync(0xffffffffu, got)) {
                    alive = false;
                    *abort_flag = 1;
                    break;
                }
                tc_fence_after();
                float s[kKeys];
#pragma unroll
                for (int q4 = 0; q4 < kKeys / 32; ++q4) {
                    uint32_t rr[32];
                    tmem_ld32(tS + q4 * 32, rr);
#pragma unroll
                    for (int e = 0; e < 32; ++e) s[q4 * 32 + e] = __uint_as_float(rr[e]);
                }
                tc_wait_ld();
                const int key0 = j * kKeys;
                if (key0 + kKeys - 1 > limit) {  // diagonal / tail tile: mask keys past the limit
#pragma unroll
                    for (int e = 0; e < kKeys; ++e)
                        if (key0 + e > limit) s[e] = -INFINITY;
                }
                float m8[8];  // eight independent max chains instead of one 128-long chain
#pragma unroll
                for (int k = 0; k < 8; ++k) m8[k] = s[k];
#pragma unroll
                for (int e = 8; e < kKeys; e += 8)
#pragma unroll
                    for (int k = 0; k < 8; ++k) m8[k] = fmaxf(m8[k], s[e + k]);
                const float mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                                       fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
                const float m_tile = mx * c;  // c > 0; -inf when the row sees no key here
                // a new running max only when it grew by more than 2^8 (lazy rescale)
                float alpha = 1.f;
                if (m_tile > m_used + kRescaleLog2) {
                    if (m_used != -INFINITY && j > 0) alpha = ex2(m_used - m_tile);
                    m_used = m_tile;
                }
                l_sum *= alpha;
                const float neg_m = (m_used == -INFINITY) ? 0.f : -m_used;  // masked s: p = 0
                const float2 c2 = make_float2(c, c), nm2 = make_float2(neg_m, neg_m);
                float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                                 make_float2(0.f, 0.f)};
#pragma unroll
                for (int h = 0; h < kKeys / 32; ++h) {  // 32 keys
                    if constexpr (Geo::kF8) {
                        // -> 8 columns of high E4M3 parts (4 keys each) at 8h, 8 of low parts at 32 + 8h
                        uint32_t hw[8], lw[8];
#pragma unroll
                        for (int e = 0; e < 32; e += 4) {
                            const float2 x0 = __ffma2_rn(make_float2(s[h * 32 + e], s[h * 32 + e + 1]), c2, nm2);
                            const float2 x1 = __ffma2_rn(make_float2(s[h * 32 + e + 2], s[h * 32 + e + 3]), c2, nm2);
                            const float2 p0 = make_float2(ex2(x0.x), ex2(x0.y)), p1 = make_float2(ex2(x1.x), ex2(x1.y));
                            acc[(e / 2) & 3] = __fadd2_rn(acc[(e / 2) & 3], p0);
                            acc[(e / 2 + 1) & 3] = __fadd2_rn(acc[(e / 2 + 1) & 3], p1);
                            split_e4m3x4(p0.x, p0.y, p1.x, p1.y, hw[e / 4], lw[e / 4]);
                        }
                        tmem_st8(tS + h * 8, hw);
                        tmem_st8(tS + 32 + h * 8, lw);
                    } else {
                        // -> 16 packed columns
                        uint32_t rr[16];
#pragma unroll
                        for (int e = 0; e < 32; e += 2) {
                            const float2 x = __ffma2_rn(make_float2(s[h * 32 + e], s[h * 32 + e + 1]), c2, nm2);
                            const float2 pp = make_float2(ex2(x.x), ex2(x.y));
                            acc[(e / 2) & 3] = __fadd2_rn(acc[(e / 2) & 3], pp);
                            rr[e / 2] = FP8 ? pack_f16x2(pp.x, pp.y) : pack_bf16x2(pp.x, pp.y);
                        }
                        tmem_st16(tS + h * 16, rr);
                    }
                }
                l_sum += ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) +
                         ((acc[2].x + acc[2].y) + (acc[3].x + acc[3].y));
                if (__any_sync(0xffffffffu, alpha != 1.f)) {
                    // O_i <- alpha * O_i (alpha = 1 on rows that keep their max).  PV_i of the
                    // previous tile has completed: it was issued before this tile's S_i, whose
                    // completion we waited for.
#pragma unroll 1
                    for (int q4 = 0; q4 < D / 32; ++q4) {
                        uint32_t rr[32];
                        tmem_ld32(tO + q4 * 32, rr);
                        tc_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) rr[e] = __float_as_uint(__uint_as_float(rr[e]) * alpha);
                        tmem_st32(tO + q4 * 32, rr);
                    }
                }
                tc_wait_st();
                tc_fence_before();
                mbar_arrive(b_pfull + 8 * wg);
            }

            Item nxt;
            const bool have_next = next_item(nxt);
            float qinv_next = 1.f;
            if (have_next) qinv_next = prologue(nxt, li + 1);
            // ---- epilogue: O / l -> bf16 -> global (valid rows only)
            bool fin = alive && mbar_wait_bounded(b_ofinal, li & 1, p.err);
            if (!fin) alive = false;
            const bool done = __all_sync(0xffffffffu, fin);
            tc_fence_after();
            const bool store = row_valid && it.valid[wg];
            const float vs = p.v_scale ? __ldg(p.v_scale + it.kvh) : 1.f;
            const float inv = (done && l_sum > 0.f) ? vs / l_sum : 0.f;
            uint4 *dst = reinterpret_cast<uint4 *>(p.out + ((size_t)(it.t_base + (store ? row : 0)) * p.Hq + it.head[wg]) * D);
#pragma unroll 1
            for (int q4 = 0; q4 < D / 32; ++q4) {
                uint32_t rr[32];
                if (done) {
                    tmem_ld32(tO + q4 * 32, rr);
                    tc_wait_ld();
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) rr[e] = 0u;
                }
                if (store) {
#pragma unroll
                    for (int v8 = 0; v8 < 4; ++v8) {
                        uint4 w;
                        w.x = pack_bf16x2(__uint_as_float(rr[v8 * 8 + 0]) * inv, __uint_as_float(rr[v8 * 8 + 1]) * inv);
                        w.y = pack_bf16x2(__uint_as_float(rr[v8 * 8 + 2]) * inv, __uint_as_float(rr[v8 * 8 + 3]) * inv);
                        w.z = pack_bf16x2(__uint_as_float(rr[v8 * 8 + 4]) * inv, __uint_as_float(rr[v8 * 8 + 5]) * inv);
                        w.w = pack_bf16x2(__uint_as_float(rr[v8 * 8 + 6]) * inv, __uint_as_float(rr[v8 * 8 + 7]) * inv);
                        dst[q4 * 4 + v8] = w;
                    }
                }
            }
            // O_i has been read: the next item's first PV_i may overwrite it
            tc_fence_before();
            mbar_arrive(b_ofree + 8 * wg);
            g += n_kv;
            ++li;
            it = nxt;
            have = have_next;
            qinv = qinv_next;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem));
    }
}

template <int D, bool FP8>
cudaError_t run(const PrefillArgs &a, const PrefillParams &p, long long items, cudaStream_t s) {
    // Q: 128-byte swizzled boxes of 64 bf16 x 128 rows (one operand slab each).  K/V: for
    // bf16 the same 128-byte swizzled 64-column boxes of one block (16 rows); for E4M3 one
    // plain box of a whole block row range (widened in shared memory by the kernel).
    // E4M3 at head dim 128: one 128-byte-swizzled box per block (a whole 128-byte row per key).
    using Geo = PGeo<D, FP8>;
    constexpr int esize = FP8 ? 1 : 2;
    CUtensorMap tq, tk, tv;
    const uint64_t slots = (uint64_t)a.num_blocks * a.block_size;
    const uint32_t box_rows = a.block_size == 8 ? 8u : (uint32_t)kPiece;
    const uint32_t inner = FP8 ? (uint32_t)D : 64u;
    constexpr bool swz = !Geo::kConv;
    if (!encode_tensor_map_3d(&tq, a.q, 2, D, a.n_q_heads, a.num_tokens, 64, 1, kRows, true) ||
        !encode_tensor_map_3d(&tk, a.k_cache, esize, D, a.n_kv_heads, slots, inner, 1, box_rows, swz) ||
        !encode_tensor_map_3d(&tv, a.v_cache, esize, D, a.n_kv_heads, slots, inner, 1, box_rows, swz))
        return cudaErrorInvalidValue;
    auto k = prefill_kernel<D, FP8>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, PGeo<D, FP8>::kSmem);
    if (e != cudaSuccess) return e;
    // persistent: one CTA per SM (shared memory allows one), items taken round robin
    const int sms = current_sm_count();
    const long long grid = items < sms ? items : sms;
    return launch_pdl(k, dim3((unsigned)grid), dim3(kThreads), PGeo<D, FP8>::kSmem, s, tq, tk, tv, p);
}

}  // namespace

cudaError_t launch_paged_prefill(const PrefillArgs &a, cudaStream_t s) {
    PrefillParams p;
    p.out = static_cast<__nv_bfloat16 *>(a.out);
    p.cu_seqlens = a.cu_seqlens;
    p.block_tables = a.block_tables;
    p.context_lens = a.context_lens;
    p.max_blocks = a.max_blocks_per_seq;
    p.bs = a.block_size;
    p.max_tokens = (int)min((long long)a.max_blocks_per_seq * a.block_size, 0x7fffffffLL);
    p.B = a.num_seqs;
    p.Hq = a.n_q_heads;
    p.Hkv = a.n_kv_heads;
    p.n_qt = (a.max_new_tokens + kRows - 1) / kRows;
    p.num_blocks = a.num_blocks;
    p.scale_log2 = a.scale * kLog2e;
    p.k_scale = a.fp8 ? a.k_scale : nullptr;
    p.v_scale = a.fp8 ? a.v_scale : nullptr;
    p.rope = a.rope;
    p.max_pos = a.max_pos;
    p.err = a.err;
    if (p.n_qt == 0) return cudaSuccess;
    const int G = p.Hq / p.Hkv;
    long long items = (G >= 2) ? (long long)p.n_qt * p.B * p.Hkv * (G / 2)
                               : (long long)((p.n_qt + 1) / 2) * p.B * p.Hq;
    if (items > 0x7fffffffLL) return cudaErrorInvalidValue;
    p.n_items = (int)items;
    cudaError_t e;
    if (a.head_dim == 128) e = a.fp8 ? run<128, true>(a, p, items, s) : run<128, false>(a, p, items, s);
    else if (a.head_dim == 64) e = a.fp8 ? run<64, true>(a, p, items, s) : run<64, false>(a, p, items, s);
    else return cudaErrorInvalidValue;
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace pkv
