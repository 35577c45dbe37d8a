// common.cuh -- device helpers shared by the libpagedkv kernels (sm_100a only).
//
// Number formats, PTX wrappers for mbarriers / TMA / named barriers, and the bounded-wait
// primitive every kernel uses.  Nothing here traps: a wait that runs out sets a flag in
// the caller-visible error word and reports failure to its caller, which finishes without
// waiting again.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libpagedkv is written for sm_100a (B200) only"
#endif

namespace pkv {

// Error-word bits (see pkv_get_error).
constexpr int kErrTimeout = 1;
constexpr int kErrBounds = 2;
constexpr int kErrPool = 4;  // a block-pool allocation the pool could not cover

// A bounded wait gives up after this long (ns).  Legitimate waits in these kernels last
// microseconds; a second means the pipeline is broken.
constexpr unsigned long long kWaitLimitNs = 1000000000ull;

// Cache rows per TMA piece: the attention kernels stream the cache in 16-token tiles of a
// sequence, whatever its physical block size (8, 16 or 32 tokens per block).
constexpr int kPiece = 16;

// ------------------------------------------------------------------------------ formats

// bf16 pair packed in a 32-bit word -> two fp32 (exact).
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ double bf16_to_f64(uint16_t b) {
    return (double)__uint_as_float(((uint32_t)b) << 16);
}

// fp64 -> bf16 with one rounding (to nearest, ties to even) of the real value.
// Round to binary32 toward zero, make the last bit sticky if anything was dropped
// (round-to-odd), then round that to bf16 to nearest even.  Rounding to odd at a width of
// at least p + 2 bits before rounding to p bits gives the correctly rounded result
// (Boldo & Melquiond, "Emulation of FMA and correctly rounded sums: proved algorithms
// using rounding to odd", IEEE TC 2008); binary32 keeps 24 bits, bf16 needs 8.
__device__ __forceinline__ uint16_t f64_to_bf16_rne(double x) {
    float f = __double2float_rz(x);
    if ((double)f != x && !isnan(x) && !isinf(f)) f = __uint_as_float(__float_as_uint(f) | 1u);
    __nv_bfloat16 b = __float2bfloat16_rn(f);
    return *reinterpret_cast<uint16_t *>(&b);
}

// OCP FP8 E4M3-FN: s.eeee.mmm, bias 7, no infinities, S.1111.111 = NaN, max 448.
// Decode is exact into fp32.
__device__ __forceinline__ float e4m3_to_f32(uint32_t c) {
    uint32_t s = (c & 0x80u) << 24, e = (c >> 3) & 15u, m = c & 7u;
    float v;
    if (e == 0) v = (float)m * 0.001953125f;                       // m/8 * 2^-6 = m * 2^-9
    else v = __uint_as_float(((e + 120u) << 23) | (m << 20));      // (1+m/8) 2^(e-7)
    return __uint_as_float(__float_as_uint(v) | s);
}

// fp64 -> E4M3 code, round to nearest even, saturating to +-448 (finite inputs).
// The magnitude is split into binade and mantissa with exact fp64 scaling; rint() rounds
// ties to even; the result is assembled from the rounded mantissa.
__device__ __forceinline__ uint32_t f64_to_e4m3(double x) {
    uint32_t sign = (__double_as_longlong(x) < 0) ? 0x80u : 0u;
    double a = fabs(x);
    if (isnan(x)) return sign | 0x7Fu;
    if (a >= 448.0) return sign | 0x7Eu;                            // satfinite
    if (a < 0.015625) {                                              // < 2^-6: subnormal grid 2^-9
        double n = rint(a * 512.0);                                  // 0..8
        if (n >= 8.0) return sign | 0x08u;                           // rounds up to 2^-6
        return sign | (uint32_t)n;
    }
    int e = ilogb(a);                                                // a in [2^e, 2^(e+1)), e in -6..8
    double n = rint(scalbn(a, 3 - e));                               // 8..16, 4 significant bits
    if (n >= 16.0) { n = 8.0; e += 1; }
    uint32_t E = (uint32_t)(e + 7), M = (uint32_t)n - 8u;
    if (E > 15u || (E == 15u && M == 7u)) return sign | 0x7Eu;       // 480 -> saturate
    return sign | (E << 3) | M;
}

// E4M3 code (round to nearest even, saturating at 448) of the exact quotient x / s for s > 0:
// the code f64_to_e4m3 gives for the fp64 quotient, computed in fp32.  Every rounding
// midpoint between two E4M3 values is an fp32 value and the fp32 quotient is correctly
// rounded, so it lies on the exact quotient's side of every midpoint unless it is one; then
// the sign of the residual x - q s (one fused multiply-add: the sign of a nonzero result is
// exact) tells where the exact quotient lies, and q moves one fp32 ulp that way, crossing no
// other midpoint.  (The fp64 quotient of a bf16 by an fp32 value is never rounded onto a
// midpoint either: that would need a quotient within 2^-53 of one, while a bf16 x differs
// from m * s, when not equal, by at least 2^-29 of it.)
// (out of line: a rare path whose fp64 code would crowd the callers' instruction cache)
static __device__ __noinline__ uint32_t e4m3_of_quotient_f64(float x, float s) {
    return f64_to_e4m3((double)x / (double)s);
}

__device__ __forceinline__ uint32_t e4m3_of_quotient(float x, float s) {
    if (!(s > 0.f) || isnan(x)) return e4m3_of_quotient_f64(x, s);  // (a NaN keeps its sign)
    float q = __fdiv_rn(x, s);
    const float a = fabsf(q);
    bool mid;
    if (a < 0.015625f) {  // E4M3 subnormal grid 2^-9: midpoints at odd multiples of 2^-10
        const float t = a * 1024.f;  // exact
        const int ti = (int)t;
        mid = (float)ti == t && (ti & 1) != 0;
    } else {  // 4 significant bits: a midpoint has bit 19 alone set below them
        mid = a < 448.f && (__float_as_uint(a) & 0xFFFFFu) == 0x80000u;
    }
    if (mid) {
        const float r = __fmaf_rn(-q, s, x);
        if (r != 0.f) {
            const bool away = (r > 0.f) == (q > 0.f);  // the exact quotient has the larger magnitude
            q = __uint_as_float(__float_as_uint(q) + (away ? 1u : 0xFFFFFFFFu));
        }
    }
    uint16_t c;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(c) : "f"(0.f), "f"(q));
    return c & 0xFFu;
}

// ------------------------------------------------------------------------------ PTX

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ unsigned long long globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete, for at most `limit_ns`.
// Returns false (and sets kErrTimeout in *err) if it gives up.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, int *err,
                                                  unsigned long long limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    unsigned long long t0 = globaltimer();
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 16; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer() - t0 > limit_ns) {
            atomicOr(err, kErrTimeout);
            return false;
        }
    }
}

// 3-D tiled TMA load global -> shared, completion counted on an mbarrier (no multicast).
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int x, int y, int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z)
        : "memory");
}

// 4-D tiled TMA load global -> shared (no multicast).
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int x, int y, int z, int w) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z), "r"(w)
        : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Programmatic dependent launch.  Every kernel of the library is launched so that it may
// be scheduled while the previous kernel on the stream drains; it then waits for that
// kernel's completion (and memory) before touching any global input, and lets the next
// kernel be scheduled as early as possible.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Named barrier among `count` threads (a multiple of 32).
__device__ __forceinline__ void named_bar(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Named barrier among `count` threads that also tells every thread whether `pred` held on
// any of them (one barrier-reduction instead of a reduction plus a barrier).
__device__ __forceinline__ bool named_bar_any(int id, int count, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(pred ? 1u : 0u), "r"(id), "r"(count)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}

__device__ __forceinline__ float4 lds128f(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr));
    return v;
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

// ------------------------------------------------------------------------------ RoPE

// Rotate the pair (x1, x2) = (x_i, x_{i+D/2}) by the table's (c, s) in fp64 and round
// each result once to bf16.  The products bf16 x fp32 are exact in fp64 (<= 32 significant
// bits), so the only roundings are the fp64 difference/sum and the final bf16 one.
__device__ __forceinline__ void rope_pair(uint16_t x1, uint16_t x2, float c, float s,
                                          uint16_t &y1, uint16_t &y2) {
    double a = bf16_to_f64(x1), b = bf16_to_f64(x2);
    double dc = (double)c, ds = (double)s;
    double r1 = __dsub_rn(__dmul_rn(a, dc), __dmul_rn(b, ds));
    double r2 = __dadd_rn(__dmul_rn(b, dc), __dmul_rn(a, ds));
    y1 = f64_to_bf16_rne(r1);
    y2 = f64_to_bf16_rne(r2);
}

// Round r = fl(a*b - p) (one FMA; p = fl(c*d) is the other product) to bf16 into *out and
// report whether that is guaranteed to equal rounding the exact a*b - c*d.
// Error: |r - exact| <= ulp(p)/2 + ulp(r)/2 < (|p| + |r|) * 2^-23.
// With y = bf16(r), r lies inside y's rounding interval, whose nearest boundary is at least
// |y| * 2^-9 - |r - y| away (half a bf16 ulp is >= |y| * 2^-9 in every binade, and larger
// than that for bf16 subnormals).  If that distance exceeds the error bound, the exact
// value rounds to y as well.  NaN/inf make the comparison false (fp64 path).
__device__ __forceinline__ bool bf16_round_checked(float r, float p, uint16_t *out) {
    const __nv_bfloat16 yb = __float2bfloat16_rn(r);
    const uint16_t bits = *reinterpret_cast<const uint16_t *>(&yb);
    const float y = __uint_as_float((uint32_t)bits << 16);
    *out = bits;
    const float room = __fmaf_rn(fabsf(y), 0x1p-9f, -fabsf(r - y));
    const float err = (fabsf(p) + fabsf(r)) * 0x1p-23f;
    return room > err;
}

// rope_pair with the same result bits, computed in fp32 whenever the bound above proves
// the fp32 value rounds like the exact one (nearly always), else in fp64.
__device__ __forceinline__ void rope_pair_fast(uint16_t x1, uint16_t x2, float c, float s,
                                               uint16_t &y1, uint16_t &y2) {
    const float a = __uint_as_float((uint32_t)x1 << 16), b = __uint_as_float((uint32_t)x2 << 16);
    const float p1 = __fmul_rn(b, s), p2 = __fmul_rn(a, s);
    const float r1 = __fmaf_rn(a, c, -p1);  // x1 cos - x2 sin
    const float r2 = __fmaf_rn(b, c, p2);   // x2 cos + x1 sin
    uint16_t o1, o2;
    const bool ok1 = bf16_round_checked(r1, p1, &o1);
    const bool ok2 = bf16_round_checked(r2, p2, &o2);
    if (ok1 && ok2) {
        y1 = o1;
        y2 = o2;
    } else {
        rope_pair(x1, x2, c, s, y1, y2);
    }
}

// Sequence owning token row t: the b with cu[b] <= t < cu[b+1] (cu is non-decreasing).
__device__ __forceinline__ int owner_seq(const int32_t *cu, int num_seqs, int t) {
    int lo = 0, hi = num_seqs - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (__ldg(cu + mid) <= t) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

#ifndef __CUDACC_RTC__
// Launch `kern` on `stream` with programmatic stream serialisation allowed (see pdl_wait).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}
#endif

}  // namespace pkv
