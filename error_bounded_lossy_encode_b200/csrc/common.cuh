// common.cuh -- stream-format constants, bound resolution and sm_100a PTX
// helpers (mbarrier, bulk async copy, bounded waits) shared by the kernels of
// libeblc.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace eblc {

// ---------------------------------------------------------------------------
// Stream format constants (version 1).  Layout: 128-byte header, one width
// byte per block (padded to 16), one (record word offset, outliers before)
// u32 pair per 4096-element chunk (padded to 16), then one record per chunk:
// the chunk's payload words followed by its outlier indices and values.
constexpr uint32_t kChunk = 4096;
constexpr uint32_t kHeaderBytes = 128;
constexpr uint32_t kMagic = 0x434C4245u;  // "EBLC"
constexpr uint32_t kVersion = 1;
constexpr uint16_t kFlagAbs = 1;
constexpr uint16_t kFlagLorenzoNd = 2;  // 2-D / 3-D Lorenzo over the array's dims (bytes 96..119: Z, Y, X)
constexpr uint16_t kFlagChunked = 4;    // chunk-cooperative codec (Diff -> Bitshuffle -> RZE), no block widths
constexpr uint16_t kFlagRre = 8;        // with kFlagChunked: RRE (repetition elimination) in place of RZE
constexpr uint64_t kMaxN = 1ull << 30;

// Device error word bits.
enum : uint32_t { kErrTimeout = 1u, kErrCapacity = 2u, kErrCorrupt = 4u, kErrRange = 8u };

__host__ __device__ constexpr uint64_t pad16(uint64_t v) { return (v + 15u) & ~uint64_t(15); }

struct Layout {
    uint64_t nb, nc, width_off, index_off, record_off;
};

__host__ __device__ inline Layout stream_layout(uint64_t n, uint32_t block) {
    Layout L;
    L.nb = (n + block - 1) / block;
    L.nc = (n + kChunk - 1) / kChunk;
    L.width_off = kHeaderBytes;
    L.index_off = L.width_off + pad16(L.nb);
    L.record_off = L.index_off + pad16(8u * L.nc);
    return L;
}

// Layout of a stream of the chunk-cooperative codec: no width bytes, one
// index entry per chunk of m elements, then the chunk records.
__host__ __device__ inline Layout chunked_layout(uint64_t n, uint32_t m) {
    Layout L;
    L.nb = 0;
    L.nc = (n + m - 1) / m;
    L.width_off = kHeaderBytes;
    L.index_off = kHeaderBytes;
    L.record_off = L.index_off + pad16(8u * L.nc);
    return L;
}

// Resolved bound of one call, plus the thresholds of the fp32 fast filter
// used by the encoder's bound test.
struct Bound {
    double eb;
    float inv2eb, step;
    float t_in, t_out;  // |x - x'| (fp32) <= t_in: certainly within eb; > t_out: certainly not
    float vmin, vmax;
    int check_range;    // 0: every finite element is known to give |x * inv2eb| < 2^30
};

// eb = rel * (vmax - vmin) (or the absolute bound), inv2eb = (float)(1/(2 eb)),
// step = (float)(2 eb), all IEEE double with round-to-nearest, then one
// rounding to float ("Pipeline specialization internals", Priming and Inverse
// declaration: the quantizer resolves the bound before the fused kernel and
// the inverse multiplies by the step 2*abs_eb).
//
// Fast filter: with d = |fl32(x - x')|, the exact |x - x'| is within a factor
// (1 +- 2^-24) of d.  d <= t_in <= eb (1 - 2^-20) therefore implies
// |x - x'| < eb, and d > t_out >= eb (1 + 2^-20) implies |x - x'| > eb by far
// more than one double ulp, so the fp64 test agrees in both cases.  Anything
// in between (and NaN) takes the fp64 test.  For eb outside [2^-120, 1e37]
// the filter is disabled (t_in = 0, t_out = inf).
__device__ inline Bound resolve_bound(int abs_mode, double bound, float vmin, float vmax, int range_given = 0) {
    Bound b;
    b.vmin = abs_mode ? 0.0f : vmin;
    b.vmax = abs_mode ? 0.0f : vmax;
    double eb = abs_mode ? bound : __dmul_rn(bound, __dsub_rn((double)vmax, (double)vmin));
    double two = __dmul_rn(2.0, eb);
    double inv = (two == 0.0) ? __longlong_as_double(0x7ff0000000000000ll) : __ddiv_rn(1.0, two);
    b.eb = eb;
    b.inv2eb = __double2float_rn(inv);
    b.step = __double2float_rn(two);
    if (eb >= 0x1p-120 && eb <= 1e37) {
        b.t_in = __double2float_rd(__dmul_rn(eb, 1.0 - 0x1p-20));
        b.t_out = __double2float_ru(__dmul_rn(eb, 1.0 + 0x1p-20));
    } else {
        b.t_in = 0.0f;
        b.t_out = __int_as_float(0x7f800000);
    }
    // Relative bound over the array's own range: every finite element lies in
    // [vmin, vmax], and float rounding is monotone, so |fl(x * inv2eb)| <=
    // fl(max(|vmin|, |vmax|) * inv2eb).  When that is below 2^30 the
    // quantizer's range test can never fail for a finite element (non-finite
    // ones fail the bound test anyway).  A range given by the caller is not
    // trusted to contain the elements: the test stays on.
    const float amax = fmaxf(fabsf(b.vmin), fabsf(b.vmax));
    b.check_range = (abs_mode || range_given) ? 1 : !(__fmul_rn(amax, b.inv2eb) < 0x1p30f);
    return b;
}

// ---------------------------------------------------------------------------
// PTX helpers.

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_init_fence() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                     smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for the phase of `bar` with the given parity to complete.  Gives up
// after limit_ns nanoseconds, records kErrTimeout in *err and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint64_t limit_ns, uint32_t *err) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
#pragma unroll 1
        for (int k = 0; k < 16; ++k)
            if (mbar_try_wait(bar, parity)) return true;
        if (globaltimer_ns() - t0 > limit_ns) {
            atomicOr(err, kErrTimeout);
            return false;
        }
    }
}

// One bulk asynchronous copy global -> shared completing on an mbarrier.
// Both addresses 16-byte aligned, bytes a multiple of 16 (not checked here;
// the callers round their ranges).  Never used with .multicast.
__device__ __forceinline__ void bulk_g2s(void *dst_smem, const void *src_gmem, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst_smem)),
        "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Tiled tensor copies global -> shared (one box of the tensor map at the
// given element coordinates, x innermost) completing on an mbarrier.  The x
// coordinate times 4 bytes is a multiple of 16 at every call site (bricks
// start at multiples of 16 elements).  Never used with .multicast.
__device__ __forceinline__ void tensor_g2s_3d(void *dst_smem, const void *tmap, int x, int y, int z, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(smem_u32(dst_smem)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tensor_g2s_2d(void *dst_smem, const void *tmap, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(smem_u32(dst_smem)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// Brick t of a multi-dimensional array {Z, Y, X} in C order over the brick
// grid: its first element's (z, y, x).  Every dim and brick count is below
// 2^30 (n <= 2^30), so 32-bit arithmetic is exact.
__host__ __device__ inline void brick_origin(uint64_t t, int nd, const uint64_t *dims, int &z, int &y, int &x) {
    const uint32_t ex = (nd == 3) ? 16u : 64u, ey = ex, ez = (nd == 3) ? 16u : 1u;
    const uint32_t gx = (uint32_t)dims[2] / ex, gy = (uint32_t)dims[1] / ey, tt = (uint32_t)t;
    const uint32_t ty = tt / gx;
    x = (int)((tt - ty * gx) * ex);
    y = (int)((ty % gy) * ey);
    z = (int)((ty / gy) * ez);
}

__device__ __forceinline__ uint64_t ld_relaxed_gpu(const uint64_t *p) {
    uint64_t v;
    asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_relaxed_gpu(uint64_t *p, uint64_t v) {
    asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Streaming store (written once, not re-read by this kernel).
__device__ __forceinline__ void st_cs_u32(uint32_t *p, uint32_t v) { __stcs(p, v); }

}  // namespace eblc
