// chunked.cu -- the chunk-cooperative codec for sm_100a: Quant -> Diff ->
// Bitshuffle -> RZE over byte chunks of 4096, 8192 or 16384 bytes of float32
// input ("Pipeline specialization internals", Chunk-cooperative path: one
// CTA owns a chunk, intermediates stay in shared memory; "nvrtc_chunk_fusion.h
// File Reference", launchNvrtcChunkFusedEncode: each chunk's coded form in a
// scratch slot with its size, then the cross-chunk scan/pack tail).
//
//   chunk_encode  one CTA per chunk, each CTA a contiguous range of chunks,
//                 each warp a contiguous run of 32-code groups in registers:
//                 the linear quantizer and the outlier test, first
//                 differences reset at the chunk start in zigzag form, the
//                 32 x 32 bit transpose of every group (lane b gets bit plane
//                 b) by a shuffle butterfly, zero elimination (a bitmap of the
//                 nonzero words by ballots, the nonzero words compacted warp
//                 by warp after one block scan; with the RRE coder the words
//                 that differ from the word before instead) or the shuffled
//                 words verbatim when that is not smaller, then the chunk's
//                 outliers in ascending order; the record goes to the chunk's
//                 scratch slot, its size to sizes[], the range's totals to
//                 part[].
//   chunk_scan    one CTA: exclusive scan of the chunk ranges' record words
//                 and outlier counts -> range bases, header, result block.
//   chunk_gather  one CTA per chunk range: the chunk index entries (a block
//                 scan from the range's base), records from scratch to their
//                 place in the stream.
//   chunk_decode  one CTA per chunk: zero elimination undone (each warp a
//                 run of bitmap words, ranks by popcounts; RRE: each word is
//                 the last kept word at or before it), the inverse
//                 transpose, zigzag undone and the prefix sum in each warp's
//                 registers, one block scan of the warps' totals,
//                 dequantization, outliers.
// No inter-CTA waits anywhere: the scan is its own launch.
#include "common.cuh"
#include "kernels.h"

namespace eblc {
namespace {

constexpr int kCT = 256;                  // threads per CTA
constexpr int kCW = kCT / 32;
constexpr uint32_t kFull = 0xffffffffu;

__device__ __forceinline__ uint32_t zz(int32_t d) { return ((uint32_t)d << 1) ^ (uint32_t)(d >> 31); }

// 32 x 32 bit-matrix transpose across the warp: on entry lane r holds row r
// (bit c = element (r, c)), on return lane c holds column c (bit r = element
// (r, c)).  Five butterfly stages, each swapping the off-diagonal j x j
// blocks between lanes r and r ^ j with one shuffle.
__device__ __forceinline__ uint32_t transpose32(uint32_t w, int ln) {
    const uint32_t masks[5] = {0x0000ffffu, 0x00ff00ffu, 0x0f0f0f0fu, 0x33333333u, 0x55555555u};
#pragma unroll
    for (int k = 0; k < 5; ++k) {
        const int j = 16 >> k;
        const uint32_t m = masks[k];
        const uint32_t p = __shfl_xor_sync(kFull, w, j);
        w = (ln & j) ? ((w & ~m) | ((p >> j) & m)) : ((w & m) | ((p & m) << j));
    }
    return w;
}
// The same transpose when the codes use bit planes 0..3 only (codes < 16):
// four ballots, lane b < 4 keeps plane b, the other lanes' planes are 0.
__device__ __forceinline__ uint32_t transpose32_low4(uint32_t d, int ln) {
    const uint32_t p0 = __ballot_sync(kFull, d & 1u), p1 = __ballot_sync(kFull, d & 2u);
    const uint32_t p2 = __ballot_sync(kFull, d & 4u), p3 = __ballot_sync(kFull, d & 8u);
    const uint32_t lo = (ln & 1) ? p1 : p0, hi = (ln & 1) ? p3 : p2;
    return (ln >= 4) ? 0u : ((ln & 2) ? hi : lo);
}

// Inverse transpose when only planes 0..nb-1 (lanes 0..nb-1) may be nonzero:
// lane l collects bit l of each plane word.
__device__ __forceinline__ uint32_t untranspose32_low(uint32_t pw, int nb, int ln) {
    uint32_t code = 0;
#pragma unroll 4
    for (int b = 0; b < nb; ++b) code |= ((__shfl_sync(kFull, pw, b) >> ln) & 1u) << b;
    return code;
}

__device__ __forceinline__ int32_t unzz(uint32_t z) { return (int32_t)((z >> 1) ^ (0u - (z & 1u))); }

// Exclusive block-wide prefix of v (every thread of the CTA calls it);
// *total receives the sum over the CTA.  tmp: kCW words of shared memory.
__device__ __forceinline__ uint32_t block_excl(uint32_t v, uint32_t *tmp, uint32_t *total) {
    const int ln = threadIdx.x % 32, w = threadIdx.x / 32;
    uint32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(kFull, incl, o);
        if (ln >= o) incl += t;
    }
    __syncthreads();  // tmp free for reuse
    if (ln == 31) tmp[w] = incl;
    __syncthreads();
    uint32_t before = 0, all = 0;
#pragma unroll
    for (int k = 0; k < kCW; ++k) {
        const uint32_t t = tmp[k];
        before += (k < w) ? t : 0u;
        all += t;
    }
    *total = all;
    return before + incl - v;
}

// Position in shared memory of word k of a chunk's shuffled words (k =
// plane * G + group, G groups of 32 codes).  For a full chunk G is 32, 64 or
// 128 and word k sits at k ^ plane: the column of one group (one word per
// plane, lanes 0..31) and a run of 32 consecutive words of one plane both
// fall in 32 distinct banks.  A ragged last chunk keeps the plain order.
__device__ __forceinline__ uint32_t phys(uint32_t k, int lg) { return lg ? (k ^ ((k >> lg) & 31u)) : k; }

// Quantized code of x and its outlier test ("Pipeline specialization
// internals", Quantization: fp32 filter with thresholds from the bound,
// fp64 test in the band between them).
__device__ __forceinline__ int32_t quant(const Bound &bd, float x, bool &o) {
    const float y = __fmul_rn(x, bd.inv2eb);
    const int32_t qq = (fabsf(y) < 0x1p30f) ? __float2int_rn(y) : 0;
    const float xr = __fmul_rn(__int2float_rn(qq), bd.step);
    const float d = fabsf(__fsub_rn(x, xr));
    o = d > bd.t_out;
    if (!o && !(d <= bd.t_in)) {
        const bool finite = fabsf(x) < __int_as_float(0x7f800000);
        o = !finite || !(fabs(__dsub_rn((double)x, (double)xr)) <= bd.eb);
    }
    return qq;
}

// Quantized code alone (the quantizer's range rule included).
__device__ __forceinline__ int32_t quant_code(const Bound &bd, float x) {
    const float y = __fmul_rn(x, bd.inv2eb);
    return (fabsf(y) < 0x1p30f) ? __float2int_rn(y) : 0;
}

// Dynamic shared memory of the encoder for chunks of m elements: the
// shuffled words, the outlier flag words, the scan's warp totals.
__host__ __device__ constexpr size_t enc_smem_bytes(uint32_t m) { return 4ull * (m + m / 32 + kCW); }

// PER = m / kCT.  CTA b codes the chunks [b K, b K + K) (K = per_range) in
// order and leaves their total record words and outliers in part[].  Warp w
// owns the PER groups of 32 codes starting at code 32 PER w of the chunk and
// keeps them in registers from the load to the bit transpose; the input of
// the CTA's next chunk is loaded as soon as the current chunk's codes are
// formed, so its latency overlaps the rest.
template <int PER, bool RRE>
__global__ void __launch_bounds__(kCT, PER == 4 ? 6 : PER == 8 ? 4 : 3) chunk_encode(const ChunkedArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    uint32_t *const sw = reinterpret_cast<uint32_t *>(smem_raw);
    uint32_t *const oflag = sw + a.m;
    uint32_t *const tmp = oflag + a.m / 32;
    const int t = threadIdx.x, ln = t % 32, w = t / 32;
    const int lg_full = 31 - __clz(a.m / 32);
    __shared__ Bound bd;
    if (t == 0) {
        const float vmin = a.abs_mode ? 0.0f : a.range[0], vmax = a.abs_mode ? 0.0f : a.range[1];
        bd = resolve_bound(a.abs_mode, a.bound, vmin, vmax);
    }
    const uint32_t first = (uint32_t)(32 * PER * w);  // the warp's first code in its chunk
    float xv[PER], xp = 0.0f;
    auto load = [&](uint64_t c) {
        const uint64_t e0 = c * a.m;
        const uint32_t cnt = (c < a.nc) ? (uint32_t)min((uint64_t)a.m, a.n - e0) : 0u;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const uint32_t j = first + 32 * i + ln;
            xv[i] = (j < cnt) ? __ldcs(a.in + e0 + j) : 0.0f;
        }
        // the code before the warp's first one (its difference), re-quantized here
        xp = (ln == 0 && first > 0 && first <= cnt) ? a.in[e0 + first - 1] : 0.0f;
    };
    const uint64_t cb = (uint64_t)blockIdx.x * a.per_range, ce = min(a.nc, cb + a.per_range);
    uint32_t tot_r = 0, tot_m = 0;  // thread 0: the range's record words and outliers
    load(cb);
    __syncthreads();
    for (uint64_t c = cb; c < ce; ++c) {
        const uint64_t e0 = c * a.m;
        const uint32_t cnt = (uint32_t)min((uint64_t)a.m, a.n - e0), mp = (cnt + 31u) & ~31u, G = mp / 32;
        const int lg = (mp == a.m) ? lg_full : 0;
        uint32_t *rec = a.scratch + c * (uint64_t)a.slot_words;
        // Quant, Diff (zigzag, reset at the chunk start) and Bitshuffle of the
        // warp's groups: lane l holds code 32 g + l; the transpose gives lane b
        // plane b's word of the group.
        // The fp32 filter settles almost every code; a warp with any element
        // not certainly within the bound (or possibly out of range) redoes
        // its group with the quantizer's range rule and the exact test.
        const uint32_t sx = (mp == a.m) ? (uint32_t)ln : 0u;  // phys(ln G + g) for this lane
        const bool chk = bd.check_range != 0;
        int32_t prev = 0;
        if (ln == 0 && first > 0 && first <= cnt) prev = quant_code(bd, xp);
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const uint32_t g = first / 32 + i, j = 32 * g + ln;
            if (g >= G) break;  // warp-uniform
            const float x = xv[i];  // 0 past the chunk's end
            const float y = __fmul_rn(x, bd.inv2eb);
            int32_t qq = __float2int_rn(y);
            const float xr = __fmul_rn(__int2float_rn(qq), bd.step);
            const bool flag = !(fabsf(__fsub_rn(x, xr)) <= bd.t_in) || (chk && !(fabsf(y) < 0x1p30f));
            bool o = false;
            if (__any_sync(kFull, flag)) qq = (j < cnt) ? quant(bd, x, o) : 0;
            int32_t left = __shfl_up_sync(kFull, qq, 1);
            if (ln == 0) left = prev;
            prev = __shfl_sync(kFull, qq, 31);
            const uint32_t d = (j < cnt) ? zz(qq - left) : 0u;
            const uint32_t fw = __ballot_sync(kFull, o);
            if (ln == 0) oflag[g] = fw;
            const uint32_t wide = __reduce_or_sync(kFull, d) >> 4;  // any code using plane 4 or above
            sw[ln * G + (g ^ sx)] = wide ? transpose32(d, ln) : transpose32_low4(d, ln);
        }
        load(c + 1 < ce ? c + 1 : a.nc);
        __syncthreads();
        // One block scan for both counts: warp w's nonzero words over its word
        // range [k0, k1) (upper 16 bits, lane 0 only) and thread t's outliers
        // in flag word t (lower 16 bits; G <= kCT).  Both totals are <= 4096.
        const uint32_t per = ((G + kCW - 1) / kCW) * 32;
        const uint32_t k0 = min(w * per, mp), k1 = min(k0 + per, mp);
        // a word is kept when it is not zero (RZE) / differs from the word
        // before it, word -1 being 0 (RRE)
        auto kept = [&](uint32_t k, uint32_t v) {
            const uint32_t pv = (RRE && k) ? sw[phys(k - 1, lg)] : 0u;
            return v != pv;
        };
        uint32_t cntw = 0;
        for (uint32_t k = k0 + ln; k < k1; k += 32) cntw += __popc(__ballot_sync(kFull, kept(k, sw[phys(k, lg)])));
        const uint32_t ow = (t < (int)G) ? __popc(oflag[t]) : 0u;
        uint32_t tot;
        const uint32_t pre = block_excl(((ln == 0 ? cntw : 0u) << 16) | ow, tmp, &tot);
        const uint32_t nnz = tot >> 16, mc = tot & 0xffffu;
        // RZE: bitmap + compacted nonzero words, or the words verbatim when
        // that is not smaller
        const bool raw = G + nnz >= mp;
        const uint32_t P = raw ? mp : G + nnz;
        if (raw) {
            for (uint32_t k = t; k < mp; k += kCT) rec[1 + k] = sw[phys(k, lg)];
        } else {
            uint32_t base = __shfl_sync(kFull, pre >> 16, 0);
            for (uint32_t k = k0 + ln; k < k1; k += 32) {
                const uint32_t v = sw[phys(k, lg)];
                const bool kp = kept(k, v);
                const uint32_t bal = __ballot_sync(kFull, kp);
                if (ln == 0) rec[1 + k / 32] = bal;  // bitmap word k / 32: bit l = word 32 (k/32) + l
                if (kp) rec[1 + G + base + __popc(bal & ((1u << ln) - 1u))] = v;
                base += __popc(bal);
            }
        }
        // outliers of the chunk, ascending: thread t writes those of flag word t
        if (t < (int)G) {
            uint32_t bits = oflag[t], q = pre & 0xffffu;
            while (bits) {
                const uint32_t e = t * 32 + (uint32_t)(__ffs(bits) - 1);
                bits &= bits - 1u;
                rec[1 + P + q] = (uint32_t)(e0 + e);
                rec[1 + P + mc + q] = __float_as_uint(a.in[e0 + e]);
                ++q;
            }
        }
        if (t == 0) {
            rec[0] = P | (raw ? 0x80000000u : 0u);
            a.sizes[c] = 1 + P + 2 * mc;
            a.outl[c] = mc;
            tot_r += 1 + P + 2 * mc;
            tot_m += mc;
        }
        __syncthreads();
    }
    if (t == 0) {
        a.part[blockIdx.x] = tot_r;
        a.part[a.nc + blockIdx.x] = tot_m;
    }
}

constexpr int kScanThreads = 1024;
constexpr int kScanWarps = kScanThreads / 32;

// Exclusive scan of the chunk ranges' totals (one CTA; part[] is replaced
// by the ranges' bases), the header of the stream, the result block.
__global__ void __launch_bounds__(kScanThreads) chunk_scan(const ChunkedArgs a) {
    __shared__ unsigned long long part_r[kScanWarps], part_m[kScanWarps];
    const int t = threadIdx.x, ln = t % 32, w = t / 32;
    const uint32_t per = (a.ranges + kScanThreads - 1) / kScanThreads;  // ranges per thread
    const uint32_t b0 = min(a.ranges, per * t), b1 = min(a.ranges, b0 + per);
    unsigned long long sr = 0, sm_ = 0;
    for (uint32_t b = b0; b < b1; ++b) {
        sr += a.part[b];
        sm_ += a.part[a.nc + b];
    }
    unsigned long long ir = sr, im = sm_;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long x = __shfl_up_sync(kFull, ir, o), y = __shfl_up_sync(kFull, im, o);
        if (ln >= o) {
            ir += x;
            im += y;
        }
    }
    if (ln == 31) {
        part_r[w] = ir;
        part_m[w] = im;
    }
    __syncthreads();
    unsigned long long r = 0, m = 0, R = 0, M = 0;
    for (int k = 0; k < kScanWarps; ++k) {
        r += (k < w) ? part_r[k] : 0ull;
        m += (k < w) ? part_m[k] : 0ull;
        R += part_r[k];
        M += part_m[k];
    }
    r += ir - sr;
    m += im - sm_;
    for (uint32_t b = b0; b < b1; ++b) {
        const uint32_t xr = a.part[b], xm = a.part[a.nc + b];
        a.part[b] = (uint32_t)r;
        a.part[a.nc + b] = (uint32_t)m;
        r += xr;
        m += xm;
    }
    const Layout L = chunked_layout(a.n, a.m);
    const bool idx_fits = L.record_off <= a.out_cap;
    if (t != 0) return;
    const float vmin = a.abs_mode ? 0.0f : a.range[0], vmax = a.abs_mode ? 0.0f : a.range[1];
    const Bound bd = resolve_bound(a.abs_mode, a.bound, vmin, vmax);
    const uint64_t W = R - 2 * M, total = L.record_off + 4 * R;
    if (total > a.out_cap || M > a.outlier_cap) atomicOr(a.err, kErrCapacity);
    a.result[0] = W;
    a.result[1] = M;
    a.result[2] = total;
    a.result[3] = R;
    a.result[4] = (uint64_t)__double_as_longlong(bd.eb);
    a.result[5] = (uint64_t)__float_as_uint(bd.step) | ((uint64_t)__float_as_uint(bd.inv2eb) << 32);
    a.result[6] = (uint64_t)__float_as_uint(bd.vmin) | ((uint64_t)__float_as_uint(bd.vmax) << 32);
    if (!idx_fits) return;
    uint32_t h[32] = {};
    const uint64_t ebits = (uint64_t)__double_as_longlong(bd.eb), bbits = (uint64_t)__double_as_longlong(a.bound);
    h[0] = kMagic;
    h[1] = kVersion | ((uint32_t)((a.abs_mode ? kFlagAbs : 0) | kFlagChunked | (a.rre ? kFlagRre : 0)) << 16);
    h[2] = (uint32_t)a.n;
    h[3] = (uint32_t)(a.n >> 32);
    h[4] = 0;  // no blocks
    h[5] = a.m;
    h[6] = (uint32_t)ebits;
    h[7] = (uint32_t)(ebits >> 32);
    h[8] = __float_as_uint(bd.inv2eb);
    h[9] = __float_as_uint(bd.step);
    h[10] = __float_as_uint(bd.vmin);
    h[11] = __float_as_uint(bd.vmax);
    h[14] = (uint32_t)a.nc;
    h[15] = (uint32_t)(a.nc >> 32);
    h[16] = (uint32_t)W;
    h[17] = (uint32_t)(W >> 32);
    h[18] = (uint32_t)M;
    h[19] = (uint32_t)(M >> 32);
    h[20] = (uint32_t)total;
    h[21] = (uint32_t)(total >> 32);
    h[22] = (uint32_t)bbits;
    h[23] = (uint32_t)(bbits >> 32);
    uint4 *dst = reinterpret_cast<uint4 *>(a.out);
    for (int j = 0; j < 8; ++j) dst[j] = make_uint4(h[4 * j], h[4 * j + 1], h[4 * j + 2], h[4 * j + 3]);
    for (uint64_t b = L.index_off + 8 * a.nc; b < L.record_off; b += 4) *reinterpret_cast<uint32_t *>(a.out + b) = 0u;
}

// CTA b: the chunk index entries of range b (a block scan of its chunks'
// sizes from the range's base, 256 chunks at a time), then the records from
// their scratch slots to their offsets, one warp per chunk.
__global__ void __launch_bounds__(kCT) chunk_gather(const ChunkedArgs a) {
    __shared__ uint32_t off_s[kCT], len_s[kCT], tmp[kCW];
    const int t = threadIdx.x, ln = t % 32, w = t / 32;
    const Layout L = chunked_layout(a.n, a.m);
    uint32_t *recs = reinterpret_cast<uint32_t *>(a.out + L.record_off);
    const uint64_t cap_words = (a.out_cap > L.record_off) ? (a.out_cap - L.record_off) / 4 : 0;
    const bool idx_fits = L.record_off <= a.out_cap;
    const uint64_t cb = (uint64_t)blockIdx.x * a.per_range, ce = min(a.nc, cb + a.per_range);
    uint32_t base_r = a.part[blockIdx.x], base_m = a.part[a.nc + blockIdx.x];
    for (uint64_t c0 = cb; c0 < ce; c0 += kCT) {
        const uint64_t c = c0 + t;
        const uint32_t s = (c < ce) ? a.sizes[c] : 0u, q = (c < ce) ? a.outl[c] : 0u;
        uint32_t tr, tm;
        const uint32_t er = block_excl(s, tmp, &tr);
        const uint32_t em = block_excl(q, tmp, &tm);
        if (c < ce && idx_fits)
            *reinterpret_cast<uint2 *>(a.out + L.index_off + 8 * c) = make_uint2(base_r + er, base_m + em);
        off_s[t] = base_r + er;
        len_s[t] = s;
        __syncthreads();
        const uint32_t nw = (uint32_t)min((uint64_t)kCT, ce - c0);
        for (uint32_t k = w; k < nw; k += kCW) {
            const uint64_t o = off_s[k];
            const uint32_t len = len_s[k];
            if (o + len > cap_words) continue;  // reported by chunk_scan (capacity)
            const uint32_t *src = a.scratch + (c0 + k) * (uint64_t)a.slot_words;
            // eight loads in flight per lane before their stores
            for (uint32_t j0 = 0; j0 < len; j0 += 8 * 32) {
                uint32_t v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const uint32_t j = j0 + 32 * u + ln;
                    v[u] = (j < len) ? __ldg(src + j) : 0u;
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const uint32_t j = j0 + 32 * u + ln;
                    if (j < len) st_cs_u32(recs + o + j, v[u]);
                }
            }
        }
        base_r += tr;
        base_m += tm;
        __syncthreads();
    }
}

// Dynamic shared memory of the decoder for chunks of m elements: the record's
// payload words, the shuffled words, the scan's warp totals and the chunk's
// record facts.
__host__ __device__ constexpr size_t dec_smem_bytes(uint32_t m) { return 4ull * (2 * m + kCW + 4); }

// PER = m / kCT.  Warp w decodes the PER groups starting at code 32 PER w:
// the transpose, zigzag and the prefix sum stay in its registers, and its
// reconstructions go out as whole 128-byte lines.  Thread 0 loads the index
// entries and the head word of the CTA's next chunk one chunk ahead; the
// payload and the first kCT outliers of a chunk come in one round of loads.
template <int PER, bool RRE>
__global__ void __launch_bounds__(kCT, PER == 4 ? 5 : PER == 8 ? 4 : 3) chunk_decode(const ChunkedDecArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    uint32_t *const pl = reinterpret_cast<uint32_t *>(smem_raw);  // payload (RZE form)
    uint32_t *const sw = pl + a.m;
    uint32_t *const tmp = sw + a.m;
    uint32_t *const info = tmp + kCW;  // P (0xffffffff: corrupt), raw, mc, record word offset
    const int t = threadIdx.x, ln = t % 32, w = t / 32;
    const int lg_full = 31 - __clz(a.m / 32);
    const Layout L = chunked_layout(a.n, a.m);
    const uint32_t *recs = reinterpret_cast<const uint32_t *>(a.in + L.record_off);
    const uint64_t R = a.W + 2 * a.mo;
    const uint32_t first = (uint32_t)(32 * PER * w);
    // thread 0: the next chunk's index entries (its own and its successor's) and head word
    uint64_t ex = 0, ey = 0, nx = 0, ny = 0;
    uint32_t head = 0;
    bool eok = false;
    auto fetch_entries = [&](uint64_t c) {
        if (c >= L.nc) return;
        const uint2 e = *reinterpret_cast<const uint2 *>(a.in + L.index_off + 8 * c);
        ex = e.x;
        ey = e.y;
        nx = R;
        ny = a.mo;
        if (c + 1 < L.nc) {
            const uint2 e2 = *reinterpret_cast<const uint2 *>(a.in + L.index_off + 8 * (c + 1));
            nx = e2.x;
            ny = e2.y;
        }
    };
    auto fetch_head = [&]() {
        eok = nx >= ex + 1 && ny >= ey && nx <= R && ny <= a.mo;
        head = eok ? recs[ex] : 0u;
    };
    if (t == 0) {
        fetch_entries(blockIdx.x);
        fetch_head();
    }
    for (uint64_t c = blockIdx.x; c < L.nc; c += gridDim.x) {
        const uint64_t e0 = c * a.m;
        const uint32_t cnt = (uint32_t)min((uint64_t)a.m, a.n - e0), mp = (cnt + 31u) & ~31u, G = mp / 32;
        const int lg = (mp == a.m) ? lg_full : 0;
        const uint32_t sx = (mp == a.m) ? (uint32_t)ln : 0u;
        if (t == 0) {
            uint32_t P = head & 0x7fffffffu, raw = head >> 31, mc = (uint32_t)(ny - ey);
            const bool ok = eok && ex + 1 + P + 2ull * mc == nx && (raw ? P == mp : (P >= G && P < mp));
            if (!ok) {
                atomicOr(a.err, kErrCorrupt);
                P = 0xffffffffu;
            }
            info[0] = P;
            info[1] = raw;
            info[2] = mc;
            info[3] = (uint32_t)ex;
            fetch_entries(c + gridDim.x);
        }
        __syncthreads();
        const uint32_t P = info[0], raw = info[1], mc = info[2];
        const uint32_t *pay = recs + info[3] + 1;
        if (P == 0xffffffffu) {  // corrupt record: skip the chunk
            if (t == 0) fetch_head();
            __syncthreads();
            continue;
        }
        uint32_t pv[PER];
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const uint32_t k = t + i * kCT;
            pv[i] = (k < P) ? pay[k] : 0u;
        }
        uint32_t oi = 0, ov = 0;
        if (t < (int)mc) {
            oi = pay[P + t];
            ov = pay[P + mc + t];
        }
        if (t == 0) fetch_head();
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const uint32_t k = t + i * kCT;
            if (k < P) {
                if (raw)
                    sw[phys(k, lg)] = pv[i];
                else
                    pl[k] = pv[i];
            }
        }
        __syncthreads();
        if (!raw) {
            // zero elimination undone: warp w expands the bitmap words [j0, j1)
            // (in order), its first nonzero word's rank the popcount of the
            // bitmap words before j0
            const uint32_t per = (G + kCW - 1) / kCW;
            const uint32_t j0 = min(w * per, G), j1 = min(j0 + per, G);
            uint32_t base = 0;
            for (uint32_t j = ln; j < j0; j += 32) base += __popc(pl[j]);
            base = __reduce_add_sync(kFull, base);
            const uint32_t lt = (1u << ln) - 1u;
            for (uint32_t j = j0; j < j1; ++j) {
                const uint32_t bw = pl[j];
                uint32_t v = 0;
                if constexpr (RRE) {
                    // each word is the last kept word at or before it (0 before the first)
                    const uint32_t r = base + __popc(bw & (lt | (1u << ln)));
                    const uint32_t idx = G + r - 1u;
                    v = (r != 0u && idx < P) ? pl[idx] : 0u;
                } else if ((bw >> ln) & 1u) {
                    const uint32_t idx = G + base + __popc(bw & lt);
                    v = (idx < P) ? pl[idx] : 0u;
                }
                sw[phys(32 * j + ln, lg)] = v;
                base += __popc(bw);
            }
            if (j1 == G && j0 < j1 && ln == 0 && G + base != P) atomicOr(a.err, kErrCorrupt);  // the bitmap must account for P
            __syncthreads();
        }
        // inverse Bitshuffle (lane b: plane b's word -> lane l: code l), zigzag
        // undone, inverse Diff: prefix sum over the chunk modulo 2^32
        uint32_t vv[PER], run = 0;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const uint32_t g = first / 32 + i;
            vv[i] = 0;
            if (g >= G) continue;  // warp-uniform
            const uint32_t pw = sw[ln * G + (g ^ sx)];
            const int nb = 32 - __clz(__ballot_sync(kFull, pw != 0u));  // planes 0..nb-1 may be nonzero
            uint32_t incl = (uint32_t)unzz(nb > 12 ? transpose32(pw, ln) : untranspose32_low(pw, nb, ln));
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t x = __shfl_up_sync(kFull, incl, o);
                if (ln >= o) incl += x;
            }
            vv[i] = run + incl;
            run += __shfl_sync(kFull, incl, 31);
        }
        uint32_t all;
        const uint32_t before = __shfl_sync(kFull, block_excl(ln == 0 ? run : 0u, tmp, &all), 0);
        float *gout = a.out + e0;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const uint32_t j = first + 32 * i + ln;
            if (j < cnt) gout[j] = __fmul_rn(__int2float_rn((int32_t)(vv[i] + before)), a.step);
        }
        __syncthreads();  // every reconstruction store of the chunk before its outliers
        if (t < (int)mc) {
            if (oi >= e0 && oi < e0 + cnt)
                a.out[oi] = __uint_as_float(ov);
            else
                atomicOr(a.err, kErrCorrupt);
        }
        for (uint32_t k = kCT + t; k < mc; k += kCT) {
            const uint32_t idx = pay[P + k], val = pay[P + mc + k];
            if (idx >= e0 && idx < e0 + cnt)
                a.out[idx] = __uint_as_float(val);
            else
                atomicOr(a.err, kErrCorrupt);
        }
    }
}

template <typename K>
int grid_for(K kernel, size_t smem, uint64_t nc, int num_sms) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kCT, smem) != cudaSuccess || per_sm < 1)
        per_sm = 1;
    const uint64_t want = (uint64_t)num_sms * per_sm;
    return (int)(nc < want ? (nc ? nc : 1) : want);
}

// One contiguous chunk range per CTA of one resident wave.
template <int PER, bool RRE>
cudaError_t chunked_encode_as(ChunkedArgs a, int num_sms, cudaStream_t stream) {
    const size_t es = enc_smem_bytes(a.m);
    cudaError_t e =
        cudaFuncSetAttribute(chunk_encode<PER, RRE>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)es);
    if (e != cudaSuccess) return e;
    const uint64_t want = (uint64_t)grid_for(chunk_encode<PER, RRE>, es, a.nc, num_sms);
    a.per_range = (uint32_t)((a.nc + want - 1) / want);
    a.ranges = a.nc ? (uint32_t)((a.nc + a.per_range - 1) / a.per_range) : 0u;
    if (a.nc) chunk_encode<PER, RRE><<<a.ranges, kCT, es, stream>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    chunk_scan<<<1, kScanThreads, 0, stream>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (a.nc) chunk_gather<<<a.ranges, kCT, 0, stream>>>(a);
    return cudaGetLastError();
}

template <int PER, bool RRE>
cudaError_t chunked_decode_as(const ChunkedDecArgs &a, uint64_t nc, int num_sms, cudaStream_t stream) {
    const size_t ds = dec_smem_bytes(a.m);
    cudaError_t e =
        cudaFuncSetAttribute(chunk_decode<PER, RRE>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ds);
    if (e != cudaSuccess) return e;
    if (nc) chunk_decode<PER, RRE><<<grid_for(chunk_decode<PER, RRE>, ds, nc, num_sms), kCT, ds, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

uint64_t chunked_slot_words(uint32_t m) { return 1 + (uint64_t)((m + 31) & ~31u) + 2ull * m; }

cudaError_t launch_chunked_encode(const ChunkedArgs &a, int num_sms, cudaStream_t stream) {
    switch (a.m * 2 + (a.rre ? 1 : 0)) {
    case 2048: return chunked_encode_as<4, false>(a, num_sms, stream);
    case 2049: return chunked_encode_as<4, true>(a, num_sms, stream);
    case 4096: return chunked_encode_as<8, false>(a, num_sms, stream);
    case 4097: return chunked_encode_as<8, true>(a, num_sms, stream);
    case 8192: return chunked_encode_as<16, false>(a, num_sms, stream);
    case 8193: return chunked_encode_as<16, true>(a, num_sms, stream);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_chunked_decode(const ChunkedDecArgs &a, int num_sms, cudaStream_t stream) {
    const uint64_t nc = (a.n + a.m - 1) / a.m;
    switch (a.m * 2 + (a.rre ? 1 : 0)) {
    case 2048: return chunked_decode_as<4, false>(a, nc, num_sms, stream);
    case 2049: return chunked_decode_as<4, true>(a, nc, num_sms, stream);
    case 4096: return chunked_decode_as<8, false>(a, nc, num_sms, stream);
    case 4097: return chunked_decode_as<8, true>(a, nc, num_sms, stream);
    case 8192: return chunked_decode_as<16, false>(a, nc, num_sms, stream);
    case 8193: return chunked_decode_as<16, true>(a, nc, num_sms, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace eblc
