// chunked.cu -- the chunk-cooperative codec for sm_100a: Quant -> Diff ->
// Bitshuffle -> RZE over byte chunks of 4096, 8192 or 16384 bytes of float32
// input ("Pipeline specialization internals", Chunk-cooperative path: one
// CTA owns a chunk, intermediates stay in shared memory; "nvrtc_chunk_fusion.h
// File Reference", launchNvrtcChunkFusedEncode: each chunk's coded form in a
// scratch slot with its size, then the cross-chunk scan/pack tail).
//
//   chunk_encode  one CTA per chunk (grid-stride), each warp a contiguous run
//                 of 32-code groups in registers: the linear quantizer and
//                 the outlier test, first differences reset at the chunk start
//                 in zigzag form, the 32 x 32 bit transpose of every group
//                 (lane b gets bit plane b) by a shuffle butterfly, zero
//                 elimination (a bitmap of the nonzero words by ballots, the
//                 nonzero words compacted warp by warp after one block scan)
//                 or the shuffled words verbatim when that is not smaller,
//                 then the chunk's outliers in ascending order; the record
//                 goes to the chunk's scratch slot, its size to sizes[].
//   chunk_scan    one CTA: exclusive scan of the record sizes and outlier
//                 counts -> chunk index, header and result block.
//   chunk_gather  records from scratch to their place in the stream.
//   chunk_decode  one CTA per chunk: zero elimination undone (ranks by
//                 popcounts), the inverse transpose, zigzag undone and the
//                 prefix sum in each warp's registers, one block scan of the
//                 warps' totals, dequantization, outliers.
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

// Dynamic shared memory of the encoder for chunks of m elements: the
// shuffled words, the outlier flag words, the scan's warp totals.
__host__ __device__ constexpr size_t enc_smem_bytes(uint32_t m) { return 4ull * (m + m / 32 + kCW); }

// PER = m / kCT.  Warp w owns the PER groups of 32 codes starting at code
// 32 PER w of the chunk and keeps them in registers from the load to the
// bit transpose; the input of the CTA's next chunk is loaded as soon as the
// current chunk's codes are formed, so its latency overlaps the rest.
template <int PER>
__global__ void __launch_bounds__(kCT) chunk_encode(const ChunkedArgs a) {
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
    load(blockIdx.x);
    __syncthreads();
    for (uint64_t c = blockIdx.x; c < a.nc; c += gridDim.x) {
        const uint64_t e0 = c * a.m;
        const uint32_t cnt = (uint32_t)min((uint64_t)a.m, a.n - e0), mp = (cnt + 31u) & ~31u, G = mp / 32;
        const int lg = (mp == a.m) ? lg_full : 0;
        uint32_t *rec = a.scratch + c * (uint64_t)a.slot_words;
        // Quant, Diff (zigzag, reset at the chunk start) and Bitshuffle of the
        // warp's groups: lane l holds code 32 g + l; the transpose gives lane b
        // plane b's word of the group.
        bool o;
        int32_t prev = 0;
        if (ln == 0 && first > 0 && first <= cnt) prev = quant(bd, xp, o);
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const uint32_t g = first / 32 + i, j = 32 * g + ln;
            if (g >= G) break;  // warp-uniform
            o = false;
            const int32_t qq = (j < cnt) ? quant(bd, xv[i], o) : 0;
            int32_t left = __shfl_up_sync(kFull, qq, 1);
            if (ln == 0) left = prev;
            prev = __shfl_sync(kFull, qq, 31);
            const uint32_t d = (j < cnt) ? zz(qq - left) : 0u;
            const uint32_t fw = __ballot_sync(kFull, o);
            if (ln == 0) oflag[g] = fw;
            sw[phys(ln * G + g, lg)] = transpose32(d, ln);
        }
        load(c + gridDim.x);
        __syncthreads();
        // One block scan for both counts: warp w's nonzero words over its word
        // range [k0, k1) (upper 16 bits, lane 0 only) and thread t's outliers
        // in flag word t (lower 16 bits; G <= kCT).  Both totals are <= 4096.
        const uint32_t per = ((G + kCW - 1) / kCW) * 32;
        const uint32_t k0 = min(w * per, mp), k1 = min(k0 + per, mp);
        uint32_t cntw = 0;
        for (uint32_t k = k0 + ln; k < k1; k += 32) cntw += __popc(__ballot_sync(kFull, sw[phys(k, lg)] != 0u));
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
                const uint32_t bal = __ballot_sync(kFull, v != 0u);
                if (ln == 0) rec[1 + k / 32] = bal;  // bitmap word k / 32: bit l = word 32 (k/32) + l
                if (v) rec[1 + G + base + __popc(bal & ((1u << ln) - 1u))] = v;
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
        }
        __syncthreads();
    }
}

constexpr int kScanThreads = 1024;
constexpr int kScanWarps = kScanThreads / 32;

// Exclusive scan of the record sizes and outlier counts over all chunks (one
// CTA), the chunk index and the header of the stream, the result block.
// Warp w takes a contiguous range of chunks, 32 at a time (coalesced): one
// pass for the warps' totals, a scan of those, a second pass for the entries.
__global__ void __launch_bounds__(kScanThreads) chunk_scan(const ChunkedArgs a) {
    __shared__ unsigned long long part_r[kScanWarps], part_m[kScanWarps];
    const int t = threadIdx.x, ln = t % 32, w = t / 32;
    const uint64_t steps = (a.nc + 32 * kScanWarps - 1) / (32 * kScanWarps);  // 32-chunk steps per warp
    const uint64_t c0 = min(a.nc, (uint64_t)w * steps * 32), c1 = min(a.nc, c0 + steps * 32);
    unsigned long long sr = 0, sm_ = 0;
#pragma unroll 4
    for (uint64_t c = c0 + ln; c < c1; c += 32) {
        sr += a.sizes[c];
        sm_ += a.outl[c];
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        sr += __shfl_xor_sync(kFull, sr, o);
        sm_ += __shfl_xor_sync(kFull, sm_, o);
    }
    if (ln == 0) {
        part_r[w] = sr;
        part_m[w] = sm_;
    }
    __syncthreads();
    unsigned long long r = 0, m = 0, R = 0, M = 0;
    for (int k = 0; k < kScanWarps; ++k) {
        r += (k < w) ? part_r[k] : 0ull;
        m += (k < w) ? part_m[k] : 0ull;
        R += part_r[k];
        M += part_m[k];
    }
    const Layout L = chunked_layout(a.n, a.m);
    const bool idx_fits = L.record_off <= a.out_cap;
    for (uint64_t cb = c0; cb < c1; cb += 32) {
        const uint64_t c = cb + ln;
        const uint32_t s = (c < c1) ? a.sizes[c] : 0u, q = (c < c1) ? a.outl[c] : 0u;
        uint32_t is = s, iq = q;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t x = __shfl_up_sync(kFull, is, o), y = __shfl_up_sync(kFull, iq, o);
            if (ln >= o) {
                is += x;
                iq += y;
            }
        }
        const uint64_t rc = r + is - s, mcc = m + iq - q;
        if (c < c1) {
            a.offs[c] = (uint32_t)rc;
            if (idx_fits) *reinterpret_cast<uint2 *>(a.out + L.index_off + 8 * c) = make_uint2((uint32_t)rc, (uint32_t)mcc);
        }
        r += __shfl_sync(kFull, is, 31);
        m += __shfl_sync(kFull, iq, 31);
    }
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
    h[1] = kVersion | ((uint32_t)((a.abs_mode ? kFlagAbs : 0) | kFlagChunked) << 16);
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

__global__ void __launch_bounds__(kCT) chunk_gather(const ChunkedArgs a) {
    const Layout L = chunked_layout(a.n, a.m);
    uint32_t *recs = reinterpret_cast<uint32_t *>(a.out + L.record_off);
    const uint64_t cap_words = (a.out_cap > L.record_off) ? (a.out_cap - L.record_off) / 4 : 0;
    for (uint64_t c = blockIdx.x; c < a.nc; c += gridDim.x) {
        const uint64_t o = a.offs[c], len = a.sizes[c];
        if (o + len > cap_words) continue;  // reported by chunk_scan (capacity)
        const uint32_t *src = a.scratch + c * (uint64_t)a.slot_words;
        for (uint64_t k = threadIdx.x; k < len; k += kCT) st_cs_u32(recs + o + k, src[k]);
    }
}

// Dynamic shared memory of the decoder for chunks of m elements: the record's
// payload words, the shuffled words, the ranks of the bitmap words, the
// scan's warp totals and the chunk's record facts.
__host__ __device__ constexpr size_t dec_smem_bytes(uint32_t m) { return 4ull * (2 * m + m / 32 + kCW + 4); }

// PER = m / kCT.  Warp w decodes the PER groups starting at code 32 PER w:
// the transpose, zigzag and the prefix sum stay in its registers, and its
// reconstructions go out as whole 128-byte lines.  Thread 0 loads the index
// entries and the head word of the CTA's next chunk one chunk ahead; the
// payload and the first kCT outliers of a chunk come in one round of loads.
template <int PER>
__global__ void __launch_bounds__(kCT) chunk_decode(const ChunkedDecArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    uint32_t *const pl = reinterpret_cast<uint32_t *>(smem_raw);  // payload (RZE form)
    uint32_t *const sw = pl + a.m;
    uint32_t *const rank = sw + a.m;
    uint32_t *const tmp = rank + a.m / 32;
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
            // ranks of the bitmap words (G <= 128: warp 0, four words per lane)
            if (w == 0) {
                uint32_t s4[4], tot = 0;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint32_t j = 4 * ln + i;
                    s4[i] = (j < G) ? __popc(pl[j]) : 0u;
                    tot += s4[i];
                }
                uint32_t incl = tot;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const uint32_t x = __shfl_up_sync(kFull, incl, o);
                    if (ln >= o) incl += x;
                }
                uint32_t r0 = incl - tot;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    if (4 * ln + i < G) rank[4 * ln + i] = r0;
                    r0 += s4[i];
                }
                if (ln == 31 && G + incl != P) atomicOr(a.err, kErrCorrupt);  // the bitmap must account for P
            }
            __syncthreads();
            for (uint32_t k = t; k < mp; k += kCT) {
                const uint32_t bw = pl[k / 32], bit = 1u << (k & 31u);
                uint32_t v = 0;
                if (bw & bit) {
                    const uint32_t idx = G + rank[k / 32] + __popc(bw & (bit - 1u));
                    v = (idx < P) ? pl[idx] : 0u;
                }
                sw[phys(k, lg)] = v;
            }
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
            uint32_t incl = (uint32_t)unzz(transpose32(sw[phys(ln * G + g, lg)], ln));
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

template <int PER>
cudaError_t chunked_encode_as(const ChunkedArgs &a, int num_sms, cudaStream_t stream) {
    const size_t es = enc_smem_bytes(a.m);
    cudaError_t e = cudaFuncSetAttribute(chunk_encode<PER>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)es);
    if (e != cudaSuccess) return e;
    if (a.nc) chunk_encode<PER><<<grid_for(chunk_encode<PER>, es, a.nc, num_sms), kCT, es, stream>>>(a);
    return cudaGetLastError();
}

template <int PER>
cudaError_t chunked_decode_as(const ChunkedDecArgs &a, uint64_t nc, int num_sms, cudaStream_t stream) {
    const size_t ds = dec_smem_bytes(a.m);
    cudaError_t e = cudaFuncSetAttribute(chunk_decode<PER>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ds);
    if (e != cudaSuccess) return e;
    if (nc) chunk_decode<PER><<<grid_for(chunk_decode<PER>, ds, nc, num_sms), kCT, ds, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

uint64_t chunked_slot_words(uint32_t m) { return 1 + (uint64_t)((m + 31) & ~31u) + 2ull * m; }

cudaError_t launch_chunked_encode(const ChunkedArgs &a, int num_sms, cudaStream_t stream) {
    cudaError_t e;
    switch (a.m) {
    case 1024: e = chunked_encode_as<4>(a, num_sms, stream); break;
    case 2048: e = chunked_encode_as<8>(a, num_sms, stream); break;
    case 4096: e = chunked_encode_as<16>(a, num_sms, stream); break;
    default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
    chunk_scan<<<1, kScanThreads, 0, stream>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (a.nc) {
        int per_sm = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, chunk_gather, kCT, 0) != cudaSuccess || per_sm < 1)
            per_sm = 1;
        const uint64_t want = (uint64_t)num_sms * per_sm;
        chunk_gather<<<(int)(a.nc < want ? a.nc : want), kCT, 0, stream>>>(a);
    }
    return cudaGetLastError();
}

cudaError_t launch_chunked_decode(const ChunkedDecArgs &a, int num_sms, cudaStream_t stream) {
    const uint64_t nc = (a.n + a.m - 1) / a.m;
    switch (a.m) {
    case 1024: return chunked_decode_as<4>(a, nc, num_sms, stream);
    case 2048: return chunked_decode_as<8>(a, nc, num_sms, stream);
    case 4096: return chunked_decode_as<16>(a, nc, num_sms, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace eblc
