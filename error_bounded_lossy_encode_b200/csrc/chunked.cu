// chunked.cu -- the chunk-cooperative codec for sm_100a: Quant -> Diff ->
// Bitshuffle -> RZE over byte chunks of 4096, 8192 or 16384 bytes of float32
// input ("Pipeline specialization internals", Chunk-cooperative path: one
// CTA owns a chunk, intermediates stay in shared memory; "nvrtc_chunk_fusion.h
// File Reference", launchNvrtcChunkFusedEncode: each chunk's coded form in a
// scratch slot with its size, then the cross-chunk scan/pack tail).
//
//   chunk_encode  one CTA per chunk (grid-stride): the linear quantizer and
//                 the outlier test, first differences reset at the chunk start
//                 in zigzag form, the 32-plane bit transpose of every group of
//                 32 codes by warp ballots, zero elimination (a bitmap of the
//                 nonzero words by ballots, the nonzero words compacted by a
//                 block scan) or the shuffled words verbatim when that is not
//                 smaller, then the chunk's outliers in ascending order; the
//                 record goes to the chunk's scratch slot, its size to sizes[].
//   chunk_scan    one CTA: exclusive scan of the record sizes and outlier
//                 counts -> chunk index, header and result block.
//   chunk_gather  records from scratch to their place in the stream.
//   chunk_decode  one CTA per chunk: zero elimination undone (ranks by
//                 popcounts), the inverse bit transpose by ballots, zigzag
//                 undone, a block-wide prefix sum, dequantization, outliers.
// No inter-CTA waits anywhere: the scan is its own launch.
#include "common.cuh"
#include "kernels.h"

namespace eblc {
namespace {

constexpr int kCT = 256;                  // threads per CTA
constexpr int kCW = kCT / 32;
constexpr uint32_t kFull = 0xffffffffu;
constexpr uint32_t kMaxM = 4096;          // largest chunk, elements

__device__ __forceinline__ uint32_t zz(int32_t d) { return ((uint32_t)d << 1) ^ (uint32_t)(d >> 31); }
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

struct __align__(16) EncShared {
    int32_t q[kMaxM];
    uint32_t sw[kMaxM];       // shuffled words, plane-major
    uint32_t oflag[kMaxM / 32];
    uint32_t tmp[kCW];
};

__global__ void __launch_bounds__(kCT) chunk_encode(const ChunkedArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    EncShared &sm = *reinterpret_cast<EncShared *>(smem_raw);
    const int t = threadIdx.x, ln = t % 32, w = t / 32;
    __shared__ Bound bd;
    if (t == 0) {
        const float vmin = a.abs_mode ? 0.0f : a.range[0], vmax = a.abs_mode ? 0.0f : a.range[1];
        bd = resolve_bound(a.abs_mode, a.bound, vmin, vmax);
    }
    __syncthreads();
    for (uint64_t c = blockIdx.x; c < a.nc; c += gridDim.x) {
        const uint64_t e0 = c * a.m;
        const uint32_t cnt = (uint32_t)min((uint64_t)a.m, a.n - e0), mp = (cnt + 31u) & ~31u, G = mp / 32;
        uint32_t *rec = a.scratch + c * (uint64_t)a.slot_words;
        for (uint32_t j = t; j < G; j += kCT) sm.oflag[j] = 0u;
        __syncthreads();
        // Quant: codes and outlier flags (fp32 filter, fp64 test in the band)
        for (uint32_t j = t; j < mp; j += kCT) {
            int32_t qq = 0;
            if (j < cnt) {
                const float x = a.in[e0 + j];
                const float y = __fmul_rn(x, bd.inv2eb);
                qq = (fabsf(y) < 0x1p30f) ? __float2int_rn(y) : 0;
                const float xr = __fmul_rn(__int2float_rn(qq), bd.step);
                const float d = fabsf(__fsub_rn(x, xr));
                bool o = d > bd.t_out;
                if (!o && !(d <= bd.t_in)) {
                    const bool finite = fabsf(x) < __int_as_float(0x7f800000);
                    o = !finite || !(fabs(__dsub_rn((double)x, (double)xr)) <= bd.eb);
                }
                if (o) atomicOr(&sm.oflag[j >> 5], 1u << (j & 31u));
            }
            sm.q[j] = qq;
        }
        __syncthreads();
        // Diff (zigzag) and Bitshuffle: warp w takes groups g = w, w + 8, ...;
        // lane l holds code 32 g + l; ballot b gives plane b's word of the group.
        for (uint32_t g = w; g < G; g += kCW) {
            const uint32_t j = g * 32 + ln;
            const uint32_t d = (j < cnt) ? zz(sm.q[j] - (j ? sm.q[j - 1] : 0)) : 0u;
            uint32_t mine = 0;
#pragma unroll
            for (int b = 0; b < 32; ++b) {
                const uint32_t pb = __ballot_sync(kFull, (d >> b) & 1u);
                if (ln == b) mine = pb;
            }
            sm.sw[ln * G + g] = mine;
        }
        __syncthreads();
        // RZE: count the nonzero words, then bitmap + compaction or verbatim
        uint32_t nz = 0;
        for (uint32_t k = t; k < mp; k += kCT) nz += sm.sw[k] != 0u;
        uint32_t nnz;
        (void)block_excl(nz, sm.tmp, &nnz);
        const uint32_t r = G + nnz;
        const bool raw = r >= mp;
        const uint32_t P = raw ? mp : r;
        if (raw) {
            for (uint32_t k = t; k < mp; k += kCT) rec[1 + k] = sm.sw[k];
        } else {
            uint32_t base = 0;
            for (uint32_t k0 = 0; k0 < mp; k0 += kCT) {  // rounds of one word per thread, in order
                const uint32_t k = k0 + t;
                const bool nzk = k < mp && sm.sw[k] != 0u;
                const uint32_t bal = __ballot_sync(kFull, nzk);
                if (k < mp && ln == 0) rec[1 + k / 32] = bal;  // bitmap word k / 32 (lane l: word 32 (k/32) + l)
                uint32_t round_total;
                const uint32_t pos = block_excl(nzk ? 1u : 0u, sm.tmp, &round_total);
                if (nzk) rec[1 + G + base + pos] = sm.sw[k];
                base += round_total;
            }
        }
        // outliers of the chunk, ascending: ranks from the flag words' popcounts
        uint32_t oc = 0;
        for (uint32_t j = t; j < G; j += kCT) oc += __popc(sm.oflag[j]);
        uint32_t mc;
        (void)block_excl(oc, sm.tmp, &mc);
        if (mc) {
            uint32_t obase = 0;
            for (uint32_t j0 = 0; j0 < G; j0 += kCT) {
                const uint32_t j = j0 + t;
                const uint32_t fw = j < G ? sm.oflag[j] : 0u;
                uint32_t round_total;
                uint32_t p = obase + block_excl(__popc(fw), sm.tmp, &round_total);
                uint32_t bits = fw;
                while (bits) {
                    const uint32_t e = j * 32 + (uint32_t)(__ffs(bits) - 1);
                    bits &= bits - 1u;
                    rec[1 + P + p] = (uint32_t)(e0 + e);
                    rec[1 + P + mc + p] = __float_as_uint(a.in[e0 + e]);
                    ++p;
                }
                obase += round_total;
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

// Exclusive scan of the record sizes and outlier counts over all chunks (one
// CTA), the chunk index and the header of the stream, the result block.
__global__ void __launch_bounds__(kScanThreads) chunk_scan(const ChunkedArgs a) {
    __shared__ unsigned long long part_r[kScanThreads / 32], part_m[kScanThreads / 32];
    const int t = threadIdx.x, ln = t % 32, w = t / 32;
    const uint64_t per = (a.nc + kScanThreads - 1) / kScanThreads;
    const uint64_t c0 = min(a.nc, per * t), c1 = min(a.nc, c0 + per);
    unsigned long long sr = 0, sm_ = 0;
    for (uint64_t c = c0; c < c1; ++c) {
        sr += a.sizes[c];
        sm_ += a.outl[c];
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
    unsigned long long br = 0, bm = 0, R = 0, M = 0;
    for (int k = 0; k < kScanThreads / 32; ++k) {
        br += (k < w) ? part_r[k] : 0ull;
        bm += (k < w) ? part_m[k] : 0ull;
        R += part_r[k];
        M += part_m[k];
    }
    unsigned long long r = br + ir - sr, m = bm + im - sm_;
    const Layout L = chunked_layout(a.n, a.m);
    const bool idx_fits = L.record_off <= a.out_cap;
    for (uint64_t c = c0; c < c1; ++c) {
        a.offs[c] = (uint32_t)r;
        if (idx_fits) *reinterpret_cast<uint2 *>(a.out + L.index_off + 8 * c) = make_uint2((uint32_t)r, (uint32_t)m);
        r += a.sizes[c];
        m += a.outl[c];
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

struct __align__(16) DecShared {
    uint32_t sw[kMaxM];
    uint32_t q[kMaxM];
    uint32_t rank[kMaxM / 32];  // nonzero words before each bitmap word
    uint32_t tmp[kCW];
    uint32_t info[4];           // P, raw, mc, record word offset
};

__global__ void __launch_bounds__(kCT) chunk_decode(const ChunkedDecArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    DecShared &sm = *reinterpret_cast<DecShared *>(smem_raw);
    const int t = threadIdx.x, ln = t % 32, w = t / 32;
    const Layout L = chunked_layout(a.n, a.m);
    const uint32_t *recs = reinterpret_cast<const uint32_t *>(a.in + L.record_off);
    const uint64_t R = a.W + 2 * a.mo;
    for (uint64_t c = blockIdx.x; c < L.nc; c += gridDim.x) {
        const uint64_t e0 = c * a.m;
        const uint32_t cnt = (uint32_t)min((uint64_t)a.m, a.n - e0), mp = (cnt + 31u) & ~31u, G = mp / 32;
        if (t == 0) {
            const uint2 ent = *reinterpret_cast<const uint2 *>(a.in + L.index_off + 8 * c);
            uint64_t nx = R, nm = a.mo;
            if (c + 1 < L.nc) {
                const uint2 e2 = *reinterpret_cast<const uint2 *>(a.in + L.index_off + 8 * (c + 1));
                nx = e2.x;
                nm = e2.y;
            }
            uint32_t ok = nx >= (uint64_t)ent.x + 1 && nm >= ent.y && nx <= R && nm <= a.mo;
            uint32_t P = 0, raw = 0, mc = 0;
            if (ok) {
                const uint32_t head = recs[ent.x];
                P = head & 0x7fffffffu;
                raw = head >> 31;
                mc = (uint32_t)(nm - ent.y);
                ok = (uint64_t)ent.x + 1 + P + 2ull * mc == nx && (raw ? P == mp : (P >= G && P < mp));
            }
            if (!ok) {
                atomicOr(a.err, kErrCorrupt);
                P = 0xffffffffu;
            }
            sm.info[0] = P;
            sm.info[1] = raw;
            sm.info[2] = mc;
            sm.info[3] = ent.x;
        }
        __syncthreads();
        const uint32_t P = sm.info[0], raw = sm.info[1], mc = sm.info[2];
        const uint32_t *pay = recs + sm.info[3] + 1;
        if (P == 0xffffffffu) {  // corrupt record: skip the chunk
            __syncthreads();
            continue;
        }
        if (raw) {
            for (uint32_t k = t; k < mp; k += kCT) sm.sw[k] = pay[k];
        } else {
            // ranks of the bitmap words (G <= 128: one warp, four words per lane)
            if (w == 0) {
                uint32_t s4[4], tot = 0;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint32_t j = 4 * ln + i;
                    s4[i] = (j < G) ? __popc(pay[j]) : 0u;
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
                    if (4 * ln + i < G) sm.rank[4 * ln + i] = r0;
                    r0 += s4[i];
                }
                if (ln == 31 && G + incl != P) atomicOr(a.err, kErrCorrupt);  // the bitmap must account for P
            }
            __syncthreads();
            for (uint32_t k = t; k < mp; k += kCT) {
                const uint32_t bw = pay[k / 32], bit = 1u << (k & 31u);
                uint32_t v = 0;
                if (bw & bit) {
                    const uint32_t idx = G + sm.rank[k / 32] + __popc(bw & (bit - 1u));
                    v = (idx < P) ? pay[idx] : 0u;
                }
                sm.sw[k] = v;
            }
        }
        __syncthreads();
        // inverse Bitshuffle: lane b holds plane b's word of group g; ballot l gives code l
        for (uint32_t g = w; g < G; g += kCW) {
            const uint32_t pw = sm.sw[ln * G + g];
            uint32_t code = 0;
#pragma unroll
            for (int l = 0; l < 32; ++l) {
                const uint32_t cb = __ballot_sync(kFull, (pw >> l) & 1u);
                if (ln == l) code = cb;
            }
            sm.q[g * 32 + ln] = (uint32_t)unzz(code);
        }
        __syncthreads();
        // inverse Diff: inclusive prefix sum over the chunk (modulo 2^32), then
        // dequantization; thread t takes codes [t * E, t * E + E)
        const uint32_t E = mp / kCT ? (mp + kCT - 1) / kCT : 1;
        const uint32_t j0 = min(t * E, mp), j1 = min(j0 + E, mp);
        uint32_t s = 0;
        for (uint32_t j = j0; j < j1; ++j) s += sm.q[j];
        uint32_t tot;
        uint32_t run = block_excl(s, sm.tmp, &tot);
        float *gout = a.out + e0;
        for (uint32_t j = j0; j < j1; ++j) {
            run += sm.q[j];
            if (j < cnt) gout[j] = __fmul_rn(__int2float_rn((int32_t)run), a.step);
        }
        __syncthreads();  // every reconstruction store of the chunk before its outliers
        const uint32_t *oi = pay + P;
        for (uint32_t k = t; k < mc; k += kCT) {
            const uint32_t idx = oi[k], val = oi[mc + k];
            if (idx >= e0 && idx < e0 + cnt)
                a.out[idx] = __uint_as_float(val);
            else
                atomicOr(a.err, kErrCorrupt);
        }
        __syncthreads();
    }
}

int grid_for(uint64_t nc, int num_sms, int per_sm) {
    const uint64_t want = (uint64_t)num_sms * per_sm;
    return (int)(nc < want ? (nc ? nc : 1) : want);
}

}  // namespace

uint64_t chunked_slot_words(uint32_t m) { return 1 + (uint64_t)((m + 31) & ~31u) + 2ull * m; }

cudaError_t launch_chunked_encode(const ChunkedArgs &a, int num_sms, cudaStream_t stream) {
    const size_t es = sizeof(EncShared);
    cudaError_t e = cudaFuncSetAttribute(chunk_encode, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)es);
    if (e != cudaSuccess) return e;
    if (a.nc) chunk_encode<<<grid_for(a.nc, num_sms, 4), kCT, es, stream>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    chunk_scan<<<1, kScanThreads, 0, stream>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (a.nc) chunk_gather<<<grid_for(a.nc, num_sms, 8), kCT, 0, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_chunked_decode(const ChunkedDecArgs &a, int num_sms, cudaStream_t stream) {
    const size_t ds = sizeof(DecShared);
    cudaError_t e = cudaFuncSetAttribute(chunk_decode, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ds);
    if (e != cudaSuccess) return e;
    const uint64_t nc = (a.n + a.m - 1) / a.m;
    if (nc) chunk_decode<<<grid_for(nc, num_sms, 4), kCT, ds, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace eblc
