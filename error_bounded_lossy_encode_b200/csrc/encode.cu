// encode.cu -- fused single-pass encoder for sm_100a.
//
// One launch turns n float32 values into the whole stream:
//   linear quantization q = rint(x * inv2eb) with the bound test and the
//   outlier side list ("Pipeline specialization internals", Roles and
//   strategies: Elementwise linear quantizer absorbed into the predictor;
//   "nvrtc_chunk_fusion.h File Reference", launchNvrtcChunkFusedEncode:
//   split-outlier side output), 1-D Lorenzo first difference reset at each
//   block (RegionLocal, region reset), zigzag (interior transform), one width
//   byte per block and fixed-length bit packing (SegmentCodec,
//   AdaptiveBitpackCoder, meta_bytes = 1), and the cross-chunk exclusive
//   scan that places every chunk record at its final offset
//   (launchGenericChunkFusion: scan/pack tail) -- here a single-pass
//   decoupled look-back instead of a separate scan and gather.
//
// CTA organisation (320 threads, 2 CTAs per SM):
//   warps 0..7  compute: each owns a contiguous 512-element slice of the
//               4096-element tile, held as warp-tiles of 32*V elements
//               (V consecutive elements per lane, V = 4, or 8 for B = 256);
//               a block of B elements spans LPB = B/V lanes.
//   warp 8      look-back: sums the warp totals of a tile, publishes the
//               tile aggregate, resolves its exclusive prefix from the
//               predecessors' status words, writes the chunk index entry
//               (and the header for the last tile).
//   warp 9      producer: claims tiles in order from a global counter and
//               streams them into a 4-stage shared-memory ring with bulk
//               async copies (cp.async.bulk, completion on mbarriers).
// Compute warps pack a tile into a shared-memory staging buffer at
// tile-local offsets, then, while the look-back of that tile resolves,
// compute the next tile; the staged words are copied to their final global
// position one tile later.  Every wait is bounded (kErrTimeout), every global
// store is checked against the caller's capacity (kErrCapacity).
#include "common.cuh"
#include "kernels.h"

namespace eblc {
namespace {

constexpr int kNW = 8;                    // compute warps
constexpr int kS = 4;                     // input stages
constexpr int kLookbackWarp = kNW;
constexpr int kThreads = (kNW + 2) * 32;
constexpr uint32_t kFull = 0xffffffffu;
constexpr uint64_t kInclBit = 1ull << 63;

struct __align__(128) EncSmem {
    float in[kS][kChunk];                 // input ring (bulk-copy destination)
    uint32_t out[2][kChunk];              // packed payload staging, double buffered
    uint8_t width[2][kChunk / 32];        // width bytes of the tile's blocks
    uint32_t totals[2][kNW][2];           // per warp: payload words, outliers
    uint32_t wprefix[2][kNW][2];          // per warp: exclusive prefix within the tile
    uint32_t info[2][4];                  // record word offset, payload words, outliers, tile
    int32_t tile_id[kS];
    uint64_t full[kS], empty[kS], computed[2], ready[2];
    Bound bound;
};

// Look-back status word: bits 0..31 record words + 1 (never 0 once
// published), bits 32..62 outliers, bit 63 set for an inclusive prefix.
__device__ __forceinline__ uint64_t pack_status(uint32_t R, uint32_t m, bool incl) {
    return (uint64_t)(R + 1u) | ((uint64_t)m << 32) | (incl ? kInclBit : 0ull);
}

template <int LPB>
__device__ __forceinline__ uint32_t group_or(uint32_t v, int g) {
    if constexpr (LPB == 32) {
        return __reduce_or_sync(kFull, v);
    } else if constexpr (LPB == 16) {
        const uint32_t a = __reduce_or_sync(kFull, g == 0 ? v : 0u);
        const uint32_t b = __reduce_or_sync(kFull, g == 1 ? v : 0u);
        return g ? b : a;
    } else {
#pragma unroll
        for (int o = LPB / 2; o > 0; o >>= 1) v |= __shfl_xor_sync(kFull, v, o);
        return v;
    }
}

__host__ __device__ constexpr int ilog2(int v) { return v <= 1 ? 0 : 1 + ilog2(v / 2); }

// Pack the lane's V codes (width w, uniform over the lane's group of LPB
// lanes) into the block's word array `dst` (shared memory): code j of the
// block occupies bits [j*w, j*w + w), least significant bit first.  Lane r
// of the group owns bits [r*V*w, (r+1)*V*w).  Lanes whose segment is
// shorter than 32 bits are first merged pairwise (shuffles) until each
// active lane holds at least 32 bits; then each word is shared by at most
// two neighbouring segments, and the earlier lane's spill word is OR-ed into
// the later lane's first word.
template <int V, int LPB>
__device__ __forceinline__ void pack_block(const uint32_t (&z)[V], uint32_t w, int r, int ln, uint32_t *dst) {
    const uint32_t L = V * w;
    uint32_t S[V + 1];
    S[0] = z[V - 1];
#pragma unroll
    for (int j = 1; j <= V; ++j) S[j] = 0u;
#pragma unroll
    for (int v = V - 2; v >= 0; --v) {
#pragma unroll
        for (int j = V - 1 - v; j >= 1; --j) S[j] = __funnelshift_lc(S[j - 1], S[j], w);
        S[0] = __funnelshift_lc(0u, S[0], w) | z[v];
    }

    uint32_t Lc = L;
    int stride = 1;
    const bool short_seg = (w != 0u) && (L < 32u);
    if (__any_sync(kFull, short_seg)) {
        constexpr int kIters = ilog2(LPB) < ilog2(32 / V) ? ilog2(LPB) : ilog2(32 / V);
#pragma unroll
        for (int it = 0; it < kIters; ++it) {
            const uint32_t o0 = __shfl_down_sync(kFull, S[0], 1 << it);
            const uint32_t o1 = __shfl_down_sync(kFull, S[1], 1 << it);
            if (short_seg && Lc < 32u) {
                if ((r & ((2 << it) - 1)) == 0) {
                    S[1] |= __funnelshift_lc(o0, o1, Lc);
                    S[0] |= o0 << Lc;
                }
                Lc <<= 1;
                stride <<= 1;
            }
        }
    }
    const bool active = (r & (stride - 1)) == 0;

    const uint32_t P = (uint32_t)r * L;  // bit offset of the segment in the block
    const uint32_t s = P & 31u, k0 = P >> 5;
#pragma unroll
    for (int j = V; j >= 1; --j) S[j] = __funnelshift_lc(S[j - 1], S[j], s);
    S[0] <<= s;
    const uint32_t nw = (s + Lc + 31u) >> 5;
    uint32_t last = S[0];
#pragma unroll
    for (int j = 1; j <= V; ++j)
        if (nw == (uint32_t)j + 1u) last = S[j];
    const int src = (r >= stride) ? ln - stride : ln;
    const uint32_t from_prev = __shfl_sync(kFull, last, src);
    if (r >= stride && s != 0u) S[0] |= from_prev;
    const bool last_shared = (r + stride < LPB) && (((P + Lc) & 31u) != 0u);
    const uint32_t nstore = nw - (last_shared ? 1u : 0u);
    if (active && w != 0u) {
#pragma unroll
        for (int j = 0; j <= V; ++j)
            if ((uint32_t)j < nstore) dst[k0 + j] = S[j];
    }
}

// Quantize, test, delta, zigzag and pack one 4096-element tile held in
// input stage s; packed words go to out[p] in this warp's region.
template <int V, int LPB>
__device__ __forceinline__ void compute_tile(EncSmem &sm, const Bound &bd, int s, int p, uint32_t valid, int cw,
                                             int ln, uint32_t &words_out, uint32_t &omask_out) {
    constexpr int kB = V * LPB;
    constexpr int kWT = 32 * V;
    constexpr int kWPW = kChunk / kWT / kNW;
    constexpr int kGroups = 32 / LPB;
    const int g = ln / LPB, r = ln % LPB;
    uint32_t *region = sm.out[p] + cw * (kWPW * kWT);
    uint32_t wo = 0, omask = 0;

#pragma unroll 1
    for (int k = 0; k < kWPW; ++k) {
        const int wt = cw * kWPW + k;
        const uint32_t e0 = wt * kWT + ln * V;
        float x[V];
#pragma unroll
        for (int h = 0; h < V / 4; ++h) {
            const float4 t = *reinterpret_cast<const float4 *>(&sm.in[s][e0 + 4 * h]);
            x[4 * h + 0] = t.x;
            x[4 * h + 1] = t.y;
            x[4 * h + 2] = t.z;
            x[4 * h + 3] = t.w;
        }
        const uint32_t blk = (uint32_t)(wt * kWT) / kB + g;  // block index within the chunk
        const int cnt = min(max((int)valid - (int)(blk * kB), 0), kB);

        int32_t q[V];
        uint32_t obits = 0, abits = 0;
#pragma unroll
        for (int v = 0; v < V; ++v) {
            const float y = __fmul_rn(x[v], bd.inv2eb);
            const int32_t qq = (fabsf(y) < 0x1p30f) ? __float2int_rn(y) : 0;
            const float xr = __fmul_rn(__int2float_rn(qq), bd.step);
            const float d = fabsf(__fsub_rn(x[v], xr));
            const bool out = d > bd.t_out;
            const bool amb = !(d <= bd.t_in) && !out;
            q[v] = qq;
            obits |= (uint32_t)out << v;
            abits |= (uint32_t)amb << v;
        }
        if (valid < kChunk) {  // ragged last tile: elements at or beyond `valid` do not exist
            const uint32_t have = (e0 >= valid) ? 0u : min(valid - e0, (uint32_t)V);
            const uint32_t vm = (have >= 32u) ? kFull : ((1u << have) - 1u);
#pragma unroll
            for (int v = 0; v < V; ++v)
                if (!((vm >> v) & 1u)) q[v] = 0;
            obits &= vm;
            abits &= vm;
        }
        if (__any_sync(kFull, abits != 0u)) {  // fp64 bound test where the fp32 filter is undecided
#pragma unroll
            for (int v = 0; v < V; ++v) {
                if ((abits >> v) & 1u) {
                    const float xr = __fmul_rn(__int2float_rn(q[v]), bd.step);
                    const bool finite = fabsf(x[v]) < __int_as_float(0x7f800000);
                    const bool ok = fabs(__dsub_rn((double)x[v], (double)xr)) <= bd.eb;
                    obits |= (uint32_t)(!finite || !ok) << v;
                }
            }
        }

        int32_t pv = __shfl_up_sync(kFull, q[V - 1], 1);
        if (r == 0) pv = 0;  // Lorenzo predecessor resets at the block start
        uint32_t z[V];
        uint32_t orz = 0;
#pragma unroll
        for (int v = 0; v < V; ++v) {
            const int32_t d = q[v] - (v ? q[v - 1] : pv);
            z[v] = ((uint32_t)d << 1) ^ (uint32_t)(d >> 31);
        }
        if (valid < kChunk) {
#pragma unroll
            for (int v = 0; v < V; ++v)
                if (e0 + v >= valid) z[v] = 0u;
        }
#pragma unroll
        for (int v = 0; v < V; ++v) orz |= z[v];
        const uint32_t w = 32u - __clz(group_or<LPB>(orz, g));
        const uint32_t bw = (w * (uint32_t)cnt + 31u) >> 5;
        uint32_t pre = 0, tot = 0;
#pragma unroll
        for (int gg = 0; gg < kGroups; ++gg) {
            const uint32_t b = __shfl_sync(kFull, bw, gg * LPB);
            pre += (gg < g) ? b : 0u;
            tot += b;
        }
        if (r == 0) sm.width[p][blk] = (uint8_t)w;
        pack_block<V, LPB>(z, w, r, ln, region + wo + pre);
        wo += tot;
        omask |= obits << (k * V);
    }
    words_out = wo;
    omask_out = omask;
}

// Copy one finished tile of this warp to its final position: payload words,
// outliers (indices then values after the tile's payload), widths.
template <int V, int LPB>
__device__ __forceinline__ bool finish_tile(EncSmem &sm, const EncodeArgs &a, const Layout &L, uint32_t iprev,
                                            int tile, int stage, uint32_t words, uint32_t omask, int cw, int ln) {
    constexpr int kB = V * LPB;
    constexpr int kWT = 32 * V;
    constexpr int kWPW = kChunk / kWT / kNW;
    const int q = iprev & 1;
    if (!mbar_wait(&sm.ready[q], (iprev >> 1) & 1, a.wait_ns, a.err)) return false;
    const uint32_t rec = sm.info[q][0], PW = sm.info[q][1], MT = sm.info[q][2];
    const uint32_t wpw = sm.wprefix[q][cw][0], wpo = sm.wprefix[q][cw][1];
    uint32_t *recs = reinterpret_cast<uint32_t *>(a.out + L.record_off);
    const uint64_t cap_words = (a.out_cap > L.record_off) ? (a.out_cap - L.record_off) / 4 : 0;
    bool over = false;

    const uint32_t *src = sm.out[q] + cw * (kWPW * kWT);
    const uint64_t w0 = (uint64_t)rec + wpw;
    for (uint32_t j = ln; j < words; j += 32) {
        if (w0 + j < cap_words)
            st_cs_u32(recs + w0 + j, src[j]);
        else
            over = true;
    }

    if (__any_sync(kFull, omask != 0u)) {
        uint32_t ord_base = 0;
#pragma unroll 1
        for (int k = 0; k < kWPW; ++k) {
            uint32_t bits = (omask >> (k * V)) & ((1u << V) - 1u);
            const uint32_t c = __popc(bits);
            uint32_t incl = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t t = __shfl_up_sync(kFull, incl, o);
                if (ln >= o) incl += t;
            }
            uint32_t ord = ord_base + incl - c;
            while (bits) {
                const int v = __ffs(bits) - 1;
                bits &= bits - 1u;
                const uint32_t e = (uint32_t)(cw * kWPW + k) * kWT + ln * V + v;
                const uint64_t pi = (uint64_t)rec + PW + wpo + ord;
                const uint64_t pv = pi + MT;
                if (pv < cap_words) {
                    recs[pi] = (uint32_t)tile * kChunk + e;
                    recs[pv] = __float_as_uint(sm.in[stage][e]);
                } else {
                    over = true;
                }
                ++ord;
            }
            ord_base += __shfl_sync(kFull, incl, 31);
        }
    }

    {  // this warp's width bytes (zeros past the last block up to the 16-byte pad)
        constexpr uint32_t kBPW = kChunk / kB / kNW;  // blocks per warp per tile
        const uint64_t b = (uint64_t)tile * (kChunk / kB) + cw * kBPW + ln;
        const uint64_t off = L.width_off + b;
        if (ln < (int)kBPW && b < pad16(L.nb)) {
            if (off < a.out_cap)
                a.out[off] = sm.width[q][cw * kBPW + ln];
            else
                over = true;
        }
    }
    if (__any_sync(kFull, over) && ln == 0) atomicOr(a.err, kErrCapacity);
    __syncwarp();
    if (ln == 0) mbar_arrive(&sm.empty[stage]);
    return true;
}

template <int V, int LPB>
__device__ void compute_warp(EncSmem &sm, const EncodeArgs &a, const Layout &L, int cw, int ln) {
    const Bound bd = sm.bound;
    int prev_tile = -1, prev_stage = 0;
    uint32_t prev_words = 0, prev_omask = 0;
    uint32_t i = 0;
    for (;; ++i) {
        const int s = i % kS, p = i & 1;
        if (!mbar_wait(&sm.full[s], (i / kS) & 1, a.wait_ns, a.err)) return;
        const int tile = sm.tile_id[s];
        if (tile < 0) break;
        const uint64_t e0 = (uint64_t)tile * kChunk;
        const uint32_t valid = (uint32_t)min((uint64_t)kChunk, a.n - e0);
        uint32_t words, omask;
        compute_tile<V, LPB>(sm, bd, s, p, valid, cw, ln, words, omask);
        const uint32_t outl = __reduce_add_sync(kFull, __popc(omask));
        if (ln == 0) {
            sm.totals[p][cw][0] = words;
            sm.totals[p][cw][1] = outl;
        }
        __syncwarp();
        if (ln == 0) mbar_arrive(&sm.computed[p]);
        if (prev_tile >= 0 &&
            !finish_tile<V, LPB>(sm, a, L, i - 1, prev_tile, prev_stage, prev_words, prev_omask, cw, ln))
            return;
        prev_tile = tile;
        prev_stage = s;
        prev_words = words;
        prev_omask = omask;
    }
    if (prev_tile >= 0) finish_tile<V, LPB>(sm, a, L, i - 1, prev_tile, prev_stage, prev_words, prev_omask, cw, ln);
}

__device__ void write_header(const EncodeArgs &a, const Layout &L, const Bound &bd, uint64_t R, uint64_t m) {
    const uint64_t W = R - 2 * m;
    const uint64_t total = L.record_off + 4 * R;
    if (total > a.out_cap || m > a.outlier_cap) atomicOr(a.err, kErrCapacity);
    a.result[0] = W;
    a.result[1] = m;
    a.result[2] = total;
    a.result[3] = R;
    a.result[4] = (uint64_t)__double_as_longlong(bd.eb);
    a.result[5] = (uint64_t)__float_as_uint(bd.step) | ((uint64_t)__float_as_uint(bd.inv2eb) << 32);
    a.result[6] = (uint64_t)__float_as_uint(bd.vmin) | ((uint64_t)__float_as_uint(bd.vmax) << 32);
    if (a.out_cap < L.record_off) return;
    uint32_t h[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) h[j] = 0u;
    const uint64_t ebits = (uint64_t)__double_as_longlong(bd.eb);
    const uint64_t bbits = (uint64_t)__double_as_longlong(a.bound);
    h[0] = kMagic;
    h[1] = kVersion | ((uint32_t)(a.abs_mode ? kFlagAbs : 0) << 16);
    h[2] = (uint32_t)a.n;
    h[3] = (uint32_t)(a.n >> 32);
    h[4] = a.block;
    h[5] = kChunk;
    h[6] = (uint32_t)ebits;
    h[7] = (uint32_t)(ebits >> 32);
    h[8] = __float_as_uint(bd.inv2eb);
    h[9] = __float_as_uint(bd.step);
    h[10] = __float_as_uint(bd.vmin);
    h[11] = __float_as_uint(bd.vmax);
    h[12] = (uint32_t)L.nb;
    h[13] = (uint32_t)(L.nb >> 32);
    h[14] = (uint32_t)L.nc;
    h[15] = (uint32_t)(L.nc >> 32);
    h[16] = (uint32_t)W;
    h[17] = (uint32_t)(W >> 32);
    h[18] = (uint32_t)m;
    h[19] = (uint32_t)(m >> 32);
    h[20] = (uint32_t)total;
    h[21] = (uint32_t)(total >> 32);
    h[22] = (uint32_t)bbits;
    h[23] = (uint32_t)(bbits >> 32);
    uint4 *dst = reinterpret_cast<uint4 *>(a.out);
#pragma unroll
    for (int j = 0; j < 8; ++j) dst[j] = make_uint4(h[4 * j], h[4 * j + 1], h[4 * j + 2], h[4 * j + 3]);
    // zero pad between the chunk index and the first record
    for (uint64_t b = L.index_off + 8 * L.nc; b < L.record_off; b += 4)
        *reinterpret_cast<uint32_t *>(a.out + b) = 0u;
}

__device__ void lookback_warp(EncSmem &sm, const EncodeArgs &a, const Layout &L, int ln) {
    for (uint32_t i = 0;; ++i) {
        const int s = i % kS, p = i & 1;
        if (!mbar_wait(&sm.full[s], (i / kS) & 1, a.wait_ns, a.err)) return;
        const int tile = sm.tile_id[s];
        if (tile < 0) break;
        if (!mbar_wait(&sm.computed[p], (i >> 1) & 1, a.wait_ns, a.err)) return;

        const uint32_t tw = (ln < kNW) ? sm.totals[p][ln][0] : 0u;
        const uint32_t to = (ln < kNW) ? sm.totals[p][ln][1] : 0u;
        uint32_t iw = tw, io = to;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t x1 = __shfl_up_sync(kFull, iw, o);
            const uint32_t x2 = __shfl_up_sync(kFull, io, o);
            if (ln >= o) {
                iw += x1;
                io += x2;
            }
        }
        const uint32_t PW = __shfl_sync(kFull, iw, 31), MT = __shfl_sync(kFull, io, 31);
        if (ln < kNW) {
            sm.wprefix[p][ln][0] = iw - tw;
            sm.wprefix[p][ln][1] = io - to;
        }
        const uint32_t Rt = PW + 2u * MT;
        const bool publish = (tile != a.stall_tile);

        uint32_t exR = 0, exM = 0;
        if (tile == 0) {
            if (ln == 0 && publish) st_relaxed_gpu(&a.status[0], pack_status(Rt, MT, true));
        } else {
            if (ln == 0 && publish) st_relaxed_gpu(&a.status[tile], pack_status(Rt, MT, false));
            int64_t base = tile - 1;
            uint64_t t0 = 0;
            uint32_t backoff = 32;
            for (;;) {
                const int64_t pi = base - ln;
                const uint64_t v = (pi >= 0) ? ld_relaxed_gpu(&a.status[pi]) : pack_status(0, 0, true);
                const uint32_t incl_mask = __ballot_sync(kFull, (v & kInclBit) != 0);
                const uint32_t none_mask = __ballot_sync(kFull, v == 0);
                const int J = incl_mask ? __ffs(incl_mask) - 1 : 32;
                const uint32_t below = (J == 32) ? kFull : ((1u << J) - 1u);
                if (none_mask & below) {
                    if (t0 == 0) t0 = globaltimer_ns();
                    if (globaltimer_ns() - t0 > a.wait_ns) {  // give up: record and move on
                        if (ln == 0) atomicOr(a.err, kErrTimeout);
                        break;
                    }
                    __nanosleep(backoff);
                    backoff = min(backoff * 2u, 1024u);
                    continue;
                }
                const bool take = (ln <= J);
                const uint32_t vr = take ? (uint32_t)(v & 0xffffffffu) - 1u : 0u;
                const uint32_t vm = take ? (uint32_t)((v >> 32) & 0x7fffffffu) : 0u;
                exR += __reduce_add_sync(kFull, vr);
                exM += __reduce_add_sync(kFull, vm);
                if (J < 32) break;
                base -= 32;
            }
            if (ln == 0 && publish) st_relaxed_gpu(&a.status[tile], pack_status(exR + Rt, exM + MT, true));
        }

        if (ln == 0) {
            sm.info[p][0] = exR;
            sm.info[p][1] = PW;
            sm.info[p][2] = MT;
            sm.info[p][3] = (uint32_t)tile;
            a.status_next[tile] = 0ull;
            const uint64_t io_off = L.index_off + 8ull * (uint64_t)tile;
            if (io_off + 8 <= a.out_cap)
                *reinterpret_cast<uint64_t *>(a.out + io_off) = (uint64_t)exR | ((uint64_t)exM << 32);
            else
                atomicOr(a.err, kErrCapacity);
            if ((uint64_t)tile == L.nc - 1)
                write_header(a, L, sm.bound, (uint64_t)exR + Rt, (uint64_t)exM + MT);
        }
        __syncwarp();
        if (ln == 0) mbar_arrive(&sm.ready[p]);
    }
}

__device__ void producer_warp(EncSmem &sm, const EncodeArgs &a, const Layout &L, int ln) {
    if (ln != 0) return;
    uint32_t issued = 0;  // stages with an outstanding fill
    uint32_t next = atomicAdd(a.counter, 1u);
    uint32_t i = 0;
    for (;; ++i) {
        const int s = i % kS;
        if (i >= kS && !mbar_wait(&sm.empty[s], ((i / kS) - 1) & 1, a.wait_ns, a.err)) break;
        const uint32_t t = next;
        if ((uint64_t)t >= L.nc) {
            sm.tile_id[s] = -1;
            mbar_arrive(&sm.full[s]);
            issued |= 1u << s;
            ++i;
            break;
        }
        next = atomicAdd(a.counter, 1u);  // claim the following tile early
        sm.tile_id[s] = (int32_t)t;
        const uint64_t e0 = (uint64_t)t * kChunk;
        const uint32_t valid = (uint32_t)min((uint64_t)kChunk, a.n - e0);
        const uint32_t bulk = (valid * 4u) & ~15u;
        for (uint32_t j = bulk / 4; j < valid; ++j) sm.in[s][j] = a.in[e0 + j];
        mbar_arrive_expect_tx(&sm.full[s], bulk);
        if (bulk) bulk_g2s(sm.in[s], a.in + e0, bulk, &sm.full[s]);
        issued |= 1u << s;
    }
    // Drain: no copy into this CTA's shared memory may still be in flight at exit.
    for (int s = 0; s < kS; ++s) {
        if (!((issued >> s) & 1u)) continue;
        const uint32_t uses = (i > (uint32_t)s) ? (i - 1 - s) / kS + 1 : 0;  // fills issued on stage s
        if (uses) mbar_wait(&sm.full[s], (uses - 1) & 1, a.wait_ns, a.err);
    }
}

template <int V, int LPB>
__global__ void __launch_bounds__(kThreads, 2) encode_kernel(const EncodeArgs a) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    EncSmem &sm = *reinterpret_cast<EncSmem *>(smem_raw);
    const int warp = threadIdx.x / 32, ln = threadIdx.x % 32;
    const Layout L = stream_layout(a.n, a.block);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kS; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], kNW);
        }
        for (int p = 0; p < 2; ++p) {
            mbar_init(&sm.computed[p], kNW);
            mbar_init(&sm.ready[p], 1);
        }
        mbar_init_fence();
        const float vmin = a.abs_mode ? 0.0f : a.range[0];
        const float vmax = a.abs_mode ? 0.0f : a.range[1];
        sm.bound = resolve_bound(a.abs_mode, a.bound, vmin, vmax);
        if (blockIdx.x == 0) {
            *a.counter_next = 0u;
            *a.err_next = 0u;
        }
    }
    __syncthreads();

    if (warp < kNW)
        compute_warp<V, LPB>(sm, a, L, warp, ln);
    else if (warp == kLookbackWarp)
        lookback_warp(sm, a, L, ln);
    else
        producer_warp(sm, a, L, ln);

    if (L.nc == 0 && blockIdx.x == 0 && threadIdx.x == 0) write_header(a, L, sm.bound, 0, 0);
}

template <int V, int LPB>
cudaError_t launch_t(const EncodeArgs &a, int num_sms, cudaStream_t stream) {
    const size_t smem = sizeof(EncSmem);
    cudaError_t e = cudaFuncSetAttribute(encode_kernel<V, LPB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const Layout L = stream_layout(a.n, a.block);
    const uint64_t want = (uint64_t)num_sms * 2;
    const int grid = (int)(L.nc == 0 ? 1 : (want < L.nc ? want : L.nc));
    encode_kernel<V, LPB><<<grid, kThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_encode(const EncodeArgs &a, int num_sms, cudaStream_t stream) {
    switch (a.block) {
        case 32: return launch_t<4, 8>(a, num_sms, stream);
        case 64: return launch_t<4, 16>(a, num_sms, stream);
        case 128: return launch_t<4, 32>(a, num_sms, stream);
        case 256: return launch_t<8, 32>(a, num_sms, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace eblc
