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
// CTA organisation (384 threads, 2 CTAs per SM, cooperative persistent grid;
// tile t = chunk t of 4096 elements is processed by CTA t mod gridDim.x):
//   warps 0..7   compute: each owns a contiguous 512-element slice of the
//                tile, held as warp-tiles of 32*V elements (V = 8 consecutive
//                elements per lane); a block of B elements spans LPB = B/V
//                lanes.  A warp packs its slice
//                into its own shared-memory ring (sized for typical packed
//                output, not the worst case) and releases the input stage at
//                once; the last warp to finish a tile publishes the tile's
//                aggregate (record words, outliers).  Packed words are copied
//                to their final position once the tile's prefix is known,
//                up to kD - 1 tiles later, so look-back latency overlaps with
//                the compute of later tiles.
//   warps 8..10  look-back and write-out (CTA tile iterations i with
//                i mod 3 = warp - 8): resolve the exclusive prefix of a tile
//                from the predecessors' status words (320 per coalesced L2
//                round trip), publish its inclusive prefix, write the chunk
//                index entry (and the header for the last tile), then copy
//                the compute warps' packed words, the outliers and the width
//                bytes to their final positions.
//   warp 11      producer: streams the CTA's tiles into a 3-stage shared-
//                memory ring with bulk async copies (cp.async.bulk,
//                completion on mbarriers).
// Every wait is bounded (kErrTimeout); every global store is checked against
// the caller's capacity (kErrCapacity).
#include "common.cuh"
#include "kernels.h"
#include "../../include/eblc.h"

namespace eblc {
namespace {

constexpr int kNW = 8;                    // compute warps
constexpr int kS = 3;                     // input stages
constexpr int kD = 8;                     // tile slots: at most kD - 1 tiles computed but not finished
constexpr int kLookbackWarps = 3;
constexpr int kProducerWarp = kNW + kLookbackWarps;
constexpr int kThreads = (kNW + kLookbackWarps + 1) * 32;
constexpr int kWindow = 10;               // look-back rows of 32 status words per round trip
constexpr uint32_t kRing = 1536;          // packed words a compute warp can hold (3 worst-case tiles)
constexpr uint32_t kWarpMax = kChunk / kNW;  // most words a warp packs for one tile
static_assert(kRing >= 3 * kWarpMax, "one pending part must always leave room for the next");
constexpr uint32_t kFull = 0xffffffffu;
constexpr uint64_t kInclBit = 1ull << 63;

struct __align__(128) EncSmem {
    float in[kS][kChunk];                 // input ring (bulk-copy destination)
    uint32_t ring[kNW][kRing];            // per compute warp: packed words awaiting their prefix
    uint32_t omask[kD][kNW][32];          // per slot, warp, lane: outlier bits
    uint8_t width[kD][kChunk / 32];       // per slot: width bytes of the tile's blocks
    uint32_t totals[kD][kNW][2];          // per slot, warp: payload words, outliers
    uint32_t ringpos[kD][kNW];            // per slot, warp: ring offset of the packed words
    int32_t slot_tile[kD];                // tile of the slot, -1 once the CTA has no more tiles
    uint32_t done[kD];                    // CTA iteration + 1 once the slot's tile is written out
    unsigned long long agg[kD];           // tile aggregate being summed: payload words | outliers << 32
    uint32_t agg_count[kD];               // compute warps that have added to agg
    int32_t tile_id[kS];
    uint64_t full[kS], empty[kS], computed[kD];
    uint64_t *st_cur, *st_next;           // this call's look-back words, the other array
    uint64_t written[kD];                 // completes once per use of the slot: its tile is written out
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
// lanes) into the block's words at `dst` (shared memory, already zeroed):
// code j of the block occupies bits [j*w, j*w + w), least significant bit
// first.  Lane r of the group owns bits [r*V*w, (r+1)*V*w): it assembles
// them in registers (NW words hold V*w bits for every width in the warp),
// shifts them to their word alignment and ORs them in.  Neighbouring lanes
// that share a word both OR into it, so no lane needs another lane's bits.
template <int V, int NW>
__device__ __forceinline__ void pack_lane(const uint32_t (&z)[V], uint32_t w, int r, uint32_t *dst) {
    uint32_t S[NW + 1];
    S[0] = z[V - 1];
#pragma unroll
    for (int j = 1; j <= NW; ++j) S[j] = 0u;
#pragma unroll
    for (int v = V - 2; v >= 0; --v) {
#pragma unroll
        for (int j = (V - 1 - v < NW - 1 ? V - 1 - v : NW - 1); j >= 1; --j)
            S[j] = __funnelshift_lc(S[j - 1], S[j], w);
        S[0] = __funnelshift_lc(0u, S[0], w) | z[v];
    }
    const uint32_t P = (uint32_t)r * V * w;  // bit offset of the segment in the block
    const uint32_t s = P & 31u;
#pragma unroll
    for (int j = NW; j >= 1; --j) S[j] = __funnelshift_lc(S[j - 1], S[j], s);
    S[0] <<= s;
    const uint32_t nw = (s + V * w + 31u) >> 5;
    uint32_t *d = dst + (P >> 5);
#pragma unroll
    for (int j = 0; j <= NW; ++j)
        if ((uint32_t)j < nw) atomicOr(d + j, S[j]);
}

// Quantize, test, delta, zigzag and pack this warp's slice of the tile in
// input stage s; packed words go to `out` (this warp's ring, room for
// kWarpMax words), width bytes to slot q.
template <int V, int LPB>
__device__ __forceinline__ void compute_tile(EncSmem &sm, const Bound &bd, int s, int q, uint32_t valid, int cw,
                                             int ln, uint32_t *out, uint32_t &words_out, uint32_t &omask_out) {
    constexpr int kB = V * LPB;
    constexpr int kWT = 32 * V;
    constexpr int kWPW = kChunk / kWT / kNW;
    constexpr int kGroups = 32 / LPB;
    const int g = ln / LPB, r = ln % LPB;
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

        int32_t q_[V];
        bool flagged = false;  // some element is not certainly within the bound
#pragma unroll
        for (int v = 0; v < V; ++v) {
            const float y = __fmul_rn(x[v], bd.inv2eb);
            const int32_t qq = (fabsf(y) < 0x1p30f) ? __float2int_rn(y) : 0;
            const float xr = __fmul_rn(__int2float_rn(qq), bd.step);
            flagged |= !(fabsf(__fsub_rn(x[v], xr)) <= bd.t_in);
            q_[v] = qq;
        }
        uint32_t vm = (1u << V) - 1u;  // elements of this lane that exist
        if (valid < kChunk) {  // ragged last tile: elements at or beyond `valid` do not exist
            const uint32_t have = (e0 >= valid) ? 0u : min(valid - e0, (uint32_t)V);
            vm = (1u << have) - 1u;
#pragma unroll
            for (int v = 0; v < V; ++v)
                if (!((vm >> v) & 1u)) q_[v] = 0;
        }
        uint32_t obits = 0;
        if (__any_sync(kFull, flagged)) {
            // Outlier test proper: certainly out beyond t_out, fp64 test in the
            // band between the fp32 filter thresholds (and for NaN).
#pragma unroll
            for (int v = 0; v < V; ++v) {
                const float xr = __fmul_rn(__int2float_rn(q_[v]), bd.step);
                const float d = fabsf(__fsub_rn(x[v], xr));
                bool out = d > bd.t_out;
                if (!out && !(d <= bd.t_in)) {
                    const bool finite = fabsf(x[v]) < __int_as_float(0x7f800000);
                    out = !finite || !(fabs(__dsub_rn((double)x[v], (double)xr)) <= bd.eb);
                }
                obits |= (uint32_t)out << v;
            }
            obits &= vm;
        }

        int32_t pv = __shfl_up_sync(kFull, q_[V - 1], 1);
        if (r == 0) pv = 0;  // Lorenzo predecessor resets at the block start
        uint32_t z[V];
        uint32_t orz = 0;
#pragma unroll
        for (int v = 0; v < V; ++v) {
            const int32_t d = q_[v] - (v ? q_[v - 1] : pv);
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
        if (r == 0) sm.width[q][blk] = (uint8_t)w;
        uint32_t *o = out + wo;
        for (uint32_t j = ln; j < tot; j += 32) o[j] = 0u;
        __syncwarp();
        const uint32_t wmax = __reduce_max_sync(kFull, w);
        if (w != 0u) {
            if (wmax * V <= 32u)
                pack_lane<V, 1>(z, w, r, o + pre);
            else if (wmax * V <= 96u)
                pack_lane<V, 3>(z, w, r, o + pre);
            else
                pack_lane<V, V>(z, w, r, o + pre);
        }
        __syncwarp();
        wo += tot;
        omask |= obits << (k * V);
    }
    words_out = wo;
    omask_out = omask;
}

__device__ __forceinline__ bool slot_done(const EncSmem &sm, uint32_t it) {
    return *reinterpret_cast<const volatile uint32_t *>(&sm.done[it % kD]) == it + 1;
}

template <int V, int LPB>
__device__ void compute_warp(EncSmem &sm, const EncodeArgs &a, int cw, int ln) {
    const Bound bd = sm.bound;
    uint32_t *ring = sm.ring[cw];
    uint32_t oldest = 0;  // oldest CTA iteration whose packed words still occupy this warp's ring
    uint32_t head = 0;    // ring offset after the newest tile's words
    uint32_t i = 0;
    for (;; ++i) {
        // Reclaim ring space of tiles already written out, then find room for a
        // worst-case tile: a free slot and kWarpMax contiguous ring words.
        uint32_t start = 0;
        for (;;) {
            while (oldest < i && slot_done(sm, oldest)) ++oldest;
            if (i - oldest <= (uint32_t)kD - 2) {
                if (oldest == i) {
                    start = 0;
                    break;
                }
                // Pending words occupy [tail, head), wrapped when head < tail.  A
                // slice never ends exactly at tail, so head == tail means that no
                // pending word is in the ring.
                const uint32_t tail = sm.ringpos[oldest % kD][cw];
                if (head >= tail) {
                    if (head + kWarpMax <= kRing) { start = head; break; }
                    if (kWarpMax < tail) { start = 0; break; }
                } else if (head + kWarpMax < tail) {
                    start = head;
                    break;
                }
            }
            // No room: sleep on the oldest pending tile's write-out (oldest < i here).
            if (!mbar_wait(&sm.written[oldest % kD], (oldest / kD) & 1, a.wait_ns, a.err)) return;
        }
        const int s = i % kS, q = i % kD;
        if (!mbar_wait(&sm.full[s], (i / kS) & 1, a.wait_ns, a.err)) return;
        const int tile = sm.tile_id[s];
        if (tile < 0) break;
        const uint64_t e0 = (uint64_t)tile * kChunk;
        const uint32_t valid = (uint32_t)min((uint64_t)kChunk, a.n - e0);
        uint32_t words, omask;
        compute_tile<V, LPB>(sm, bd, s, q, valid, cw, ln, ring + start, words, omask);
        const uint32_t outl = __reduce_add_sync(kFull, __popc(omask));
        sm.omask[q][cw][ln] = omask;
        __syncwarp();
        if (ln == 0) {
            mbar_arrive(&sm.empty[s]);  // the input stage is free again
            sm.totals[q][cw][0] = words;
            sm.totals[q][cw][1] = outl;
            sm.ringpos[q][cw] = start;
            if (cw == 0) sm.slot_tile[q] = tile;
            // The last warp to finish the tile publishes its aggregate at once, so
            // successors' look-backs never wait for this CTA's look-back warps.
            atomicAdd(&sm.agg[q], (unsigned long long)words | ((unsigned long long)outl << 32));
            __threadfence_block();
            if (atomicAdd(&sm.agg_count[q], 1u) == kNW - 1) {
                __threadfence_block();
                const unsigned long long t = atomicExch(&sm.agg[q], 0ull);
                sm.agg_count[q] = 0;
                const uint32_t PW = (uint32_t)t, MT = (uint32_t)(t >> 32);
                if (tile != a.stall_tile)
                    st_relaxed_gpu(&sm.st_cur[tile], pack_status(PW + 2u * MT, MT, tile == 0));
            }
            mbar_arrive(&sm.computed[q]);
        }
        head = start + words;
    }
    // Tell the look-back warps that this CTA has no more tiles: iterations
    // i .. i + kLookbackWarps - 1 get tile -1.  Their slots must be free of
    // pending tiles first.
    while (i - oldest > (uint32_t)(kD - kLookbackWarps)) {
        if (!slot_done(sm, oldest) &&
            !mbar_wait(&sm.written[oldest % kD], (oldest / kD) & 1, a.wait_ns, a.err))
            return;
        ++oldest;
    }
    if (ln == 0) {
        if (cw == 0)
            for (int j = 0; j < kLookbackWarps; ++j) sm.slot_tile[(i + j) % kD] = -1;
        __threadfence_block();
        for (int j = 0; j < kLookbackWarps; ++j) mbar_arrive(&sm.computed[(i + j) % kD]);
    }
}

// Write the tile of CTA iteration `it` (slot q) to its final position once
// its prefix (record word offset rec, payload words PW, outliers MT) is
// known: every compute warp's packed words from its ring, the outliers
// (indices then values after the tile's payload; values read back from the
// input array) and the width bytes.  Lane c < kNW of this warp holds compute
// warp c's exclusive prefix (words wpw, outliers wpo) within the tile.
template <int V, int LPB>
__device__ __forceinline__ void write_tile(EncSmem &sm, const EncodeArgs &a, const Layout &L, int q, int tile,
                                           uint32_t rec, uint32_t PW, uint32_t MT, uint32_t wpw, uint32_t wpo,
                                           int ln) {
    constexpr int kB = V * LPB;
    constexpr int kWT = 32 * V;
    constexpr int kWPW = kChunk / kWT / kNW;
    uint32_t *recs = reinterpret_cast<uint32_t *>(a.out + L.record_off);
    const uint64_t cap_words = (a.out_cap > L.record_off) ? (a.out_cap - L.record_off) / 4 : 0;
    bool over = false;
    const float *xin = a.in + (uint64_t)tile * kChunk;
#pragma unroll 1
    for (int c = 0; c < kNW; ++c) {
        const uint32_t words = sm.totals[q][c][0], pos = sm.ringpos[q][c], mc = sm.totals[q][c][1];
        const uint64_t w0 = (uint64_t)rec + __shfl_sync(kFull, wpw, c);
        const uint32_t *src = sm.ring[c] + pos;
        uint32_t *dst = recs + w0;
        // words that fit in the caller's capacity (all of them unless it is too small)
        const uint32_t lim = (w0 >= cap_words) ? 0u : (uint32_t)min((uint64_t)words, cap_words - w0);
        over |= lim < words;
        for (uint32_t j = ln; j < lim; j += 32) st_cs_u32(dst + j, src[j]);
        const uint32_t obase = __shfl_sync(kFull, wpo, c);
        if (mc != 0u) {
            const uint32_t omask = sm.omask[q][c][ln];
            uint32_t ord_base = 0;
#pragma unroll 1
            for (int k = 0; k < kWPW; ++k) {
                uint32_t bits = (omask >> (k * V)) & ((1u << V) - 1u);
                const uint32_t cnt = __popc(bits);
                uint32_t incl = cnt;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const uint32_t t = __shfl_up_sync(kFull, incl, o);
                    if (ln >= o) incl += t;
                }
                uint32_t ord = ord_base + incl - cnt;
                while (bits) {
                    const int v = __ffs(bits) - 1;
                    bits &= bits - 1u;
                    const uint32_t e = (uint32_t)(c * kWPW + k) * kWT + ln * V + v;
                    const uint64_t pi = (uint64_t)rec + PW + obase + ord;
                    const uint64_t pv = pi + MT;
                    if (pv < cap_words) {
                        recs[pi] = (uint32_t)tile * kChunk + e;
                        recs[pv] = __float_as_uint(__ldg(xin + e));
                    } else {
                        over = true;
                    }
                    ++ord;
                }
                ord_base += __shfl_sync(kFull, incl, 31);
            }
        }
    }
    {  // width bytes of the tile's blocks, zeros past the last block up to the 16-byte pad
        constexpr uint32_t K = kChunk / kB;
        const uint64_t b0 = (uint64_t)tile * K;
        const uint64_t bend = min(b0 + K, pad16(L.nb));
        const uint32_t nwords = (uint32_t)((bend - b0) / 4);
        const uint32_t *ws = reinterpret_cast<const uint32_t *>(sm.width[q]);
        uint32_t *wd = reinterpret_cast<uint32_t *>(a.out + L.width_off + b0);
        const uint64_t room = (a.out_cap > L.width_off + b0) ? (a.out_cap - L.width_off - b0) / 4 : 0;
        const uint32_t nw = (uint32_t)min((uint64_t)nwords, room);
        over |= nw < nwords;
        for (uint32_t j = ln; j < nw; j += 32) wd[j] = ws[j];
    }
    if (__any_sync(kFull, over) && ln == 0) atomicOr(a.err, kErrCapacity);
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

// Exclusive prefix (record words, outliers) of `tile` from its predecessors'
// status words, nearest first, stopping at the nearest inclusive prefix.
// Tile `stop` (-1 before tile 0) is known to have the inclusive prefix
// `known` (status word form), so no status word at or below it is read.  One
// L2 round trip reads kWindow rows of 32 consecutive status words (row j,
// lane l: predecessor tile - 1 - 32 j - l), coalesced.  Every tile between
// the inclusive prefix found and `tile` must have published at least its
// aggregate: polls the nearest missing one with back-off (bounded by
// wait_ns, and given up at once when another wait of the launch has timed
// out), then reads the window again.
__device__ __forceinline__ void look_back(const EncodeArgs &a, const uint64_t *status, int tile, int stop,
                                          uint64_t known, int ln, uint32_t &exR, uint32_t &exM) {
    exR = 0;
    exM = 0;
    int base = tile - 1;  // nearest predecessor not yet summed
    uint64_t t0 = 0;
    uint32_t backoff = 32;
    while (base > stop - 1) {
        uint64_t v[kWindow];
#pragma unroll
        for (int j = 0; j < kWindow; ++j) {
            const int p = base - 32 * j - ln;
            v[j] = (p > stop) ? ld_relaxed_gpu(&status[p]) : (p == stop ? known : pack_status(0, 0, true));
        }
        uint32_t sr = 0, sm_ = 0;
        int found = 0, miss_row = -1;
        uint32_t miss_lanes = 0;
#pragma unroll
        for (int j = 0; j < kWindow; ++j) {
            const uint32_t inc = __ballot_sync(kFull, (v[j] & kInclBit) != 0ull);
            const uint32_t mis = __ballot_sync(kFull, v[j] == 0ull);
            if (!found && miss_row < 0) {
                const uint32_t upto = inc ? (inc ^ (inc - 1u)) : kFull;  // lanes through the first inclusive
                if (mis & upto) {
                    miss_row = j;
                    miss_lanes = mis & upto;
                } else {
                    if ((upto >> ln) & 1u) {
                        sr += (uint32_t)(v[j] & 0xffffffffu) - 1u;
                        sm_ += (uint32_t)((v[j] >> 32) & 0x7fffffffu);
                    }
                    found = inc != 0u;
                }
            }
        }
        if (miss_row >= 0) {
            const uint64_t *w = &status[base - 32 * miss_row - (__ffs(miss_lanes) - 1)];
            if (t0 == 0) t0 = globaltimer_ns();
            while (ld_relaxed_gpu(w) == 0) {
                if (globaltimer_ns() - t0 > a.wait_ns ||
                    (*reinterpret_cast<volatile uint32_t *>(a.err) & kErrTimeout)) {  // give up: record, move on
                    if (ln == 0) atomicOr(a.err, kErrTimeout);
                    return;
                }
                __nanosleep(backoff);
                backoff = min(backoff * 2u, 512u);
            }
            __syncwarp();
            continue;
        }
        exR += __reduce_add_sync(kFull, sr);
        exM += __reduce_add_sync(kFull, sm_);
        if (found) return;
        base -= 32 * kWindow;
    }
}

template <int V, int LPB>
__device__ void lookback_warp(EncSmem &sm, const EncodeArgs &a, const Layout &L, int lw, int ln) {
    for (uint32_t i = lw;; i += kLookbackWarps) {
        const int q = i % kD;
        if (!mbar_wait(&sm.computed[q], (i / kD) & 1, a.wait_ns, a.err)) return;
        const int tile = sm.slot_tile[q];
        if (tile < 0) break;

        const uint32_t tw = (ln < kNW) ? sm.totals[q][ln][0] : 0u;
        const uint32_t to = (ln < kNW) ? sm.totals[q][ln][1] : 0u;
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
        const uint32_t Rt = PW + 2u * MT;
        const bool publish = (tile != a.stall_tile);

        uint32_t exR = 0, exM = 0;
        if (tile != 0) {  // the aggregate is already published by the compute warps
            // Start once this CTA has also computed its next tile: by then the
            // other CTAs have almost always published this tile's predecessors
            // of the same wave, so the look-back rarely has to wait.  This wait
            // cannot close a cycle: a compute warp at iteration i + 1 never
            // needs tile i written out, because with a single pending part of
            // at most kWarpMax words a ring of 3 * kWarpMax words always has
            // kWarpMax contiguous free words.
            if (!mbar_wait(&sm.computed[(i + 1) % kD], ((i + 1) / kD) & 1, a.wait_ns, a.err)) return;
            look_back(a, sm.st_cur, tile, -1, pack_status(0, 0, true), ln, exR, exM);
            if (ln == 0 && publish) st_relaxed_gpu(&sm.st_cur[tile], pack_status(exR + Rt, exM + MT, true));
        }
        if (ln == 0) {
            sm.st_next[tile] = 0ull;
            const uint64_t io_off = L.index_off + 8ull * (uint64_t)tile;
            if (io_off + 8 <= a.out_cap)
                *reinterpret_cast<uint64_t *>(a.out + io_off) = (uint64_t)exR | ((uint64_t)exM << 32);
            else
                atomicOr(a.err, kErrCapacity);
            if ((uint64_t)tile == L.nc - 1)
                write_header(a, L, sm.bound, (uint64_t)exR + Rt, (uint64_t)exM + MT);
        }
        write_tile<V, LPB>(sm, a, L, q, tile, exR, PW, MT, iw - tw, io - to, ln);
        __syncwarp();
        if (ln == 0) {
            __threadfence_block();
            *reinterpret_cast<volatile uint32_t *>(&sm.done[q]) = i + 1;
            mbar_arrive(&sm.written[q]);
        }
    }
}

// Tile t is processed by CTA t mod gridDim.x, in increasing t.  The grid is
// launched cooperatively (all CTAs resident at once), so every tile a
// look-back waits for belongs to a running CTA that reaches it without
// waiting on anything later: the look-back cannot deadlock.
__device__ void producer_warp(EncSmem &sm, const EncodeArgs &a, const Layout &L, int ln) {
    if (ln != 0) return;
    uint32_t i = 0;
    for (;; ++i) {
        const int s = i % kS;
        if (i >= kS && !mbar_wait(&sm.empty[s], ((i / kS) - 1) & 1, a.wait_ns, a.err)) break;
        const uint64_t t = (uint64_t)blockIdx.x + (uint64_t)i * gridDim.x;
        if (t >= L.nc) {
            sm.tile_id[s] = -1;
            mbar_arrive(&sm.full[s]);
            ++i;
            break;
        }
        sm.tile_id[s] = (int32_t)t;
        const uint64_t e0 = t * kChunk;
        const uint32_t valid = (uint32_t)min((uint64_t)kChunk, a.n - e0);
        const uint32_t bulk = (valid * 4u) & ~15u;
        for (uint32_t j = bulk / 4; j < valid; ++j) sm.in[s][j] = a.in[e0 + j];
        mbar_arrive_expect_tx(&sm.full[s], bulk);
        if (bulk) bulk_g2s(sm.in[s], a.in + e0, bulk, &sm.full[s]);
    }
    // Drain: no copy into this CTA's shared memory may still be in flight at exit.
    for (int s = 0; s < kS; ++s) {
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
        for (int q = 0; q < kD; ++q) {
            mbar_init(&sm.computed[q], kNW);
            mbar_init(&sm.written[q], 1);
            sm.done[q] = 0u;
            sm.agg[q] = 0ull;
            sm.agg_count[q] = 0u;
        }
        mbar_init_fence();
        const float vmin = a.abs_mode ? 0.0f : a.range[0];
        const float vmax = a.abs_mode ? 0.0f : a.range[1];
        sm.bound = resolve_bound(a.abs_mode, a.bound, vmin, vmax);
        const uint64_t par = *a.epoch & 1u;
        sm.st_cur = a.status + par * a.ntiles;
        sm.st_next = a.status + (par ^ 1u) * a.ntiles;
    }
    __syncthreads();

    if (warp < kNW)
        compute_warp<V, LPB>(sm, a, warp, ln);
    else if (warp < kProducerWarp)
        lookback_warp<V, LPB>(sm, a, L, warp - kNW, ln);
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
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, encode_kernel<V, LPB>, kThreads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const Layout L = stream_layout(a.n, a.block);
    const uint64_t resident = (uint64_t)per_sm * (uint64_t)num_sms;
    const int grid = (int)(L.nc == 0 ? 1 : (resident < L.nc ? resident : L.nc));
    EncodeArgs args = a;
    void *params[] = {&args};
    return cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(encode_kernel<V, LPB>), dim3(grid),
                                       dim3(kThreads), params, smem, stream);
}

constexpr int kFinishThreads = 256;

__global__ void __launch_bounds__(kFinishThreads) finish_kernel(const FinishArgs f) {
    const uint32_t err = *f.err;
    if (err != 0u)
        for (uint64_t j = threadIdx.x; j < f.status_words; j += kFinishThreads) f.status[j] = 0ull;
    __syncthreads();  // every thread has read err before thread 0 clears it
    if (threadIdx.x != 0) return;
    f.result[7] = err;
    *f.err = 0u;
    *f.epoch += 1u;
    if (f.user) {
        const uint32_t status = (err & kErrTimeout)    ? (uint32_t)EBLC_TIMEOUT
                                : (err & kErrCapacity) ? (uint32_t)EBLC_CAPACITY
                                : (err & kErrCorrupt)  ? (uint32_t)EBLC_CORRUPT
                                                       : (uint32_t)EBLC_OK;
        f.user[0] = f.result[2];  // stream bytes
        f.user[1] = f.result[0];  // payload words
        f.user[2] = f.result[1];  // outliers
        f.user[3] = status;
    }
}

}  // namespace

cudaError_t launch_finish(const FinishArgs &f, cudaStream_t stream) {
    finish_kernel<<<1, kFinishThreads, 0, stream>>>(f);
    return cudaGetLastError();
}

cudaError_t launch_encode(const EncodeArgs &a, int num_sms, cudaStream_t stream) {
    switch (a.block) {
        case 32: return launch_t<8, 4>(a, num_sms, stream);
        case 64: return launch_t<8, 8>(a, num_sms, stream);
        case 128: return launch_t<8, 16>(a, num_sms, stream);
        case 256: return launch_t<8, 32>(a, num_sms, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace eblc
