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
#ifndef EBLC_ENC_SLOTS
#define EBLC_ENC_SLOTS 12
#endif
constexpr int kD = EBLC_ENC_SLOTS;        // tile slots: at most kD - 1 tiles computed but not finished
#ifndef EBLC_ENC_LB
#define EBLC_ENC_LB 3
#endif
constexpr int kLookbackWarps = EBLC_ENC_LB;  // look-back and write-out warps
constexpr int kProducerWarp = kNW + kLookbackWarps;
constexpr int kThreads = (kNW + kLookbackWarps + 1) * 32;
constexpr int kWindow = 10;               // look-back rows of 32 status words per round trip
constexpr uint32_t kRing = 1760;          // packed words a compute warp can hold (the rest of the CTA's shared memory)
constexpr uint32_t kWarpMax = kChunk / kNW;  // most words a warp packs for one tile
// A compute warp short of ring room waits only for the write-out of its own
// earlier tiles, whose look-backs wait only for lower tiles: no cycle.  The
// ring holds several typical tiles per warp so the compute warps can run
// ahead of the look-back (kRing >= 2 kWarpMax lets a worst-case tile follow a
// pending one without waiting).  A warp starts a tile only with kWarpMax
// contiguous free words, so the ring's size sets how many wide tiles can
// wait for their write-out; it takes what two CTAs per SM leave after the
// input stages and the 12 slots' bookkeeping.
static_assert(kRing >= 2 * kWarpMax, "a worst-case part must fit beside a pending one");
constexpr uint32_t kFull = 0xffffffffu;
constexpr uint64_t kInclBit = 1ull << 63;

struct __align__(128) EncSmem {
    float in[kS][kChunk];                 // input ring (bulk-copy destination)
    uint32_t ring[kNW][kRing];            // per compute warp: packed words awaiting their prefix
    uint16_t omask[kD][kNW][32];          // per slot, warp, lane: outlier bits (2 warp-tiles x 8);
                                          // for 2-D / 3-D bricks the slot's 4096-bit C-order bitmap
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

// Two CTAs per SM: 228 KB of shared memory per SM, 1 KB of it reserved per CTA.
static_assert(sizeof(EncSmem) <= 233472 / 2 - 1024, "two encoder CTAs must fit on an SM");

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

// ---------------------------------------------------------------------------
// Fast path for full tiles (all 4096 elements present, so every block holds
// B elements): V = 8 consecutive elements per lane, so a lane's 8 codes form
// one 8w-bit segment that starts at bit r*8w of its block (r = lane within
// the block), a multiple of 8.  Every output word is written by exactly one
// lane with a plain store: the lane whose segment ends in a word that the
// next lane's segment continues hands its part of that word to the next lane
// (one shuffle), and the next lane writes the whole word.  For w >= 2 at most
// two lanes share a word; w = 1 (four 8-bit segments per word) is combined
// within each quad of lanes first.

// Shift the lane's segment (NG words, least significant first) left by s
// bits (s = 0, 8, 16, 24) into NG + 1 words.
template <int NG>
__device__ __forceinline__ void shift_segment(const uint32_t (&G)[NG], uint32_t s, uint32_t (&W)[NG + 1]) {
    W[0] = G[0] << s;
#pragma unroll
    for (int j = 1; j < NG; ++j) W[j] = __funnelshift_l(G[j - 1], G[j], s);
    W[NG] = __funnelshift_l(G[NG - 1], 0u, s);
}

// Write the lane's words W[0..NW) (already shifted by s, the segment's bit
// offset within its first word) to dst[0..): words the lane owns are stored,
// the partial last word goes to the next lane.  E = s + 8w is the bit offset
// of the segment's end from dst[0].
template <int NW>
__device__ __forceinline__ void emit_segment(uint32_t (&W)[NW], uint32_t s, uint32_t w, uint32_t *dst) {
    const uint32_t E = s + 8u * w;
    const uint32_t own = E >> 5;  // words that end inside this lane's segment
    uint32_t last = W[0];         // the word holding the segment's end (partial when E % 32 != 0)
#pragma unroll
    for (int j = 1; j < NW; ++j)
        if ((uint32_t)j == own) last = W[j];
    const uint32_t prev = __shfl_up_sync(kFull, last, 1);
    if (s != 0u) W[0] |= prev;  // s != 0 never happens for the first lane of a block
    if (__any_sync(kFull, w == 1u)) {
        // 8-bit segments: a word holds the segments of a whole quad of lanes.
        uint32_t v = W[0];
        v |= __shfl_xor_sync(kFull, v, 1);
        v |= __shfl_xor_sync(kFull, v, 2);
        if (w == 1u) W[0] = v;
    }
    // own <= NW - 1 (E <= 24 + 8w and NW words span it), so the top word is
    // never whole: at most words 0 .. NW - 2 are stored here.
#pragma unroll
    for (int j = 0; j < NW - 1; ++j)
        if ((uint32_t)j < own) dst[j] = W[j];
}

// Segment of 8 codes of width w <= 8 (at most 64 bits) in two words.
__device__ __forceinline__ void segment64(const uint32_t (&z)[8], uint32_t w, uint32_t (&G)[2]) {
    const uint32_t pw = 1u << w, pw2 = pw * pw;
    const uint32_t u0 = (z[0] + z[1] * pw) + (z[2] + z[3] * pw) * pw2;  // 4w <= 32 bits
    const uint32_t u1 = (z[4] + z[5] * pw) + (z[6] + z[7] * pw) * pw2;
    const uint64_t g = (uint64_t)u0 | ((uint64_t)u1 << (4u * w));
    G[0] = (uint32_t)g;
    G[1] = (uint32_t)(g >> 32);
}

// Segment of 8 codes of width w <= 16 (at most 128 bits) in four words.
__device__ __forceinline__ void segment128(const uint32_t (&z)[8], uint32_t w, uint32_t (&G)[4]) {
    const uint32_t pw = 1u << w;
    const uint32_t p0 = z[0] + z[1] * pw, p1 = z[2] + z[3] * pw;  // 2w <= 32 bits
    const uint32_t p2 = z[4] + z[5] * pw, p3 = z[6] + z[7] * pw;
    const uint64_t u0 = (uint64_t)p0 | ((uint64_t)p1 << (2u * w));  // 4w <= 64 bits
    const uint64_t u1 = (uint64_t)p2 | ((uint64_t)p3 << (2u * w));
    // u1 << 4w into three words, in two clamped funnel shifts of a + b = 4w bits
    const uint32_t a = min(4u * w, 32u), b = 4u * w - a;
    const uint32_t l1 = (uint32_t)u1, h1 = (uint32_t)(u1 >> 32);
    const uint32_t A0 = __funnelshift_lc(0u, l1, a), A1 = __funnelshift_lc(l1, h1, a);
    const uint32_t A2 = __funnelshift_lc(h1, 0u, a);
    G[0] = (uint32_t)u0 | __funnelshift_lc(0u, A0, b);
    G[1] = (uint32_t)(u0 >> 32) | __funnelshift_lc(A0, A1, b);
    G[2] = __funnelshift_lc(A1, A2, b);
    G[3] = __funnelshift_lc(A2, 0u, b);
}

// Segment of 8 codes of width w <= 32 (at most 256 bits) in eight words:
// Horner over the codes from the top one down.
__device__ __forceinline__ void segment256(const uint32_t (&z)[8], uint32_t w, uint32_t (&G)[8]) {
    G[0] = z[7];
#pragma unroll
    for (int j = 1; j < 8; ++j) G[j] = 0u;
#pragma unroll
    for (int v = 6; v >= 0; --v) {
#pragma unroll
        for (int j = (7 - v < 7 ? 7 - v : 7); j >= 1; --j) G[j] = __funnelshift_lc(G[j - 1], G[j], w);
        G[0] = __funnelshift_lc(0u, G[0], w) | z[v];
    }
}

// Group width and the exclusive prefix / total of the group words within
// one warp-tile (units of w: a full block of width w holds kB * w / 32
// words), plus the width bytes of the warp-tile's blocks written to wb.
template <int LPB>
__device__ __forceinline__ void group_prefix(uint32_t w, int g, int r, int ln, uint8_t *wb, uint32_t &pre_w,
                                             uint32_t &tot_w) {
    if constexpr (LPB == 32) {
        pre_w = 0;
        tot_w = w;
        if (ln == 0) wb[0] = (uint8_t)w;
    } else if constexpr (LPB == 16) {
        const uint32_t o = __shfl_xor_sync(kFull, w, 16);
        pre_w = g ? o : 0u;
        tot_w = w + o;
        if (ln == 0) *reinterpret_cast<uint16_t *>(wb) = (uint16_t)(w | (o << 8));
    } else if constexpr (LPB == 8) {
        // one byte per block: sums of up to four widths (<= 128) stay in a byte
        const uint32_t W4 = __reduce_or_sync(kFull, r == 0 ? w << (8 * g) : 0u);
        pre_w = ((W4 * 0x01010100u) >> (8 * g)) & 0xffu;
        tot_w = (W4 * 0x01010101u) >> 24;
        if (ln == 0) *reinterpret_cast<uint32_t *>(wb) = W4;
    } else {  // LPB == 4: eight blocks, widths of blocks 0-3 and 4-7 in two words
        const uint32_t lo = __reduce_or_sync(kFull, (r == 0 && g < 4) ? w << (8 * g) : 0u);
        const uint32_t hi = __reduce_or_sync(kFull, (r == 0 && g >= 4) ? w << (8 * (g - 4)) : 0u);
        const uint32_t tlo = (lo * 0x01010101u) >> 24;
        const uint32_t wd = (g < 4) ? lo : hi;
        pre_w = ((wd * 0x01010100u) >> (8 * (g & 3))) & 0xffu;
        if (g >= 4) pre_w += tlo;
        tot_w = tlo + ((hi * 0x01010101u) >> 24);
        if (ln == 0) *reinterpret_cast<uint2 *>(wb) = make_uint2(lo, hi);
    }
}

// Quantize 8 elements (q = rint(x * inv2eb) when |x * inv2eb| < 2^30, else 0)
// and set obits (bit v: element v is an outlier: non-finite, or |x - x'| >
// eb in fp64).  The fp32 filter decides almost every element; a warp with any
// element in the band between the thresholds (or a NaN, or an out-of-range y
// when kCheckRange) takes the exact path for all its lanes.
template <bool kCheckRange>
__device__ __forceinline__ void quantize8(const float (&x)[8], const Bound &bd, int32_t (&q)[8], uint32_t &obits) {
    bool flagged = false;  // some element is not certainly within the bound (or out of range)
#pragma unroll
    for (int v = 0; v < 8; ++v) {
        const float y = __fmul_rn(x[v], bd.inv2eb);
        const int32_t qq = __float2int_rn(y);
        const float xr = __fmul_rn(__int2float_rn(qq), bd.step);
        flagged |= !(fabsf(__fsub_rn(x[v], xr)) <= bd.t_in);
        if (kCheckRange) flagged |= !(fabsf(y) < 0x1p30f);
        q[v] = qq;
    }
    obits = 0;
    if (__any_sync(kFull, flagged)) {
        // Rare: redo the quantizer with its range rule and take the outlier
        // test proper (fp64 in the band between the filter thresholds).
#pragma unroll
        for (int v = 0; v < 8; ++v) {
            const float y = __fmul_rn(x[v], bd.inv2eb);
            const int32_t qq = (fabsf(y) < 0x1p30f) ? __float2int_rn(y) : 0;
            const float xr = __fmul_rn(__int2float_rn(qq), bd.step);
            const float d = fabsf(__fsub_rn(x[v], xr));
            bool o = d > bd.t_out;
            if (!o && !(d <= bd.t_in)) {
                const bool finite = fabsf(x[v]) < __int_as_float(0x7f800000);
                o = !finite || !(fabs(__dsub_rn((double)x[v], (double)xr)) <= bd.eb);
            }
            obits |= (uint32_t)o << v;
            q[v] = qq;
        }
    }
}

__device__ __forceinline__ uint32_t zigzag(int32_t d) { return ((uint32_t)d << 1) ^ (uint32_t)(d >> 31); }

// Block widths, their width bytes (at wb) and the bit packing of one
// warp-tile's zigzag codes (8 per lane, in block order; a block of 8 * LPB
// codes spans LPB lanes) into out, the warp-tile's first payload word.
// Returns the warp-tile's payload words.
template <int LPB>
__device__ __forceinline__ uint32_t pack_warp_tile(const uint32_t (&z)[8], int g, int r, int ln, uint8_t *wb,
                                                   uint32_t *out) {
    constexpr uint32_t kWordsPerW = 8 * LPB / 32;  // words of a full block per unit of width
    uint32_t orz = 0;
#pragma unroll
    for (int v = 0; v < 8; ++v) orz |= z[v];
    const uint32_t w = 32u - __clz(group_or<LPB>(orz, g));
    uint32_t pre_w, tot_w;
    group_prefix<LPB>(w, g, r, ln, wb, pre_w, tot_w);
    // this lane's segment starts at bit r*8w of its block: word (r*w)/4, bit 8*((r*w)%4)
    const uint32_t rw = (uint32_t)r * w;
    uint32_t *dst = out + kWordsPerW * pre_w + (rw >> 2);
    const uint32_t sh = (rw & 3u) << 3;
    const uint32_t wmax = __reduce_max_sync(kFull, w);
    if (wmax <= 8u) {
        if (wmax != 0u) {
            uint32_t G[2], W[3];
            segment64(z, w, G);
            shift_segment<2>(G, sh, W);
            emit_segment<3>(W, sh, w, dst);
        }
    } else if (wmax <= 16u) {
        uint32_t G[4], W[5];
        segment128(z, w, G);
        shift_segment<4>(G, sh, W);
        emit_segment<5>(W, sh, w, dst);
    } else {
        uint32_t G[8], W[9];
        segment256(z, w, G);
        shift_segment<8>(G, sh, W);
        emit_segment<9>(W, sh, w, dst);
    }
    return kWordsPerW * tot_w;
}

template <int LPB, bool kCheckRange>
__device__ __forceinline__ void compute_tile_fast(EncSmem &sm, const Bound &bd, int s, int q, int cw, int ln,
                                                  uint32_t *out, uint32_t &words_out, uint32_t &omask_out) {
    constexpr int V = 8;
    constexpr int kB = V * LPB;
    constexpr int kWT = 32 * V;
    constexpr int kWPW = kChunk / kWT / kNW;
    const int g = ln / LPB, r = ln % LPB;
    uint32_t wo = 0, omask = 0;

#pragma unroll 1
    for (int k = 0; k < kWPW; ++k) {
        const int wt = cw * kWPW + k;
        const uint32_t e0 = wt * kWT + ln * V;
        float x[V];
        {
            const float4 t0 = *reinterpret_cast<const float4 *>(&sm.in[s][e0]);
            const float4 t1 = *reinterpret_cast<const float4 *>(&sm.in[s][e0 + 4]);
            x[0] = t0.x; x[1] = t0.y; x[2] = t0.z; x[3] = t0.w;
            x[4] = t1.x; x[5] = t1.y; x[6] = t1.z; x[7] = t1.w;
        }
        int32_t q_[V];
        uint32_t obits;
        quantize8<kCheckRange>(x, bd, q_, obits);
        int32_t pv = __shfl_up_sync(kFull, q_[V - 1], 1);
        if (r == 0) pv = 0;  // Lorenzo predecessor resets at the block start
        uint32_t z[V];
#pragma unroll
        for (int v = 0; v < V; ++v) z[v] = zigzag(q_[v] - (v ? q_[v - 1] : pv));
        wo += pack_warp_tile<LPB>(z, g, r, ln, &sm.width[q][(uint32_t)(wt * kWT) / kB], out + wo);
        omask |= obits << (k * V);
    }
    words_out = wo;
    omask_out = omask;
}

// ---------------------------------------------------------------------------
// Multi-dimensional Lorenzo tiles (ND = 2 or 3).  A tile is a brick of
// 16 x 16 x 16 (3-D) or 64 x 64 (2-D) elements, copied into the input stage
// by a tensor copy in C order (x fastest).  Blocks are taken in C order
// within the brick and codes in C order within a block, so each lane still
// holds 8 consecutive codes of its block and everything after the predictor
// (zigzag, widths, packing, the tile's record) is the 1-D path's.
//   3-D, B = 64  (4x4x4):  lane r: plane r/2, rows 2(r%2), 2(r%2)+1, 4 x each
//   3-D, B = 256 (4x8x8):  lane r: plane r/8, row r%8, 8 x
//   2-D, B = 64  (8x8):    lane r: row r, 8 x
//   2-D, B = 256 (16x16):  lane r: row r/2, x half r%2 (8 x)
// The predictor is the first difference along x, then y, then z within the
// block, neighbours outside the block taken as 0.
template <int ND, int LPB>
struct NdGeom {
    static constexpr int kBrickX = (ND == 3) ? 16 : 64;       // brick row length (elements)
    static constexpr int kBrickY = (ND == 3) ? 16 : 64;
    static constexpr int kBZ = (ND == 3) ? 4 : 1;             // block edges
    static constexpr int kBY = (ND == 3) ? (LPB == 8 ? 4 : 8) : (LPB == 8 ? 8 : 16);
    static constexpr int kBX = (ND == 3) ? (LPB == 8 ? 4 : 8) : (LPB == 8 ? 8 : 16);
    static constexpr int kKX = kBrickX / kBX, kKY = kBrickY / kBY;  // blocks per brick along x, y
    static_assert(kBZ * kBY * kBX == 8 * LPB, "block = 8 codes per lane");
    // Brick-local (z, y, x) of the first code of row `row` (0 or 1) of lane
    // r in block bi; codes of a row are consecutive in x.
    __device__ static void origin(int bi, int r, int row, int &z, int &y, int &x) {
        const int bx = bi % kKX, by = (bi / kKX) % kKY, bz = bi / (kKX * kKY);
        if constexpr (ND == 3 && LPB == 8) {
            z = bz * 4 + (r >> 1); y = by * 4 + ((r & 1) << 1) + row; x = bx * 4;
        } else if constexpr (ND == 3) {
            z = bz * 4 + (r >> 3); y = by * 8 + (r & 7); x = bx * 8;
        } else if constexpr (LPB == 8) {
            z = 0; y = by * 8 + r; x = bx * 8;
        } else {
            z = 0; y = by * 16 + (r >> 1); x = bx * 16 + ((r & 1) << 3);
        }
    }
    __device__ static int index(int z, int y, int x) { return (z * kBrickY + y) * kBrickX + x; }
};

// d = Lorenzo residuals of the lane's 8 codes q (slot v = row v / RX, x v % RX).
template <int ND, int LPB>
__device__ __forceinline__ void nd_delta(const int32_t (&q)[8], int r, uint32_t (&d)[8]) {
    int32_t a[8], b[8];
    if constexpr (ND == 3 && LPB == 8) {  // two rows of 4
#pragma unroll
        for (int v = 0; v < 8; ++v) a[v] = q[v] - ((v & 3) ? q[v - 1] : 0);
        // y: row 1 minus row 0; row 0 minus the row above it (lane r-1's row 1, unless y = 0)
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const int32_t up = __shfl_up_sync(kFull, a[v + 4], 1);
            b[v] = a[v] - ((r & 1) ? up : 0);
            b[v + 4] = a[v + 4] - a[v];
        }
        // z: minus the same rows one plane up (lane r-2), unless z = 0
#pragma unroll
        for (int v = 0; v < 8; ++v) {
            const int32_t up = __shfl_up_sync(kFull, b[v], 2);
            d[v] = (uint32_t)(b[v] - ((r >= 2) ? up : 0));
        }
    } else if constexpr (ND == 3) {  // one row of 8, y = r % 8, z = r / 8
#pragma unroll
        for (int v = 0; v < 8; ++v) a[v] = q[v] - (v ? q[v - 1] : 0);
#pragma unroll
        for (int v = 0; v < 8; ++v) {
            const int32_t up = __shfl_up_sync(kFull, a[v], 1);
            b[v] = a[v] - ((r & 7) ? up : 0);
        }
#pragma unroll
        for (int v = 0; v < 8; ++v) {
            const int32_t up = __shfl_up_sync(kFull, b[v], 8);
            d[v] = (uint32_t)(b[v] - ((r >= 8) ? up : 0));
        }
    } else if constexpr (LPB == 8) {  // 2-D 8x8: one row of 8, y = r
#pragma unroll
        for (int v = 0; v < 8; ++v) a[v] = q[v] - (v ? q[v - 1] : 0);
#pragma unroll
        for (int v = 0; v < 8; ++v) {
            const int32_t up = __shfl_up_sync(kFull, a[v], 1);
            d[v] = (uint32_t)(a[v] - (r ? up : 0));
        }
    } else {  // 2-D 16x16: half a row of 8, y = r / 2, x half r % 2
        const int32_t left = __shfl_up_sync(kFull, q[7], 1);  // x - 1 of the lane's first code, lane r-1
#pragma unroll
        for (int v = 0; v < 8; ++v) a[v] = q[v] - (v ? q[v - 1] : ((r & 1) ? left : 0));
#pragma unroll
        for (int v = 0; v < 8; ++v) {
            const int32_t up = __shfl_up_sync(kFull, a[v], 2);
            d[v] = (uint32_t)(a[v] - ((r >= 2) ? up : 0));
        }
    }
}

template <int ND, int LPB, bool kCheckRange>
__device__ __forceinline__ void compute_tile_nd(EncSmem &sm, const Bound &bd, int s, int q, int cw, int ln,
                                                uint32_t *out, uint32_t &words_out, uint32_t &omask_out) {
    using Gm = NdGeom<ND, LPB>;
    constexpr int kB = 8 * LPB;
    constexpr int kWT = 256;
    constexpr int kWPW = kChunk / kWT / kNW;
    constexpr int RX = (ND == 3 && LPB == 8) ? 4 : 8;  // codes per row of a lane
    const int g = ln / LPB, r = ln % LPB;
    uint32_t wo = 0, outl = 0;
    uint32_t *bitmap = reinterpret_cast<uint32_t *>(&sm.omask[q][0][0]);  // brick C order, 4096 bits
#pragma unroll 1
    for (int k = 0; k < kWPW; ++k) {
        const int wt = cw * kWPW + k;
        const int bi = wt * (kWT / kB) + g;  // block within the brick
        float x[8];
        int z0, y0, x0;
        Gm::origin(bi, r, 0, z0, y0, x0);
        if constexpr (RX == 4) {
            int z1, y1, x1;
            Gm::origin(bi, r, 1, z1, y1, x1);
            const float4 t0 = *reinterpret_cast<const float4 *>(&sm.in[s][Gm::index(z0, y0, x0)]);
            const float4 t1 = *reinterpret_cast<const float4 *>(&sm.in[s][Gm::index(z1, y1, x1)]);
            x[0] = t0.x; x[1] = t0.y; x[2] = t0.z; x[3] = t0.w;
            x[4] = t1.x; x[5] = t1.y; x[6] = t1.z; x[7] = t1.w;
        } else {
            const float *row = &sm.in[s][Gm::index(z0, y0, x0)];
            const float4 t0 = *reinterpret_cast<const float4 *>(row);
            const float4 t1 = *reinterpret_cast<const float4 *>(row + 4);
            x[0] = t0.x; x[1] = t0.y; x[2] = t0.z; x[3] = t0.w;
            x[4] = t1.x; x[5] = t1.y; x[6] = t1.z; x[7] = t1.w;
        }
        int32_t q_[8];
        uint32_t obits;
        quantize8<kCheckRange>(x, bd, q_, obits);
        if (obits) {  // rare: mark the outliers in the tile's C-order bitmap
#pragma unroll
            for (int v = 0; v < 8; ++v)
                if ((obits >> v) & 1u) {
                    int zz, yy, xx;
                    Gm::origin(bi, r, v / RX, zz, yy, xx);
                    const int p = Gm::index(zz, yy, xx + v % RX);
                    atomicOr(&bitmap[p >> 5], 1u << (p & 31));
                }
        }
        outl += __popc(obits);
        uint32_t dd[8], z[8];
        nd_delta<ND, LPB>(q_, r, dd);
#pragma unroll
        for (int v = 0; v < 8; ++v) z[v] = zigzag((int32_t)dd[v]);
        wo += pack_warp_tile<LPB>(z, g, r, ln, &sm.width[q][(uint32_t)(wt * kWT) / kB], out + wo);
    }
    words_out = wo;
    omask_out = outl;  // only the count is used for multi-dimensional tiles (the bitmap holds the positions)
}

__device__ __forceinline__ bool slot_done(const EncSmem &sm, uint32_t it) {
    return *reinterpret_cast<const volatile uint32_t *>(&sm.done[it % kD]) == it + 1;
}

template <int V, int LPB, int ND>
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
        uint32_t words, omask, outl;
        if constexpr (ND != 0) {  // every tile is a full brick; outliers go to the slot's bitmap
            if (bd.check_range)
                compute_tile_nd<ND, LPB, true>(sm, bd, s, q, cw, ln, ring + start, words, omask);
            else
                compute_tile_nd<ND, LPB, false>(sm, bd, s, q, cw, ln, ring + start, words, omask);
            outl = __reduce_add_sync(kFull, omask);
        } else {
            if (valid == kChunk) {
                if (bd.check_range)
                    compute_tile_fast<LPB, true>(sm, bd, s, q, cw, ln, ring + start, words, omask);
                else
                    compute_tile_fast<LPB, false>(sm, bd, s, q, cw, ln, ring + start, words, omask);
            } else {
                compute_tile<V, LPB>(sm, bd, s, q, valid, cw, ln, ring + start, words, omask);
            }
            outl = __reduce_add_sync(kFull, __popc(omask));
            sm.omask[q][cw][ln] = (uint16_t)omask;  // kWPW * V = 16 bits
        }
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

constexpr uint32_t kHeavySlice = 16;  // outliers in a slice from which write_slice_heavy takes it

// One compute warp's slice of a full tile with many outliers (write_tile_fast
// below takes the others): the lanes that have outliers reload their inputs
// for both warp-tiles first, so those L2 round trips overlap the payload copy,
// then the ranked outlier stores.  Kept out of line so that the common path's
// code is not shaped by it.
template <int V>
__device__ __noinline__ void write_slice_heavy(const uint32_t *src, uint32_t *dst, uint32_t words, uint32_t om,
                                               uint32_t *recs, uint32_t ord, uint32_t MT, const float *xin,
                                               uint32_t i_tile, int c, int ln) {
    constexpr int kWT = 32 * V;
    constexpr int kWPW = kChunk / kWT / kNW;
    float4 xr[kWPW][2];
#pragma unroll
    for (int k = 0; k < kWPW; ++k) {
        const uint32_t e_loc = (uint32_t)(c * kWPW + k) * kWT + ln * V;
        if ((om >> (k * V)) & ((1u << V) - 1u)) {
            xr[k][0] = __ldg(reinterpret_cast<const float4 *>(xin + e_loc));
            xr[k][1] = __ldg(reinterpret_cast<const float4 *>(xin + e_loc + 4));
        }
    }
    uint32_t j = ln;
    for (; j + 32 < words; j += 64) {
        const uint32_t v0 = src[j], v1 = src[j + 32];
        st_cs_u32(dst + j, v0);
        st_cs_u32(dst + j + 32, v1);
    }
    if (j < words) st_cs_u32(dst + j, src[j]);
#pragma unroll
    for (int k = 0; k < kWPW; ++k) {
        const uint32_t bits = (om >> (k * V)) & ((1u << V) - 1u);
        const uint32_t cnt = __popc(bits);
        uint32_t incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t t = __shfl_up_sync(kFull, incl, o);
            if (ln >= o) incl += t;
        }
        if (bits != 0u) {
            const float xv[V] = {xr[k][0].x, xr[k][0].y, xr[k][0].z, xr[k][0].w,
                                 xr[k][1].x, xr[k][1].y, xr[k][1].z, xr[k][1].w};
            uint32_t p = ord + incl - cnt;
            const uint32_t i0 = i_tile + (uint32_t)(c * kWPW + k) * kWT + ln * V;
#pragma unroll
            for (int v = 0; v < V; ++v) {
                if ((bits >> v) & 1u) {
                    recs[p] = i0 + v;
                    recs[p + MT] = __float_as_uint(xv[v]);
                    ++p;
                }
            }
        }
        ord += __shfl_sync(kFull, incl, 31);
    }
}

// write_tile for a full tile whose whole record (and its width bytes) fits
// in the caller's capacity, checked once by the caller: no per-store checks.
// Outliers: per warp-tile of a compute warp's slice, one warp scan of the
// lanes' outlier counts gives every outlier its rank, and the lanes that have
// outliers reload their 8 inputs with two coalesced 16-byte loads (the tile
// was read moments ago, so they come from L2).
template <int V, int LPB>
__device__ __forceinline__ void write_tile_fast(EncSmem &sm, const EncodeArgs &a, const Layout &L, int q, int tile,
                                                uint32_t rec, uint32_t PW, uint32_t MT, uint32_t wpw, uint32_t wpo,
                                                int ln) {
    constexpr int kB = V * LPB;
    constexpr int kWT = 32 * V;
    constexpr int kWPW = kChunk / kWT / kNW;
    static_assert(V == 8, "the outlier reload reads two float4 per lane");
    uint32_t *recs = reinterpret_cast<uint32_t *>(a.out + L.record_off);
    const float *xin = a.in + (uint64_t)tile * kChunk;
#pragma unroll 1
    for (int c = 0; c < kNW; ++c) {
        const uint32_t words = sm.totals[q][c][0], pos = sm.ringpos[q][c], mc = sm.totals[q][c][1];
        const uint32_t *src = sm.ring[c] + pos;
        uint32_t *dst = recs + (rec + __shfl_sync(kFull, wpw, c));
        if (mc >= kHeavySlice) {
            write_slice_heavy<V>(src, dst, words, sm.omask[q][c][ln], recs, rec + PW + __shfl_sync(kFull, wpo, c),
                                 MT, xin, (uint32_t)tile * kChunk, c, ln);
            continue;
        }
        uint32_t j = ln;
        for (; j + 32 < words; j += 64) {
            const uint32_t v0 = src[j], v1 = src[j + 32];
            st_cs_u32(dst + j, v0);
            st_cs_u32(dst + j + 32, v1);
        }
        if (j < words) st_cs_u32(dst + j, src[j]);
        if (mc != 0u) {
            const uint32_t om = sm.omask[q][c][ln];
            uint32_t ord = rec + PW + __shfl_sync(kFull, wpo, c);  // index slot of the slice's first outlier
#pragma unroll 1
            for (int k = 0; k < kWPW; ++k) {
                const uint32_t bits = (om >> (k * V)) & ((1u << V) - 1u);
                const uint32_t cnt = __popc(bits);
                uint32_t incl = cnt;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const uint32_t t = __shfl_up_sync(kFull, incl, o);
                    if (ln >= o) incl += t;
                }
                const uint32_t e_loc = (uint32_t)(c * kWPW + k) * kWT + ln * V;
                if (bits != 0u) {
                    const float4 x0 = __ldg(reinterpret_cast<const float4 *>(xin + e_loc));
                    const float4 x1 = __ldg(reinterpret_cast<const float4 *>(xin + e_loc + 4));
                    const float xv[V] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                    uint32_t p = ord + incl - cnt;
                    const uint32_t i0 = (uint32_t)tile * kChunk + e_loc;
#pragma unroll
                    for (int v = 0; v < V; ++v) {
                        if ((bits >> v) & 1u) {
                            recs[p] = i0 + v;
                            recs[p + MT] = __float_as_uint(xv[v]);
                            ++p;
                        }
                    }
                }
                ord += __shfl_sync(kFull, incl, 31);
            }
        }
    }
    {  // width bytes of the tile's blocks (a full tile holds K of them, K a multiple of 16)
        constexpr uint32_t K = kChunk / kB;
        const uint32_t *ws = reinterpret_cast<const uint32_t *>(sm.width[q]);
        uint32_t *wd = reinterpret_cast<uint32_t *>(a.out + L.width_off + (uint64_t)tile * K);
        for (uint32_t j = ln; j < K / 4; j += 32) wd[j] = ws[j];
    }
}

// write_tile for a multi-dimensional brick: the compute warps' packed words
// (capacity checked per warp part), then the outliers, ranked in C order
// through the slot's bitmap (lane l holds bits 128 l .. 128 l + 127 of the
// brick), their values reloaded from the input (L2), and the bitmap cleared
// for the slot's next tile; then the width bytes.
template <int ND, int LPB>
__device__ __forceinline__ void write_tile_nd(EncSmem &sm, const EncodeArgs &a, const Layout &L, int q, int tile,
                                              uint32_t rec, uint32_t PW, uint32_t MT, uint32_t wpw, int ln) {
    constexpr int kB = 8 * LPB;
    uint32_t *recs = reinterpret_cast<uint32_t *>(a.out + L.record_off);
    const uint64_t cap_words = (a.out_cap > L.record_off) ? (a.out_cap - L.record_off) / 4 : 0;
    bool over = false;
#pragma unroll 1
    for (int c = 0; c < kNW; ++c) {
        const uint32_t words = sm.totals[q][c][0], pos = sm.ringpos[q][c];
        const uint64_t w0 = (uint64_t)rec + __shfl_sync(kFull, wpw, c);
        const uint32_t *src = sm.ring[c] + pos;
        uint32_t *dst = recs + w0;
        const uint32_t lim = (w0 >= cap_words) ? 0u : (uint32_t)min((uint64_t)words, cap_words - w0);
        over |= lim < words;
        for (uint32_t j = ln; j < lim; j += 32) st_cs_u32(dst + j, src[j]);
    }
    if (MT != 0u) {
        uint32_t *bm = reinterpret_cast<uint32_t *>(&sm.omask[q][0][0]) + 4 * ln;
        const uint4 b4 = *reinterpret_cast<const uint4 *>(bm);
        const uint32_t cnt = __popc(b4.x) + __popc(b4.y) + __popc(b4.z) + __popc(b4.w);
        uint32_t incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t t = __shfl_up_sync(kFull, incl, o);
            if (ln >= o) incl += t;
        }
        int bz, by, bx;
        brick_origin((uint64_t)tile, ND, a.dims, bz, by, bx);
        uint64_t pi = (uint64_t)rec + PW + (incl - cnt);  // index slot of this lane's first outlier
        const uint32_t wv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            uint32_t bits = wv[k];
            while (bits) {
                const int b = __ffs(bits) - 1;
                bits &= bits - 1u;
                const int p = (4 * ln + k) * 32 + b;  // position in the brick, C order
                int z, y, x;
                if constexpr (ND == 3) {
                    z = p >> 8; y = (p >> 4) & 15; x = p & 15;
                } else {
                    z = 0; y = p >> 6; x = p & 63;
                }
                const uint64_t idx = (((uint64_t)(bz + z) * a.dims[1]) + (uint64_t)(by + y)) * a.dims[2] + (uint64_t)(bx + x);
                if (pi + MT < cap_words) {
                    recs[pi] = (uint32_t)idx;
                    recs[pi + MT] = __float_as_uint(__ldg(a.in + idx));
                } else {
                    over = true;
                }
                ++pi;
            }
        }
        *reinterpret_cast<uint4 *>(bm) = make_uint4(0u, 0u, 0u, 0u);
    }
    {  // width bytes of the brick's blocks
        constexpr uint32_t K = kChunk / kB;
        const uint32_t *ws = reinterpret_cast<const uint32_t *>(sm.width[q]);
        uint32_t *wd = reinterpret_cast<uint32_t *>(a.out + L.width_off + (uint64_t)tile * K);
        const uint64_t end = L.width_off + (uint64_t)(tile + 1) * K;
        if (end <= a.out_cap) {
            for (uint32_t j = ln; j < K / 4; j += 32) wd[j] = ws[j];
        } else {
            over = true;
        }
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
    h[1] = kVersion | ((uint32_t)((a.abs_mode ? kFlagAbs : 0) | (a.nd ? kFlagLorenzoNd : 0)) << 16);
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
    if (a.nd) {  // dims Z, Y, X at bytes 96..119
        for (int d = 0; d < 3; ++d) {
            h[24 + 2 * d] = (uint32_t)a.dims[d];
            h[25 + 2 * d] = (uint32_t)(a.dims[d] >> 32);
        }
    }
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
// aggregate: polls the farthest missing one with back-off (bounded by
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
            if (!found) {
                const uint32_t upto = inc ? (inc ^ (inc - 1u)) : kFull;  // lanes through the first inclusive
                if (mis & upto) {  // the farthest row with a missing predecessor so far
                    miss_row = j;
                    miss_lanes = mis & upto;
                }
                if ((upto >> ln) & 1u) {
                    sr += (uint32_t)(v[j] & 0xffffffffu) - 1u;
                    sm_ += (uint32_t)((v[j] >> 32) & 0x7fffffffu);
                }
                found = inc != 0u;
            }
        }
        if (miss_row >= 0) {
            // Wait for the farthest predecessor that has not published: tiles of
            // a wave finish in no particular order, so by the time it has, the
            // nearer ones almost always have too, and one more read of the
            // window suffices (waiting for the nearest one first costs a round
            // trip per missing predecessor).
            const uint64_t *w = &status[base - 32 * miss_row - (31 - __clz(miss_lanes))];
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

template <int V, int LPB, int ND>
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
            // The look-back waits only for aggregates of lower tiles, which
            // their CTAs publish as soon as they have computed them; the compute
            // warps meanwhile run up to kD - 2 tiles ahead of the write-out, so
            // a wave's tiles are rarely still missing by the time it is read.
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
        if constexpr (ND != 0) {
            write_tile_nd<ND, LPB>(sm, a, L, q, tile, exR, PW, MT, iw - tw, ln);
        } else {
            constexpr uint32_t K = kChunk / (V * LPB);
            const uint64_t rec_end = L.record_off + 4ull * ((uint64_t)exR + Rt);
            const uint64_t wid_end = L.width_off + (uint64_t)(tile + 1) * K;
            const bool full = (uint64_t)(tile + 1) * kChunk <= a.n;
            if (full && rec_end <= a.out_cap && wid_end <= a.out_cap)
                write_tile_fast<V, LPB>(sm, a, L, q, tile, exR, PW, MT, iw - tw, io - to, ln);
            else
                write_tile<V, LPB>(sm, a, L, q, tile, exR, PW, MT, iw - tw, io - to, ln);
        }
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
template <int ND>
__device__ void producer_warp(EncSmem &sm, const EncodeArgs &a, const Layout &L, int ln) {
    if (ln != 0) return;
    // Tensor copies want a 128-byte aligned shared destination; the stages are
    // laid out for that, and a launch where it does not hold reports an error
    // and ends (every tile marked absent) instead of issuing the copy.
    const bool tensor_ok = ND == 0 || (smem_u32(&sm.in[0][0]) & 127u) == 0;
    if (!tensor_ok) atomicOr(a.err, kErrCorrupt);
    uint32_t i = 0;
    for (;; ++i) {
        const int s = i % kS;
        if (i >= kS && !mbar_wait(&sm.empty[s], ((i / kS) - 1) & 1, a.wait_ns, a.err)) break;
        const uint64_t t = (uint64_t)blockIdx.x + (uint64_t)i * gridDim.x;
        if (t >= L.nc || !tensor_ok) {
            sm.tile_id[s] = -1;
            mbar_arrive(&sm.full[s]);
            ++i;
            break;
        }
        sm.tile_id[s] = (int32_t)t;
        if constexpr (ND != 0) {  // a whole brick by one tensor copy, C order in the stage
            int z, y, x;
            brick_origin(t, ND, a.dims, z, y, x);
            mbar_arrive_expect_tx(&sm.full[s], kChunk * 4u);
            if constexpr (ND == 3)
                tensor_g2s_3d(sm.in[s], &a.tmap, x, y, z, &sm.full[s]);
            else
                tensor_g2s_2d(sm.in[s], &a.tmap, x, y, &sm.full[s]);
            continue;
        }
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

template <int V, int LPB, int ND>
__global__ void __launch_bounds__(kThreads, 2) encode_kernel(const __grid_constant__ EncodeArgs a) {
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
        if (ND != 0)  // the outlier bitmaps of the slots start clear
            for (int j = 0; j < kD * kNW * 32; ++j) (&sm.omask[0][0][0])[j] = 0;
        float vmin = a.abs_mode ? 0.0f : a.range[0] + 0.0f;  // + 0: -0 reads as +0
        float vmax = a.abs_mode ? 0.0f : a.range[1] + 0.0f;
        if (!a.abs_mode && a.range_given && blockIdx.x == 0 &&
            !(fabsf(vmin) < __int_as_float(0x7f800000) && fabsf(vmax) < __int_as_float(0x7f800000) && vmin <= vmax))
            atomicOr(a.err, kErrRange);
        sm.bound = resolve_bound(a.abs_mode, a.bound, vmin, vmax, a.range_given);
        const uint64_t par = *a.epoch & 1u;
        sm.st_cur = a.status + par * a.ntiles;
        sm.st_next = a.status + (par ^ 1u) * a.ntiles;
    }
    __syncthreads();

    if (warp < kNW)
        compute_warp<V, LPB, ND>(sm, a, warp, ln);
    else if (warp < kProducerWarp)
        lookback_warp<V, LPB, ND>(sm, a, L, warp - kNW, ln);
    else
        producer_warp<ND>(sm, a, L, ln);

    if (L.nc == 0 && blockIdx.x == 0 && threadIdx.x == 0) write_header(a, L, sm.bound, 0, 0);
}

template <int V, int LPB, int ND>
cudaError_t launch_t(const EncodeArgs &a, int num_sms, cudaStream_t stream) {
    const size_t smem = sizeof(EncSmem);
    cudaError_t e = cudaFuncSetAttribute(encode_kernel<V, LPB, ND>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, encode_kernel<V, LPB, ND>, kThreads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const Layout L = stream_layout(a.n, a.block);
    const uint64_t resident = (uint64_t)per_sm * (uint64_t)num_sms;
    const int grid = (int)(L.nc == 0 ? 1 : (resident < L.nc ? resident : L.nc));
    EncodeArgs args = a;
    void *params[] = {&args};
    return cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(encode_kernel<V, LPB, ND>), dim3(grid),
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
                                : (err & kErrRange)    ? (uint32_t)EBLC_INVALID_ARG
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
        case 32: return a.nd ? cudaErrorInvalidValue : launch_t<8, 4, 0>(a, num_sms, stream);
        case 64: return a.nd == 3 ? launch_t<8, 8, 3>(a, num_sms, stream)
                      : a.nd == 2 ? launch_t<8, 8, 2>(a, num_sms, stream)
                                  : launch_t<8, 8, 0>(a, num_sms, stream);
        case 128: return a.nd ? cudaErrorInvalidValue : launch_t<8, 16, 0>(a, num_sms, stream);
        case 256: return a.nd == 3 ? launch_t<8, 32, 3>(a, num_sms, stream)
                       : a.nd == 2 ? launch_t<8, 32, 2>(a, num_sms, stream)
                                   : launch_t<8, 32, 0>(a, num_sms, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace eblc
