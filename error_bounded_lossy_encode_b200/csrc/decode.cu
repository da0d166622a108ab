// decode.cu -- fused decoder for sm_100a.
//
// The exact inverse of the encoder ("Pipeline specialization internals",
// Inverse declaration and the device policy contract: coder decode ->
// undelta (plain first-difference inverse, a prefix sum restarting at every
// block) -> linear dequantization x' = code * step, step = 2*eb), followed
// by writing each chunk's outliers back over the reconstruction.
//
// The chunk index gives every chunk's record offset, so chunks decode
// independently: no scan, no inter-CTA communication, no scratch memory.
//
// CTA organisation (288 threads, 4 CTAs per SM, persistent grid, chunk
// t handled by CTA t mod grid):
//   warps 0..7  compute: warp-tiles of 32*V elements (V consecutive
//               elements per lane; a block of B elements spans B/V lanes).
//               Each lane reads its bits straight from the staged record,
//               extracts its codes, undoes zigzag, and the block prefix sum
//               is a lane-serial sum plus a segmented warp scan.
//   warp 8      producer: reads the chunk index and streams each record
//               (payload, and the outlier list when it fits) and the
//               chunk's width bytes into a 2-stage shared-memory ring with
//               bulk async copies completing on mbarriers.
// The reconstruction is stored straight from registers (128-bit coalesced
// streaming stores); a chunk's outliers are then written over it in global
// memory, after an mbarrier of the compute warps (bounded wait) orders them
// behind every reconstruction store of the chunk.
#include "common.cuh"
#include "kernels.h"

namespace eblc {
namespace {

constexpr int kNW = 8;
constexpr int kS = 2;
constexpr int kThreads = (kNW + 1) * 32;
constexpr uint32_t kFull = 0xffffffffu;
constexpr uint32_t kStagedOutliers = 1024;                 // outliers staged with the payload
constexpr uint32_t kRecWords = kChunk + 2 * kStagedOutliers + 4 + 16;  // + alignment + over-read slack

struct __align__(128) DecSmem {
    uint32_t rec[kS][kRecWords];
    uint8_t width[kS][kChunk / 32];
    uint32_t info[kS][8];  // tile (or -1), valid, PW, mt, adj, staged, rec, corrupt
    uint64_t full[kS], empty[kS];
    uint64_t stored;       // compute warps: a chunk's reconstruction stores are done (one phase per use)
};

template <int LPB>
__device__ __forceinline__ uint32_t group_scan_excl(uint32_t v, int r, uint32_t &incl_out) {
    uint32_t incl = v;
#pragma unroll
    for (int o = 1; o < LPB; o <<= 1) {
        const uint32_t t = __shfl_up_sync(kFull, incl, o);
        if (r >= o) incl += t;
    }
    incl_out = incl;
    return incl - v;
}

// Width of this lane's block and the exclusive prefix / total of the widths
// of the warp-tile's blocks (wb: their width bytes in shared memory), read as
// one word per lane instead of a shuffle per block.  Widths above 32 exist
// only in corrupt streams: they are clamped to 32 (per byte, so the byte
// sums below stay under 256) and reported through `raw_over`.
template <int LPB>
__device__ __forceinline__ void widths_of_tile(const uint8_t *wb, int g, uint32_t &w, uint32_t &pre, uint32_t &tot,
                                               bool &raw_over) {
    if constexpr (LPB == 32) {
        const uint32_t raw = wb[0];
        raw_over = raw > 32u;
        w = min(raw, 32u);
        pre = 0;
        tot = w;
    } else if constexpr (LPB == 16) {
        const uint32_t raw = *reinterpret_cast<const uint16_t *>(wb);
        const uint32_t c = __vminu4(raw, 0x2020u);
        raw_over = ((raw >> (8 * g)) & 0xffu) > 32u;
        const uint32_t w0 = c & 0xffu, w1 = c >> 8;
        w = g ? w1 : w0;
        pre = g ? w0 : 0u;
        tot = w0 + w1;
    } else if constexpr (LPB == 8) {
        const uint32_t raw = *reinterpret_cast<const uint32_t *>(wb);
        const uint32_t c = __vminu4(raw, 0x20202020u);
        raw_over = ((raw >> (8 * g)) & 0xffu) > 32u;
        w = (c >> (8 * g)) & 0xffu;
        pre = ((c * 0x01010100u) >> (8 * g)) & 0xffu;
        tot = (c * 0x01010101u) >> 24;
    } else {  // LPB == 4: eight blocks in two words
        const uint2 raw = *reinterpret_cast<const uint2 *>(wb);
        const uint32_t lo = __vminu4(raw.x, 0x20202020u), hi = __vminu4(raw.y, 0x20202020u);
        const uint32_t rw = (g < 4) ? raw.x : raw.y, cw = (g < 4) ? lo : hi;
        raw_over = ((rw >> (8 * (g & 3))) & 0xffu) > 32u;
        const uint32_t tlo = (lo * 0x01010101u) >> 24;
        w = (cw >> (8 * (g & 3))) & 0xffu;
        pre = ((cw * 0x01010100u) >> (8 * (g & 3))) & 0xffu;
        if (g >= 4) pre += tlo;
        tot = tlo + ((hi * 0x01010101u) >> 24);
    }
}

// Multi-dimensional Lorenzo blocks (nd = 2, 3): the lane's residuals d (8
// codes in block order, the encoder's lane layout: 3-D 4x4x4 two rows of 4;
// 3-D 4x8x8 and 2-D 8x8 one row of 8; 2-D 16x16 half a row) summed back --
// inclusive prefix sums along x, then y, then z within the block, by
// segmented warp scans -- dequantized and stored at their places in the
// array.  Block bi (C order within the brick) of the brick whose first
// element is (bz, by, bx).
template <int ND, int LPB>
__device__ __forceinline__ void nd_store(const DecodeArgs &a, int bz, int by, int bx, uint32_t bi, int r,
                                         const uint32_t (&d)[8]) {
    constexpr int kBX = (ND == 3) ? (LPB == 8 ? 4 : 8) : (LPB == 8 ? 8 : 16);
    constexpr int kBY = (ND == 3) ? (LPB == 8 ? 4 : 8) : (LPB == 8 ? 8 : 16);
    constexpr int kKX = ((ND == 3) ? 16 : 64) / kBX, kKY = ((ND == 3) ? 16 : 64) / kBY;
    uint32_t q[8];
    int zo, yo, xo;  // the lane's first code, within the block
    if constexpr (ND == 3 && LPB == 8) {
#pragma unroll
        for (int v = 0; v < 8; ++v) q[v] = d[v] + ((v & 3) ? q[v - 1] : 0u);  // x, per row of 4
#pragma unroll
        for (int v = 0; v < 4; ++v) q[v + 4] += q[v];                            // y, within the lane
#pragma unroll
        for (int v = 0; v < 4; ++v) {                                             // y, rows 0-1 of lane r-1
            const uint32_t up = __shfl_up_sync(kFull, q[v + 4], 1);
            if (r & 1) { q[v] += up; q[v + 4] += up; }
        }
#pragma unroll
        for (int o = 2; o <= 4; o <<= 1)                                         // z: planes at lane stride 2
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                const uint32_t up = __shfl_up_sync(kFull, q[v], o);
                if (r >= o) q[v] += up;
            }
        zo = r >> 1; yo = (r & 1) << 1; xo = 0;
    } else if constexpr (ND == 3) {
#pragma unroll
        for (int v = 0; v < 8; ++v) q[v] = d[v] + (v ? q[v - 1] : 0u);
#pragma unroll
        for (int o = 1; o <= 4; o <<= 1)                                         // y: rows at lane stride 1
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                const uint32_t up = __shfl_up_sync(kFull, q[v], o);
                if ((r & 7) >= o) q[v] += up;
            }
#pragma unroll
        for (int o = 8; o <= 16; o <<= 1)                                        // z: planes at lane stride 8
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                const uint32_t up = __shfl_up_sync(kFull, q[v], o);
                if (r >= o) q[v] += up;
            }
        zo = r >> 3; yo = r & 7; xo = 0;
    } else if constexpr (LPB == 8) {
#pragma unroll
        for (int v = 0; v < 8; ++v) q[v] = d[v] + (v ? q[v - 1] : 0u);
#pragma unroll
        for (int o = 1; o <= 4; o <<= 1)
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                const uint32_t up = __shfl_up_sync(kFull, q[v], o);
                if (r >= o) q[v] += up;
            }
        zo = 0; yo = r; xo = 0;
    } else {
#pragma unroll
        for (int v = 0; v < 8; ++v) q[v] = d[v] + (v ? q[v - 1] : 0u);
        const uint32_t left = __shfl_up_sync(kFull, q[7], 1);                    // x: first half of the row
        if (r & 1) {
#pragma unroll
            for (int v = 0; v < 8; ++v) q[v] += left;
        }
#pragma unroll
        for (int o = 2; o <= 16; o <<= 1)                                        // y: rows at lane stride 2
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                const uint32_t up = __shfl_up_sync(kFull, q[v], o);
                if (r >= o) q[v] += up;
            }
        zo = 0; yo = r >> 1; xo = (r & 1) << 3;
    }
    float y[8];
#pragma unroll
    for (int v = 0; v < 8; ++v) y[v] = __fmul_rn(__int2float_rn((int32_t)q[v]), a.step);
    const int kx = (int)(bi % kKX), ky = (int)((bi / kKX) % kKY), kz = (int)(bi / (kKX * kKY));
    const uint64_t z = (uint64_t)(bz + kz * ((ND == 3) ? 4 : 1) + zo);
    const uint64_t yy = (uint64_t)(by + ky * kBY + yo), x = (uint64_t)(bx + kx * kBX + xo);
    float *row = a.out + (z * a.dims[1] + yy) * a.dims[2] + x;
    if constexpr (ND == 3 && LPB == 8) {  // two rows of 4
        __stcs(reinterpret_cast<float4 *>(row), make_float4(y[0], y[1], y[2], y[3]));
        __stcs(reinterpret_cast<float4 *>(row + a.dims[2]), make_float4(y[4], y[5], y[6], y[7]));
    } else {
        __stcs(reinterpret_cast<float4 *>(row), make_float4(y[0], y[1], y[2], y[3]));
        __stcs(reinterpret_cast<float4 *>(row + 4), make_float4(y[4], y[5], y[6], y[7]));
    }
}

template <int V, int LPB, int ND>
__device__ void compute_warp(DecSmem &sm, const DecodeArgs &a, int cw, int ln) {
    constexpr int kB = V * LPB;
    constexpr int kWT = 32 * V;
    constexpr int kWPW = kChunk / kWT / kNW;
    constexpr int kEPL = kB / 32;  // payload words per unit of width for a full block
    const int g = ln / LPB, r = ln % LPB;
    const int tid = cw * 32 + ln;
    uint32_t stored_uses = 0;  // phases of sm.stored this warp has waited for (the same for every warp)

    for (uint32_t i = 0;; ++i) {
        const int s = i % kS;
        if (!mbar_wait(&sm.full[s], (i / kS) & 1, a.wait_ns, a.err)) return;
        const int tile = (int)sm.info[s][0];
        if (tile < 0) break;
        const uint32_t valid = sm.info[s][1], PW = sm.info[s][2], mt = sm.info[s][3], adj = sm.info[s][4];
        const bool staged = sm.info[s][5] != 0, corrupt = sm.info[s][7] != 0;
        const uint32_t *rec = sm.rec[s] + adj;
        const uint8_t *wid = sm.width[s];
        float *const gout = a.out + (uint64_t)tile * kChunk;
        int bz = 0, by = 0, bx = 0;  // the brick's first element (multi-dimensional tiles)
        if constexpr (ND != 0) brick_origin((uint64_t)tile, ND, a.dims, bz, by, bx);

        // widths of the chunk's blocks before this warp's first block
        const uint32_t blk0 = (uint32_t)(cw * kWPW * kWT) / kB;
        uint32_t before = 0;
        for (uint32_t b = ln; b < blk0; b += 32) before += wid[b];
        before = __reduce_add_sync(kFull, before);

        if (!corrupt) {
#pragma unroll 1
            for (int k = 0; k < kWPW; ++k) {
                const int wt = cw * kWPW + k;
                const uint32_t e0 = wt * kWT + ln * V;
                uint32_t w, pre, tot;
                bool over;  // widths above 32 are reported once per chunk, below
                widths_of_tile<LPB>(wid + (uint32_t)(wt * kWT) / kB, g, w, pre, tot, over);
                (void)over;
                // bit position of this lane's first code in the chunk payload
                const uint32_t bit0 = 32u * kEPL * (before + pre) + (uint32_t)r * V * w;
                const uint32_t mask = (w == 32u) ? kFull : ((1u << w) - 1u);
                int32_t c[V];
                uint32_t dv[V];  // the residuals (the 1-D path also keeps their running sum in c)
                uint32_t run = 0;
                // The lane's codes occupy bits [bit0, bit0 + 8w) of the staged
                // payload.  For narrow blocks the lane loads the few words that
                // hold them once and shifts the codes out of registers; wider
                // blocks read two words per code.  Every word index is clamped
                // into the stage (lim words from rec): a valid stream's codes
                // lie in its payload, far below the clamp, so it never acts;
                // a corrupt stream's widths can only make the lane read other
                // words of the stage, and the per-chunk payload check below
                // reports it.
                const uint32_t wmax = __reduce_max_sync(kFull, w);
                const uint32_t lim = kRecWords - adj, sh0 = bit0 & 31u;
                if (wmax <= 8u) {
                    static_assert(V == 8, "narrow path: 8 codes of <= 8 bits fit in 64 bits");
                    const uint32_t wd0 = min(bit0 >> 5, lim - 3u);
                    uint32_t lo = __funnelshift_r(rec[wd0], rec[wd0 + 1], sh0);
                    uint32_t hi = __funnelshift_r(rec[wd0 + 1], rec[wd0 + 2], sh0);
#pragma unroll
                    for (int v = 0; v < V; ++v) {
                        const uint32_t zz = lo & mask;
                        lo = __funnelshift_r(lo, hi, w);
                        hi >>= w;
                        const uint32_t d = (zz >> 1) ^ (0u - (zz & 1u));  // inverse zigzag
                        dv[v] = d;
                        run += d;
                        c[v] = (int32_t)run;
                    }
                } else if (wmax <= 16u) {
                    // 8 codes of <= 16 bits: 128 bits, shifted out of four words
                    const uint32_t wd0 = min(bit0 >> 5, lim - 5u);
                    uint32_t g0 = __funnelshift_r(rec[wd0], rec[wd0 + 1], sh0);
                    uint32_t g1 = __funnelshift_r(rec[wd0 + 1], rec[wd0 + 2], sh0);
                    uint32_t g2 = __funnelshift_r(rec[wd0 + 2], rec[wd0 + 3], sh0);
                    uint32_t g3 = __funnelshift_r(rec[wd0 + 3], rec[wd0 + 4], sh0);
#pragma unroll
                    for (int v = 0; v < V; ++v) {
                        const uint32_t zz = g0 & mask;
                        g0 = __funnelshift_r(g0, g1, w);
                        g1 = __funnelshift_r(g1, g2, w);
                        g2 = __funnelshift_r(g2, g3, w);
                        g3 >>= w;
                        const uint32_t d = (zz >> 1) ^ (0u - (zz & 1u));  // inverse zigzag
                        dv[v] = d;
                        run += d;
                        c[v] = (int32_t)run;
                    }
                } else {
#pragma unroll
                    for (int v = 0; v < V; ++v) {
                        const uint32_t b = bit0 + v * w;
                        const uint32_t wd = min(b >> 5, lim - 2u);
                        const uint32_t zz = __funnelshift_r(rec[wd], rec[wd + 1], b & 31u) & mask;
                        const uint32_t d = (zz >> 1) ^ (0u - (zz & 1u));  // inverse zigzag
                        dv[v] = d;
                        run += d;
                        c[v] = (int32_t)run;
                    }
                }
                if constexpr (ND != 0) {
                    nd_store<ND, LPB>(a, bz, by, bx, (uint32_t)(wt * kWT) / kB + g, r, dv);
                    before += tot;
                    continue;
                }
                uint32_t incl;
                const uint32_t ex = group_scan_excl<LPB>(run, r, incl);
                float y[V];
#pragma unroll
                for (int v = 0; v < V; ++v) y[v] = __fmul_rn(__int2float_rn((int32_t)((uint32_t)c[v] + ex)), a.step);

                if (e0 + V <= valid) {
#pragma unroll
                    for (int h = 0; h < V / 4; ++h)
                        __stcs(reinterpret_cast<float4 *>(gout + e0 + 4 * h),
                               make_float4(y[4 * h], y[4 * h + 1], y[4 * h + 2], y[4 * h + 3]));
                } else {
#pragma unroll
                    for (int v = 0; v < V; ++v)
                        if (e0 + v < valid) gout[e0 + v] = y[v];
                }
                before += tot;
            }
            // the chunk's widths must be at most 32, and its payload must hold
            // exactly the words they call for
            if (cw == kNW - 1) {
                const uint32_t nblk = (valid + kB - 1) / kB;
                uint32_t sum = 0, wbig = 0;
                for (uint32_t b = ln; b + 1 < nblk; b += 32) {
                    sum += min((uint32_t)wid[b], 32u);
                    wbig = max(wbig, (uint32_t)wid[b]);
                }
                sum = __reduce_add_sync(kFull, sum);
                const uint32_t last_cnt = valid - (nblk - 1) * kB;
                const uint32_t wl = min((uint32_t)wid[nblk - 1], 32u);
                const bool too_wide = __any_sync(kFull, wbig > 32u) || wid[nblk - 1] > 32u;
                if (ln == 0 && (too_wide || kEPL * sum + (wl * last_cnt + 31u) / 32u != PW))
                    atomicOr(a.err, kErrCorrupt);
            }
        }

        if (mt != 0 && !corrupt) {
            // Every compute thread's reconstruction stores of this chunk come
            // before any outlier store: each warp arrives (release) once its
            // lanes' stores are done and waits (acquire) for all kNW warps.
            // The wait is bounded like every other: a warp that gave up
            // earlier never arrives, so the others record kErrTimeout and
            // return instead of waiting for good.
            __syncwarp();
            if (ln == 0) mbar_arrive(&sm.stored);
            if (!mbar_wait(&sm.stored, stored_uses & 1u, a.wait_ns, a.err)) return;
            ++stored_uses;
            const uint32_t *gidx = reinterpret_cast<const uint32_t *>(a.in + stream_layout(a.n, a.block).record_off) +
                                   sm.info[s][6] + PW;
            for (uint32_t k = tid; k < mt; k += kNW * 32) {
                const uint32_t idx = staged ? rec[PW + k] : gidx[k];
                const uint32_t val = staged ? rec[PW + mt + k] : gidx[mt + k];
                if constexpr (ND != 0) {  // the index must lie in this brick (32-bit: n <= 2^30)
                    const uint32_t X = (uint32_t)a.dims[2], Y = (uint32_t)a.dims[1];
                    const uint32_t row = idx / X, xx = idx - row * X, zz = row / Y, yy = row - zz * Y;
                    const uint32_t ez = (ND == 3) ? 16 : 1, exy = (ND == 3) ? 16 : 64;
                    if (idx < a.n && zz >= (uint32_t)bz && zz < bz + ez && yy >= (uint32_t)by && yy < by + exy &&
                        xx >= (uint32_t)bx && xx < bx + exy)
                        a.out[idx] = __uint_as_float(val);
                    else
                        atomicOr(a.err, kErrCorrupt);
                } else {
                    const uint64_t e = (uint64_t)idx - (uint64_t)tile * kChunk;
                    if (idx >= (uint64_t)tile * kChunk && e < valid)
                        gout[e] = __uint_as_float(val);
                    else
                        atomicOr(a.err, kErrCorrupt);
                }
            }
        }
        __syncwarp();
        if (ln == 0) mbar_arrive(&sm.empty[s]);
    }
}

__device__ void producer_warp(DecSmem &sm, const DecodeArgs &a, int ln) {
    if (ln != 0) return;
    const Layout L = stream_layout(a.n, a.block);
    const uint64_t R = a.W + 2 * a.m;
    const uint32_t K = kChunk / a.block;  // blocks per chunk
    const uint64_t total16 = a.total & ~uint64_t(15);
    // The chunk index entries of a chunk and of the one after it, for the
    // chunk of iteration i; those of iteration i + 1 are loaded one iteration
    // ahead, so a stage fill waits for its bulk copy only, not for an index
    // read before it.
    auto index_pair = [&](uint64_t t, uint2 &ent, uint2 &nx) {
        ent = make_uint2(0u, 0u);
        nx = make_uint2((uint32_t)R, (uint32_t)a.m);
        if (t < L.nc) ent = *reinterpret_cast<const uint2 *>(a.in + L.index_off + 8 * t);
        if (t + 1 < L.nc) nx = *reinterpret_cast<const uint2 *>(a.in + L.index_off + 8 * (t + 1));
    };
    uint2 ent_ahead, nx_ahead;
    index_pair(blockIdx.x, ent_ahead, nx_ahead);
    uint32_t i = 0;
    for (;; ++i) {
        const int s = i % kS;
        const uint64_t t = (uint64_t)blockIdx.x + (uint64_t)i * gridDim.x;
        const uint2 ent = ent_ahead;
        uint64_t rec_next = (t + 1 < L.nc) ? nx_ahead.x : R, bef_next = (t + 1 < L.nc) ? nx_ahead.y : a.m;
        index_pair(t + gridDim.x, ent_ahead, nx_ahead);  // next iteration's entries, in flight meanwhile
        if (i >= kS && !mbar_wait(&sm.empty[s], ((i / kS) - 1) & 1, a.wait_ns, a.err)) break;
        if (t >= L.nc) {
            sm.info[s][0] = (uint32_t)-1;
            mbar_arrive(&sm.full[s]);
            ++i;
            break;
        }
        const uint64_t e0 = t * kChunk;
        const uint32_t valid = (uint32_t)min((uint64_t)kChunk, a.n - e0);
        uint32_t corrupt = 0, PW = 0, mt = 0;
        if (rec_next < ent.x || bef_next < ent.y || rec_next > R || bef_next > a.m) {
            corrupt = 1;
        } else {
            mt = (uint32_t)(bef_next - ent.y);
            const uint64_t rw = rec_next - ent.x;
            if (rw < 2ull * mt || rw - 2ull * mt > valid) corrupt = 1;
            else PW = (uint32_t)(rw - 2ull * mt);
        }
        if (corrupt) {
            atomicOr(a.err, kErrCorrupt);
            mt = 0;
            PW = 0;
        }
        const uint32_t staged = (mt <= kStagedOutliers) ? 1u : 0u;
        const uint64_t start = L.record_off + 4ull * ent.x;
        const uint64_t a0 = start & ~uint64_t(15);
        const uint32_t adj = (uint32_t)((start - a0) / 4);
        const uint64_t end = start + 4ull * (PW + (staged ? 2ull * mt : 0ull));
        uint64_t a1 = (end + 15) & ~uint64_t(15);
        if (a1 > total16) a1 = total16;
        if (a1 < a0) a1 = a0;
        const uint32_t bulk = corrupt ? 0u : (uint32_t)(a1 - a0);
        if (!corrupt)
            for (uint64_t b = a1; b < end; b += 4)  // ragged end of the stream: plain loads
                sm.rec[s][(b - a0) / 4] = *reinterpret_cast<const uint32_t *>(a.in + b);
        const uint64_t wb0 = L.width_off + t * K;
        const uint64_t wleft = pad16(L.nb) - t * K;
        const uint32_t wbytes = (uint32_t)(wleft < K ? wleft : K);

        sm.info[s][0] = (uint32_t)t;
        sm.info[s][1] = valid;
        sm.info[s][2] = PW;
        sm.info[s][3] = mt;
        sm.info[s][4] = adj;
        sm.info[s][5] = staged;
        sm.info[s][6] = ent.x;
        sm.info[s][7] = corrupt;
        mbar_arrive_expect_tx(&sm.full[s], bulk + wbytes);
        if (bulk) bulk_g2s(sm.rec[s], a.in + a0, bulk, &sm.full[s]);
        bulk_g2s(sm.width[s], a.in + wb0, wbytes, &sm.full[s]);
    }
    for (int s = 0; s < kS; ++s) {
        const uint32_t uses = (i > (uint32_t)s) ? (i - 1 - s) / kS + 1 : 0;
        if (uses) mbar_wait(&sm.full[s], (uses - 1) & 1, a.wait_ns, a.err);
    }
}

template <int V, int LPB, int ND>
__global__ void __launch_bounds__(kThreads, 4) decode_kernel(const DecodeArgs a) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    DecSmem &sm = *reinterpret_cast<DecSmem *>(smem_raw);
    const int warp = threadIdx.x / 32, ln = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kS; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], kNW);
        }
        mbar_init(&sm.stored, kNW);
        mbar_init_fence();
    }
    __syncthreads();
    if (warp < kNW)
        compute_warp<V, LPB, ND>(sm, a, warp, ln);
    else
        producer_warp(sm, a, ln);
}

template <int V, int LPB, int ND>
cudaError_t launch_t(const DecodeArgs &a, int num_sms, cudaStream_t stream) {
    const size_t smem = sizeof(DecSmem);
    cudaError_t e =
        cudaFuncSetAttribute(decode_kernel<V, LPB, ND>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const uint64_t nc = (a.n + kChunk - 1) / kChunk;
    if (nc == 0) return cudaSuccess;
    const uint64_t want = (uint64_t)num_sms * 4;
    const int grid = (int)(want < nc ? want : nc);
    decode_kernel<V, LPB, ND><<<grid, kThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs &a, int num_sms, cudaStream_t stream) {
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
