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

template <int V, int LPB>
__device__ void compute_warp(DecSmem &sm, const DecodeArgs &a, int cw, int ln) {
    constexpr int kB = V * LPB;
    constexpr int kWT = 32 * V;
    constexpr int kWPW = kChunk / kWT / kNW;
    constexpr int kGroups = 32 / LPB;
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
                const uint32_t blk = (uint32_t)(wt * kWT) / kB + g;
                uint32_t w = wid[blk];
                if (w > 32u) {
                    if (r == 0 && blk * kB < valid) atomicOr(a.err, kErrCorrupt);
                    w = 32u;
                }
                uint32_t pre = 0, tot = 0;
#pragma unroll
                for (int gg = 0; gg < kGroups; ++gg) {
                    const uint32_t b = __shfl_sync(kFull, w, gg * LPB);
                    pre += (gg < g) ? b : 0u;
                    tot += b;
                }
                // bit position of this lane's first code in the chunk payload
                const uint32_t bit0 = 32u * kEPL * (before + pre) + (uint32_t)r * V * w;
                const uint32_t mask = (w == 32u) ? kFull : ((1u << w) - 1u);
                int32_t c[V];
                uint32_t run = 0;
                // Every word this lane reads lies in the staged record (widths
                // checked above): one test for the lane instead of one per code.
                const bool inside = ((bit0 + V * w) >> 5) + 1 < kRecWords - adj;
                if (__all_sync(kFull, inside)) {
#pragma unroll
                    for (int v = 0; v < V; ++v) {
                        const uint32_t b = bit0 + v * w;
                        const uint32_t wd = b >> 5;
                        const uint32_t zz = __funnelshift_r(rec[wd], rec[wd + 1], b & 31u) & mask;
                        const uint32_t d = (zz >> 1) ^ (0u - (zz & 1u));  // inverse zigzag
                        run += d;
                        c[v] = (int32_t)run;
                    }
                } else {
#pragma unroll
                    for (int v = 0; v < V; ++v) {
                        const uint32_t b = bit0 + v * w;
                        const uint32_t wd = b >> 5;
                        const uint32_t zz = (wd + 1 < kRecWords - adj)
                                                ? (__funnelshift_r(rec[wd], rec[wd + 1], b & 31u) & mask)
                                                : 0u;
                        const uint32_t d = (zz >> 1) ^ (0u - (zz & 1u));  // inverse zigzag
                        run += d;
                        c[v] = (int32_t)run;
                    }
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
            // the chunk's payload must hold exactly the words its widths call for
            if (cw == kNW - 1) {
                const uint32_t nblk = (valid + kB - 1) / kB;
                uint32_t sum = 0;
                for (uint32_t b = ln; b + 1 < nblk; b += 32) sum += min((uint32_t)wid[b], 32u);
                sum = __reduce_add_sync(kFull, sum);
                const uint32_t last_cnt = valid - (nblk - 1) * kB;
                const uint32_t wl = min((uint32_t)wid[nblk - 1], 32u);
                if (ln == 0 && kEPL * sum + (wl * last_cnt + 31u) / 32u != PW) atomicOr(a.err, kErrCorrupt);
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
                const uint64_t e = (uint64_t)idx - (uint64_t)tile * kChunk;
                if (idx >= (uint64_t)tile * kChunk && e < valid)
                    gout[e] = __uint_as_float(val);
                else
                    atomicOr(a.err, kErrCorrupt);
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
    uint32_t i = 0;
    for (;; ++i) {
        const int s = i % kS;
        if (i >= kS && !mbar_wait(&sm.empty[s], ((i / kS) - 1) & 1, a.wait_ns, a.err)) break;
        const uint64_t t = (uint64_t)blockIdx.x + (uint64_t)i * gridDim.x;
        if (t >= L.nc) {
            sm.info[s][0] = (uint32_t)-1;
            mbar_arrive(&sm.full[s]);
            ++i;
            break;
        }
        const uint64_t e0 = t * kChunk;
        const uint32_t valid = (uint32_t)min((uint64_t)kChunk, a.n - e0);
        const uint2 ent = *reinterpret_cast<const uint2 *>(a.in + L.index_off + 8 * t);
        uint64_t rec_next = R, bef_next = a.m;
        if (t + 1 < L.nc) {
            const uint2 nx = *reinterpret_cast<const uint2 *>(a.in + L.index_off + 8 * (t + 1));
            rec_next = nx.x;
            bef_next = nx.y;
        }
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

template <int V, int LPB>
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
        compute_warp<V, LPB>(sm, a, warp, ln);
    else
        producer_warp(sm, a, ln);
}

template <int V, int LPB>
cudaError_t launch_t(const DecodeArgs &a, int num_sms, cudaStream_t stream) {
    const size_t smem = sizeof(DecSmem);
    cudaError_t e =
        cudaFuncSetAttribute(decode_kernel<V, LPB>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const uint64_t nc = (a.n + kChunk - 1) / kChunk;
    if (nc == 0) return cudaSuccess;
    const uint64_t want = (uint64_t)num_sms * 4;
    const int grid = (int)(want < nc ? want : nc);
    decode_kernel<V, LPB><<<grid, kThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs &a, int num_sms, cudaStream_t stream) {
    switch (a.block) {
        case 32: return launch_t<8, 4>(a, num_sms, stream);
        case 64: return launch_t<8, 8>(a, num_sms, stream);
        case 128: return launch_t<8, 16>(a, num_sms, stream);
        case 256: return launch_t<8, 32>(a, num_sms, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace eblc
