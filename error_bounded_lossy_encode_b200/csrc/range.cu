// range.cu -- value range (min, max) over the finite elements.
//
// "Pipeline specialization internals", Priming: the quantizer runs a
// value-range scan and resolves the bound before the fused kernel, because a
// relative bound eb = rel * (max - min) must be known before any code is
// produced.  This is the compulsory first read of the input in relative mode.
//
// HBM-bound: 4 bytes read per element, no writes.  Persistent grid of one
// wave of 256-thread CTAs; each thread keeps 16 float4 loads in flight.
// The array is walked from its end to its start so the lowest addresses are
// the last read and are still in L2 when the encoder starts at tile 0: the
// lowest kKeep4 float4 (48 MiB) are loaded with the normal L2 policy and a
// 256-byte L2 prefetch hint, everything above with evict-first streaming
// loads, so the streamed part does not push the kept part out of L2.
#include "common.cuh"
#include "kernels.h"

namespace eblc {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 16;
constexpr uint64_t kKeep4 = 3ull << 20;  // float4 at the array's start kept in L2 for the encoder

__device__ __forceinline__ void fold(float v, float &lo, float &hi) {
    // +-Inf become NaN, which fminf / fmaxf ignore (as they ignore NaN itself)
    const float f = (fabsf(v) < __int_as_float(0x7f800000)) ? v : __int_as_float(0x7fffffff);
    lo = fminf(lo, f);
    hi = fmaxf(hi, f);
}

__device__ __forceinline__ float4 ld_nc_256(const float4 *p) {
    float4 v;
    asm volatile("ld.global.nc.L2::256B.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p));
    return v;
}

__global__ void __launch_bounds__(kThreads) range_kernel(RangeArgs a) {
    float lo = __int_as_float(0x7f800000), hi = __int_as_float(0xff800000);
    const float4 *in4 = reinterpret_cast<const float4 *>(a.in);
    const uint64_t n4 = a.n / 4;
    const uint64_t stride = (uint64_t)gridDim.x * kThreads;
    const uint64_t tid = (uint64_t)blockIdx.x * kThreads + threadIdx.x;

    for (uint64_t base = 0; base < n4; base += stride * kUnroll) {
        float4 v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const uint64_t i = base + u * stride + tid;
            const uint64_t j = n4 - 1 - i;
            v[u] = (i < n4) ? ((j < kKeep4) ? ld_nc_256(in4 + j) : __ldcs(in4 + j)) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const uint64_t i = base + u * stride + tid;
            if (i < n4) {
                fold(v[u].x, lo, hi);
                fold(v[u].y, lo, hi);
                fold(v[u].z, lo, hi);
                fold(v[u].w, lo, hi);
            }
        }
    }
    if (blockIdx.x == 0 && threadIdx.x < (a.n & 3)) fold(a.in[n4 * 4 + threadIdx.x], lo, hi);

#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    __shared__ float2 warp_part[kThreads / 32];
    __shared__ bool is_last;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (lane == 0) warp_part[warp] = make_float2(lo, hi);
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < kThreads / 32; ++w) {
            lo = fminf(lo, warp_part[w].x);
            hi = fmaxf(hi, warp_part[w].y);
        }
        a.partials[blockIdx.x] = make_float2(lo, hi);
        __threadfence();
        const uint32_t done = atomicAdd(a.counter, 1u);
        is_last = (done == gridDim.x - 1);
    }
    __syncthreads();
    if (!is_last) return;

    // Last CTA: fold the per-CTA partials (in CTA order) and publish.
    __threadfence();
    lo = __int_as_float(0x7f800000);
    hi = __int_as_float(0xff800000);
    for (uint32_t i = threadIdx.x; i < gridDim.x; i += kThreads) {
        const float2 p = __ldcg(a.partials + i);
        lo = fminf(lo, p.x);
        hi = fmaxf(hi, p.y);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    __syncthreads();
    if (lane == 0) warp_part[warp] = make_float2(lo, hi);
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < kThreads / 32; ++w) {
            lo = fminf(lo, warp_part[w].x);
            hi = fmaxf(hi, warp_part[w].y);
        }
        if (!(lo <= hi)) {  // no finite element
            lo = 0.0f;
            hi = 0.0f;
        }
        a.range_out[0] = __fadd_rn(lo, 0.0f);  // canonical +0 for a zero end
        a.range_out[1] = __fadd_rn(hi, 0.0f);
        *a.counter = 0;
    }
}

}  // namespace

// One wave of resident CTAs (occupancy is set by the registers of the
// 16-deep load unroll), at most 8 per SM.
int range_grid(int num_sms) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, range_kernel, kThreads, 0) != cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    return num_sms * (per_sm < 8 ? per_sm : 8);
}

cudaError_t launch_range(const RangeArgs &a, int grid, cudaStream_t stream) {
    range_kernel<<<grid, kThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace eblc
