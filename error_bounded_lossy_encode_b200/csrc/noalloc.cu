// noalloc.cu -- eblc_compress_noalloc: compress without any device memory
// allocation by the library.
//
// Some callers cannot call cudaMalloc: code running under an allocator that
// owns all device memory (a framework caching allocator or a memory pool
// that must not be bypassed), code inside a region where allocation is
// forbidden or would synchronise the device, and callers that must not grow
// the device footprint behind their back.  They can still compress with this
// entry point: it needs no plan, and the scratch the range and encode kernels
// use (look-back status words, error words, range partials,
// the result block) lives in one file-scope __device__ array of fixed size,
// which every GPU that loads this library holds until the process exits.
// The caller passes the input and the output buffer, as with eblc_compress.
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/eblc.h"
#include "common.cuh"
#include "kernels.h"

using namespace eblc;

namespace {

constexpr uint64_t kMaxTiles = EBLC_NOALLOC_MAX_N / kChunk;
constexpr int kMaxRangeParts = 4096;
constexpr int kMaxDevices = 64;

struct NoallocScratch {
    // cleared at the start of every call
    uint32_t err;
    uint32_t epoch;          // stays 0: every call uses look-back array 0, cleared here
    uint32_t range_counter;
    uint32_t pad[5];
    uint64_t result[8];
    float range[4];          // vmin, vmax: zero when the range kernel does not run (n == 0)
    // written before being read within a call
    float2 partials[kMaxRangeParts];
    uint64_t status[2][kMaxTiles];
};
constexpr size_t kClearBytes = offsetof(NoallocScratch, partials);

static __device__ __align__(256) NoallocScratch g_noalloc_scratch;

std::mutex g_setup_mutex;
NoallocScratch *g_scratch_ptr[kMaxDevices] = {};

// Device address of the array on the current device.  Host code must not use
// &g_noalloc_scratch directly (it is a host-side stand-in, not a device
// address); the address comes from cudaGetSymbolAddress, once per device.
cudaError_t scratch_on_current_device(int dev, NoallocScratch **out) {
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_ptr[dev]) {
        NoallocScratch *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void **>(&p), g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" EBLC_API eblc_status_t eblc_compress_noalloc(const float *d_in, uint64_t n, uint32_t block, int abs_mode,
                                                        double bound, void *d_out, size_t out_capacity,
                                                        void *stream, size_t *compressed_bytes, void *h_sidecar) {
    if (compressed_bytes) *compressed_bytes = 0;
    if (n > EBLC_NOALLOC_MAX_N) {
        std::fprintf(stderr, "[eblc] eblc_compress_noalloc: n = %llu exceeds the no-allocation limit of %llu "
                             "elements; use a plan (eblc_plan_create + eblc_compress)\n",
                     (unsigned long long)n, (unsigned long long)EBLC_NOALLOC_MAX_N);
        return EBLC_UNSUPPORTED;
    }
    if (block != 32 && block != 64 && block != 128 && block != 256) return EBLC_UNSUPPORTED;
    if (!(bound >= 0.0) || bound > 1.7976931348623157e308) return EBLC_INVALID_ARG;
    if (!d_out || (n && !d_in) || !aligned16(d_out) || (d_in && !aligned16(d_in))) return EBLC_INVALID_ARG;
    if (h_sidecar && (reinterpret_cast<uintptr_t>(h_sidecar) & 7u)) return EBLC_INVALID_ARG;
    const Layout L = stream_layout(n, block);
    if (out_capacity < L.record_off) return EBLC_CAPACITY;

    int dev = 0, major = 0, minor = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return EBLC_CUDA_ERROR;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return EBLC_CUDA_ERROR;
    if (major != 10 || minor != 0 || sms <= 0 || range_grid(sms) > kMaxRangeParts) return EBLC_UNSUPPORTED;
    NoallocScratch *S = nullptr;
    if (scratch_on_current_device(dev, &S) != cudaSuccess) return EBLC_CUDA_ERROR;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const uint64_t ntiles = L.nc;
    if (cudaMemsetAsync(S, 0, kClearBytes, st) != cudaSuccess) return EBLC_CUDA_ERROR;
    if (ntiles && cudaMemsetAsync(S->status[0], 0, 8 * ntiles, st) != cudaSuccess) return EBLC_CUDA_ERROR;
    if (!abs_mode && n > 0) {
        RangeArgs ra{d_in, n, S->partials, &S->range_counter, S->range};
        if (launch_range(ra, range_grid(sms), st) != cudaSuccess) return EBLC_CUDA_ERROR;
    }
    EncodeArgs ea{};
    ea.in = d_in;
    ea.n = n;
    ea.out = static_cast<uint8_t *>(d_out);
    ea.out_cap = out_capacity;
    ea.block = block;
    ea.abs_mode = abs_mode ? 1 : 0;
    ea.bound = bound;
    ea.range = S->range;
    ea.status = &S->status[0][0];
    ea.ntiles = kMaxTiles;
    ea.epoch = &S->epoch;
    ea.err = &S->err;
    ea.result = S->result;
    ea.outlier_cap = n;
    ea.stall_tile = -1;
    ea.wait_ns = 2000ull * 1000000ull;
    if (launch_encode(ea, sms, st) != cudaSuccess) return EBLC_CUDA_ERROR;

    struct {
        uint64_t result[8];
        uint32_t err;
    } rb;
    if (cudaMemcpyAsync(rb.result, S->result, sizeof(rb.result), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaMemcpyAsync(&rb.err, &S->err, sizeof(rb.err), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return EBLC_CUDA_ERROR;
    if (compressed_bytes) *compressed_bytes = (size_t)rb.result[2];
    if (h_sidecar) {
        eblc_sidecar_t sc{};
        sc.magic = kMagic;
        sc.version = (uint16_t)kVersion;
        sc.flags = (uint16_t)(abs_mode ? kFlagAbs : 0);
        sc.block = block;
        sc.chunk = kChunk;
        sc.n = n;
        sc.total_bytes = rb.result[2];
        sc.payload_words = rb.result[0];
        sc.n_outliers = rb.result[1];
        std::memcpy(&sc.eb, &rb.result[4], 8);
        const uint32_t stepbits = (uint32_t)rb.result[5], invbits = (uint32_t)(rb.result[5] >> 32);
        std::memcpy(&sc.step, &stepbits, 4);
        std::memcpy(&sc.inv2eb, &invbits, 4);
        std::memcpy(h_sidecar, &sc, sizeof(sc));
    }
    if (rb.err & kErrTimeout) return EBLC_TIMEOUT;
    if (rb.err & kErrCapacity) return EBLC_CAPACITY;
    return EBLC_OK;
}
