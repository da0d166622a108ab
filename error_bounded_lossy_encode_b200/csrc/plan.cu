// plan.cu -- host side of the libeblc C ABI (include/eblc.h): option
// parsing, sizing, plan-owned scratch, launch sequence, result readback.
//
// The interface follows "DevitoComp provider interface" (Provider layout:
// plan_create with an options string, dims/strides slowest to fastest in
// elements, HOST/CUDA/HIP execution descriptor with an optional stream,
// a host sidecar ready on return, device work that may stay queued, a
// payload alignment reported through the limits, UNSUPPORTED for what a
// provider does not do).  Compress ends with one stream synchronisation,
// as "nvrtc_chunk_fusion.h File Reference" describes for
// launchGenericChunkFusion (the archive length and the outlier count are
// read back after a stream sync).
#include <algorithm>
#include <atomic>
#include <cerrno>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <string>

#include <cudaTypedefs.h>  // PFN_cuTensorMapEncodeTiled

#include "../../include/eblc.h"
#include "common.cuh"
#include "kernels.h"

using namespace eblc;

namespace {

constexpr uint64_t kPayloadAlignment = 16;
constexpr uint64_t kSidecarBytes = 64;
constexpr uint64_t kSidecarAlignment = 8;
static_assert(sizeof(eblc_sidecar_t) == 64, "sidecar layout");
static_assert(sizeof(eblc_limits_t) == 72, "limits layout");
static_assert(sizeof(eblc_execution_t) == 16, "execution descriptor layout");

bool log_enabled() {
    static const bool on = [] {
        const char *e = std::getenv("EBLC_LOG");
        return e && *e && std::strcmp(e, "0") != 0;
    }();
    return on;
}

#define EBLC_LOG(...)                              \
    do {                                           \
        if (log_enabled()) {                       \
            std::fprintf(stderr, "[eblc] " __VA_ARGS__); \
            std::fputc('\n', stderr);              \
        }                                          \
    } while (0)

// Device scratch owned by a plan: look-back status words (two arrays, used
// alternately by consecutive calls as the device-side call counter says),
// error word, range partials, readback block.
struct Readback {
    uint64_t result[8];  // W, m, total, R, eb bits, step|inv2eb, vmin|vmax, the call's error bits
    uint32_t err;        // error word of the running call (cleared by the finish kernel)
    uint32_t epoch;      // calls finished on the device: selects the look-back array
};

// Per-call device timing (option timing=1): a start/end event pair around
// each kernel launch and one pair around the whole call (first launch to the
// end of the result readback).
struct Timing {
    bool on = false;
    cudaEvent_t ev[8] = {};
    const char *name[3] = {};
    int count = 0;
};

}  // namespace

struct eblc_plan_s {
    int device = 0;
    int num_sms = 0;
    uint64_t n = 0;
    uint32_t block = 128;
    int abs_mode = 0;
    double bound = 1e-4;
    uint64_t outlier_cap = 0;
    uint64_t wait_ns = 2000ull * 1000000ull;
    int64_t stall_tile = -1;
    int nd = 0;                     // option lorenzo=nd: 2 or 3 (the plan's rank), 0 for the 1-D path
    uint32_t chunked_m = 0;         // option codec=chunked: elements per chunk (1024, 2048, 4096), else 0
    int opt_chunked = 0;            // options as parsed (resolved by plan_create)
    int opt_coder = -1;             // option coder=: -1 unset, 0 rze, 1 rre (codec=chunked only)
    int chunked_rre = 0;            // codec=chunked with the RRE coder
    uint32_t opt_chunk_bytes = 0;
    uint32_t *chunk_scratch = nullptr;  // codec=chunked: nc record slots, then sizes, outlier counts, range totals
    uint64_t dims[3] = {0, 0, 0};   // {Z, Y, X} of a multi-dimensional plan (Z = 1 for 2-D)
    uint64_t stall_call = 0;        // the compress call (0-based) that stall_tile applies to
    uint64_t calls = 0;             // compress calls enqueued so far
    Layout L{};
    uint64_t max_bytes = 0;

    void *scratch = nullptr;
    uint64_t *status = nullptr;     // 2 x ntiles look-back words
    uint64_t ntiles = 0;
    Readback *d_rb = nullptr;       // device copy of the readback block
    uint32_t *dec_err = nullptr;
    float2 *partials = nullptr;
    uint32_t *range_counter = nullptr;
    float *range = nullptr;
    int range_grid = 0;
    Readback *h_rb = nullptr;       // pinned
    uint32_t *h_err = nullptr;      // pinned

    // HOST execution: device staging, allocated on first use
    float *stage_in = nullptr;
    uint8_t *stage_out = nullptr;
    cudaStream_t host_stream = nullptr;

    Timing timing;
};

namespace {

struct DeviceGuard {
    int prev = -1;
    bool ok = true;
    explicit DeviceGuard(int dev) {
        if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
        if (prev != dev) ok = cudaSetDevice(dev) == cudaSuccess;
    }
    ~DeviceGuard() {
        if (prev >= 0) cudaSetDevice(prev);
    }
};

eblc_status_t cuda_status(cudaError_t e, const char *what) {
    if (e == cudaSuccess) return EBLC_OK;
    EBLC_LOG("%s: %s", what, cudaGetErrorString(e));
    return (e == cudaErrorMemoryAllocation) ? EBLC_NOMEM : EBLC_CUDA_ERROR;
}

bool parse_double(const std::string &s, double *out) {
    if (s.empty()) return false;
    errno = 0;
    char *end = nullptr;
    const double v = std::strtod(s.c_str(), &end);
    if (errno != 0 || end != s.c_str() + s.size()) return false;
    *out = v;
    return true;
}

bool parse_int(const std::string &s, int64_t *out) {
    if (s.empty()) return false;
    errno = 0;
    char *end = nullptr;
    const long long v = std::strtoll(s.c_str(), &end, 10);
    if (errno != 0 || end != s.c_str() + s.size()) return false;
    *out = v;
    return true;
}

std::string trim(const std::string &s) {
    size_t a = 0, b = s.size();
    while (a < b && (s[a] == ' ' || s[a] == '\t')) ++a;
    while (b > a && (s[b - 1] == ' ' || s[b - 1] == '\t')) --b;
    return s.substr(a, b - a);
}

eblc_status_t parse_options(const char *options, eblc_plan_s *p, bool *timing) {
    p->abs_mode = 0;
    p->bound = 1e-4;  // default relative bound ("Pipeline specialization internals", Priming)
    p->block = 128;
    *timing = false;
    if (!options) return EBLC_OK;
    const std::string all(options);
    double v;
    if (parse_double(trim(all), &v)) {  // a bare decimal is a relative bound
        if (!std::isfinite(v) || v < 0) return EBLC_INVALID_ARG;
        p->bound = v;
        return EBLC_OK;
    }
    size_t pos = 0;
    bool have_bound = false;
    while (pos <= all.size()) {
        size_t comma = all.find(',', pos);
        if (comma == std::string::npos) comma = all.size();
        const std::string item = trim(all.substr(pos, comma - pos));
        pos = comma + 1;
        if (item.empty()) {
            if (comma == all.size()) break;
            continue;
        }
        const size_t eq = item.find('=');
        if (eq == std::string::npos) return EBLC_INVALID_ARG;
        const std::string key = trim(item.substr(0, eq)), val = trim(item.substr(eq + 1));
        int64_t iv = 0;
        if (key == "rel" || key == "abs") {
            if (have_bound || !parse_double(val, &v) || !std::isfinite(v) || v < 0) return EBLC_INVALID_ARG;
            p->abs_mode = (key == "abs");
            p->bound = v;
            have_bound = true;
        } else if (key == "block") {
            if (!parse_int(val, &iv)) return EBLC_INVALID_ARG;
            if (iv != 32 && iv != 64 && iv != 128 && iv != 256) return EBLC_UNSUPPORTED;
            p->block = (uint32_t)iv;
        } else if (key == "outlier_cap") {
            if (!parse_int(val, &iv) || iv < 0) return EBLC_INVALID_ARG;
            p->outlier_cap = (uint64_t)iv;  // clamped to n by the caller
        } else if (key == "codec") {
            if (val == "chunked") p->opt_chunked = 1;
            else if (val != "lorenzo") return EBLC_INVALID_ARG;
        } else if (key == "coder") {  // zero elimination of the chunked codec: rze or rre
            if (val == "rze") p->opt_coder = 0;
            else if (val == "rre") p->opt_coder = 1;
            else return EBLC_INVALID_ARG;
        } else if (key == "chunk") {  // bytes of float32 input per chunk of the chunked codec
            if (!parse_int(val, &iv)) return EBLC_INVALID_ARG;
            if (iv != 4096 && iv != 8192 && iv != 16384) return EBLC_UNSUPPORTED;
            p->opt_chunk_bytes = (uint32_t)iv;
        } else if (key == "lorenzo") {
            if (val == "nd") p->nd = -1;  // resolved against the dims by the caller
            else if (val != "1d") return EBLC_INVALID_ARG;
        } else if (key == "timing") {
            if (!parse_int(val, &iv)) return EBLC_INVALID_ARG;
            *timing = iv != 0;
        } else if (key == "wait_ms") {
            if (!parse_int(val, &iv) || iv <= 0 || iv > 600000) return EBLC_INVALID_ARG;
            p->wait_ns = (uint64_t)iv * 1000000ull;
        } else if (key == "stall_tile") {
            if (!parse_int(val, &iv) || iv < -1) return EBLC_INVALID_ARG;
            p->stall_tile = iv;
        } else if (key == "stall_call") {
            if (!parse_int(val, &iv) || iv < 0) return EBLC_INVALID_ARG;
            p->stall_call = (uint64_t)iv;
        } else {
            return EBLC_UNSUPPORTED;
        }
    }
    return EBLC_OK;
}

template <typename T>
T *carve(uint8_t *base, size_t *off, size_t count) {
    *off = (*off + 255) & ~size_t(255);
    T *p = reinterpret_cast<T *>(reinterpret_cast<uintptr_t>(base) + *off);
    *off += count * sizeof(T);
    return p;
}

void destroy(eblc_plan_s *p) {
    if (!p) return;
    DeviceGuard g(p->device);
    for (cudaEvent_t &e : p->timing.ev)
        if (e) cudaEventDestroy(e);
    if (p->scratch) cudaFree(p->scratch);
    if (p->chunk_scratch) cudaFree(p->chunk_scratch);
    if (p->stage_in) cudaFree(p->stage_in);
    if (p->stage_out) cudaFree(p->stage_out);
    if (p->host_stream) cudaStreamDestroy(p->host_stream);
    if (p->h_rb) cudaFreeHost(p->h_rb);
    if (p->h_err) cudaFreeHost(p->h_err);
    delete p;
}

bool aligned16(const void *ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

void timing_begin(eblc_plan_s *p, cudaStream_t st) {
    p->timing.count = 0;
    if (p->timing.on) cudaEventRecord(p->timing.ev[6], st);
}

void timing_end(eblc_plan_s *p, cudaStream_t st) {
    if (p->timing.on) cudaEventRecord(p->timing.ev[7], st);
}

void timing_mark(eblc_plan_s *p, cudaStream_t st, bool start, const char *name) {
    if (!p->timing.on) return;
    Timing &t = p->timing;
    if (start) {
        if (t.count >= 3) return;
        t.name[t.count] = name;
        cudaEventRecord(t.ev[2 * t.count], st);
    } else {
        cudaEventRecord(t.ev[2 * t.count + 1], st);
        ++t.count;
    }
}

eblc_status_t ensure_host_staging(eblc_plan_s *p) {
    if (p->stage_in) return EBLC_OK;
    eblc_status_t s = cuda_status(cudaMalloc(&p->stage_in, std::max<uint64_t>(4 * p->n, 16)), "cudaMalloc");
    if (s == EBLC_OK) s = cuda_status(cudaMalloc(&p->stage_out, p->max_bytes), "cudaMalloc");
    if (s == EBLC_OK) s = cuda_status(cudaStreamCreateWithFlags(&p->host_stream, cudaStreamNonBlocking), "stream");
    if (s != EBLC_OK) {
        if (p->stage_in) cudaFree(p->stage_in);
        if (p->stage_out) cudaFree(p->stage_out);
        p->stage_in = nullptr;
        p->stage_out = nullptr;
    }
    return s;
}

// Queue the compress kernels on `st` (device pointers).
// call_events: record the "call" timing pair around this enqueue (false when
// the caller brackets a larger span, e.g. the HOST kind's copies).
// d_user: NULL for the synchronous calls (the result block is copied to the
// pinned readback), else the caller's device result record (no copy back).
// Tiled tensor map of a multi-dimensional plan's input at d_in: dims {X, Y[, Z]}
// innermost first, a brick (16^3, or 64x64 in 2-D) per box, no swizzle, so a
// box lands in shared memory in C order.  The encoder is taken from the
// driver once per process.
eblc_status_t encode_tensor_map(const eblc_plan_s *p, const float *d_in, CUtensorMap *out) {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            f = nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }();
    if (!fn) return EBLC_CUDA_ERROR;
    const cuuint32_t rank = (cuuint32_t)p->nd;
    cuuint64_t gdim[3] = {p->dims[2], p->dims[1], p->dims[0]};
    cuuint64_t gstride[2] = {p->dims[2] * 4, p->dims[2] * p->dims[1] * 4};  // bytes, of dims 1 and 2
    cuuint32_t box[3] = {(p->nd == 3) ? 16u : 64u, (p->nd == 3) ? 16u : 64u, 16u};
    cuuint32_t estride[3] = {1, 1, 1};
    const CUresult r = fn(out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, rank, const_cast<float *>(d_in), gdim, gstride, box,
                          estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        EBLC_LOG("cuTensorMapEncodeTiled failed (%d)", (int)r);
        return EBLC_CUDA_ERROR;
    }
    return EBLC_OK;
}

// given_range: NULL, or a device float[2] {vmin, vmax} that replaces the
// value range of d_in (relative bound; the range kernel is not run).
eblc_status_t enqueue_compress(eblc_plan_s *p, cudaStream_t st, const float *d_in, uint8_t *d_out, uint64_t cap,
                               bool call_events = true, uint64_t *d_user = nullptr,
                               const float *given_range = nullptr) {
    if (call_events)
        timing_begin(p, st);
    else
        p->timing.count = 0;
    if (!p->abs_mode && p->n > 0 && !given_range) {
        RangeArgs ra{d_in, p->n, p->partials, p->range_counter, p->range};
        timing_mark(p, st, true, "range");
        eblc_status_t s = cuda_status(launch_range(ra, p->range_grid, st), "range launch");
        timing_mark(p, st, false, nullptr);
        if (s != EBLC_OK) return s;
    }
    if (p->chunked_m) {
        const uint64_t slot = chunked_slot_words(p->chunked_m);
        ChunkedArgs ca{};
        ca.in = d_in;
        ca.n = p->n;
        ca.m = p->chunked_m;
        ca.nc = p->L.nc;
        ca.abs_mode = p->abs_mode;
        ca.bound = p->bound;
        ca.range = given_range ? given_range : p->range;
        ca.scratch = p->chunk_scratch;
        ca.slot_words = (uint32_t)slot;
        ca.sizes = p->chunk_scratch ? p->chunk_scratch + p->L.nc * slot : nullptr;
        ca.outl = ca.sizes ? ca.sizes + p->L.nc : nullptr;
        ca.part = ca.outl ? ca.outl + p->L.nc : nullptr;
        ca.rre = p->chunked_rre;
        ca.out = d_out;
        ca.out_cap = cap;
        ca.result = p->d_rb->result;
        ca.err = &p->d_rb->err;
        ca.outlier_cap = p->outlier_cap;
        timing_mark(p, st, true, "encode");
        eblc_status_t s = cuda_status(launch_chunked_encode(ca, p->num_sms, st), "chunked encode launch");
        timing_mark(p, st, false, nullptr);
        if (s != EBLC_OK) return s;
        FinishArgs fa{p->d_rb->result, &p->d_rb->err, &p->d_rb->epoch, d_user, p->status, 2 * p->ntiles};
        if ((s = cuda_status(launch_finish(fa, st), "finish launch")) != EBLC_OK) return s;
        if (!d_user)
            s = cuda_status(cudaMemcpyAsync(p->h_rb, p->d_rb, sizeof(Readback), cudaMemcpyDeviceToHost, st),
                            "readback");
        if (call_events) timing_end(p, st);
        return s;
    }
    EncodeArgs ea{};
    ea.in = d_in;
    ea.n = p->n;
    ea.out = d_out;
    ea.out_cap = cap;
    ea.block = p->block;
    ea.abs_mode = p->abs_mode;
    ea.bound = p->bound;
    ea.range = given_range ? given_range : p->range;
    ea.range_given = given_range ? 1 : 0;
    ea.status = p->status;
    ea.ntiles = p->ntiles;
    ea.epoch = &p->d_rb->epoch;
    ea.err = &p->d_rb->err;
    ea.result = p->d_rb->result;
    ea.outlier_cap = p->outlier_cap;
    ea.stall_tile = (p->calls++ == p->stall_call) ? p->stall_tile : -1;
    ea.wait_ns = p->wait_ns;
    ea.nd = p->nd;
    for (int d = 0; d < 3; ++d) ea.dims[d] = p->dims[d];
    if (p->nd && p->n > 0) {
        eblc_status_t t = encode_tensor_map(p, d_in, &ea.tmap);
        if (t != EBLC_OK) return t;
    }
    timing_mark(p, st, true, "encode");
    eblc_status_t s = cuda_status(launch_encode(ea, p->num_sms, st), "encode launch");
    timing_mark(p, st, false, nullptr);
    if (s != EBLC_OK) return s;
    FinishArgs fa{p->d_rb->result, &p->d_rb->err, &p->d_rb->epoch, d_user, p->status, 2 * p->ntiles};
    if ((s = cuda_status(launch_finish(fa, st), "finish launch")) != EBLC_OK) return s;
    if (!d_user)
        s = cuda_status(cudaMemcpyAsync(p->h_rb, p->d_rb, sizeof(Readback), cudaMemcpyDeviceToHost, st), "readback");
    if (call_events) timing_end(p, st);
    return s;
}

// The plan's decoder: the block codec or the chunked one.
cudaError_t launch_plan_decode(const eblc_plan_s *p, const DecodeArgs &da, cudaStream_t st) {
    if (!p->chunked_m) return launch_decode(da, p->num_sms, st);
    ChunkedDecArgs ca{};
    ca.in = da.in;
    ca.n = da.n;
    ca.m = p->chunked_m;
    ca.W = da.W;
    ca.mo = da.m;
    ca.step = da.step;
    ca.out = da.out;
    ca.err = da.err;
    ca.rre = p->chunked_rre;
    return launch_chunked_decode(ca, p->num_sms, st);
}

eblc_status_t finish_compress(eblc_plan_s *p, size_t *compressed_bytes, void *h_sidecar) {
    const Readback &rb = *p->h_rb;
    const uint32_t err = (uint32_t)rb.result[7];
    const uint64_t total = rb.result[2];
    if (compressed_bytes) *compressed_bytes = (size_t)total;
    if (h_sidecar) {
        eblc_sidecar_t sc{};
        sc.magic = kMagic;
        sc.version = (uint16_t)kVersion;
        sc.flags = (uint16_t)((p->abs_mode ? kFlagAbs : 0) | (p->nd ? kFlagLorenzoNd : 0) |
                              (p->chunked_m ? kFlagChunked : 0) | (p->chunked_rre ? kFlagRre : 0));
        sc.block = p->block;
        sc.chunk = p->chunked_m ? p->chunked_m : kChunk;
        sc.n = p->n;
        sc.total_bytes = total;
        sc.payload_words = rb.result[0];
        sc.n_outliers = rb.result[1];
        uint64_t ebits = rb.result[4];
        std::memcpy(&sc.eb, &ebits, 8);
        const uint32_t stepbits = (uint32_t)rb.result[5], invbits = (uint32_t)(rb.result[5] >> 32);
        std::memcpy(&sc.step, &stepbits, 4);
        std::memcpy(&sc.inv2eb, &invbits, 4);
        std::memcpy(h_sidecar, &sc, sizeof(sc));
    }
    if (err & kErrTimeout) return EBLC_TIMEOUT;
    if (err & kErrRange) return EBLC_INVALID_ARG;
    if (err & kErrCapacity) return EBLC_CAPACITY;
    if (err & kErrCorrupt) return EBLC_CORRUPT;
    return EBLC_OK;
}

struct StreamInfo {
    uint64_t total, W, m;
    float step;
};

// Validate the sidecar (or the header it was rebuilt from) against the plan.
eblc_status_t check_stream(const eblc_plan_s *p, const eblc_sidecar_t &sc, size_t compressed_bytes,
                           StreamInfo *info) {
    if (sc.magic != kMagic || sc.version != kVersion) return EBLC_CORRUPT;
    if (sc.chunk != (p->chunked_m ? p->chunked_m : kChunk)) return p->chunked_m ? EBLC_INVALID_ARG : EBLC_CORRUPT;
    if (((sc.flags & kFlagChunked) != 0) != (p->chunked_m != 0)) return EBLC_INVALID_ARG;  // the plan's codec
    if (((sc.flags & kFlagRre) != 0) != (p->chunked_rre != 0)) return EBLC_INVALID_ARG;     // and its coder
    if (sc.n != p->n || sc.block != p->block) return EBLC_INVALID_ARG;
    if (((sc.flags & kFlagLorenzoNd) != 0) != (p->nd != 0)) return EBLC_INVALID_ARG;  // the plan's predictor
    if (sc.payload_words > sc.n + 32 * p->L.nc || sc.n_outliers > sc.n) return EBLC_CORRUPT;
    const uint64_t total = p->L.record_off + 4 * (sc.payload_words + 2 * sc.n_outliers);
    if (total != sc.total_bytes || compressed_bytes < total) return EBLC_CORRUPT;
    info->total = total;
    info->W = sc.payload_words;
    info->m = sc.n_outliers;
    info->step = sc.step;
    return EBLC_OK;
}

// Rebuild a sidecar from the 128-byte stream header.
eblc_sidecar_t sidecar_from_header(const uint8_t *h) {
    eblc_sidecar_t sc{};
    auto u16 = [&](int o) { uint16_t v; std::memcpy(&v, h + o, 2); return v; };
    auto u32 = [&](int o) { uint32_t v; std::memcpy(&v, h + o, 4); return v; };
    auto u64 = [&](int o) { uint64_t v; std::memcpy(&v, h + o, 8); return v; };
    sc.magic = u32(0);
    sc.version = u16(4);
    sc.flags = u16(6);
    sc.n = u64(8);
    sc.block = u32(16);
    sc.chunk = u32(20);
    std::memcpy(&sc.eb, h + 24, 8);
    std::memcpy(&sc.inv2eb, h + 32, 4);
    std::memcpy(&sc.step, h + 36, 4);
    sc.payload_words = u64(64);
    sc.n_outliers = u64(72);
    sc.total_bytes = u64(80);
    return sc;
}

eblc_status_t device_error_status(uint32_t err) {
    if (err & kErrTimeout) return EBLC_TIMEOUT;
    if (err & kErrCorrupt) return EBLC_CORRUPT;
    if (err & kErrCapacity) return EBLC_CAPACITY;
    return EBLC_OK;
}

}  // namespace

// ---------------------------------------------------------------------------
extern "C" {

EBLC_API uint32_t eblc_abi_version(void) { return EBLC_ABI_VERSION; }

EBLC_API const char *eblc_status_string(eblc_status_t s) {
    switch (s) {
        case EBLC_OK: return "ok";
        case EBLC_UNSUPPORTED: return "unsupported";
        case EBLC_INVALID_ARG: return "invalid argument";
        case EBLC_CAPACITY: return "capacity exceeded";
        case EBLC_CORRUPT: return "corrupt stream";
        case EBLC_CUDA_ERROR: return "CUDA error";
        case EBLC_TIMEOUT: return "device wait timed out";
        case EBLC_NOMEM: return "out of memory";
    }
    return "unknown status";
}

EBLC_API eblc_status_t eblc_plan_create(eblc_plan_t *out, int rank, const int64_t *dims, const int64_t *strides,
                                        const char *options) {
    if (!out) return EBLC_INVALID_ARG;
    *out = nullptr;
    if (rank < 1 || rank > 8 || !dims) return EBLC_INVALID_ARG;
    bool zero = false, too_big = false;
    uint64_t n = 1;
    for (int i = 0; i < rank; ++i) {
        if (dims[i] < 0) return EBLC_INVALID_ARG;
        if (dims[i] == 0) zero = true;
        else if (!too_big && n > kMaxN / (uint64_t)dims[i]) too_big = true;
        else if (!too_big) n *= (uint64_t)dims[i];
    }
    if (zero) n = 0;
    else if (too_big || n > kMaxN) return EBLC_UNSUPPORTED;
    if (strides && n > 0) {  // only C-contiguous layouts (strides in elements, slowest to fastest)
        int64_t expect = 1;
        for (int i = rank - 1; i >= 0; --i) {
            if (dims[i] != 1 && strides[i] != expect) return EBLC_UNSUPPORTED;
            expect *= dims[i];
        }
    }

    eblc_plan_s *p = new (std::nothrow) eblc_plan_s;
    if (!p) return EBLC_NOMEM;
    p->outlier_cap = UINT64_MAX;
    bool timing = false;
    eblc_status_t s = parse_options(options, p, &timing);
    if (s != EBLC_OK) {
        delete p;
        return s;
    }
    p->n = n;
    if ((p->opt_chunk_bytes || p->opt_coder >= 0) && !p->opt_chunked) {  // chunk= and coder= belong to codec=chunked
        delete p;
        return EBLC_INVALID_ARG;
    }
    if (p->opt_chunked) {
        if (p->nd) {  // one codec per plan
            delete p;
            return EBLC_UNSUPPORTED;
        }
        p->chunked_m = (p->opt_chunk_bytes ? p->opt_chunk_bytes : 16384) / 4;
        p->chunked_rre = p->opt_coder == 1;
        p->block = 0;  // no blocks: the stream has no width bytes
    }
    if (p->nd) {  // multi-dimensional Lorenzo: rank 2 or 3, dims multiples of the brick, block 64 or 256
        const int r = rank;
        const uint64_t be = (r == 3) ? 16 : 64;
        bool ok = (r == 2 || r == 3) && (p->block == 64 || p->block == 256);
        for (int i = 0; ok && i < r; ++i) ok = dims[i] > 0 && (uint64_t)dims[i] % be == 0;
        if (!ok) {
            EBLC_LOG("lorenzo=nd needs rank 2 or 3, block 64 or 256, dims multiples of %s",
                     r == 3 ? "16" : "64");
            delete p;
            return EBLC_UNSUPPORTED;
        }
        p->nd = r;
        p->dims[0] = (r == 3) ? (uint64_t)dims[0] : 1;
        p->dims[1] = (uint64_t)dims[r - 2];
        p->dims[2] = (uint64_t)dims[r - 1];
    }
    p->outlier_cap = std::min<uint64_t>(p->outlier_cap, n);
    if (p->chunked_m) {
        p->L = chunked_layout(n, p->chunked_m);
        // per chunk: a head word and at most its codes padded to 32, then the outliers
        p->max_bytes = p->L.record_off + 4 * (p->L.nc + n + 31 * p->L.nc + 2 * p->outlier_cap);
    } else {
        p->L = stream_layout(n, p->block);
        p->max_bytes = p->L.record_off + 4 * (n + 2 * p->outlier_cap);
    }

    if ((s = cuda_status(cudaGetDevice(&p->device), "cudaGetDevice")) != EBLC_OK) {
        delete p;
        return s;
    }
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, p->device);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, p->device);
    cudaDeviceGetAttribute(&p->num_sms, cudaDevAttrMultiProcessorCount, p->device);
    if (major != 10 || minor != 0 || p->num_sms <= 0) {
        EBLC_LOG("device %d is sm_%d%d; libeblc is compiled for sm_100a only", p->device, major, minor);
        delete p;
        return EBLC_UNSUPPORTED;
    }
    p->range_grid = range_grid(p->num_sms);

    const size_t ntiles = std::max<uint64_t>(p->L.nc, 1);
    p->ntiles = ntiles;
    size_t off = 0;
    uint8_t *base = nullptr;  // first pass computes the size
    for (int pass = 0; pass < 2; ++pass) {
        off = 0;
        p->status = carve<uint64_t>(base, &off, 2 * ntiles);
        p->d_rb = carve<Readback>(base, &off, 1);
        p->dec_err = carve<uint32_t>(base, &off, 1);
        p->partials = carve<float2>(base, &off, p->range_grid);
        p->range_counter = carve<uint32_t>(base, &off, 1);
        p->range = carve<float>(base, &off, 2);
        if (pass == 0) {
            if ((s = cuda_status(cudaMalloc(&p->scratch, off), "cudaMalloc scratch")) != EBLC_OK) {
                p->scratch = nullptr;
                destroy(p);
                return s;
            }
            base = static_cast<uint8_t *>(p->scratch);
        }
    }
    if (p->chunked_m && p->L.nc) {  // record slots of the chunked codec, then sizes, outlier counts, range totals
        const uint64_t words = p->L.nc * (chunked_slot_words(p->chunked_m) + 4);
        if ((s = cuda_status(cudaMalloc(&p->chunk_scratch, 4 * words), "cudaMalloc chunk scratch")) != EBLC_OK) {
            p->chunk_scratch = nullptr;
            destroy(p);
            return s;
        }
    }
    if ((s = cuda_status(cudaMemset(p->scratch, 0, off), "cudaMemset")) != EBLC_OK ||
        (s = cuda_status(cudaMallocHost(&p->h_rb, sizeof(Readback)), "cudaMallocHost")) != EBLC_OK ||
        (s = cuda_status(cudaMallocHost(&p->h_err, 256), "cudaMallocHost")) != EBLC_OK) {
        destroy(p);
        return s;
    }
    if (timing) {
        p->timing.on = true;
        for (cudaEvent_t &e : p->timing.ev)
            if ((s = cuda_status(cudaEventCreate(&e), "cudaEventCreate")) != EBLC_OK) {
                destroy(p);
                return s;
            }
    }
    if ((s = cuda_status(cudaDeviceSynchronize(), "plan init")) != EBLC_OK) {
        destroy(p);
        return s;
    }
    *out = p;
    return EBLC_OK;
}

EBLC_API eblc_status_t eblc_plan_get_limits(eblc_plan_t p, eblc_limits_t *out) {
    if (!p || !out) return EBLC_INVALID_ARG;
    std::memset(out, 0, sizeof(*out));
    out->n = p->n;
    out->block = p->block;
    out->chunk = p->chunked_m ? p->chunked_m : kChunk;
    out->max_compressed_bytes = p->max_bytes;
    out->payload_alignment = kPayloadAlignment;
    out->sidecar_bytes = kSidecarBytes;
    out->sidecar_alignment = kSidecarAlignment;
    out->outlier_capacity = p->outlier_cap;
    out->bound = p->bound;
    out->abs_mode = p->abs_mode;
    return EBLC_OK;
}

EBLC_API eblc_status_t eblc_compress(eblc_plan_t p, const eblc_execution_t *exec, const float *d_in, void *d_out,
                                     size_t out_capacity, size_t *compressed_bytes, void *h_sidecar) {
    if (!p || !exec) return EBLC_INVALID_ARG;
    if (compressed_bytes) *compressed_bytes = 0;
    if (exec->kind == EBLC_EXECUTION_HIP) return EBLC_UNSUPPORTED;
    if (exec->kind != EBLC_EXECUTION_CUDA && exec->kind != EBLC_EXECUTION_HOST) return EBLC_INVALID_ARG;
    if (!d_out || (p->n && !d_in)) return EBLC_INVALID_ARG;
    if (!aligned16(d_out) || (d_in && !aligned16(d_in))) return EBLC_INVALID_ARG;
    if (h_sidecar && (reinterpret_cast<uintptr_t>(h_sidecar) % kSidecarAlignment)) return EBLC_INVALID_ARG;
    if (out_capacity < p->L.record_off) return EBLC_CAPACITY;
    DeviceGuard g(p->device);
    if (!g.ok) return EBLC_CUDA_ERROR;
    eblc_status_t s;
    if (exec->kind == EBLC_EXECUTION_CUDA) {
        cudaStream_t st = static_cast<cudaStream_t>(exec->stream);
        if ((s = enqueue_compress(p, st, d_in, static_cast<uint8_t *>(d_out), out_capacity)) != EBLC_OK) return s;
        if ((s = cuda_status(cudaStreamSynchronize(st), "compress sync")) != EBLC_OK) return s;
        return finish_compress(p, compressed_bytes, h_sidecar);
    }
    // HOST: host pointers, same kernels on plan-owned device staging.  The
    // "call" timing pair spans the input copy through the stream copy back.
    if ((s = ensure_host_staging(p)) != EBLC_OK) return s;
    cudaStream_t st = p->host_stream;
    const uint64_t cap = std::min<uint64_t>(out_capacity, p->max_bytes);
    timing_begin(p, st);
    if (p->n && (s = cuda_status(cudaMemcpyAsync(p->stage_in, d_in, 4 * p->n, cudaMemcpyHostToDevice, st), "h2d")) !=
                    EBLC_OK)
        return s;
    if ((s = enqueue_compress(p, st, p->stage_in, p->stage_out, cap, false)) != EBLC_OK) return s;
    if ((s = cuda_status(cudaStreamSynchronize(st), "compress sync")) != EBLC_OK) return s;
    size_t total = 0;
    s = finish_compress(p, &total, h_sidecar);
    if (compressed_bytes) *compressed_bytes = total;
    if (s != EBLC_OK) return s;
    eblc_status_t c = cuda_status(cudaMemcpyAsync(d_out, p->stage_out, total, cudaMemcpyDeviceToHost, st), "d2h");
    timing_end(p, st);
    if (c == EBLC_OK) c = cuda_status(cudaStreamSynchronize(st), "d2h sync");
    return c;
}

EBLC_API eblc_status_t eblc_compress_async(eblc_plan_t p, const eblc_execution_t *exec, const float *d_in,
                                           void *d_out, size_t out_capacity, eblc_async_result_t *d_result) {
    static_assert(sizeof(eblc_async_result_t) == 32, "async result record is 4 words");
    if (!p || !exec || !d_result) return EBLC_INVALID_ARG;
    if (exec->kind == EBLC_EXECUTION_HIP) return EBLC_UNSUPPORTED;
    if (exec->kind != EBLC_EXECUTION_CUDA) return EBLC_INVALID_ARG;
    if (!d_out || (p->n && !d_in)) return EBLC_INVALID_ARG;
    if (!aligned16(d_out) || (d_in && !aligned16(d_in)) || (reinterpret_cast<uintptr_t>(d_result) & 7u))
        return EBLC_INVALID_ARG;
    if (out_capacity < p->L.record_off) return EBLC_CAPACITY;
    if (p->chunked_m) return EBLC_UNSUPPORTED;  // the chunked codec has its synchronous calls only
    DeviceGuard g(p->device);
    if (!g.ok) return EBLC_CUDA_ERROR;
    cudaStream_t st = static_cast<cudaStream_t>(exec->stream);
    // Under stream capture no timing events are recorded (the graph replays
    // the kernels only).
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) return EBLC_CUDA_ERROR;
    const bool timed = p->timing.on;
    if (cs != cudaStreamCaptureStatusNone) p->timing.on = false;
    const eblc_status_t s = enqueue_compress(p, st, d_in, static_cast<uint8_t *>(d_out), out_capacity, true,
                                             reinterpret_cast<uint64_t *>(d_result));
    p->timing.on = timed;
    return s;
}

EBLC_API eblc_status_t eblc_value_range(eblc_plan_t p, const eblc_execution_t *exec, const float *d_in,
                                        float *d_range) {
    if (!p || !exec || !d_range) return EBLC_INVALID_ARG;
    if (exec->kind == EBLC_EXECUTION_HIP || exec->kind == EBLC_EXECUTION_HOST) return EBLC_UNSUPPORTED;
    if (exec->kind != EBLC_EXECUTION_CUDA) return EBLC_INVALID_ARG;
    if ((p->n && !d_in) || (d_in && !aligned16(d_in)) || (reinterpret_cast<uintptr_t>(d_range) & 3u))
        return EBLC_INVALID_ARG;
    DeviceGuard g(p->device);
    if (!g.ok) return EBLC_CUDA_ERROR;
    cudaStream_t st = static_cast<cudaStream_t>(exec->stream);
    if (p->n == 0) return cuda_status(cudaMemsetAsync(d_range, 0, 2 * sizeof(float), st), "range clear");
    RangeArgs ra{d_in, p->n, p->partials, p->range_counter, d_range};
    return cuda_status(launch_range(ra, p->range_grid, st), "range launch");
}

EBLC_API eblc_status_t eblc_compress_range(eblc_plan_t p, const eblc_execution_t *exec, const float *d_in,
                                           const float *d_range, void *d_out, size_t out_capacity,
                                           size_t *compressed_bytes, void *h_sidecar) {
    if (!p || !exec || !d_range) return EBLC_INVALID_ARG;
    if (compressed_bytes) *compressed_bytes = 0;
    if (exec->kind == EBLC_EXECUTION_HIP || exec->kind == EBLC_EXECUTION_HOST) return EBLC_UNSUPPORTED;
    if (exec->kind != EBLC_EXECUTION_CUDA) return EBLC_INVALID_ARG;
    if (p->abs_mode) return EBLC_INVALID_ARG;  // a value range only matters for a relative bound
    if (p->chunked_m) return EBLC_UNSUPPORTED;
    if (!d_out || (p->n && !d_in)) return EBLC_INVALID_ARG;
    if (!aligned16(d_out) || (d_in && !aligned16(d_in)) || (reinterpret_cast<uintptr_t>(d_range) & 3u))
        return EBLC_INVALID_ARG;
    if (h_sidecar && (reinterpret_cast<uintptr_t>(h_sidecar) % kSidecarAlignment)) return EBLC_INVALID_ARG;
    if (out_capacity < p->L.record_off) return EBLC_CAPACITY;
    DeviceGuard g(p->device);
    if (!g.ok) return EBLC_CUDA_ERROR;
    cudaStream_t st = static_cast<cudaStream_t>(exec->stream);
    eblc_status_t s;
    if ((s = enqueue_compress(p, st, d_in, static_cast<uint8_t *>(d_out), out_capacity, true, nullptr, d_range)) !=
        EBLC_OK)
        return s;
    if ((s = cuda_status(cudaStreamSynchronize(st), "compress sync")) != EBLC_OK) return s;
    return finish_compress(p, compressed_bytes, h_sidecar);
}

EBLC_API eblc_status_t eblc_decompress(eblc_plan_t p, const eblc_execution_t *exec, const void *d_in,
                                       size_t compressed_bytes, const void *h_sidecar, float *d_out) {
    if (!p || !exec) return EBLC_INVALID_ARG;
    if (exec->kind == EBLC_EXECUTION_HIP) return EBLC_UNSUPPORTED;
    if (exec->kind != EBLC_EXECUTION_CUDA && exec->kind != EBLC_EXECUTION_HOST) return EBLC_INVALID_ARG;
    if (!d_in || (p->n && !d_out)) return EBLC_INVALID_ARG;
    if (!aligned16(d_in) || (d_out && !aligned16(d_out))) return EBLC_INVALID_ARG;
    if (compressed_bytes < kHeaderBytes) return EBLC_CORRUPT;
    DeviceGuard g(p->device);
    if (!g.ok) return EBLC_CUDA_ERROR;
    const bool host = exec->kind == EBLC_EXECUTION_HOST;
    cudaStream_t st = static_cast<cudaStream_t>(exec->stream);
    eblc_status_t s;
    eblc_sidecar_t sc{};
    if (h_sidecar) {
        std::memcpy(&sc, h_sidecar, sizeof(sc));
    } else if (host) {
        sc = sidecar_from_header(static_cast<const uint8_t *>(d_in));
    } else {
        uint8_t *hb = reinterpret_cast<uint8_t *>(p->h_err) + 64;  // pinned scratch for the header copy
        if ((s = cuda_status(cudaMemcpyAsync(hb, d_in, kHeaderBytes, cudaMemcpyDeviceToHost, st), "header")) !=
                EBLC_OK ||
            (s = cuda_status(cudaStreamSynchronize(st), "header sync")) != EBLC_OK)
            return s;
        sc = sidecar_from_header(hb);
    }
    StreamInfo info{};
    if ((s = check_stream(p, sc, compressed_bytes, &info)) != EBLC_OK) return s;

    DecodeArgs da{};
    da.total = info.total;
    da.n = p->n;
    da.block = p->block;
    da.W = info.W;
    da.m = info.m;
    da.step = info.step;
    da.err = p->dec_err;
    da.wait_ns = p->wait_ns;
    da.nd = p->nd;
    for (int d = 0; d < 3; ++d) da.dims[d] = p->dims[d];
    if (!host) {
        da.in = static_cast<const uint8_t *>(d_in);
        da.out = d_out;
        timing_begin(p, st);
        timing_mark(p, st, true, "decode");
        s = cuda_status(launch_plan_decode(p, da, st), "decode launch");
        timing_mark(p, st, false, nullptr);
        timing_end(p, st);
        return s;
    }
    if (info.total > p->max_bytes) return EBLC_CAPACITY;  // larger than this plan's staging
    if ((s = ensure_host_staging(p)) != EBLC_OK) return s;
    st = p->host_stream;
    da.in = p->stage_out;
    da.out = p->stage_in;
    timing_begin(p, st);  // the "call" pair spans the stream copy in through the output copy back
    if ((s = cuda_status(cudaMemcpyAsync(p->stage_out, d_in, info.total, cudaMemcpyHostToDevice, st), "h2d")) !=
        EBLC_OK)
        return s;
    timing_mark(p, st, true, "decode");
    s = cuda_status(launch_plan_decode(p, da, st), "decode launch");
    timing_mark(p, st, false, nullptr);
    if (s != EBLC_OK) return s;
    if (p->n && (s = cuda_status(cudaMemcpyAsync(d_out, p->stage_in, 4 * p->n, cudaMemcpyDeviceToHost, st),
                                 "d2h")) != EBLC_OK)
        return s;
    timing_end(p, st);
    if ((s = cuda_status(cudaMemcpyAsync(p->h_err, p->dec_err, 4, cudaMemcpyDeviceToHost, st), "err")) != EBLC_OK ||
        (s = cuda_status(cudaMemsetAsync(p->dec_err, 0, 4, st), "err clear")) != EBLC_OK ||
        (s = cuda_status(cudaStreamSynchronize(st), "decompress sync")) != EBLC_OK)
        return s;
    return device_error_status(*p->h_err);
}

EBLC_API eblc_status_t eblc_check(eblc_plan_t p, const eblc_execution_t *exec) {
    if (!p) return EBLC_INVALID_ARG;
    DeviceGuard g(p->device);
    if (!g.ok) return EBLC_CUDA_ERROR;
    cudaStream_t st = (exec && exec->kind == EBLC_EXECUTION_CUDA) ? static_cast<cudaStream_t>(exec->stream)
                      : p->host_stream;
    eblc_status_t s;
    if ((s = cuda_status(cudaMemcpyAsync(p->h_err, p->dec_err, 4, cudaMemcpyDeviceToHost, st), "err")) != EBLC_OK ||
        (s = cuda_status(cudaMemsetAsync(p->dec_err, 0, 4, st), "err clear")) != EBLC_OK ||
        (s = cuda_status(cudaStreamSynchronize(st), "check sync")) != EBLC_OK)
        return s;
    return device_error_status(*p->h_err);
}

EBLC_API eblc_status_t eblc_plan_kernel_times(eblc_plan_t p, eblc_kernel_time_t *out, int cap, int *count) {
    if (!p || !count || (cap > 0 && !out)) return EBLC_INVALID_ARG;
    *count = 0;
    if (!p->timing.on) return EBLC_UNSUPPORTED;
    DeviceGuard g(p->device);
    const int nk = p->timing.count;
    int k = 0;
    for (int i = 0; i <= nk && k < cap; ++i) {  // the kernels, then the whole call
        const bool call = (i == nk);
        cudaEvent_t a = call ? p->timing.ev[6] : p->timing.ev[2 * i];
        cudaEvent_t b = call ? p->timing.ev[7] : p->timing.ev[2 * i + 1];
        float ms = 0.f;
        eblc_status_t s = cuda_status(cudaEventSynchronize(b), "event sync");
        if (s == EBLC_OK) s = cuda_status(cudaEventElapsedTime(&ms, a, b), "event time");
        if (s != EBLC_OK) return s;
        std::memset(&out[k], 0, sizeof(out[k]));
        std::strncpy(out[k].name, call ? "call" : p->timing.name[i], sizeof(out[k].name) - 1);
        out[k].ms = ms;
        out[k].launches = call ? (uint32_t)nk : 1u;
        ++k;
    }
    *count = k;
    return EBLC_OK;
}

EBLC_API void eblc_plan_destroy(eblc_plan_t p) { destroy(p); }

}  // extern "C"
