/*
 * eblc.h -- C ABI of libeblc, a B200 (sm_100a) error-bounded lossy
 * compressor for float32 arrays.
 *
 * The hot path is one fused block-local pipeline: linear quantizer ->
 * 1-D Lorenzo predictor reset at each block -> zigzag -> adaptive
 * fixed-length bitpack, with an outlier side list, and a cross-block scan
 * that places every block at its final offset in one stream; plus its exact
 * inverse.  Every element of the reconstruction x' satisfies
 * |x - x'| <= eb (tested in IEEE double), non-finite elements and elements
 * that would break the bound are stored losslessly in the outlier list.
 *
 * Sources (page title, section):
 *   "DevitoComp provider interface" -- "Configuring the error tolerance"
 *     (a non-negative relative error fixed at plan creation, passed as a
 *     decimal string or NULL for the provider default), "Provider layout"
 *     (plan_create with an options string; dims and strides in
 *     slowest-to-fastest order, strides in elements; HOST / CUDA / HIP
 *     execution descriptor with an optional native stream; per-snapshot
 *     host sidecar ready on return; device work may stay queued; providers
 *     report payload alignment through a limits struct and may return
 *     UNSUPPORTED), "Dummy provider" (contiguous float32 tensors; a maximum
 *     compressed size).
 *   FZGPUModules "Pipeline specialization internals" -- "Roles and
 *     strategies", "Forward declaration", "Inverse declaration", "Priming:
 *     the fused runner bypasses execute()" (default bound 1e-4; the inverse
 *     must read the resolved bound), "The device policy contract".
 *   "nvrtc_chunk_fusion.h File Reference" -- launchNvrtcChunkFusedEncode and
 *     launchGenericChunkFusion (outlier side output: uint32 indices + values;
 *     the cross-chunk scan/pack tail returns the archive byte length after a
 *     stream synchronisation).
 *
 * Threading and streams: a plan may be used by one host thread and one
 * stream at a time (it owns the scratch memory of its calls).  All device
 * pointers must belong to the device that was current at eblc_plan_create.
 *
 * Errors: every call returns an eblc_status_t; no C++ exception crosses this
 * ABI and nothing aborts the process.  Device-side faults that the kernels
 * detect (corrupt stream, capacity, a bounded wait that ran out) are
 * reported through a device error word, read by eblc_compress (which
 * synchronises) or by eblc_check.
 */
#ifndef EBLC_H
#define EBLC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(_WIN32)
#define EBLC_API
#else
#define EBLC_API __attribute__((visibility("default")))
#endif

#define EBLC_ABI_VERSION 1u

typedef enum {
    EBLC_OK = 0,
    EBLC_UNSUPPORTED = 1,  /* execution kind, layout or option not supported      */
    EBLC_INVALID_ARG = 2,  /* bad pointer, size, alignment or option value          */
    EBLC_CAPACITY = 3,     /* output buffer or outlier capacity too small           */
    EBLC_CORRUPT = 4,      /* stream or sidecar malformed (host or device detected) */
    EBLC_CUDA_ERROR = 5,   /* a CUDA runtime call failed                            */
    EBLC_TIMEOUT = 6,      /* a bounded device-side wait ran out                    */
    EBLC_NOMEM = 7         /* host or device allocation failed                      */
} eblc_status_t;

typedef enum {
    /* Host pointers.  The call is synchronous.  The work still runs on the
     * GPU: the plan copies the input to device staging buffers, runs the
     * same kernels, and copies the result back (no CPU code path).
     * num_threads and stream are ignored.  Pinned host memory is fastest.  */
    EBLC_EXECUTION_HOST = 0,
    /* Device pointers on the plan's device, work queued on `stream`
     * (a cudaStream_t; NULL = the legacy default stream).                   */
    EBLC_EXECUTION_CUDA = 1,
    /* Not supported: returns EBLC_UNSUPPORTED.                              */
    EBLC_EXECUTION_HIP = 2
} eblc_execution_kind_t;

typedef struct {
    int32_t kind;        /* eblc_execution_kind_t                     */
    int32_t num_threads; /* ignored                                   */
    void *stream;        /* cudaStream_t for EBLC_EXECUTION_CUDA      */
} eblc_execution_t;

typedef struct eblc_plan_s *eblc_plan_t;

typedef struct {
    uint64_t n;                    /* elements per snapshot (product of dims)             */
    uint32_t block;                /* block size B (elements), one of 32, 64, 128, 256    */
    uint32_t chunk;                /* elements per chunk record (4096)                    */
    uint64_t max_compressed_bytes; /* worst-case stream size for this plan                */
    uint64_t payload_alignment;    /* required alignment of stream and float buffers (16) */
    uint64_t sidecar_bytes;        /* size of the host sidecar (64)                       */
    uint64_t sidecar_alignment;    /* alignment of the host sidecar (8)                   */
    uint64_t outlier_capacity;     /* most outliers a stream may hold (default n)         */
    double bound;                  /* error bound requested (relative or absolute)        */
    int32_t abs_mode;              /* 1 if `bound` is absolute, 0 if relative             */
    int32_t reserved;
} eblc_limits_t;

/* Host sidecar written by eblc_compress (64 bytes, 8-byte aligned, little
 * endian).  It repeats the stream header fields that a decompressing caller
 * needs to validate sizes without reading device memory.                    */
typedef struct {
    uint32_t magic;         /* 0x434C4245 ("EBLC")                   */
    uint16_t version;       /* stream version (1)                    */
    uint16_t flags;         /* bit0: absolute bound; bit1: 2-D / 3-D
                               Lorenzo (lorenzo=nd); bit2: chunked
                               codec (codec=chunked); bit3: its RRE
                               coder (coder=rre)                     */
    uint32_t block;         /* B (0 for the chunked codec)           */
    uint32_t chunk;         /* elements per chunk: 4096, or the
                               chunked codec's 1024 / 2048 / 4096    */
    uint64_t n;             /* elements                              */
    uint64_t total_bytes;   /* stream length                         */
    uint64_t payload_words; /* W                                     */
    uint64_t n_outliers;    /* m                                     */
    double eb;              /* resolved absolute bound               */
    float step;             /* dequantisation step (float)(2 eb)     */
    float inv2eb;           /* quantisation factor (float)(1/(2 eb)) */
} eblc_sidecar_t;

/* Device timing of the last call, recorded when the plan was created with
 * the option "timing=1": CUDA events on the call's stream around each kernel
 * launch, plus one entry "call" from the first launch to the end of the
 * call's last device operation (for compress: the result readback).  For
 * the HOST execution kind "call" spans the host-to-device copy of the input
 * through the device-to-host copy of the output.                           */
typedef struct {
    char name[24];      /* "range", "encode", "decode", "call"          */
    float ms;           /* elapsed device time                          */
    uint32_t launches;  /* 1 for a kernel; kernels in the call for "call" */
} eblc_kernel_time_t;

/* Version of this ABI (EBLC_ABI_VERSION).                                   */
EBLC_API uint32_t eblc_abi_version(void);

/* Static description of a status code.                                      */
EBLC_API const char *eblc_status_string(eblc_status_t status);

/*
 * Create a plan for float32 snapshots of shape dims[0..rank) (slowest to
 * fastest).  strides (in elements, slowest to fastest) may be NULL for
 * C-contiguous data; any non-contiguous stride gives EBLC_UNSUPPORTED.  The
 * data are coded as one flat sequence in C order (unless lorenzo=nd, below).
 * Requires 1 <= rank <= 8,
 * dims >= 0 and n = prod(dims) <= 2^30.
 *
 * options: NULL -> relative bound 1e-4, block 128.  A bare decimal ("1e-3")
 * is a relative bound.  Otherwise comma-separated key=value:
 *   rel=<x>          relative bound, eb = x * (max - min) over the finite
 *                    elements of each snapshot (x finite, >= 0)
 *   abs=<x>          absolute bound eb = x (finite, >= 0)
 *   block=<B>        32 | 64 | 128 | 256 (default 128)
 *   outlier_cap=<k>  most outliers per stream (default n); more gives
 *                    EBLC_CAPACITY
 *   lorenzo=nd       2-D / 3-D Lorenzo predictor over the plan's own dims
 *                    (rank 2 {Y, X} or rank 3 {Z, Y, X}, each a multiple of 64
 *                    (2-D) or 16 (3-D); block 64 or 256, i.e. 8x8 / 16x16
 *                    or 4x4x4 / 4x8x8 elements), reset at every block face;
 *                    bricks of 64x64 or 16x16x16 elements take the place of
 *                    the 4096-element chunks.  Otherwise EBLC_UNSUPPORTED.
 *                    Default lorenzo=1d: the data coded as one flat sequence
 *   codec=chunked    the chunk-cooperative codec instead of the block codec:
 *                    per chunk of `chunk` bytes of input, the quantization
 *                    codes' first differences (zigzag form), bit-shuffled
 *                    (32 bit planes per group of 32 codes) and zero-eliminated
 *                    (a bitmap of the nonzero words, then those words), or
 *                    kept verbatim when that is not smaller.  Not with
 *                    lorenzo=nd; eblc_compress_async and eblc_compress_range
 *                    return EBLC_UNSUPPORTED for such plans.  ("Pipeline
 *                    specialization internals", Chunk-cooperative path.)
 *   chunk=<bytes>    4096 | 8192 | 16384 (default 16384), with codec=chunked
 *   coder=rze|rre    with codec=chunked: zero elimination (default) or
 *                    repetition elimination (a bitmap of the words that
 *                    differ from the word before, the first word's
 *                    predecessor being 0, then those words); a plan decodes
 *                    only streams of its own coder (else EBLC_INVALID_ARG)
 *   timing=1         record per-kernel device times (eblc_plan_kernel_times)
 *   wait_ms=<t>      limit of device-side waits in milliseconds (default 2000)
 *   stall_tile=<t>   test hook: tile t of one compress call never publishes
 *                    its scan value, so later tiles' waits run out and the
 *                    call returns EBLC_TIMEOUT (default off); the plan's
 *                    later calls are unaffected
 *   stall_call=<k>   the compress call (0-based, counted per plan) that
 *                    stall_tile applies to (default 0)
 * The plan allocates its device scratch here (cudaMalloc on the current
 * device).  *out is NULL on failure.
 */
EBLC_API eblc_status_t eblc_plan_create(eblc_plan_t *out, int rank, const int64_t *dims,
                                        const int64_t *strides, const char *options);

/* Sizes and alignment rules of a plan.                                      */
EBLC_API eblc_status_t eblc_plan_get_limits(eblc_plan_t plan, eblc_limits_t *out);

/*
 * Compress one snapshot.
 *   d_in          n float32 values (device pointer for CUDA kind, host pointer
 *                 for HOST kind), 16-byte aligned; caller owned, not modified.
 *   d_out         output buffer of out_capacity bytes, 16-byte aligned
 *                 (device or host pointer by kind); caller owned.
 *   out_capacity  bytes available at d_out.  If the stream does not fit the
 *                 call returns EBLC_CAPACITY and nothing beyond out_capacity
 *                 is written; max_compressed_bytes always fits.
 *   compressed_bytes  receives the stream length.
 *   h_sidecar     host buffer of sidecar_bytes (8-byte aligned) receiving an
 *                 eblc_sidecar_t; may be NULL.
 * The call synchronises the stream once at the end (the length and the
 * sidecar must be ready on return).  Stream layout: see the stream format
 * notes shipped with this library (header, widths, chunk index, one record
 * per 4096-element chunk holding its payload words then its outliers).
 */
EBLC_API eblc_status_t eblc_compress(eblc_plan_t plan, const eblc_execution_t *exec, const float *d_in,
                                     void *d_out, size_t out_capacity, size_t *compressed_bytes,
                                     void *h_sidecar);

/* Device-written result of eblc_compress_async (4 words, 8-byte aligned).  */
typedef struct eblc_async_result_t {
    uint64_t compressed_bytes;  /* stream length; with EBLC_CAPACITY the length the
                                   stream needs                                    */
    uint64_t payload_words;     /* W                                               */
    uint64_t n_outliers;        /* m                                               */
    uint32_t status;            /* eblc_status_t of the device work: EBLC_OK,
                                   EBLC_CAPACITY or EBLC_TIMEOUT                   */
    uint32_t reserved;
} eblc_async_result_t;

/*
 * Compress one snapshot without synchronising the host: every step is
 * queued on exec->stream (CUDA kind only) and the call returns at once; the
 * stream length, the counts and the device status are written to *d_result
 * (device memory, or host memory mapped into the device) by the last queued
 * kernel.  There is no host synchronisation, memory allocation or host read
 * inside, so the call may be captured into a CUDA graph and the graph
 * replayed: the plan keeps its per-call state (which of its two look-back
 * arrays a call uses) on the device.  Sources: FZGPUModules "Architecture",
 * MemoryPool (CUDA Graph capture of a pipeline with a preallocated pool);
 * "DevitoComp provider interface", Provider layout (device work may stay
 * queued when the call returns).  No sidecar is produced: build one
 * from the stream header, or pass NULL to eblc_decompress (which then reads
 * the header, synchronising once).
 *   d_in, d_out, out_capacity  as for eblc_compress (device pointers)
 *   d_result   8-byte aligned record, valid once the stream reaches it
 * Returns EBLC_OK when the work was queued (argument errors and a capacity
 * below the fixed sections are reported at once); the outcome of the device
 * work is d_result->status.  Calls on one plan are serialised by the stream
 * order like every plan call; with timing=1 per-kernel times are recorded
 * unless the stream is capturing.
 */
EBLC_API eblc_status_t eblc_compress_async(eblc_plan_t plan, const eblc_execution_t *exec, const float *d_in,
                                           void *d_out, size_t out_capacity, eblc_async_result_t *d_result);

/*
 * Value range of one snapshot: d_range[0] = vmin, d_range[1] = vmax over the
 * finite elements of d_in (each +0 where the value is a zero; both 0 when no
 * element is finite, or n = 0).  This is the range a relative bound is
 * relative to ("Pipeline specialization internals", Priming: the value-range
 * scan that resolves the bound before the fused kernel).
 *   d_in     n float32 values in device memory, 16-byte aligned
 *   d_range  device float[2], 4-byte aligned, caller owned
 * CUDA kind only (HOST and HIP: EBLC_UNSUPPORTED).  Queued on exec->stream;
 * no synchronisation.  Uses the plan's scratch, like its other calls.
 *
 * With eblc_compress_range this codes an array split across processes (one
 * contiguous part per GPU) under one relative bound: each process computes
 * its part's range here, the processes combine them (minimum of vmin,
 * maximum of vmax: one small all-reduce, which is the caller's, e.g. NCCL
 * through torch.distributed), and each compresses its part under the
 * combined range ("DevitoComp provider interface", Validating a private
 * provider: the provider runs inside an MPI-run consumer).
 */
EBLC_API eblc_status_t eblc_value_range(eblc_plan_t plan, const eblc_execution_t *exec, const float *d_in,
                                        float *d_range);

/*
 * eblc_compress with the value range given instead of taken from d_in: the
 * bound is eb = rel * (vmax - vmin) with {vmin, vmax} = d_range[0..1] read
 * from device memory by the encoder (relative-bound plans only, else
 * EBLC_INVALID_ARG).  Meant for one part of a larger array, with the range of
 * the whole (see eblc_value_range); outlier indices in the stream count from
 * the part's first element, and the stream decodes on its own with
 * eblc_decompress.  When the parts are cut at multiples of 4096 elements,
 * their width bytes, payload words and outlier values are those of the whole
 * array's stream for the same chunks.
 *   d_range  device float[2], 4-byte aligned; must be finite with
 *            vmin <= vmax, else the call returns EBLC_INVALID_ARG (checked
 *            on the device, reported after the closing synchronisation)
 * Other arguments, synchronisation and sidecar as for eblc_compress; CUDA
 * kind only.
 */
EBLC_API eblc_status_t eblc_compress_range(eblc_plan_t plan, const eblc_execution_t *exec, const float *d_in,
                                           const float *d_range, void *d_out, size_t out_capacity,
                                           size_t *compressed_bytes, void *h_sidecar);

/*
 * Decompress one snapshot.
 *   d_in              the stream (compressed_bytes long, 16-byte aligned).
 *   h_sidecar         the sidecar eblc_compress returned with this stream
 *                     (may be NULL; then the stream header is copied to the
 *                     host, which synchronises the stream).
 *   d_out             n float32 values, 16-byte aligned, caller owned.
 * With the CUDA kind and a sidecar the work stays queued on the stream (no
 * synchronisation); device-detected corruption is reported by eblc_check.
 * The stream must have been produced with the same n and block; the bound
 * is read from the stream, never from the plan.
 */
EBLC_API eblc_status_t eblc_decompress(eblc_plan_t plan, const eblc_execution_t *exec, const void *d_in,
                                       size_t compressed_bytes, const void *h_sidecar, float *d_out);

/* Synchronise exec->stream and return (then clear) the status recorded by
 * the device during this plan's calls since the last check.                */
EBLC_API eblc_status_t eblc_check(eblc_plan_t plan, const eblc_execution_t *exec);

/* Device times of the last compress / decompress (option timing=1): one
 * entry per kernel, then the whole call.  Synchronises on the recorded
 * events.  Writes at most cap entries and sets *count to the number
 * written; EBLC_UNSUPPORTED if the plan records no timing.                 */
EBLC_API eblc_status_t eblc_plan_kernel_times(eblc_plan_t plan, eblc_kernel_time_t *out, int cap, int *count);

/* Release the plan and its device memory.  NULL is allowed.                */
EBLC_API void eblc_plan_destroy(eblc_plan_t plan);

/* Largest n accepted by eblc_compress_noalloc: 2^26 elements (256 MiB of
 * float32).  Its scratch is one fixed device array of about 280 KB.        */
#define EBLC_NOALLOC_MAX_N (1ull << 26)

/*
 * Compress one array without allocating any device memory.  The paper has
 * no counterpart to this entry point.  It is for callers that cannot call
 * cudaMalloc: code running under an allocator that owns all device memory,
 * code inside a region where an allocation is forbidden or would
 * synchronise the device, and callers that must not grow the device
 * footprint behind their back.  No plan is needed; the result is
 * byte-identical to eblc_plan_create(n, "rel=|abs=<bound>,block=<block>")
 * followed by eblc_compress.
 *   d_in, n        n float32 values in device memory, 16-byte aligned;
 *                  n <= EBLC_NOALLOC_MAX_N, else EBLC_UNSUPPORTED (a message
 *                  goes to stderr)
 *   block          32, 64, 128 or 256
 *   abs_mode, bound  absolute (abs_mode != 0) or relative bound, finite >= 0
 *   d_out, out_capacity  caller-owned device output, 16-byte aligned
 *   stream         cudaStream_t (NULL: the legacy default stream)
 *   compressed_bytes, h_sidecar  as for eblc_compress (h_sidecar may be NULL)
 * The scratch of the range and encode kernels is a file-scope __device__
 * array that every GPU that loads this library holds until the process
 * exits.  The first call on a device does a one-time set-up: it looks up
 * that array's device address (cudaGetSymbolAddress) with the device
 * current.  Make that first call before any stream capture begins.
 * Every call on a device shares the array and each call clears what must
 * start at zero (including the value range when n is 0), so calls that
 * overlap on the GPU (other streams, other host threads) race: serialise
 * them.  Like eblc_compress, the call ends by copying the result to the
 * host and synchronising `stream`.
 */
EBLC_API eblc_status_t eblc_compress_noalloc(const float *d_in, uint64_t n, uint32_t block, int abs_mode,
                                             double bound, void *d_out, size_t out_capacity, void *stream,
                                             size_t *compressed_bytes, void *h_sidecar);

#ifdef __cplusplus
}
#endif

#endif /* EBLC_H */
