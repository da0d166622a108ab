// kernels.h -- host-side launch interface of the libeblc kernels (internal).
#pragma once

#include <cstdint>
#include <cuda.h>  // CUtensorMap (the tensor map itself is encoded on the host)
#include <cuda_runtime.h>

namespace eblc {

// Value range over the finite elements ("Pipeline specialization
// internals", Priming: the quantizer's value-range scan before the fused
// kernel).  Writes range_out[0] = vmin, range_out[1] = vmax (each
// canonicalised so -0 reads as +0; both 0 when nothing is finite).
struct RangeArgs {
    const float *in;   // n floats, 16-byte aligned
    uint64_t n;
    float2 *partials;  // one per CTA of the grid
    uint32_t *counter; // zero on entry; the last CTA resets it
    float *range_out;  // 2 floats
};
int range_grid(int num_sms);
cudaError_t launch_range(const RangeArgs &a, int grid, cudaStream_t stream);

// Fused encode with single-pass decoupled look-back.  One launch writes the
// whole stream: header, widths, chunk index and every chunk record.
struct EncodeArgs {
    const float *in;          // n floats, 16-byte aligned
    uint64_t n;
    uint8_t *out;             // stream buffer, 16-byte aligned
    uint64_t out_cap;         // bytes available at out
    uint32_t block;           // 32, 64, 128, 256
    int abs_mode;
    double bound;             // relative or absolute bound as requested
    const float *range;       // vmin, vmax (relative mode): from the range kernel, or given by the caller
    int range_given;          // 1: `range` comes from the caller (checked: finite, vmin <= vmax)
    uint64_t *status;         // look-back words: two arrays of ntiles; the call uses array
                              // (*epoch & 1), zero on entry, and clears the other one
    uint64_t ntiles;          // stride between the two arrays
    const uint32_t *epoch;    // call counter on the device (advanced by the finish kernel)
    uint32_t *err;            // error word, zero on entry
    uint64_t *result;         // [W, m, total, R, eb, step|inv2eb, vmin|vmax] written by the last tile
    uint64_t outlier_cap;
    int64_t stall_tile;       // test hook (-1: off)
    uint64_t wait_ns;         // limit of every device-side wait
    // Multi-dimensional Lorenzo (nd = 2 or 3; 0: the 1-D path): the array's
    // dims {Z, Y, X} (Z = 1 for 2-D), each a multiple of the brick edge, and
    // a tiled tensor map of `in` with a 16x16x16 (3-D) or 64x64 (2-D) box.
    int nd;
    uint64_t dims[3];
    CUtensorMap tmap;
};
cudaError_t launch_encode(const EncodeArgs &a, int num_sms, cudaStream_t stream);

// After the encoder on the same stream: result[7] = the call's error word,
// which it then clears; advances the call counter; when `user` is set,
// writes the caller's result record (compressed bytes, payload words,
// outliers, status code); and when the call failed (a wait that ran out
// leaves look-back words behind) zeroes both look-back arrays, so the plan's
// next call starts clean.
struct FinishArgs {
    uint64_t *result;         // the encoder's result block (8 words)
    uint32_t *err;
    uint32_t *epoch;
    uint64_t *user;           // NULL, or 4 words: total, W, m, status | reserved << 32
    uint64_t *status;         // both look-back arrays
    uint64_t status_words;    // their total length
};
cudaError_t launch_finish(const FinishArgs &f, cudaStream_t stream);

// Fused decode: widths + chunk records -> reconstruction with the chunk's
// outliers written back.
struct DecodeArgs {
    const uint8_t *in;        // stream, 16-byte aligned
    uint64_t total;           // stream length (validated on the host)
    uint64_t n;
    uint32_t block;
    uint64_t W, m;            // payload words and outliers (from the sidecar)
    float step;
    float *out;               // n floats, 16-byte aligned
    uint32_t *err;            // sticky error word (kErrCorrupt, kErrTimeout)
    uint64_t wait_ns;
    int nd;                   // as EncodeArgs::nd
    uint64_t dims[3];         // {Z, Y, X} when nd != 0
};
cudaError_t launch_decode(const DecodeArgs &a, int num_sms, cudaStream_t stream);

// Chunk-cooperative codec (Quant -> Diff -> Bitshuffle -> RZE): chunks of m
// = 1024, 2048 or 4096 elements.  One launch sequence writes the stream:
// encode (CTA b codes the contiguous chunk range b: each chunk's record into
// its scratch slot of chunked_slot_words(m) words, its size and outlier
// count, the range's totals), scan (the ranges' bases, header, result
// block), gather (per range: chunk index entries, records to their offsets).
struct ChunkedArgs {
    const float *in;          // n floats
    uint64_t n;
    uint32_t m;               // elements per chunk
    uint64_t nc;
    int abs_mode;
    double bound;
    const float *range;       // vmin, vmax (relative mode)
    uint32_t *scratch;        // nc slots
    uint32_t slot_words;
    uint32_t *sizes, *outl;   // nc each: record words, outliers
    uint32_t *part;           // 2 nc: per chunk range, record words [0, nc) and outliers [nc, 2 nc)
    int rre;                  // coder: 0 RZE, 1 RRE
    uint32_t ranges, per_range;  // set by the launcher: chunk ranges, chunks per range
    uint8_t *out;
    uint64_t out_cap;
    uint64_t *result;         // as EncodeArgs::result
    uint32_t *err;
    uint64_t outlier_cap;
};
uint64_t chunked_slot_words(uint32_t m);
cudaError_t launch_chunked_encode(const ChunkedArgs &a, int num_sms, cudaStream_t stream);

struct ChunkedDecArgs {
    const uint8_t *in;        // stream, 16-byte aligned
    uint64_t n;
    uint32_t m;
    uint64_t W, mo;           // payload words (record head words included) and outliers
    float step;
    float *out;
    uint32_t *err;
    int rre;                  // coder: 0 RZE, 1 RRE
};
cudaError_t launch_chunked_decode(const ChunkedDecArgs &a, int num_sms, cudaStream_t stream);

}  // namespace eblc
