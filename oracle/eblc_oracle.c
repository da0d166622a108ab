/*
 * eblc_oracle.c -- plain, slow, scalar CPU oracle of the error-bounded lossy
 * encoding (linear quantizer -> 1-D Lorenzo predictor reset per block ->
 * zigzag -> adaptive fixed-length bitpack, with an outlier side list and a
 * cross-block scan/pack into one archive), and of its exact inverse.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the package smoke check and
 * the CPU-baseline leg of the benchmark load this library.  The product (the
 * CUDA library) never includes, links or calls anything in this directory, and
 * this file includes nothing of the product: every constant and layout rule
 * below is written out here on its own.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fPIC -shared
 * (no FMA contraction, IEEE single/double arithmetic, round-to-nearest-even).
 *
 * Sources (page title, section):
 *   [SPEC]  FZGPUModules "Pipeline specialization internals":
 *           "Roles and strategies" (Elementwise linear quantizer, RegionLocal
 *           1-D Lorenzo with region reset, SegmentCodec adaptive bitpack,
 *           WarpRegister block = 32*EPL elements);
 *           "Forward declaration" (block_size % 32 == 0, block = 32*EPL, the
 *           float inv2eb slot; the quantizer quantizes inline in delta());
 *           "Inverse declaration" (dequant step = 2*abs_eb; plain
 *           first-difference undelta);
 *           "Priming: the fused runner bypasses execute()" (value-range scan
 *           and bound resolution before the fused kernel; default bound 1e-4;
 *           the inverse must read the resolved bound);
 *           "The device policy contract" (coder meta_bytes = 1 per block;
 *           decode(meta, base, count, ...); Zigzag as an interior transform);
 *           "Validation requirements" (byte-identical archives, partial final
 *           block).
 *   [NVRTC] "nvrtc_chunk_fusion.h File Reference": launchNvrtcChunkFusedEncode
 *           and launchGenericChunkFusion (split-outlier side output: uint32
 *           index array + value array with an append counter; cross-chunk
 *           scan/pack tail returning the archive byte length).
 *   [DEVITO] "DevitoComp provider interface": "Configuring the error
 *           tolerance" (non-negative relative error fixed at plan creation).
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - relative error is relative to the value range (max - min) over the
 *     finite elements; with no finite element the range is 0;
 *   - y = x * inv2eb in float, q = round-half-even(y) when |y| < 2^30, else 0;
 *   - outlier test: x non-finite, or fp64 |x - x'| > eb, x' = (float)q * step;
 *     the code q stays in the stream even for an outlier;
 *   - zigzag is the textbook map d >= 0 -> 2d, d < 0 -> -2d - 1;
 *   - width = bit length of the OR of the block's zigzag codes (0..32), one
 *     byte per block; the payload of a block is ceil(w*cnt/32) little-endian
 *     u32 words holding code j at bits [j*w, j*w + w), least significant first;
 *   - the partial final block holds only its cnt real elements;
 *   - outliers are stored sorted by index, value as raw float32 bits, each
 *     in the record of the 4096-element chunk that holds it;
 *   - at most 2^30 elements per stream (record offsets are 32-bit words).
 *
 * Stream layout, version 1 (all little-endian):
 *   header, 128 bytes:
 *     0 u32 magic 0x434C4245 ("EBLC")   4 u16 version = 1   6 u16 flags
 *     (bit0: absolute bound)            8 u64 n             16 u32 block B
 *     20 u32 chunk = 4096               24 f64 eb           32 f32 inv2eb
 *     36 f32 step                       40 f32 vmin         44 f32 vmax
 *     48 u64 nb (blocks)                56 u64 nc (chunks)  64 u64 W (payload
 *     words)                            72 u64 m (outliers) 80 u64 total bytes
 *     88 f64 bound as requested (relative or absolute)      96..127 zero
 *   128:  u8 width[nb], zero padded to a multiple of 16 bytes
 *   I0:   per chunk c (elements [4096c, 4096c + 4096)), a u32 pair: the word
 *         offset of the chunk's record from P0, and the number of outliers
 *         before the chunk's first element; zero padded to 16
 *   P0:   one record per chunk, in order: the payload words of the chunk's
 *         blocks, then u32 idx[m_c] (ascending element index), then u32
 *         val[m_c] (float32 bits) of the chunk's m_c outliers.
 *   total = P0 + 4 * (W + 2m).
 */
#include <fenv.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_MAGIC 0x434C4245u
#define ORC_VERSION 1u
#define ORC_CHUNK 4096u
#define ORC_HEADER_BYTES 128u
#define ORC_FLAG_ABS 1u
#define ORC_FLAG_LORENZO_ND 2u    /* 2-D / 3-D Lorenzo over the array's own dims */
#define ORC_FLAG_CHUNKED 4u       /* chunk-cooperative codec: Diff -> Bitshuffle -> RZE */
#define ORC_FLAG_RRE 8u           /* with the chunked codec: RRE in place of RZE */

/* error codes returned as negative values */
#define ORC_ERR_ARG (-1)
#define ORC_ERR_CAPACITY (-2)     /* output buffer too small               */
#define ORC_ERR_OUTLIER_CAP (-3)  /* more outliers than the stated capacity */
#define ORC_ERR_CORRUPT (-4)
#define ORC_ERR_NOMEM (-5)

static uint64_t pad16(uint64_t v) { return (v + 15u) / 16u * 16u; }

static void put_u16(uint8_t *p, uint16_t v) { p[0] = (uint8_t)v; p[1] = (uint8_t)(v >> 8); }
static void put_u32(uint8_t *p, uint32_t v) {
    for (int i = 0; i < 4; ++i) p[i] = (uint8_t)(v >> (8 * i));
}
static void put_u64(uint8_t *p, uint64_t v) {
    for (int i = 0; i < 8; ++i) p[i] = (uint8_t)(v >> (8 * i));
}
static void put_f32(uint8_t *p, float v) { uint32_t u; memcpy(&u, &v, 4); put_u32(p, u); }
static void put_f64(uint8_t *p, double v) { uint64_t u; memcpy(&u, &v, 8); put_u64(p, u); }
static uint16_t get_u16(const uint8_t *p) { return (uint16_t)(p[0] | (p[1] << 8)); }
static uint32_t get_u32(const uint8_t *p) {
    uint32_t v = 0;
    for (int i = 3; i >= 0; --i) v = (v << 8) | p[i];
    return v;
}
static uint64_t get_u64(const uint8_t *p) {
    uint64_t v = 0;
    for (int i = 7; i >= 0; --i) v = (v << 8) | p[i];
    return v;
}
static float get_f32(const uint8_t *p) { uint32_t u = get_u32(p); float v; memcpy(&v, &u, 4); return v; }
static double get_f64(const uint8_t *p) { uint64_t u = get_u64(p); double v; memcpy(&v, &u, 8); return v; }

/* ------------------------------------------------------------------------ */
/* Step 1. Value range over the finite elements ([SPEC] Priming: the
 * quantizer's value-range scan).  Sequential min/max; each end is then
 * canonicalised with "+ 0.0f" so that -0.0 reads as +0.0.  Returns 1 if any
 * element is finite, else 0 (and the range is [0, 0]).                      */
int orc_value_range(const float *x, uint64_t n, float *vmin_out, float *vmax_out) {
    int any = 0;
    float lo = 0.0f, hi = 0.0f;
    for (uint64_t i = 0; i < n; ++i) {
        float v = x[i];
        if (!isfinite(v)) continue;
        if (!any) {
            lo = v;
            hi = v;
            any = 1;
        } else {
            if (v < lo) lo = v;
            if (v > hi) hi = v;
        }
    }
    *vmin_out = lo + 0.0f;
    *vmax_out = hi + 0.0f;
    return any;
}

/* Step 2. Bound resolution ([SPEC] Priming; Inverse declaration: dequant step
 * 2*abs_eb; Forward declaration: the float inv2eb slot).  All in IEEE double,
 * round to nearest, then rounded once to float.                             */
void orc_resolve_bound(int abs_mode, double bound, float vmin, float vmax,
                       double *eb_out, float *inv2eb_out, float *step_out) {
    double eb;
    if (abs_mode)
        eb = bound;
    else
        eb = bound * ((double)vmax - (double)vmin);
    double two_eb = 2.0 * eb;
    double inv = (two_eb == 0.0) ? INFINITY : 1.0 / two_eb;
    *eb_out = eb;
    *inv2eb_out = (float)inv;
    *step_out = (float)two_eb;
}

/* Step 3. Linear quantization of one element ([SPEC] Roles and strategies:
 * the linear quantizer is Elementwise, absorbed into the predictor).        */
static int32_t quant_code(float x, float inv2eb) {
    float y = x * inv2eb;
    if (!(fabsf(y) < 1073741824.0f)) /* 2^30; false for NaN and +-Inf */
        return 0;
    return (int32_t)nearbyintf(y); /* round half to even (FE_TONEAREST) */
}

static float dequant(int32_t q, float step) { return (float)q * step; }

/* Outlier test for one element ([NVRTC] split-outlier side output).        */
static int outlier_test(float x, float xr, double eb) {
    if (!isfinite(x)) return 1;
    return !(fabs((double)x - (double)xr) <= eb);
}

/* Quantize a whole array; exposed so the tests can pin step 3 alone.        */
void orc_quantize(const float *x, uint64_t n, float inv2eb, float step, double eb,
                  int32_t *q_out, uint8_t *outlier_out) {
    for (uint64_t i = 0; i < n; ++i) {
        int32_t q = quant_code(x[i], inv2eb);
        q_out[i] = q;
        outlier_out[i] = (uint8_t)outlier_test(x[i], dequant(q, step), eb);
    }
}

/* Step 5. Zigzag (textbook): d >= 0 -> 2d, d < 0 -> -2d - 1.                */
uint32_t orc_zigzag(int32_t d) {
    int64_t v = d;
    if (v >= 0) return (uint32_t)(2 * v);
    return (uint32_t)(-2 * v - 1);
}

int32_t orc_unzigzag(uint32_t z) {
    if ((z & 1u) == 0) return (int32_t)(z / 2u);
    return (int32_t)(-(int64_t)(z / 2u) - 1);
}

/* Step 6a. Block width: bit length of the OR of the codes (0..32).          */
uint32_t orc_block_width(const uint32_t *z, uint32_t cnt) {
    uint32_t acc = 0, w = 0;
    for (uint32_t j = 0; j < cnt; ++j) acc |= z[j];
    while (acc != 0) {
        ++w;
        acc >>= 1;
    }
    return w;
}

uint32_t orc_block_words(uint32_t w, uint32_t cnt) {
    return (uint32_t)(((uint64_t)w * cnt + 31u) / 32u);
}

/* Step 6b. Fixed-length pack: code j at bits [j*w, j*w+w) of the block's
 * word array, least significant bit first.  words[] must hold
 * orc_block_words(w, cnt) words; it is cleared here.                        */
void orc_pack_block(const uint32_t *z, uint32_t cnt, uint32_t w, uint32_t *words) {
    uint32_t nw = orc_block_words(w, cnt);
    for (uint32_t k = 0; k < nw; ++k) words[k] = 0;
    if (w == 0) return;
    for (uint32_t j = 0; j < cnt; ++j) {
        uint64_t pos = (uint64_t)j * w;
        uint64_t k = pos / 32u;
        uint32_t sh = (uint32_t)(pos % 32u);
        uint64_t v = (uint64_t)z[j] << sh;
        words[k] |= (uint32_t)v;
        if ((v >> 32) != 0) words[k + 1] |= (uint32_t)(v >> 32);
    }
}

void orc_unpack_block(const uint32_t *words, uint32_t cnt, uint32_t w, uint32_t *z) {
    uint32_t nw = orc_block_words(w, cnt);
    uint64_t mask = (w == 32) ? 0xFFFFFFFFull : ((1ull << w) - 1ull);
    for (uint32_t j = 0; j < cnt; ++j) {
        if (w == 0) {
            z[j] = 0;
            continue;
        }
        uint64_t pos = (uint64_t)j * w;
        uint64_t k = pos / 32u;
        uint32_t sh = (uint32_t)(pos % 32u);
        uint64_t v = words[k];
        if (k + 1 < nw) v |= (uint64_t)words[k + 1] << 32;
        z[j] = (uint32_t)((v >> sh) & mask);
    }
}

/* ------------------------------------------------------------------------ */
/* Section offsets of a stream with nb blocks, nc chunks, W payload words and
 * m outliers.                                                               */
typedef struct {
    uint64_t width_off, index_off, record_off, total;
} orc_layout;

static orc_layout layout_of(uint64_t nb, uint64_t nc, uint64_t W, uint64_t m) {
    orc_layout L;
    L.width_off = ORC_HEADER_BYTES;
    L.index_off = L.width_off + pad16(nb);
    L.record_off = L.index_off + pad16(8u * nc);
    L.total = L.record_off + 4u * (W + 2u * m);
    return L;
}

static int block_ok(uint32_t b) { return b == 32 || b == 64 || b == 128 || b == 256; }

#define ORC_MAX_N (1ull << 30)

/* Worst-case stream size: every block at width 32 and outlier_cap outliers. */
uint64_t orc_max_compressed_bytes(uint64_t n, uint32_t block, uint64_t outlier_cap) {
    if (!block_ok(block)) return 0;
    uint64_t nb = (n + block - 1) / block;
    uint64_t nc = (n + ORC_CHUNK - 1) / ORC_CHUNK;
    return layout_of(nb, nc, n, outlier_cap).total;
}

/* ------------------------------------------------------------------------ */
/* Compress x[0..n) into out[0..out_cap).  Returns the stream length, or a
 * negative ORC_ERR_* code.  More outliers than outlier_cap is an error.
 * `range` (relative bound only): NULL to take the value range of x itself
 * (step 1), else {vmin, vmax} given by the caller.                         */
static int64_t compress_with(const float *x, uint64_t n, uint32_t block, int abs_mode, double bound,
                             const float *range, uint64_t outlier_cap, uint8_t *out, uint64_t out_cap) {
    if (!block_ok(block) || !(bound >= 0.0) || !isfinite(bound)) return ORC_ERR_ARG;
    if (n > ORC_MAX_N) return ORC_ERR_ARG;
    if (fegetround() != FE_TONEAREST) return ORC_ERR_ARG;

    /* steps 1-2 */
    float vmin = 0.0f, vmax = 0.0f;
    if (!abs_mode && range) {
        vmin = range[0] + 0.0f;
        vmax = range[1] + 0.0f;
    } else if (!abs_mode) {
        orc_value_range(x, n, &vmin, &vmax);
    }
    double eb;
    float inv2eb, step;
    orc_resolve_bound(abs_mode, bound, vmin, vmax, &eb, &inv2eb, &step);

    uint64_t nb = (n + block - 1) / block;
    uint64_t nc = (n + ORC_CHUNK - 1) / ORC_CHUNK;

    /* step 3: codes and outlier flags for every element */
    int32_t *q = (int32_t *)malloc((n ? n : 1) * sizeof(int32_t));
    uint8_t *flag = (uint8_t *)malloc(n ? n : 1);
    uint8_t *width = (uint8_t *)malloc(nb ? nb : 1);
    uint32_t *block_words = (uint32_t *)malloc((nb ? nb : 1) * sizeof(uint32_t));
    if (!q || !flag || !width || !block_words) {
        free(q); free(flag); free(width); free(block_words);
        return ORC_ERR_NOMEM;
    }
    orc_quantize(x, n, inv2eb, step, eb, q, flag);

    uint64_t m = 0;
    for (uint64_t i = 0; i < n; ++i) m += flag[i];

    /* steps 4-6a: per block delta (reset at the block start), zigzag, width */
    uint32_t z[256];
    uint64_t W = 0;
    for (uint64_t b = 0; b < nb; ++b) {
        uint64_t first = b * block;
        uint32_t cnt = (uint32_t)((n - first < block) ? (n - first) : block);
        int32_t prev = 0; /* Lorenzo predecessor resets to 0 at each block */
        for (uint32_t j = 0; j < cnt; ++j) {
            int32_t cur = q[first + j];
            z[j] = orc_zigzag(cur - prev); /* |q| < 2^30 so no overflow */
            prev = cur;
        }
        width[b] = (uint8_t)orc_block_width(z, cnt);
        block_words[b] = orc_block_words(width[b], cnt);
        W += block_words[b];
    }

    orc_layout L = layout_of(nb, nc, W, m);
    int64_t status = (int64_t)L.total;
    if (m > outlier_cap) status = ORC_ERR_OUTLIER_CAP;
    else if (L.total > out_cap) status = ORC_ERR_CAPACITY;
    if (status < 0) {
        free(q); free(flag); free(width); free(block_words);
        return status;
    }

    memset(out, 0, L.total);
    /* header */
    put_u32(out + 0, ORC_MAGIC);
    put_u16(out + 4, (uint16_t)ORC_VERSION);
    put_u16(out + 6, (uint16_t)(abs_mode ? ORC_FLAG_ABS : 0u));
    put_u64(out + 8, n);
    put_u32(out + 16, block);
    put_u32(out + 20, ORC_CHUNK);
    put_f64(out + 24, eb);
    put_f32(out + 32, inv2eb);
    put_f32(out + 36, step);
    put_f32(out + 40, vmin);
    put_f32(out + 44, vmax);
    put_u64(out + 48, nb);
    put_u64(out + 56, nc);
    put_u64(out + 64, W);
    put_u64(out + 72, m);
    put_u64(out + 80, L.total);
    put_f64(out + 88, bound);

    /* widths */
    memcpy(out + L.width_off, width, nb);

    /* step 6b + step 8, chunk by chunk: the chunk index entry (record word
     * offset, outliers so far), then each block packed at the scanned word
     * offset, then the chunk's outliers ([NVRTC] split-outlier side output,
     * index array then value array; step 7).                               */
    uint64_t rec = 0, outl_before = 0, blocks_per_chunk = ORC_CHUNK / block;
    uint32_t words[256];
    for (uint64_t c = 0; c < nc; ++c) {
        put_u32(out + L.index_off + 8 * c, (uint32_t)rec);
        put_u32(out + L.index_off + 8 * c + 4, (uint32_t)outl_before);
        uint64_t b_end = (c + 1) * blocks_per_chunk < nb ? (c + 1) * blocks_per_chunk : nb;
        for (uint64_t b = c * blocks_per_chunk; b < b_end; ++b) {
            uint64_t first = b * block;
            uint32_t cnt = (uint32_t)((n - first < block) ? (n - first) : block);
            int32_t prev = 0;
            for (uint32_t j = 0; j < cnt; ++j) {
                int32_t cur = q[first + j];
                z[j] = orc_zigzag(cur - prev);
                prev = cur;
            }
            orc_pack_block(z, cnt, width[b], words);
            for (uint32_t k = 0; k < block_words[b]; ++k)
                put_u32(out + L.record_off + 4 * (rec + k), words[k]);
            rec += block_words[b];
        }
        uint64_t e_first = c * ORC_CHUNK;
        uint64_t e_end = e_first + ORC_CHUNK < n ? e_first + ORC_CHUNK : n;
        uint64_t mc = 0;
        for (uint64_t i = e_first; i < e_end; ++i) mc += flag[i];
        uint64_t k = 0;
        for (uint64_t i = e_first; i < e_end; ++i) {
            if (!flag[i]) continue;
            uint32_t bits;
            memcpy(&bits, &x[i], 4);
            put_u32(out + L.record_off + 4 * (rec + k), (uint32_t)i);
            put_u32(out + L.record_off + 4 * (rec + mc + k), bits);
            ++k;
        }
        rec += 2 * mc;
        outl_before += mc;
    }

    free(q); free(flag); free(width); free(block_words);
    return (int64_t)L.total;
}

int64_t orc_compress(const float *x, uint64_t n, uint32_t block, int abs_mode, double bound,
                     uint64_t outlier_cap, uint8_t *out, uint64_t out_cap) {
    return compress_with(x, n, block, abs_mode, bound, NULL, outlier_cap, out, out_cap);
}

/* One contiguous part of a larger array, coded under the relative bound of
 * the whole: eb = rel * (vmax - vmin) with the whole array's value range
 * {vmin, vmax} given by the caller instead of the part's own ([SPEC]
 * Priming: the bound is resolved from a value range before any code is
 * produced; "DevitoComp provider interface", Validating a private provider:
 * the provider runs under an MPI-run consumer, one part of the domain per
 * process).  vmin <= vmax, both finite, else ORC_ERR_ARG.  With the part's
 * own range this is orc_compress.                                           */
int64_t orc_compress_range(const float *x, uint64_t n, uint32_t block, double rel, float vmin, float vmax,
                           uint64_t outlier_cap, uint8_t *out, uint64_t out_cap) {
    if (!isfinite(vmin) || !isfinite(vmax) || !(vmin <= vmax)) return ORC_ERR_ARG;
    const float range[2] = {vmin, vmax};
    return compress_with(x, n, block, 0, rel, range, outlier_cap, out, out_cap);
}

/* ------------------------------------------------------------------------ */
/* Multi-dimensional Lorenzo ([SPEC] Roles and strategies: a RegionLocal
 * predictor is one whose values may depend on others within a fixed logical
 * region, with no dependency across regions; the 1-D Lorenzo predictor with
 * region reset is the one the pages print).  Reading for 2-D / 3-D data
 * (the pages print no multi-dimensional predictor): the region is a block of
 * the array's own dims -- bz x by x bx elements -- and the predictor is the
 * classical Lorenzo stencil over the quantization codes, with every
 * neighbour outside the block taken as 0 (the region reset):
 *   d(i,j,k) = sum over a,b,c in {0,1} of (-1)^(a+b+c) q(i-a, j-b, k-c),
 * i.e. the first difference along x, then y, then z.  Its inverse is the
 * inclusive prefix sum along each axis of the block.  d is taken modulo
 * 2^32 (two's complement), so the inverse is exact even where a sum of
 * eight codes would not fit in 32 bits.
 *
 * Layout reading: a chunk is a brick of 16 x 16 x 16 elements (3-D) or
 * 64 x 64 (2-D), the array's dims must be multiples of the brick, bricks are
 * taken in C order over the brick grid, blocks in C order within a brick,
 * codes in C order within a block; the header's bytes 96..119 hold Z, Y, X
 * (Z = 1 for 2-D).  Outlier indices are the elements' C-order indices in
 * the whole array, ascending within each brick.  Blocks: 64 -> 4x4x4 (3-D)
 * or 8x8 (2-D); 256 -> 4x8x8 (3-D) or 16x16 (2-D).                        */
int orc_nd_edges(int rank, uint32_t block, uint32_t be[3], uint32_t ce[3]) {
    if (rank == 3) {
        ce[0] = ce[1] = ce[2] = 16;
        if (block == 64) { be[0] = 4; be[1] = 4; be[2] = 4; return 1; }
        if (block == 256) { be[0] = 4; be[1] = 8; be[2] = 8; return 1; }
    } else if (rank == 2) {
        ce[0] = 1; ce[1] = ce[2] = 64;
        if (block == 64) { be[0] = 1; be[1] = 8; be[2] = 8; return 1; }
        if (block == 256) { be[0] = 1; be[1] = 16; be[2] = 16; return 1; }
    }
    return 0;
}

/* Flat C-order index of element e (block order) of block `b` (brick order)
 * for dims d[3], block edges be[3], brick edges ce[3].                      */
static uint64_t nd_flat(uint64_t b, uint32_t e, const uint64_t d[3], const uint32_t be[3], const uint32_t ce[3]) {
    uint64_t kz = ce[0] / be[0], ky = ce[1] / be[1], kx = ce[2] / be[2];
    uint64_t bpc = kz * ky * kx;
    uint64_t c = b / bpc, bi = b % bpc;
    uint64_t gx = d[2] / ce[2], gy = d[1] / ce[1];
    uint64_t cz = c / (gy * gx), cy = (c / gx) % gy, cx = c % gx;
    uint64_t iz = bi / (ky * kx), iy = (bi / kx) % ky, ix = bi % kx;
    uint64_t ez = e / (be[1] * be[2]), ey = (e / be[2]) % be[1], ex = e % be[2];
    uint64_t z = cz * ce[0] + iz * be[0] + ez;
    uint64_t y = cy * ce[1] + iy * be[1] + ey;
    uint64_t x = cx * ce[2] + ix * be[2] + ex;
    return (z * d[1] + y) * d[2] + x;
}

/* Lorenzo residuals of one block: q[] in block order -> d[] (as int32,
 * modulo 2^32), neighbours outside the block are 0.                        */
void orc_lorenzo_block(const int32_t *q, const uint32_t be[3], int32_t *d) {
    for (uint32_t i = 0; i < be[0]; ++i)
        for (uint32_t j = 0; j < be[1]; ++j)
            for (uint32_t k = 0; k < be[2]; ++k) {
                uint32_t acc = 0;
                for (uint32_t a = 0; a < 2; ++a)
                    for (uint32_t b = 0; b < 2; ++b)
                        for (uint32_t c = 0; c < 2; ++c) {
                            if (a > i || b > j || c > k) continue; /* outside the block: 0 */
                            uint32_t v = (uint32_t)q[((i - a) * be[1] + (j - b)) * be[2] + (k - c)];
                            acc = ((a + b + c) & 1u) ? acc - v : acc + v;
                        }
                d[(i * be[1] + j) * be[2] + k] = (int32_t)acc;
            }
}

/* Inverse: inclusive prefix sums along x, then y, then z (modulo 2^32).    */
void orc_unlorenzo_block(const int32_t *d, const uint32_t be[3], int32_t *q) {
    uint32_t nb = be[0] * be[1] * be[2];
    for (uint32_t e = 0; e < nb; ++e) q[e] = d[e];
    for (uint32_t i = 0; i < be[0]; ++i)
        for (uint32_t j = 0; j < be[1]; ++j)
            for (uint32_t k = 1; k < be[2]; ++k) {
                uint32_t e = (i * be[1] + j) * be[2] + k;
                q[e] = (int32_t)((uint32_t)q[e] + (uint32_t)q[e - 1]);
            }
    for (uint32_t i = 0; i < be[0]; ++i)
        for (uint32_t j = 1; j < be[1]; ++j)
            for (uint32_t k = 0; k < be[2]; ++k) {
                uint32_t e = (i * be[1] + j) * be[2] + k;
                q[e] = (int32_t)((uint32_t)q[e] + (uint32_t)q[e - be[2]]);
            }
    for (uint32_t i = 1; i < be[0]; ++i)
        for (uint32_t j = 0; j < be[1]; ++j)
            for (uint32_t k = 0; k < be[2]; ++k) {
                uint32_t e = (i * be[1] + j) * be[2] + k;
                q[e] = (int32_t)((uint32_t)q[e] + (uint32_t)q[e - be[1] * be[2]]);
            }
}

/* Compress an array of dims {Z, Y, X} (rank 3) or {1, Y, X} (rank 2) with
 * the multi-dimensional Lorenzo predictor.  Same steps and stream as
 * orc_compress otherwise.  Returns the stream length or ORC_ERR_*.        */
int64_t orc_compress_lorenzo(const float *x, int rank, const uint64_t dims[3], uint32_t block, int abs_mode,
                             double bound, uint64_t outlier_cap, uint8_t *out, uint64_t out_cap) {
    uint32_t be[3], ce[3];
    if (!orc_nd_edges(rank, block, be, ce) || !(bound >= 0.0) || !isfinite(bound)) return ORC_ERR_ARG;
    if ((rank == 2 && dims[0] != 1) || dims[0] % ce[0] || dims[1] % ce[1] || dims[2] % ce[2]) return ORC_ERR_ARG;
    if (dims[0] > ORC_MAX_N || dims[1] > ORC_MAX_N || dims[2] > ORC_MAX_N) return ORC_ERR_ARG;
    uint64_t n = dims[0] * dims[1] * dims[2];
    if (n > ORC_MAX_N) return ORC_ERR_ARG;
    if (fegetround() != FE_TONEAREST) return ORC_ERR_ARG;

    float vmin = 0.0f, vmax = 0.0f;
    if (!abs_mode) orc_value_range(x, n, &vmin, &vmax);
    double eb;
    float inv2eb, step;
    orc_resolve_bound(abs_mode, bound, vmin, vmax, &eb, &inv2eb, &step);

    uint64_t nb = n / block, nc = n / ORC_CHUNK, bpc = ORC_CHUNK / block;
    int32_t *q = (int32_t *)malloc((n ? n : 1) * sizeof(int32_t));
    uint8_t *flag = (uint8_t *)malloc(n ? n : 1);
    uint8_t *width = (uint8_t *)malloc(nb ? nb : 1);
    if (!q || !flag || !width) {
        free(q); free(flag); free(width);
        return ORC_ERR_NOMEM;
    }
    orc_quantize(x, n, inv2eb, step, eb, q, flag);
    uint64_t m = 0, W = 0;
    for (uint64_t i = 0; i < n; ++i) m += flag[i];

    int32_t qb[256], db[256];
    uint32_t z[256], words[256];
    for (uint64_t b = 0; b < nb; ++b) {  /* widths */
        for (uint32_t e = 0; e < block; ++e) qb[e] = q[nd_flat(b, e, dims, be, ce)];
        orc_lorenzo_block(qb, be, db);
        for (uint32_t e = 0; e < block; ++e) z[e] = orc_zigzag(db[e]);
        width[b] = (uint8_t)orc_block_width(z, block);
        W += orc_block_words(width[b], block);
    }
    orc_layout L = layout_of(nb, nc, W, m);
    int64_t status = (int64_t)L.total;
    if (m > outlier_cap) status = ORC_ERR_OUTLIER_CAP;
    else if (L.total > out_cap) status = ORC_ERR_CAPACITY;
    if (status < 0) {
        free(q); free(flag); free(width);
        return status;
    }
    memset(out, 0, L.total);
    put_u32(out + 0, ORC_MAGIC);
    put_u16(out + 4, (uint16_t)ORC_VERSION);
    put_u16(out + 6, (uint16_t)((abs_mode ? ORC_FLAG_ABS : 0u) | ORC_FLAG_LORENZO_ND));
    put_u64(out + 8, n);
    put_u32(out + 16, block);
    put_u32(out + 20, ORC_CHUNK);
    put_f64(out + 24, eb);
    put_f32(out + 32, inv2eb);
    put_f32(out + 36, step);
    put_f32(out + 40, vmin);
    put_f32(out + 44, vmax);
    put_u64(out + 48, nb);
    put_u64(out + 56, nc);
    put_u64(out + 64, W);
    put_u64(out + 72, m);
    put_u64(out + 80, L.total);
    put_f64(out + 88, bound);
    put_u64(out + 96, dims[0]);
    put_u64(out + 104, dims[1]);
    put_u64(out + 112, dims[2]);
    memcpy(out + L.width_off, width, nb);

    uint64_t rec = 0, before = 0;
    for (uint64_t c = 0; c < nc; ++c) {
        put_u32(out + L.index_off + 8 * c, (uint32_t)rec);
        put_u32(out + L.index_off + 8 * c + 4, (uint32_t)before);
        for (uint64_t b = c * bpc; b < (c + 1) * bpc; ++b) {
            for (uint32_t e = 0; e < block; ++e) qb[e] = q[nd_flat(b, e, dims, be, ce)];
            orc_lorenzo_block(qb, be, db);
            for (uint32_t e = 0; e < block; ++e) z[e] = orc_zigzag(db[e]);
            orc_pack_block(z, block, width[b], words);
            uint32_t nw = orc_block_words(width[b], block);
            for (uint32_t k = 0; k < nw; ++k) put_u32(out + L.record_off + 4 * (rec + k), words[k]);
            rec += nw;
        }
        /* the brick's outliers, ascending C-order index: z, then y, then x */
        uint64_t gx = dims[2] / ce[2], gy = dims[1] / ce[1];
        uint64_t z0 = c / (gy * gx) * ce[0], y0 = (c / gx) % gy * ce[1], x0 = c % gx * ce[2];
        uint64_t mc = 0, k = 0;
        for (uint64_t zz = z0; zz < z0 + ce[0]; ++zz)
            for (uint64_t yy = y0; yy < y0 + ce[1]; ++yy)
                for (uint64_t xx = x0; xx < x0 + ce[2]; ++xx) mc += flag[(zz * dims[1] + yy) * dims[2] + xx];
        for (uint64_t zz = z0; zz < z0 + ce[0]; ++zz)
            for (uint64_t yy = y0; yy < y0 + ce[1]; ++yy)
                for (uint64_t xx = x0; xx < x0 + ce[2]; ++xx) {
                    uint64_t i = (zz * dims[1] + yy) * dims[2] + xx;
                    if (!flag[i]) continue;
                    uint32_t bits;
                    memcpy(&bits, &x[i], 4);
                    put_u32(out + L.record_off + 4 * (rec + k), (uint32_t)i);
                    put_u32(out + L.record_off + 4 * (rec + mc + k), bits);
                    ++k;
                }
        rec = rec + 2 * mc;   /* the brick's outlier indices and values */
        before = before + mc;
    }
    free(q); free(flag); free(width);
    return (int64_t)L.total;
}

/* ------------------------------------------------------------------------ */
/* Parsed header, exposed for the tests.                                     */
typedef struct {
    uint32_t magic, version, flags, block, chunk, pad;
    uint64_t n, nb, nc, W, m, total;
    double eb, bound;
    float inv2eb, step, vmin, vmax;
    uint64_t width_off, index_off, record_off;
    uint64_t dims[3];  /* Z, Y, X of a multi-dimensional Lorenzo stream, else 0 */
} orc_header;

int orc_parse_header(const uint8_t *s, uint64_t bytes, orc_header *h) {
    memset(h, 0, sizeof(*h));
    if (bytes < ORC_HEADER_BYTES) return ORC_ERR_CORRUPT;
    h->magic = get_u32(s + 0);
    h->version = get_u16(s + 4);
    h->flags = get_u16(s + 6);
    h->n = get_u64(s + 8);
    h->block = get_u32(s + 16);
    h->chunk = get_u32(s + 20);
    h->eb = get_f64(s + 24);
    h->inv2eb = get_f32(s + 32);
    h->step = get_f32(s + 36);
    h->vmin = get_f32(s + 40);
    h->vmax = get_f32(s + 44);
    h->nb = get_u64(s + 48);
    h->nc = get_u64(s + 56);
    h->W = get_u64(s + 64);
    h->m = get_u64(s + 72);
    h->total = get_u64(s + 80);
    h->bound = get_f64(s + 88);
    h->dims[0] = get_u64(s + 96);
    h->dims[1] = get_u64(s + 104);
    h->dims[2] = get_u64(s + 112);
    if ((h->flags & ORC_FLAG_RRE) && !(h->flags & ORC_FLAG_CHUNKED)) return ORC_ERR_CORRUPT;  /* RRE codes chunks only */
    if (h->flags & ORC_FLAG_CHUNKED) {
        if (h->magic != ORC_MAGIC || h->version != ORC_VERSION || h->block != 0 ||
            (h->chunk != 1024 && h->chunk != 2048 && h->chunk != 4096) || (h->flags & ORC_FLAG_LORENZO_ND) ||
            h->n > ORC_MAX_N || h->nb != 0 || h->nc != (h->n + h->chunk - 1) / h->chunk ||
            h->W > h->n + 32 * h->nc || h->m > h->n || h->dims[0] || h->dims[1] || h->dims[2])
            return ORC_ERR_CORRUPT;
        orc_layout L = layout_of(0, h->nc, h->W, h->m);
        if (L.total != h->total || h->total > bytes) return ORC_ERR_CORRUPT;
        h->width_off = L.width_off;
        h->index_off = L.index_off;
        h->record_off = L.record_off;
        return 0;
    }
    if (h->magic != ORC_MAGIC || h->version != ORC_VERSION || !block_ok(h->block) ||
        h->chunk != ORC_CHUNK)
        return ORC_ERR_CORRUPT;
    if (h->flags & ORC_FLAG_LORENZO_ND) {
        uint32_t be[3], ce[3];
        int rank = h->dims[0] == 1 ? 2 : 3;
        if (!orc_nd_edges(rank, h->block, be, ce) || h->dims[0] * h->dims[1] * h->dims[2] != h->n ||
            h->dims[0] % ce[0] || h->dims[1] % ce[1] || h->dims[2] % ce[2])
            return ORC_ERR_CORRUPT;
    } else if (h->dims[0] || h->dims[1] || h->dims[2]) {
        return ORC_ERR_CORRUPT;
    }
    if (h->n > ORC_MAX_N || h->nb != (h->n + h->block - 1) / h->block ||
        h->nc != (h->n + ORC_CHUNK - 1) / ORC_CHUNK || h->W > h->n || h->m > h->n)
        return ORC_ERR_CORRUPT;
    orc_layout L = layout_of(h->nb, h->nc, h->W, h->m);
    if (L.total != h->total || h->total > bytes) return ORC_ERR_CORRUPT;
    h->width_off = L.width_off;
    h->index_off = L.index_off;
    h->record_off = L.record_off;
    return 0;
}

/* Inverse ([SPEC] Inverse declaration; device policy contract: decode ->
 * undelta -> dequant code * 2eb), then each chunk's outliers are written
 * back over the reconstruction.                                            */
static int decompress_nd(const uint8_t *s, const orc_header *h, float *out);
static int decompress_chunked(const uint8_t *s, const orc_header *h, float *out);

int orc_decompress(const uint8_t *s, uint64_t bytes, float *out, uint64_t n_expected) {
    orc_header h;
    int rc = orc_parse_header(s, bytes, &h);
    if (rc != 0) return rc;
    if (h.n != n_expected) return ORC_ERR_ARG;
    if (h.flags & ORC_FLAG_LORENZO_ND) return decompress_nd(s, &h, out);
    if (h.flags & ORC_FLAG_CHUNKED) return decompress_chunked(s, &h, out);

    uint32_t words[256], z[256];
    uint64_t blocks_per_chunk = ORC_CHUNK / h.block;
    uint64_t R = h.W + 2 * h.m, W_seen = 0;
    for (uint64_t c = 0; c < h.nc; ++c) {
        uint64_t rec = get_u32(s + h.index_off + 8 * c);
        uint64_t before = get_u32(s + h.index_off + 8 * c + 4);
        uint64_t rec_next = (c + 1 < h.nc) ? get_u32(s + h.index_off + 8 * (c + 1)) : R;
        uint64_t after = (c + 1 < h.nc) ? get_u32(s + h.index_off + 8 * (c + 1) + 4) : h.m;
        if (rec_next < rec || after < before || rec_next > R || after > h.m) return ORC_ERR_CORRUPT;
        uint64_t mc = after - before;
        uint64_t word_off = rec;
        uint64_t b_end = (c + 1) * blocks_per_chunk < h.nb ? (c + 1) * blocks_per_chunk : h.nb;
        for (uint64_t b = c * blocks_per_chunk; b < b_end; ++b) {
            uint64_t first = b * h.block;
            uint32_t cnt = (uint32_t)((h.n - first < h.block) ? (h.n - first) : h.block);
            uint32_t w = s[h.width_off + b];
            if (w > 32) return ORC_ERR_CORRUPT;
            uint32_t nw = orc_block_words(w, cnt);
            if (word_off + nw > rec_next) return ORC_ERR_CORRUPT;
            for (uint32_t k = 0; k < nw; ++k)
                words[k] = get_u32(s + h.record_off + 4 * (word_off + k));
            orc_unpack_block(words, cnt, w, z);
            int64_t qv = 0; /* undelta: running sum restarting at each block */
            for (uint32_t j = 0; j < cnt; ++j) {
                qv += orc_unzigzag(z[j]);
                int32_t q = (int32_t)(uint32_t)(uint64_t)qv;
                out[first + j] = dequant(q, h.step);
            }
            word_off += nw;
        }
        if (word_off + 2 * mc != rec_next) return ORC_ERR_CORRUPT;
        W_seen += word_off - rec;
        uint64_t e_first = c * ORC_CHUNK;
        uint64_t e_end = e_first + ORC_CHUNK < h.n ? e_first + ORC_CHUNK : h.n;
        for (uint64_t k = 0; k < mc; ++k) {
            uint32_t i = get_u32(s + h.record_off + 4 * (word_off + k));
            uint32_t bits = get_u32(s + h.record_off + 4 * (word_off + mc + k));
            if (i < e_first || i >= e_end) return ORC_ERR_CORRUPT;
            memcpy(&out[i], &bits, 4);
        }
    }
    if (W_seen != h.W) return ORC_ERR_CORRUPT;
    return 0;
}

/* Inverse of orc_compress_lorenzo: per brick, each block's codes unpacked,
 * the Lorenzo residuals summed back (inclusive prefix sums along x, y, z
 * within the block), dequantized and placed at their C-order positions;
 * then the brick's outliers written back.                                  */
static int decompress_nd(const uint8_t *s, const orc_header *h, float *out) {
    uint32_t be[3], ce[3];
    int rank = h->dims[0] == 1 ? 2 : 3;
    if (!orc_nd_edges(rank, h->block, be, ce)) return ORC_ERR_CORRUPT;
    uint32_t words[256], z[256];
    int32_t d[256], q[256];
    uint64_t bpc = ORC_CHUNK / h->block, R = h->W + 2 * h->m, W_seen = 0;
    uint64_t gx = h->dims[2] / ce[2], gy = h->dims[1] / ce[1];
    for (uint64_t c = 0; c < h->nc; ++c) {
        uint64_t rec = get_u32(s + h->index_off + 8 * c);
        uint64_t before = get_u32(s + h->index_off + 8 * c + 4);
        uint64_t rec_next = (c + 1 < h->nc) ? get_u32(s + h->index_off + 8 * (c + 1)) : R;
        uint64_t after = (c + 1 < h->nc) ? get_u32(s + h->index_off + 8 * (c + 1) + 4) : h->m;
        if (rec_next < rec || after < before || rec_next > R || after > h->m) return ORC_ERR_CORRUPT;
        uint64_t mc = after - before, word_off = rec;
        for (uint64_t b = c * bpc; b < (c + 1) * bpc; ++b) {
            uint32_t w = s[h->width_off + b];
            if (w > 32) return ORC_ERR_CORRUPT;
            uint32_t nw = orc_block_words(w, h->block);
            if (word_off + nw > rec_next) return ORC_ERR_CORRUPT;
            for (uint32_t k = 0; k < nw; ++k) words[k] = get_u32(s + h->record_off + 4 * (word_off + k));
            orc_unpack_block(words, h->block, w, z);
            for (uint32_t e = 0; e < h->block; ++e) d[e] = orc_unzigzag(z[e]);
            orc_unlorenzo_block(d, be, q);
            for (uint32_t e = 0; e < h->block; ++e) out[nd_flat(b, e, h->dims, be, ce)] = dequant(q[e], h->step);
            word_off += nw;
        }
        if (word_off + 2 * mc != rec_next) return ORC_ERR_CORRUPT;
        W_seen += word_off - rec;
        uint64_t z0 = c / (gy * gx) * ce[0], y0 = (c / gx) % gy * ce[1], x0 = c % gx * ce[2];
        for (uint64_t k = 0; k < mc; ++k) {
            uint32_t i = get_u32(s + h->record_off + 4 * (word_off + k));
            uint32_t bits = get_u32(s + h->record_off + 4 * (word_off + mc + k));
            uint64_t xx = i % h->dims[2], yy = (i / h->dims[2]) % h->dims[1], zz = i / (h->dims[2] * h->dims[1]);
            if (i >= h->n || zz < z0 || zz >= z0 + ce[0] || yy < y0 || yy >= y0 + ce[1] || xx < x0 ||
                xx >= x0 + ce[2])
                return ORC_ERR_CORRUPT;
            memcpy(&out[i], &bits, 4);
        }
    }
    if (W_seen != h->W) return ORC_ERR_CORRUPT;
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Chunk-cooperative codec ("Pipeline specialization internals",
 * Chunk-cooperative path: one CTA owns a byte chunk of 4096, 8192 or 16384
 * bytes, a Quant -> Diff -> Bitshuffle -> RZE chain; "nvrtc_chunk_fusion.h
 * File Reference", launchNvrtcChunkFusedEncode: each chunk's coded form lands
 * in a scratch slot of CHUNK_BYTES with its size, then a cross-chunk scan
 * packs them into one archive, the outliers leaving through a side list).
 * The pages name the ops and give no definitions; readings:
 *   - chunk: CHUNK_BYTES of float32 input, m = CHUNK_BYTES / 4 elements (the
 *     last chunk may be shorter);
 *   - Quant: the linear quantizer and outlier rule of the main path;
 *   - Diff: first difference of the codes within the chunk (0 before its
 *     first code), taken to zigzag form so that small differences of either
 *     sign leave the high bit planes zero;
 *   - Bitshuffle: the chunk's codes, zero-padded to mp = a multiple of 32, in
 *     groups of 32; bit b of code l of group g is bit l of word b*(mp/32) + g
 *     (32 bit planes, each mp/32 words);
 *   - RZE (zero elimination): one bitmap bit per shuffled word (bit j of the
 *     bitmap: word j is not zero; mp/32 bitmap words, least significant bit
 *     first), then the nonzero words in order;
 *   - RRE (repetition elimination), the coder chosen in place of RZE: one
 *     bitmap bit per shuffled word (bit j: word j differs from word j - 1,
 *     word -1 being 0), then the words that differ, in order; a word whose
 *     bit is clear equals the word before it, so each word is the last kept
 *     word at or before it (0 before the first).  RZE is RRE with every
 *     predecessor taken as 0;
 *   - a chunk whose coded form is not smaller than its mp shuffled words keeps
 *     the shuffled words verbatim, so a coded chunk never exceeds its input;
 *   - record of a chunk: one word P | raw << 31 (P payload words follow),
 *     the payload, then the chunk's outlier indices and values (ascending
 *     index), located by the chunk index as in the main format.          */
void orc_bitshuffle(const uint32_t *in, uint32_t mp, uint32_t *out) {
    uint32_t G = mp / 32;
    for (uint32_t b = 0; b < 32; ++b)
        for (uint32_t g = 0; g < G; ++g) {
            uint32_t word = 0;
            for (uint32_t l = 0; l < 32; ++l) word |= ((in[g * 32 + l] >> b) & 1u) << l;
            out[b * G + g] = word;
        }
}

void orc_unbitshuffle(const uint32_t *in, uint32_t mp, uint32_t *out) {
    uint32_t G = mp / 32;
    for (uint32_t g = 0; g < G; ++g)
        for (uint32_t l = 0; l < 32; ++l) {
            uint32_t code = 0;
            for (uint32_t b = 0; b < 32; ++b) code |= ((in[b * G + g] >> l) & 1u) << b;
            out[g * 32 + l] = code;
        }
}

/* Zero elimination of mp words (mp a multiple of 32): returns the words
 * written to out (mp / 32 bitmap words, then the nonzero words).           */
uint32_t orc_rze(const uint32_t *in, uint32_t mp, uint32_t *out) {
    uint32_t nbm = mp / 32, k = nbm;
    for (uint32_t i = 0; i < nbm; ++i) out[i] = 0;
    for (uint32_t j = 0; j < mp; ++j)
        if (in[j] != 0) {
            out[j / 32] |= 1u << (j % 32);
            out[k++] = in[j];
        }
    return k;
}

/* Inverse: from `avail` words at in, mp words to out.  Returns the words
 * consumed, or -1 if the bitmap calls for more words than avail.           */
int64_t orc_unrze(const uint32_t *in, uint64_t avail, uint32_t mp, uint32_t *out) {
    uint32_t nbm = mp / 32;
    if (avail < nbm) return -1;
    uint64_t k = nbm;
    for (uint32_t j = 0; j < mp; ++j) {
        if ((in[j / 32] >> (j % 32)) & 1u) {
            if (k >= avail) return -1;
            out[j] = in[k++];
        } else {
            out[j] = 0;
        }
    }
    return (int64_t)k;
}

/* Repetition elimination of mp words (mp a multiple of 32): returns the
 * words written to out (mp / 32 bitmap words, then the words that differ
 * from their predecessor, the predecessor of word 0 being 0).              */
uint32_t orc_rre(const uint32_t *in, uint32_t mp, uint32_t *out) {
    uint32_t nbm = mp / 32, k = nbm;
    for (uint32_t i = 0; i < nbm; ++i) out[i] = 0;
    for (uint32_t j = 0; j < mp; ++j) {
        uint32_t pred = j ? in[j - 1] : 0u;
        if (in[j] != pred) {
            out[j >> 5] |= 1u << (j & 31u);
            out[k++] = in[j];
        }
    }
    return k;
}

/* Inverse: from `avail` words at in, mp words to out (a clear bit repeats
 * the word before).  Returns the words consumed, or -1 if the bitmap calls
 * for more words than avail.                                               */
int64_t orc_unrre(const uint32_t *in, uint64_t avail, uint32_t mp, uint32_t *out) {
    uint32_t nbm = mp / 32;
    if (avail < nbm) return -1;
    uint64_t k = nbm;
    uint32_t last = 0;
    for (uint32_t j = 0; j < mp; ++j) {
        if ((in[j / 32] >> (j % 32)) & 1u) {
            if (k >= avail) return -1;
            last = in[k++];
        }
        out[j] = last;
    }
    return (int64_t)k;
}

static int chunk_bytes_ok(uint32_t cb) { return cb == 4096 || cb == 8192 || cb == 16384; }

uint64_t orc_max_chunked_bytes(uint64_t n, uint32_t chunk_bytes, uint64_t outlier_cap) {
    if (!chunk_bytes_ok(chunk_bytes)) return 0;
    uint64_t m = chunk_bytes / 4, nc = (n + m - 1) / m;
    return layout_of(0, nc, nc + n + 31 * nc, outlier_cap).total;
}

/* coder 0: RZE, 1: RRE. */
int64_t orc_compress_chunked_coder(const float *x, uint64_t n, uint32_t chunk_bytes, int coder, int abs_mode,
                                   double bound, uint64_t outlier_cap, uint8_t *out, uint64_t out_cap) {
    if (!chunk_bytes_ok(chunk_bytes) || !(bound >= 0.0) || !isfinite(bound)) return ORC_ERR_ARG;
    if (coder != 0 && coder != 1) return ORC_ERR_ARG;
    if (n > ORC_MAX_N) return ORC_ERR_ARG;
    if (fegetround() != FE_TONEAREST) return ORC_ERR_ARG;
    float vmin = 0.0f, vmax = 0.0f;
    if (!abs_mode) orc_value_range(x, n, &vmin, &vmax);
    double eb;
    float inv2eb, step;
    orc_resolve_bound(abs_mode, bound, vmin, vmax, &eb, &inv2eb, &step);

    uint32_t mc_max = chunk_bytes / 4;
    uint64_t nc = (n + mc_max - 1) / mc_max;
    int32_t *q = (int32_t *)malloc((n ? n : 1) * sizeof(int32_t));
    uint8_t *flag = (uint8_t *)malloc(n ? n : 1);
    uint32_t *d = (uint32_t *)malloc(4096 * 4), *sh = (uint32_t *)malloc(4096 * 4);
    uint32_t *rz = (uint32_t *)malloc((4096 + 128) * 4);
    if (!q || !flag || !d || !sh || !rz) {
        free(q); free(flag); free(d); free(sh); free(rz);
        return ORC_ERR_NOMEM;
    }
    orc_quantize(x, n, inv2eb, step, eb, q, flag);
    uint64_t m = 0, W = 0;
    for (uint64_t i = 0; i < n; ++i) m += flag[i];
    for (int pass = 0; pass < 2; ++pass) {
        /* pass 0 sizes every chunk; pass 1 writes the stream */
        orc_layout L = layout_of(0, nc, W, m);
        if (pass == 1) {
            int64_t status = (int64_t)L.total;
            if (m > outlier_cap) status = ORC_ERR_OUTLIER_CAP;
            else if (L.total > out_cap) status = ORC_ERR_CAPACITY;
            if (status < 0) {
                free(q); free(flag); free(d); free(sh); free(rz);
                return status;
            }
            memset(out, 0, L.total);
            put_u32(out + 0, ORC_MAGIC);
            put_u16(out + 4, (uint16_t)ORC_VERSION);
            put_u16(out + 6, (uint16_t)((abs_mode ? ORC_FLAG_ABS : 0u) | ORC_FLAG_CHUNKED | (coder ? ORC_FLAG_RRE : 0u)));
            put_u64(out + 8, n);
            put_u32(out + 16, 0);
            put_u32(out + 20, mc_max);
            put_f64(out + 24, eb);
            put_f32(out + 32, inv2eb);
            put_f32(out + 36, step);
            put_f32(out + 40, vmin);
            put_f32(out + 44, vmax);
            put_u64(out + 48, 0);
            put_u64(out + 56, nc);
            put_u64(out + 64, W);
            put_u64(out + 72, m);
            put_u64(out + 80, L.total);
            put_f64(out + 88, bound);
        }
        uint64_t rec = 0, before = 0;
        for (uint64_t c = 0; c < nc; ++c) {
            uint64_t e0 = c * mc_max, e1 = e0 + mc_max < n ? e0 + mc_max : n;
            uint32_t cnt = (uint32_t)(e1 - e0), mp = (cnt + 31) / 32 * 32;
            int32_t prev = 0;  /* Diff: 0 before the chunk's first code */
            for (uint32_t j = 0; j < mp; ++j) {
                if (j < cnt) {
                    d[j] = orc_zigzag(q[e0 + j] - prev);
                    prev = q[e0 + j];
                } else {
                    d[j] = 0;
                }
            }
            orc_bitshuffle(d, mp, sh);
            uint32_t r = coder ? orc_rre(sh, mp, rz) : orc_rze(sh, mp, rz);
            int raw = r >= mp;
            uint32_t P = raw ? mp : r;
            uint64_t mc = 0;
            for (uint64_t i = e0; i < e1; ++i) mc += flag[i];
            if (pass == 0) {
                W += 1 + P;
                continue;
            }
            put_u32(out + L.index_off + 8 * c, (uint32_t)rec);
            put_u32(out + L.index_off + 8 * c + 4, (uint32_t)before);
            uint8_t *rp = out + L.record_off + 4 * rec;
            put_u32(rp, P | (raw ? 0x80000000u : 0u));
            for (uint32_t k = 0; k < P; ++k) put_u32(rp + 4 * (1 + k), raw ? sh[k] : rz[k]);
            uint64_t k = 0;
            for (uint64_t i = e0; i < e1; ++i) {
                if (!flag[i]) continue;
                uint32_t bits;
                memcpy(&bits, &x[i], 4);
                put_u32(rp + 4 * (1 + P + k), (uint32_t)i);
                put_u32(rp + 4 * (1 + P + mc + k), bits);
                ++k;
            }
            rec = rec + 1 + P + 2 * mc;
            before = before + mc;
        }
        if (pass == 1) {
            free(q); free(flag); free(d); free(sh); free(rz);
            return (int64_t)L.total;
        }
    }
    return ORC_ERR_ARG; /* not reached */
}

int64_t orc_compress_chunked(const float *x, uint64_t n, uint32_t chunk_bytes, int abs_mode, double bound,
                             uint64_t outlier_cap, uint8_t *out, uint64_t out_cap) {
    return orc_compress_chunked_coder(x, n, chunk_bytes, 0, abs_mode, bound, outlier_cap, out, out_cap);
}

static int decompress_chunked(const uint8_t *s, const orc_header *h, float *out) {
    uint32_t rec_words[4096 + 129], sh[4096], d[4096];
    uint64_t R = h->W + 2 * h->m, W_seen = 0;
    for (uint64_t c = 0; c < h->nc; ++c) {
        uint64_t rec = get_u32(s + h->index_off + 8 * c);
        uint64_t before = get_u32(s + h->index_off + 8 * c + 4);
        uint64_t rec_next = (c + 1 < h->nc) ? get_u32(s + h->index_off + 8 * (c + 1)) : R;
        uint64_t after = (c + 1 < h->nc) ? get_u32(s + h->index_off + 8 * (c + 1) + 4) : h->m;
        if (rec_next < rec || after < before || rec_next > R || after > h->m) return ORC_ERR_CORRUPT;
        uint64_t mc = after - before, e0 = c * h->chunk, e1 = e0 + h->chunk < h->n ? e0 + h->chunk : h->n;
        uint32_t cnt = (uint32_t)(e1 - e0), mp = (cnt + 31) / 32 * 32;
        if (rec_next - rec < 1 + 2 * mc) return ORC_ERR_CORRUPT;
        uint32_t head = get_u32(s + h->record_off + 4 * rec), P = head & 0x7fffffffu;
        int raw = (head >> 31) != 0;
        if (1 + (uint64_t)P + 2 * mc != rec_next - rec || P > mp + mp / 32) return ORC_ERR_CORRUPT;
        for (uint32_t k = 0; k < P; ++k) rec_words[k] = get_u32(s + h->record_off + 4 * (rec + 1 + k));
        if (raw) {
            if (P != mp) return ORC_ERR_CORRUPT;
            memcpy(sh, rec_words, 4 * mp);
        } else if (((h->flags & ORC_FLAG_RRE) ? orc_unrre(rec_words, P, mp, sh) : orc_unrze(rec_words, P, mp, sh)) !=
                   (int64_t)P) {
            return ORC_ERR_CORRUPT;
        }
        orc_unbitshuffle(sh, mp, d);
        int64_t qv = 0; /* inverse Diff: running sum from 0 at the chunk start */
        for (uint32_t j = 0; j < cnt; ++j) {
            qv += orc_unzigzag(d[j]);
            out[e0 + j] = dequant((int32_t)(uint32_t)(uint64_t)qv, h->step);
        }
        W_seen += 1 + P;
        uint64_t o = rec + 1 + P;
        for (uint64_t k = 0; k < mc; ++k) {
            uint32_t i = get_u32(s + h->record_off + 4 * (o + k));
            uint32_t bits = get_u32(s + h->record_off + 4 * (o + mc + k));
            if (i < e0 || i >= e1) return ORC_ERR_CORRUPT;
            memcpy(&out[i], &bits, 4);
        }
    }
    if (W_seen != h->W) return ORC_ERR_CORRUPT;
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Block-level view for the tests: widths and per-block zigzag codes of the
 * whole array under given parameters (no stream assembly).                 */
void orc_block_codes(const float *x, uint64_t n, uint32_t block, float inv2eb,
                     uint32_t *z_out, uint8_t *width_out) {
    uint64_t nb = (n + block - 1) / block;
    for (uint64_t b = 0; b < nb; ++b) {
        uint64_t first = b * block;
        uint32_t cnt = (uint32_t)((n - first < block) ? (n - first) : block);
        int32_t prev = 0;
        for (uint32_t j = 0; j < cnt; ++j) {
            int32_t cur = quant_code(x[first + j], inv2eb);
            z_out[first + j] = orc_zigzag(cur - prev);
            prev = cur;
        }
        width_out[b] = (uint8_t)orc_block_width(z_out + first, cnt);
    }
}
