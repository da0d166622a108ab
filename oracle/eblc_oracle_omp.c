/*
 * eblc_oracle_omp.c -- the oracle's compress and decompress spread over all
 * host cores with OpenMP, for the benchmark's all-core CPU baseline.
 *
 * TEST INFRASTRUCTURE ONLY, like eblc_oracle.c (which this file includes, so
 * that every step -- value range, bound resolution, quantizer, outlier test,
 * zigzag, width, pack, unpack -- is the plain oracle's own function).  Only the
 * order of the work differs:
 *   - the value range is a parallel min/max reduction over the finite
 *     elements (min and max do not depend on the order; the same "+ 0.0f"
 *     canonicalisation follows, so -0 reads as +0 either way);
 *   - quantization, the per-block widths and each chunk's payload and outlier
 *     counts run in parallel over elements, blocks and chunks;
 *   - one sequential exclusive scan over the chunks gives every chunk record
 *     its offset (the oracle's running `rec` and `outl_before`), then the
 *     chunks are written in parallel, each exactly as the oracle writes it.
 * The stream is therefore byte-identical to orc_compress's, which the CPU
 * tests check.  Decompress decodes the chunks in parallel, each through the
 * oracle's own per-block steps.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fopenmp -fPIC -shared
 */
#include "eblc_oracle.c"

#include <omp.h>

int orc_omp_threads(void) { return omp_get_max_threads(); }

/* Value range over the finite elements, as orc_value_range, in parallel. */
static int omp_value_range(const float *x, uint64_t n, float *vmin_out, float *vmax_out) {
    int any = 0;
    float lo = INFINITY, hi = -INFINITY;
#pragma omp parallel for reduction(min : lo) reduction(max : hi) reduction(| : any) schedule(static)
    for (uint64_t i = 0; i < n; ++i) {
        float v = x[i];
        if (!isfinite(v)) continue;
        any = 1;
        if (v < lo) lo = v;
        if (v > hi) hi = v;
    }
    if (!any) lo = hi = 0.0f;
    *vmin_out = lo + 0.0f;
    *vmax_out = hi + 0.0f;
    return any;
}

int64_t orc_compress_omp(const float *x, uint64_t n, uint32_t block, int abs_mode, double bound,
                         uint64_t outlier_cap, uint8_t *out, uint64_t out_cap) {
    if (!block_ok(block) || !(bound >= 0.0) || !isfinite(bound)) return ORC_ERR_ARG;
    if (n > ORC_MAX_N) return ORC_ERR_ARG;
    if (fegetround() != FE_TONEAREST) return ORC_ERR_ARG;

    float vmin = 0.0f, vmax = 0.0f;
    if (!abs_mode) omp_value_range(x, n, &vmin, &vmax);
    double eb;
    float inv2eb, step;
    orc_resolve_bound(abs_mode, bound, vmin, vmax, &eb, &inv2eb, &step);

    uint64_t nb = (n + block - 1) / block;
    uint64_t nc = (n + ORC_CHUNK - 1) / ORC_CHUNK;
    uint64_t bpc = ORC_CHUNK / block;
    int32_t *q = (int32_t *)malloc((n ? n : 1) * sizeof(int32_t));
    uint8_t *flag = (uint8_t *)malloc(n ? n : 1);
    uint8_t *width = (uint8_t *)malloc(nb ? nb : 1);
    uint32_t *block_words = (uint32_t *)malloc((nb ? nb : 1) * sizeof(uint32_t));
    uint64_t *crec = (uint64_t *)malloc((nc + 1) * sizeof(uint64_t));   /* record word offset per chunk */
    uint64_t *cout = (uint64_t *)malloc((nc + 1) * sizeof(uint64_t));   /* outliers before each chunk  */
    if (!q || !flag || !width || !block_words || !crec || !cout) {
        free(q); free(flag); free(width); free(block_words); free(crec); free(cout);
        return ORC_ERR_NOMEM;
    }

#pragma omp parallel for schedule(static)
    for (uint64_t c = 0; c < nc; ++c) {
        uint64_t e0 = c * ORC_CHUNK, e1 = e0 + ORC_CHUNK < n ? e0 + ORC_CHUNK : n;
        orc_quantize(x + e0, e1 - e0, inv2eb, step, eb, q + e0, flag + e0);
        uint64_t words = 0, mc = 0;
        uint32_t z[256];
        uint64_t b_end = (c + 1) * bpc < nb ? (c + 1) * bpc : nb;
        for (uint64_t b = c * bpc; b < b_end; ++b) {
            uint64_t first = b * block;
            uint32_t cnt = (uint32_t)((n - first < block) ? (n - first) : block);
            int32_t prev = 0;
            for (uint32_t j = 0; j < cnt; ++j) {
                z[j] = orc_zigzag(q[first + j] - prev);
                prev = q[first + j];
            }
            width[b] = (uint8_t)orc_block_width(z, cnt);
            block_words[b] = orc_block_words(width[b], cnt);
            words += block_words[b];
        }
        for (uint64_t i = e0; i < e1; ++i) mc += flag[i];
        crec[c] = words + 2 * mc;
        cout[c] = mc;
    }
    uint64_t W = 0, m = 0, rec = 0;
    for (uint64_t c = 0; c < nc; ++c) {  /* exclusive scan over the chunks */
        uint64_t r = crec[c], mc = cout[c];
        crec[c] = rec;
        cout[c] = m;
        rec += r;
        m += mc;
        W += r - 2 * mc;
    }

    orc_layout L = layout_of(nb, nc, W, m);
    int64_t status = (int64_t)L.total;
    if (m > outlier_cap) status = ORC_ERR_OUTLIER_CAP;
    else if (L.total > out_cap) status = ORC_ERR_CAPACITY;
    if (status < 0) {
        free(q); free(flag); free(width); free(block_words); free(crec); free(cout);
        return status;
    }
    memset(out, 0, L.total);
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
    memcpy(out + L.width_off, width, nb);

#pragma omp parallel for schedule(static)
    for (uint64_t c = 0; c < nc; ++c) {
        uint64_t rec_c = crec[c];
        put_u32(out + L.index_off + 8 * c, (uint32_t)rec_c);
        put_u32(out + L.index_off + 8 * c + 4, (uint32_t)cout[c]);
        uint32_t z[256], words[256];
        uint64_t b_end = (c + 1) * bpc < nb ? (c + 1) * bpc : nb;
        for (uint64_t b = c * bpc; b < b_end; ++b) {
            uint64_t first = b * block;
            uint32_t cnt = (uint32_t)((n - first < block) ? (n - first) : block);
            int32_t prev = 0;
            for (uint32_t j = 0; j < cnt; ++j) {
                z[j] = orc_zigzag(q[first + j] - prev);
                prev = q[first + j];
            }
            orc_pack_block(z, cnt, width[b], words);
            for (uint32_t k = 0; k < block_words[b]; ++k)
                put_u32(out + L.record_off + 4 * (rec_c + k), words[k]);
            rec_c += block_words[b];
        }
        uint64_t e0 = c * ORC_CHUNK, e1 = e0 + ORC_CHUNK < n ? e0 + ORC_CHUNK : n;
        uint64_t mc = 0, k = 0;
        for (uint64_t i = e0; i < e1; ++i) mc += flag[i];
        for (uint64_t i = e0; i < e1; ++i) {
            if (!flag[i]) continue;
            uint32_t bits;
            memcpy(&bits, &x[i], 4);
            put_u32(out + L.record_off + 4 * (rec_c + k), (uint32_t)i);
            put_u32(out + L.record_off + 4 * (rec_c + mc + k), bits);
            ++k;
        }
    }
    free(q); free(flag); free(width); free(block_words); free(crec); free(cout);
    return (int64_t)L.total;
}

/* Decompress with the chunks decoded in parallel (each chunk record is
 * located by the chunk index).  Returns 0 or a negative ORC_ERR_* code.   */
int orc_decompress_omp(const uint8_t *s, uint64_t bytes, float *out, uint64_t n_expected) {
    orc_header h;
    int rc = orc_parse_header(s, bytes, &h);
    if (rc != 0) return rc;
    if (h.n != n_expected) return ORC_ERR_ARG;
    uint64_t bpc = ORC_CHUNK / h.block, R = h.W + 2 * h.m, W_seen = 0;
    int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad) reduction(+ : W_seen)
    for (uint64_t c = 0; c < h.nc; ++c) {
        uint32_t words[256], z[256];
        uint64_t rec = get_u32(s + h.index_off + 8 * c);
        uint64_t before = get_u32(s + h.index_off + 8 * c + 4);
        uint64_t rec_next = (c + 1 < h.nc) ? get_u32(s + h.index_off + 8 * (c + 1)) : R;
        uint64_t after = (c + 1 < h.nc) ? get_u32(s + h.index_off + 8 * (c + 1) + 4) : h.m;
        if (rec_next < rec || after < before || rec_next > R || after > h.m) { bad = 1; continue; }
        uint64_t mc = after - before, word_off = rec;
        uint64_t b_end = (c + 1) * bpc < h.nb ? (c + 1) * bpc : h.nb;
        for (uint64_t b = c * bpc; b < b_end && !bad; ++b) {
            uint64_t first = b * h.block;
            uint32_t cnt = (uint32_t)((h.n - first < h.block) ? (h.n - first) : h.block);
            uint32_t w = s[h.width_off + b];
            uint32_t nw = w > 32 ? 0 : orc_block_words(w, cnt);
            if (w > 32 || word_off + nw > rec_next) { bad = 1; break; }
            for (uint32_t k = 0; k < nw; ++k) words[k] = get_u32(s + h.record_off + 4 * (word_off + k));
            orc_unpack_block(words, cnt, w, z);
            int64_t qv = 0;
            for (uint32_t j = 0; j < cnt; ++j) {
                qv += orc_unzigzag(z[j]);
                out[first + j] = dequant((int32_t)(uint32_t)(uint64_t)qv, h.step);
            }
            word_off += nw;
        }
        if (bad || word_off + 2 * mc != rec_next) { bad = 1; continue; }
        W_seen += word_off - rec;
        uint64_t e0 = c * ORC_CHUNK, e1 = e0 + ORC_CHUNK < h.n ? e0 + ORC_CHUNK : h.n;
        for (uint64_t k = 0; k < mc; ++k) {
            uint32_t i = get_u32(s + h.record_off + 4 * (word_off + k));
            uint32_t bits = get_u32(s + h.record_off + 4 * (word_off + mc + k));
            if (i < e0 || i >= e1) { bad = 1; break; }
            memcpy(&out[i], &bits, 4);
        }
    }
    return (bad || W_seen != h.W) ? ORC_ERR_CORRUPT : 0;
}
