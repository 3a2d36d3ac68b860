/*
 * saw_oracle.c -- plain, slow CPU oracle for SAW-INT4 paged INT4 KV-cache compression.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls this file:
 * only the tests, the smoke check and the CPU-baseline leg of the benchmark do.  It shares
 * no code, header, table or constant generator with the CUDA library.
 *
 * What it computes (source pages, all describing the same method):
 *   - "SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World LLM Serving"
 *     (podcast-summary page, Research Findings): token-wise INT4 quantization combined with a
 *     block-diagonal Hadamard rotation; a fused rotation-quantization kernel writes straight into
 *     a paged KV-cache layout; the cache must stay compatible with paged memory, regular access
 *     and fused attention.
 *   - "Memory compression method reducing KV-cache size..." (idea page, Core Innovation and
 *     Summary): the same method restated.
 *   - "BitDecoding-FP4" (abstract): Hadamard rotation against key outliers under token-wise
 *     scaling; stacked-query attention over paged caches.
 * The pages give no formula.  The fixed build parameters used here are: Hadamard block B = 128
 * (B = D for the 64-wide head vectors, which hold no 128-point block), normalised by 1/sqrt(B),
 * applied as an fp32 butterfly (natural Sylvester order, stages h = 1, 2, ..., B/2, no FMA
 * contraction: this file is compiled with -ffp-contract=off);
 * asymmetric per-(token, kv-head) scale = (max - min) / 15 and zero = min computed in fp32 and
 * stored as fp16; code = clamp(rint((y - min) / scale), 0, 15); two codes per byte, the even
 * index in the low nibble; 16-token pages.
 *
 * Readings where the pages are silent:
 *   - a vector whose fp32 scale is 0 (all elements equal) stores scale +0 and all codes 0;
 *   - a zero minimum is stored as +0 (the stored zero point is min + 0.0f);
 *   - page layout: codes   uint8 [num_pages][Hkv][2 (K,V)][page_size][D/2],
 *                  scales  fp16  [num_pages][Hkv][2 (K,V)][page_size][2 (scale, zero)];
 *   - decode: q is rotated by the same normalised Hadamard, scores use sm_scale, softmax over
 *     the seq_len valid tokens, and the output is rotated back by the same (self-inverse)
 *     normalised Hadamard; query head hq reads kv head hq / (Hq / Hkv).
 * The decode reference runs entirely in fp64 on the dequantised cache.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define ORACLE_HADAMARD_BLOCK 128

/* ---- scalar conversions -------------------------------------------------------------- */

/* bf16 -> fp32 is exact: the bf16 bits are the high half of the fp32 bits. */
float oracle_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* fp32 -> fp16 bits, IEEE round-to-nearest-even (overflow -> inf, subnormals kept). */
uint16_t oracle_f32_to_f16_bits(float x)
{
    _Float16 h = (_Float16)x;
    uint16_t b;
    memcpy(&b, &h, sizeof b);
    return b;
}

/* fp16 bits -> fp64, exact widening. */
double oracle_f16_bits_to_f64(uint16_t b)
{
    _Float16 h;
    memcpy(&h, &b, sizeof h);
    return (double)h;
}

/* ---- rotation ----------------------------------------------------------------------- */

/* Normalised Hadamard transform of one block of n = 2^m fp32 values, in place.
 * Sylvester butterfly: for h = 1, 2, 4, ..., n/2 and every j with (j & h) == 0,
 *     (x[j], x[j+h]) <- (x[j] + x[j+h], x[j] - x[j+h]),
 * then every element is multiplied by the fp32 constant 1/sqrt(n).  Each step is one IEEE
 * fp32 add, subtract or multiply, in exactly this order. */
void oracle_fwht_f32(float *x, int n)
{
    for (int h = 1; h < n; h <<= 1) {
        for (int j = 0; j < n; j++) {
            if ((j & h) == 0) {
                float a = x[j];
                float b = x[j + h];
                x[j] = a + b;
                x[j + h] = a - b;
            }
        }
    }
    const float c = (float)(1.0 / sqrt((double)n));
    for (int j = 0; j < n; j++)
        x[j] = x[j] * c;
}

/* Width of the diagonal blocks for a head vector of length D: the 128-point block, or the
 * whole vector when it is shorter (D = 64: the 64-point transform, normalised by 1/sqrt(64)). */
static int oracle_block(int D) { return D < ORACLE_HADAMARD_BLOCK ? D : ORACLE_HADAMARD_BLOCK; }

/* Block-diagonal rotation of a head vector of length D (64, or a multiple of 128): each
 * block is rotated independently. */
void oracle_rotate_f32(float *x, int D)
{
    const int B = oracle_block(D);
    for (int b = 0; b < D; b += B)
        oracle_fwht_f32(x + b, B);
}

/* Same transform in fp64 (used on the decode side, where the reference is fp64). */
void oracle_fwht_f64(double *x, int n)
{
    for (int h = 1; h < n; h <<= 1) {
        for (int j = 0; j < n; j++) {
            if ((j & h) == 0) {
                double a = x[j];
                double b = x[j + h];
                x[j] = a + b;
                x[j + h] = a - b;
            }
        }
    }
    const double c = 1.0 / sqrt((double)n);
    for (int j = 0; j < n; j++)
        x[j] = x[j] * c;
}

void oracle_rotate_f64(double *x, int D)
{
    const int B = oracle_block(D);
    for (int b = 0; b < D; b += B)
        oracle_fwht_f64(x + b, B);
}

/* ---- token-wise asymmetric INT4 quantizer -------------------------------------------- */

/* Quantize one vector y[0..n) (n even).  Writes n/2 packed bytes, and the fp16 bits of the
 * scale and of the zero point.  Also returns the fp32 scale and min through out-pointers
 * (may be NULL) so that tests can check the error bound against the unrounded values. */
void oracle_quantize_vec(const float *y, int n, uint8_t *packed, uint16_t *scale_h,
                         uint16_t *zero_h, float *scale_f32, float *min_f32)
{
    float mn = y[0];
    float mx = y[0];
    for (int i = 1; i < n; i++) {
        if (y[i] < mn)
            mn = y[i];
        if (y[i] > mx)
            mx = y[i];
    }
    float scale = (mx - mn) / 15.0f;
    int degenerate = (scale == 0.0f);
    if (degenerate)
        scale = 0.0f; /* canonical +0 */

    for (int j = 0; j < n / 2; j++) {
        int code[2];
        for (int e = 0; e < 2; e++) {
            if (degenerate) {
                code[e] = 0;
            } else {
                float q = (y[2 * j + e] - mn) / scale;
                float r = rintf(q); /* default rounding mode: nearest, ties to even */
                if (r < 0.0f)
                    r = 0.0f;
                if (r > 15.0f)
                    r = 15.0f;
                code[e] = (int)r;
            }
        }
        packed[j] = (uint8_t)(code[0] | (code[1] << 4));
    }
    *scale_h = oracle_f32_to_f16_bits(scale);
    *zero_h = oracle_f32_to_f16_bits(mn + 0.0f); /* a zero minimum is stored as +0 */
    if (scale_f32)
        *scale_f32 = scale;
    if (min_f32)
        *min_f32 = mn;
}

/* ---- fused rotate + quantize + scatter into the paged cache -------------------------- */

/* k, v: bf16 bits [T][Hkv][D].  slot_mapping: int64 [T]; slot < 0 means "skip this token".
 * kv_pages: uint8 [num_pages][Hkv][2][page_size][D/2].  scales: fp16 bits
 * [num_pages][Hkv][2][page_size][2].  rotate = 0 gives the plain-INT4 variant (H = I).
 * Returns the number of tokens whose slot was >= num_pages * page_size (those are skipped). */
int64_t oracle_rotate_quantize_paged(const uint16_t *k, const uint16_t *v,
                                     const int64_t *slot_mapping, int64_t T, int Hkv, int D,
                                     int page_size, int64_t num_pages, uint8_t *kv_pages,
                                     uint16_t *scales, int rotate, int nthreads)
{
    int64_t bad = 0;
    const int64_t nslots = num_pages * (int64_t)page_size;
#pragma omp parallel for schedule(static) num_threads(nthreads) reduction(+ : bad)
    for (int64_t t = 0; t < T; t++) {
        int64_t slot = slot_mapping[t];
        if (slot < 0)
            continue;
        if (slot >= nslots) {
            bad += 1;
            continue;
        }
        int64_t page = slot / page_size;
        int64_t off = slot % page_size;
        float y[1024];
        for (int h = 0; h < Hkv; h++) {
            for (int sel = 0; sel < 2; sel++) {
                const uint16_t *src = (sel == 0 ? k : v) + ((size_t)t * Hkv + h) * D;
                for (int d = 0; d < D; d++)
                    y[d] = oracle_bf16_to_f32(src[d]);
                if (rotate)
                    oracle_rotate_f32(y, D);
                size_t row = (((size_t)page * Hkv + h) * 2 + sel) * page_size + off;
                oracle_quantize_vec(y, D, kv_pages + row * (D / 2), &scales[row * 2],
                                    &scales[row * 2 + 1], NULL, NULL);
            }
        }
    }
    return bad;
}

/* ---- decode attention over the INT4 paged cache, fp64 -------------------------------- */

/* Dequantise the head vector stored at (page, kv head h, sel, off) into y[0..D) in fp64:
 * y[d] = zero + code[d] * scale, with the stored fp16 scale and zero widened exactly. */
void oracle_dequant_row_f64(const uint8_t *kv_pages, const uint16_t *scales, int Hkv, int D,
                            int page_size, int64_t page, int h, int sel, int off, double *y)
{
    size_t row = (((size_t)page * Hkv + h) * 2 + sel) * page_size + off;
    const uint8_t *codes = kv_pages + row * (D / 2);
    double scale = oracle_f16_bits_to_f64(scales[row * 2]);
    double zero = oracle_f16_bits_to_f64(scales[row * 2 + 1]);
    for (int j = 0; j < D / 2; j++) {
        y[2 * j] = zero + (double)(codes[j] & 0xF) * scale;
        y[2 * j + 1] = zero + (double)(codes[j] >> 4) * scale;
    }
}

/* q: bf16 bits [S][Hq][D].  block_table: int32 [S][max_blocks].  seq_lens: int32 [S].
 * out: fp64 [S][Hq][D].  For each (seq s, query head hq) with kv head h = hq / (Hq / Hkv):
 *   q_r = H q (rotate != 0) or q,
 *   s_t = sm_scale * <q_r, k_t>    for the seq_lens[s] tokens t (dequantised k_t),
 *   p   = softmax(s),
 *   o_r = sum_t p_t v_t,
 *   out = H o_r (rotate != 0) or o_r.
 * A sequence with seq_lens[s] <= 0 gets an all-zero output. */
void oracle_decode_fp64(const uint16_t *q, const uint8_t *kv_pages, const uint16_t *scales,
                        const int32_t *block_table, int max_blocks, const int32_t *seq_lens,
                        int S, int Hq, int Hkv, int D, int page_size, double sm_scale,
                        int rotate, double *out, int nthreads)
{
    const int G = Hq / Hkv;
#pragma omp parallel for collapse(2) schedule(dynamic) num_threads(nthreads)
    for (int s = 0; s < S; s++) {
        for (int hq = 0; hq < Hq; hq++) {
            const int h = hq / G;
            const int L = seq_lens[s];
            double qr[1024], kv[1024], o[1024];
            double *dst = out + ((size_t)s * Hq + hq) * D;
            if (L <= 0) {
                for (int d = 0; d < D; d++)
                    dst[d] = 0.0;
                continue;
            }
            const uint16_t *qs = q + ((size_t)s * Hq + hq) * D;
            for (int d = 0; d < D; d++)
                qr[d] = (double)oracle_bf16_to_f32(qs[d]);
            if (rotate)
                oracle_rotate_f64(qr, D);

            /* pass 1: scores and their maximum */
            double m = -INFINITY;
            for (int t = 0; t < L; t++) {
                int64_t page = block_table[(size_t)s * max_blocks + t / page_size];
                oracle_dequant_row_f64(kv_pages, scales, Hkv, D, page_size, page, h, 0,
                                       t % page_size, kv);
                double acc = 0.0;
                for (int d = 0; d < D; d++)
                    acc += qr[d] * kv[d];
                double sc = sm_scale * acc;
                if (sc > m)
                    m = sc;
            }
            /* pass 2: softmax weights and the weighted sum of values */
            double l = 0.0;
            for (int d = 0; d < D; d++)
                o[d] = 0.0;
            for (int t = 0; t < L; t++) {
                int64_t page = block_table[(size_t)s * max_blocks + t / page_size];
                oracle_dequant_row_f64(kv_pages, scales, Hkv, D, page_size, page, h, 0,
                                       t % page_size, kv);
                double acc = 0.0;
                for (int d = 0; d < D; d++)
                    acc += qr[d] * kv[d];
                double p = exp(sm_scale * acc - m);
                l += p;
                oracle_dequant_row_f64(kv_pages, scales, Hkv, D, page_size, page, h, 1,
                                       t % page_size, kv);
                for (int d = 0; d < D; d++)
                    o[d] += p * kv[d];
            }
            for (int d = 0; d < D; d++)
                o[d] /= l;
            if (rotate)
                oracle_rotate_f64(o, D);
            for (int d = 0; d < D; d++)
                dst[d] = o[d];
        }
    }
}

/* ---- the BF16 paged-cache baseline ----------------------------------------------------- */
/*
 * The uncompressed cache the INT4 format is measured against ("SAW-INT4", Research Findings:
 * its serving throughput gain is relative to a 16-bit KV cache; "BitDecoding-FP4", abstract:
 * the speedup over BF16 KV decoding).  Layout (reading: the INT4 layout with 16-bit elements):
 * kv_bf16 uint16 [num_pages][Hkv][2 (K,V)][page_size][D]; no scale, no rotation.
 */

/* Scatter T tokens of bf16 K and V into the bf16 pages.  A negative slot is skipped; a slot
 * beyond the cache is skipped and counted.  Returns the count. */
int64_t oracle_append_bf16(const uint16_t *k, const uint16_t *v, const int64_t *slot_mapping,
                           int64_t T, int Hkv, int D, int page_size, int64_t num_pages,
                           uint16_t *kv_bf16)
{
    int64_t bad = 0;
    for (int64_t t = 0; t < T; t++) {
        const int64_t slot = slot_mapping[t];
        if (slot < 0)
            continue;
        if (slot >= num_pages * page_size) {
            bad++;
            continue;
        }
        const int64_t page = slot / page_size, off = slot % page_size;
        for (int h = 0; h < Hkv; h++)
            for (int sel = 0; sel < 2; sel++) {
                const uint16_t *src = (sel ? v : k) + ((size_t)t * Hkv + h) * D;
                uint16_t *dst = kv_bf16 + ((((size_t)page * Hkv + h) * 2 + sel) * page_size + off) * D;
                for (int d = 0; d < D; d++)
                    dst[d] = src[d];
            }
    }
    return bad;
}

/* fp64 decode attention over the bf16 cache: s_t = sm_scale <q, k_t>, softmax over the
 * seq_len valid tokens, out = sum_t p_t v_t; query head hq reads kv head hq / (Hq / Hkv). */
void oracle_decode_bf16_fp64(const uint16_t *q, const uint16_t *kv_bf16,
                             const int32_t *block_table, int max_blocks, const int32_t *seq_lens,
                             int S, int Hq, int Hkv, int D, int page_size, double sm_scale,
                             double *out, int nthreads)
{
    const int G = Hq / Hkv;
#pragma omp parallel for collapse(2) schedule(dynamic) num_threads(nthreads)
    for (int s = 0; s < S; s++) {
        for (int hq = 0; hq < Hq; hq++) {
            const int h = hq / G;
            const int L = seq_lens[s];
            double qd[1024], o[1024];
            double *dst = out + ((size_t)s * Hq + hq) * D;
            if (L <= 0) {
                for (int d = 0; d < D; d++)
                    dst[d] = 0.0;
                continue;
            }
            for (int d = 0; d < D; d++)
                qd[d] = (double)oracle_bf16_to_f32(q[((size_t)s * Hq + hq) * D + d]);
            double m = -INFINITY;
            for (int t = 0; t < L; t++) {
                const int64_t page = block_table[(size_t)s * max_blocks + t / page_size];
                const uint16_t *kr = kv_bf16 + ((((size_t)page * Hkv + h) * 2 + 0) * page_size + t % page_size) * D;
                double acc = 0.0;
                for (int d = 0; d < D; d++)
                    acc += qd[d] * (double)oracle_bf16_to_f32(kr[d]);
                if (sm_scale * acc > m)
                    m = sm_scale * acc;
            }
            double l = 0.0;
            for (int d = 0; d < D; d++)
                o[d] = 0.0;
            for (int t = 0; t < L; t++) {
                const int64_t page = block_table[(size_t)s * max_blocks + t / page_size];
                const size_t base = (((size_t)page * Hkv + h) * 2) * page_size + t % page_size;
                const uint16_t *kr = kv_bf16 + base * D;
                const uint16_t *vr = kv_bf16 + (base + page_size) * D;
                double acc = 0.0;
                for (int d = 0; d < D; d++)
                    acc += qd[d] * (double)oracle_bf16_to_f32(kr[d]);
                const double p = exp(sm_scale * acc - m);
                l += p;
                for (int d = 0; d < D; d++)
                    o[d] += p * (double)oracle_bf16_to_f32(vr[d]);
            }
            for (int d = 0; d < D; d++)
                dst[d] = o[d] / l;
        }
    }
}

/* ---- full-precision sink / recent window beside the INT4 cache -------------------------- */
/*
 * "InnerQ: Hardware-Aware Tuning-Free Quantization of KV Cache for Large Language Models",
 * Abstract and Figure 2: a small high-precision window of attention-sink tokens and recent
 * tokens is kept beside the quantized cache; the attention over the quantized part and over the
 * window are computed separately and merged.  Readings (the pages give no layout):
 *   - positions p < w_sink of a sequence of L tokens are sinks and positions
 *     p >= max(w_sink, L - w_recent) are recent; both stay in bf16 in the window, the others are
 *     quantized (rotated INT4) -- a sequence has min(L, W) window tokens and max(0, L - W)
 *     quantized ones (W = w_sink + w_recent);
 *   - window slot of position p: p for a sink, w_sink + (p - w_sink) mod w_recent for a recent
 *     token; window slot i lives in bf16 page win_table[s][i / 16] at offset i mod 16 (the layout
 *     of the bf16 baseline cache), so the occupied slots are always 0 .. min(L, W) - 1;
 *   - the quantized tokens form their own paged INT4 sequence: position p is quantized index
 *     j = p - w_sink, stored in page block_table[s][j / 16] at offset j mod 16.
 * The reference attends in the original (unrotated) domain: each quantized key and value is
 * dequantized and rotated back by the same normalised Hadamard transform, then one softmax runs
 * over the window tokens and the quantized tokens together (the merged result the figure
 * describes).  fp64 throughout. */
static void oracle_window_token(const uint16_t *win_kv, const int32_t *win_table, int win_blocks,
                                const uint8_t *kv_pages, const uint16_t *scales,
                                const int32_t *block_table, int max_blocks, int s, int h,
                                int Hkv, int D, int page_size, int L_w, int t, int sel,
                                int rotate, double *y)
{
    if (t < L_w) {   /* window slot t */
        const int64_t page = win_table[(size_t)s * win_blocks + t / page_size];
        const uint16_t *r = win_kv + ((((size_t)page * Hkv + h) * 2 + sel) * page_size + t % page_size) * D;
        for (int d = 0; d < D; d++)
            y[d] = (double)oracle_bf16_to_f32(r[d]);
    } else {         /* quantized index j */
        const int j = t - L_w;
        const int64_t page = block_table[(size_t)s * max_blocks + j / page_size];
        oracle_dequant_row_f64(kv_pages, scales, Hkv, D, page_size, page, h, sel, j % page_size, y);
        if (rotate)
            oracle_rotate_f64(y, D);
    }
}

void oracle_decode_window_fp64(const uint16_t *q, const uint16_t *win_kv, const int32_t *win_table,
                               int win_blocks, const uint8_t *kv_pages, const uint16_t *scales,
                               const int32_t *block_table, int max_blocks, const int32_t *seq_lens,
                               int S, int Hq, int Hkv, int D, int page_size, int w_sink,
                               int w_recent, double sm_scale, int rotate, double *out, int nthreads)
{
    const int G = Hq / Hkv;
    const int W = w_sink + w_recent;
#pragma omp parallel for collapse(2) schedule(dynamic) num_threads(nthreads)
    for (int s = 0; s < S; s++) {
        for (int hq = 0; hq < Hq; hq++) {
            const int h = hq / G;
            const int L = seq_lens[s];
            double qd[1024], kv[1024], o[1024];
            double *dst = out + ((size_t)s * Hq + hq) * D;
            if (L <= 0) {
                for (int d = 0; d < D; d++)
                    dst[d] = 0.0;
                continue;
            }
            const int L_w = L < W ? L : W;
            const int n = L_w + (L > W ? L - W : 0);   /* every token once */
            for (int d = 0; d < D; d++)
                qd[d] = (double)oracle_bf16_to_f32(q[((size_t)s * Hq + hq) * D + d]);
            double m = -INFINITY;
            for (int t = 0; t < n; t++) {
                oracle_window_token(win_kv, win_table, win_blocks, kv_pages, scales, block_table,
                                    max_blocks, s, h, Hkv, D, page_size, L_w, t, 0, rotate, kv);
                double acc = 0.0;
                for (int d = 0; d < D; d++)
                    acc += qd[d] * kv[d];
                if (sm_scale * acc > m)
                    m = sm_scale * acc;
            }
            double l = 0.0;
            for (int d = 0; d < D; d++)
                o[d] = 0.0;
            for (int t = 0; t < n; t++) {
                oracle_window_token(win_kv, win_table, win_blocks, kv_pages, scales, block_table,
                                    max_blocks, s, h, Hkv, D, page_size, L_w, t, 0, rotate, kv);
                double acc = 0.0;
                for (int d = 0; d < D; d++)
                    acc += qd[d] * kv[d];
                const double p = exp(sm_scale * acc - m);
                l += p;
                oracle_window_token(win_kv, win_table, win_blocks, kv_pages, scales, block_table,
                                    max_blocks, s, h, Hkv, D, page_size, L_w, t, 1, rotate, kv);
                for (int d = 0; d < D; d++)
                    o[d] += p * kv[d];
            }
            for (int d = 0; d < D; d++)
                dst[d] = o[d] / l;
        }
    }
}

/* ---- chunked-prefill attention over the INT4 cache ------------------------------------- */
/*
 * The read step for a chunk of new tokens whose K/V are already in the paged cache ("SAW-INT4",
 * Research Findings: the quantized cache must serve attention over paged memory; a prefill
 * chunk is the multi-query case).  Sequence s has C_s = q_start[s + 1] - q_start[s] query
 * tokens, the last C_s of its seq_lens[s] cached tokens: query i (row q_start[s] + i of q / out)
 * sits at position L - C + i and attends causally to cache tokens 0 .. L - C + i.  Rotation,
 * dequantization and the fp64 evaluation are those of oracle_decode_fp64.
 */
void oracle_prefill_fp64(const uint16_t *q, const int32_t *q_start, const uint8_t *kv_pages,
                         const uint16_t *scales, const int32_t *block_table, int max_blocks,
                         const int32_t *seq_lens, int S, int Hq, int Hkv, int D, int page_size,
                         double sm_scale, int rotate, double *out, int nthreads)
{
    const int G = Hq / Hkv;
    const int64_t total = q_start[S];
#pragma omp parallel for collapse(2) schedule(dynamic) num_threads(nthreads)
    for (int64_t row = 0; row < total; row++) {
        for (int hq = 0; hq < Hq; hq++) {
            int s = 0;
            while (q_start[s + 1] <= row)
                s++;
            const int C = q_start[s + 1] - q_start[s];
            const int i = (int)(row - q_start[s]);
            const int L = seq_lens[s] - C + i + 1;   /* tokens this query sees */
            const int h = hq / G;
            double qr[1024], kv[1024], o[1024];
            double *dst = out + ((size_t)row * Hq + hq) * D;
            for (int d = 0; d < D; d++)
                qr[d] = (double)oracle_bf16_to_f32(q[((size_t)row * Hq + hq) * D + d]);
            if (rotate)
                oracle_rotate_f64(qr, D);
            double m = -INFINITY;
            for (int t = 0; t < L; t++) {
                const int64_t page = block_table[(size_t)s * max_blocks + t / page_size];
                oracle_dequant_row_f64(kv_pages, scales, Hkv, D, page_size, page, h, 0,
                                       t % page_size, kv);
                double acc = 0.0;
                for (int d = 0; d < D; d++)
                    acc += qr[d] * kv[d];
                if (sm_scale * acc > m)
                    m = sm_scale * acc;
            }
            double l = 0.0;
            for (int d = 0; d < D; d++)
                o[d] = 0.0;
            for (int t = 0; t < L; t++) {
                const int64_t page = block_table[(size_t)s * max_blocks + t / page_size];
                oracle_dequant_row_f64(kv_pages, scales, Hkv, D, page_size, page, h, 0,
                                       t % page_size, kv);
                double acc = 0.0;
                for (int d = 0; d < D; d++)
                    acc += qr[d] * kv[d];
                const double p = exp(sm_scale * acc - m);
                l += p;
                oracle_dequant_row_f64(kv_pages, scales, Hkv, D, page_size, page, h, 1,
                                       t % page_size, kv);
                for (int d = 0; d < D; d++)
                    o[d] += p * kv[d];
            }
            for (int d = 0; d < D; d++)
                o[d] /= l;
            if (rotate)
                oracle_rotate_f64(o, D);
            for (int d = 0; d < D; d++)
                dst[d] = o[d];
        }
    }
}
