/*
 * Host checks of the two arithmetic shortcuts the GPU quantizer takes in place of IEEE divides
 * (test infrastructure; built and run by tests/test_quant_arith.py with gcc, strict IEEE fp32
 * on x86-64 SSE, no contraction).
 *
 *   div15   scale = RN(x / 15) for x >= 0 computed as q0 = RN(x c), e = fma(-q0, 15, x),
 *           q1 = fma(e, c, q0) with c = RN(1/15): the correction step of P. Markstein,
 *           "Computation of elementary functions on the IBM RISC System/6000 processor",
 *           IBM J. Res. Dev. 34(1), 1990.  Checked for EVERY non-negative finite fp32 x.
 *
 *   codes   code = rint(RN((y - min) / s)) (clamped to [0, 15]) computed without a divide:
 *           t = RN(d r16 + 2^23 + 2^15), r16 ~ 2^16 / s; the code is bits 16..19 of t unless the
 *           low 16 bits of t are zero (a grid value exactly half-way between two codes), where
 *           the sign of the exact remainder E = fma(-m, s, d) against s ulp(m) / 2 (m the
 *           half-integer next to the quotient) decides.  r16 is emulated pessimistically: a
 *           reciprocal with relative error up to 2^-21 (the GPU's is within 2^-23), refined by one
 *           Newton step, as the kernel refines its hardware reciprocal.  Vectors mix Gaussian
 *           fp32 (rotated-like), raw bf16, small integers and tiny multiples (exact half-way
 *           quotients), wide magnitude ranges, outlier channels, and quotients within a few ulps
 *           of k + 1/2.  Scales outside [2^-100, 2^100] take the IEEE divide in the kernel and
 *           are skipped here.
 *
 * usage: quant_arith_check div15 | codes N_VECTORS     exit status 0 when nothing differs
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static float as_f(uint32_t b) { float x; memcpy(&x, &b, 4); return x; }
static uint32_t as_u(float x) { uint32_t b; memcpy(&b, &x, 4); return b; }

static int check_div15(void)
{
    const float c = 1.0f / 15.0f;
    long long bad = 0;
#pragma omp parallel for reduction(+ : bad) schedule(static)
    for (long long i = 0; i < 0x7F800000ll; i++) {
        const float x = as_f((uint32_t)i);
        const float want = x / 15.0f;
        const float q0 = x * c;
        const float e = fmaf(-q0, 15.0f, x);
        const float q1 = fmaf(e, c, q0);
        if (as_u(q1) != as_u(want))
            bad++;
    }
    printf("div15: %lld non-negative finite fp32 dividends, %lld mismatches\n", 0x7F800000ll, bad);
    return bad != 0;
}

/* xorshift64 stream per vector: deterministic, independent of the thread count */
typedef struct { uint64_t s; } rng;
static uint64_t next(rng *r) { r->s ^= r->s << 13; r->s ^= r->s >> 7; r->s ^= r->s << 17; return r->s; }
static double unif(rng *r) { return (double)(next(r) >> 11) * (1.0 / 9007199254740992.0); }
static float gauss(rng *r)
{
    const double a = unif(r), b = unif(r);
    return (float)(sqrt(-2.0 * log(a + 1e-300)) * cos(6.283185307179586 * b));
}
static float round_bf16(float x)
{
    const uint32_t b = as_u(x);
    return as_f((b + 0x7FFFu + ((b >> 16) & 1u)) & 0xFFFF0000u);
}

static int code_ieee(float d, float s)
{
    float k = rintf(d / s);
    if (k < 0.0f) k = 0.0f;
    if (k > 15.0f) k = 15.0f;
    return (int)k;
}

static const float kGridMagic = 8421376.0f; /* 2^23 + 2^15 */

static int code_grid(float d, float s, float r16, long long *flagged)
{
    const uint32_t t = as_u(fmaf(d, r16, kGridMagic));
    const int cand = (int)((t >> 16) & 15u);
    if ((t & 0xFFFFu) != 0)
        return cand;
    (*flagged)++;
    const float m = (float)cand - 0.5f;
    const float e = fmaf(-m, s, d);
    const float half_ulp = as_f((as_u(m) & 0x7F800000u) - (24u << 23));
    return (int)(fabsf(e) <= s * half_ulp ? rintf(m) : m + copysignf(0.5f, e));
}

/* all codes of one vector; returns the number of mismatches */
static long long vector_codes(const float *y, int n, rng *r, long long *total, long long *flagged)
{
    float mn = y[0], mx = y[0];
    for (int i = 1; i < n; i++) {
        if (y[i] < mn) mn = y[i];
        if (y[i] > mx) mx = y[i];
    }
    const float s = (mx - mn) / 15.0f;
    if (!(s >= 0x1p-100f && s <= 0x1p100f))
        return 0;
    const double rel = (unif(r) * 2.0 - 1.0) * 0x1p-21;
    const float r0 = (float)((1.0 / (double)s) * (1.0 + rel));
    const float e = fmaf(-s, r0, 1.0f);
    const float r0s = r0 * 65536.0f;
    const float r16 = fmaf(r0s, e, r0s);
    long long bad = 0;
    for (int i = 0; i < n; i++) {
        const float d = y[i] - mn;
        (*total)++;
        if (code_ieee(d, s) != code_grid(d, s, r16, flagged))
            bad++;
    }
    return bad;
}

static int check_codes(long long nvec)
{
    long long total = 0, flagged = 0, bad = 0;
#pragma omp parallel for reduction(+ : total, flagged, bad) schedule(dynamic, 4096)
    for (long long v = 0; v < nvec; v++) {
        rng r = {0x9E3779B97F4A7C15ull ^ (uint64_t)(v + 1) * 0xD1B54A32D192ED03ull};
        for (int w = 0; w < 8; w++)
            next(&r);
        float y[128];
        const int kind = (int)(v % 6);
        for (int i = 0; i < 128; i++) {
            float x;
            switch (kind) {
            case 0: x = gauss(&r); break;
            case 1: x = round_bf16(gauss(&r)); break;
            case 2: x = (float)((int)(next(&r) % 31) - 15); break;
            case 3: x = round_bf16(gauss(&r) * (float)pow(10.0, (int)(next(&r) % 7) - 3)); break;
            case 4: x = (float)((int)(next(&r) % 7) - 3) * 0x1p-40f; break;
            default: x = gauss(&r) * 30.0f * (i < 4 ? 1.0f : 0.05f); break;
            }
            y[i] = x;
        }
        if (kind == 2 || kind == 4) {
            /* exact half-way quotients: min 0, max 15, the rest k + 1/2 (times 2^-40) */
            y[0] = 0.0f;
            y[1] = 15.0f;
            for (int i = 2; i < 128; i++)
                y[i] = (float)(next(&r) % 15) + 0.5f;
            if (kind == 4)
                for (int i = 0; i < 128; i++)
                    y[i] *= 0x1p-40f;
        }
        bad += vector_codes(y, 128, &r, &total, &flagged);
        if (v % 3 == 0) {
            /* quotients within 4 ulps of k + 1/2 */
            const float s0 = (float)(0.1 + unif(&r));
            y[0] = 0.0f;
            y[1] = 15.0f * s0;
            for (int i = 2; i < 128; i++) {
                const float q = (float)(next(&r) % 15) + 0.5f;
                y[i] = as_f(as_u(q * s0) + (uint32_t)((int)(next(&r) % 9) - 4));
            }
            bad += vector_codes(y, 128, &r, &total, &flagged);
        }
    }
    printf("codes: %lld elements, %lld at an exact half-way grid value, %lld mismatches\n", total,
           flagged, bad);
    return bad != 0;
}

int main(int argc, char **argv)
{
    if (argc >= 2 && strcmp(argv[1], "div15") == 0)
        return check_div15();
    if (argc >= 3 && strcmp(argv[1], "codes") == 0)
        return check_codes(atoll(argv[2]));
    fprintf(stderr, "usage: %s div15 | codes N_VECTORS\n", argv[0]);
    return 2;
}
