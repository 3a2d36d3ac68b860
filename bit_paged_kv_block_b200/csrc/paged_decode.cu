// paged_decode.cu -- decode attention over the INT4 paged KV cache (split-K, GQA-stacked).
//
// The read side of "SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World LLM
// Serving" (Research Findings: the quantized cache must keep fused attention execution over
// paged memory with regular access), with the query heads of one kv head stacked into one
// tensor-core tile as in "BitDecoding-FP4" (abstract: stacked query MMA on paged KV caches).
// Because H is orthogonal and symmetric, <q, k> = <Hq, Hk> and sum p_t v_t = H sum p_t (H v_t):
// the kernel rotates q once, attends over the rotated codes and rotates the output back.
//
// Work split.  A (sequence s, kv head h) pair is a segment of n = ceil(len_s / 16) pages.  All
// segments are laid end to end (seq-major, then kv head) in a cost space where a segment costs
// n + kKappa (kKappa pages' worth of per-segment work: query rotation and output rotation), and
// that cost range is cut into W equal slices, one per warp of a persistent grid.  Each warp
// owns the contiguous run of pages whose cost positions fall in its slice and works on it
// independently: no barrier, atomic or fence between warps.  A segment that lies entirely in one
// warp's run is finished by that warp; the pieces of a segment split across warps are written to
// the workspace (slot segment + warp, unique because both orders are monotone) and combined by
// a second kernel (paged_decode_merge_kernel), launched as a programmatic dependent.
//
// Per page (16 tokens x one kv head, 2 KiB of codes + 128 B of scales), per warp:
//   * one elected lane queues a 2-D tensor copy of the 32 code rows (64B swizzle, so the K
//     reads and the transposed V reads below are bank-conflict free) and a 1-D bulk copy of the
//     scales into a 4-stage ring, completion on an mbarrier (bounded wait), three pages ahead;
//   * S^T[16 tok x 8 heads] = K_codes[16 x 128] . Q^T with mma.m16n8k16 (fp16 in, fp32 acc):
//     the codes are exact fp16 subnormals, and s = scale * acc + zero * sum(q) in fp32;
//   * online softmax in the log2 domain (q carries sm_scale * log2 e);
//   * O^T[128 d x 8 heads] += V_codes^T . P'^T with P' = p * scale_V in fp16 and the zero
//     point added in fp32 through sum_t p_t zero_t.
// The work split, the piece loop, the split-K slots and the merge kernel are generic over the
// page format and live in decode_common.cuh; this file is the INT4 page format (Int4Format).
// The query of the next segment is bulk-copied into a per-warp buffer while the current one is
// processed.  The query dimension d of QK and the value dimension of PV are consumed in a
// permuted order (both sides permuted alike), which lets every thread unpack whole 32-bit code
// words; the final inverse rotation undoes it.
#include <cfloat>
#include <cudaTypedefs.h>

#include "decode_common.cuh"
#include "saw_device.cuh"
#include "saw_internal.h"

namespace saw {
namespace {

using namespace decode;

// K + V codes of one (page, kv head): 2 x 16 rows of D / 2 bytes
__host__ __device__ constexpr int code_bytes(int d) { return 2 * kPageSize * d / 2; }
constexpr int kScaleBytes = 2 * kPageSize * 4;          // K + V (scale, zero) fp16 pairs
// 1/sqrt(B) of the rotation block B = min(D, 128): fp32(1/sqrt(128)), or 1/8 for D = 64
__host__ __device__ constexpr float hadamard_c(int d) { return d == 64 ? 0.125f : 0.0883883461356163f; }

// Unpack one 32-bit word of packed codes (bytes b0..b3, low nibble first) into four fp16x2
// registers by masking alone: a nibble left in the low mantissa bits of an fp16 with a zero
// exponent is the subnormal n * 2^-24 (low nibble) or 16 n * 2^-24 = n * 2^-20 (high nibble),
// exactly.  y[0] = (b0.lo, b2.lo), y[1] = (b0.hi, b2.hi), y[2] = (b1.lo, b3.lo),
// y[3] = (b1.hi, b3.hi).  The powers of two are folded into q (high nibbles use q / 16) and into
// the scales, so the tensor-core products are exact.
__device__ __forceinline__ void unpack_codes(uint32_t w, uint32_t y[4])
{
    const uint32_t w8 = w >> 8;
    y[0] = w & 0x000F000Fu;
    y[1] = w & 0x00F000F0u;
    y[2] = w8 & 0x000F000Fu;
    y[3] = w8 & 0x00F000F0u;
}

constexpr float kLowNibble = 16777216.0f;   // 2^24: undoes the low-nibble subnormal scale
constexpr float kHighNibble = 1048576.0f;   // 2^20: undoes the high-nibble subnormal scale

__device__ __forceinline__ float2 h2_to_f2(uint32_t u)
{
    return __half22float2(u32_as_half2(u));
}

// Rotated, scaled query of one segment as fp16 mma B fragments, from the raw bf16 queries of
// its nheads <= 8 heads in shared memory ([nheads][kD] at qbuf).
// Thread (g, t) owns query head g of the group and d in [kQ t, kQ t + kQ), kQ = kD / 4.  The
// rotation is the Hadamard transform of each block of B = min(kD, 128) elements of d (for
// kD = 256 the two halves are independent blocks, as the quantizer rotates them).
template <bool kRotate, int kD>
__device__ __forceinline__ void load_query(const DecodeParams &p, uint32_t qbuf, int nheads, int g,
                                           int t, uint32_t bq[kD / 16][2], float sq_out[2])
{
    constexpr int kQ = kD / 4;
    constexpr int kBlock = kD < 128 ? kD : 128;
    float x[kQ];
    if (g < nheads) {
#pragma unroll
        for (int c = 0; c < kQ / 8; c++) {
            const uint4 u = lds128(qbuf + g * (kD * 2) + 2 * kQ * t + 16 * c);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int k = 0; k < 4; k++) {
                x[8 * c + 2 * k] = __uint_as_float(w[k] << 16);
                x[8 * c + 2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
            }
        }
    } else {
#pragma unroll
        for (int l = 0; l < kQ; l++)
            x[l] = 0.0f;
    }
    // Hadamard butterfly (skipped for the plain INT4 cache): the low log2(kQ) bits of d in
    // registers, the remaining bits of the block across lanes t ^ 1 (and t ^ 2 for kD <= 128).
#pragma unroll
    for (int hb = 1; kRotate && hb < kQ; hb <<= 1)
#pragma unroll
        for (int l = 0; l < kQ; l++)
            if ((l & hb) == 0) {
                const float a = x[l], b = x[l + hb];
                x[l] = a + b;
                x[l + hb] = a - b;
            }
#pragma unroll
    for (int lb = 1; kRotate && kQ * lb < kBlock; lb <<= 1) {
        const bool high = (t & lb) != 0;
#pragma unroll
        for (int l = 0; l < kQ; l++) {
            const float o = __shfl_xor_sync(0xFFFFFFFFu, x[l], lb);
            x[l] = high ? o - x[l] : x[l] + o;
        }
    }
    // Even d pair with low nibbles (weight 2^-24), odd d with high nibbles (weight 2^-20): odd
    // entries carry q / 16 so that every product is q_d * code_d * 2^-24.  sum(q) runs over all
    // kD elements: one (scale, zero) pair covers the whole head vector.
    float sq = 0.0f;
    __half hq[kQ];
#pragma unroll
    for (int l = 0; l < kQ; l++) {
        const float qv = x[l] * p.q_mult;
        hq[l] = __float2half_rn((l & 1) ? qv * 0.0625f : qv);
        sq += (l & 1) ? 16.0f * __half2float(hq[l]) : __half2float(hq[l]);
    }
    sq += __shfl_xor_sync(0xFFFFFFFFu, sq, 1);
    sq += __shfl_xor_sync(0xFFFFFFFFu, sq, 2);
    // k-step (i, e): k slots (2t, 2t+1 | 2t+8, 2t+9) <-> d = kQ t + 8i + 2e + (0, 4 | 1, 5)
#pragma unroll
    for (int i = 0; i < kQ / 8; i++)
#pragma unroll
        for (int e = 0; e < 2; e++) {
            const int l0 = 8 * i + 2 * e;
            bq[2 * i + e][0] = half2_as_u32(__halves2half2(hq[l0], hq[l0 + 4]));
            bq[2 * i + e][1] = half2_as_u32(__halves2half2(hq[l0 + 1], hq[l0 + 5]));
        }
    // thread (g, t) needs sum(q) of heads 2t and 2t + 1 (held by lanes 4 (2t) and 4 (2t + 1))
    sq_out[0] = __shfl_sync(0xFFFFFFFFu, sq, 8 * t);
    sq_out[1] = __shfl_sync(0xFFFFFFFFu, sq, 8 * t + 4);
}

// Byte offset of 16-byte chunk c of code row r in a staged page: rows of kD / 2 bytes with the
// tensor copy's swizzle (32B for 32-byte rows: chunk ^ bit 2 of the row; 64B for 64-byte rows:
// chunk ^ bits 1-2 of the row; 128B for 128-byte rows: chunk ^ bits 0-2 of the row).
template <int kD>
__device__ __forceinline__ uint32_t code_offset(int r, int c)
{
    const int sw = kD == 64 ? (r >> 2) & 1 : kD == 128 ? (r >> 1) & 3 : r & 7;
    return static_cast<uint32_t>(r * (kD / 2) + ((c ^ sw) << 4));
}

// The logits of one page (log2 domain): S^T = K . Q^T over its 16 tokens (rows g, g + 8), then
// s = scale * acc + zero * sum(q) per (token, query column); tokens a column may not see get
// -inf.  kMask: tokens [0, mask.valid) of the page exist and column e (block row 2t + e) sees
// tokens [0, mask.col[e]).
template <bool kMask, int kD>
__device__ __forceinline__ void page_logits(uint32_t cbase, uint32_t sbase, const PageMask &mask,
                                            const uint32_t bq[kD / 16][2], const float sq[2],
                                            int lane, float s[4])
{
    const int g = lane >> 2, t = lane & 3;
    constexpr int kWords = kD / 32;   // 32-bit code words of one row per thread

    // Thread t reads the kD / 4 codes of d in [kD/4 t, kD/4 (t + 1)) of rows g and g + 8: for
    // kD >= 128 whole 16-byte chunks (within each quarter warp the two rows land in disjoint
    // banks), for kD = 64 half a chunk (each half warp reads four whole 32-byte rows).
    uint32_t kw0[kWords], kw1[kWords];
    if constexpr (kD == 64) {
        const uint32_t off = static_cast<uint32_t>(8 * (t & 1));
        const uint2 k0 = lds64(cbase + code_offset<kD>(g, t >> 1) + off);
        const uint2 k1 = lds64(cbase + code_offset<kD>(g + 8, t >> 1) + off);
        kw0[0] = k0.x;
        kw0[1] = k0.y;
        kw1[0] = k1.x;
        kw1[1] = k1.y;
    } else {
#pragma unroll
        for (int hf = 0; hf < kD / 128; hf++) {
            const int c = (kD / 128) * t + hf;
            const uint4 k0 = lds128(cbase + code_offset<kD>(g, c));
            const uint4 k1 = lds128(cbase + code_offset<kD>(g + 8, c));
            kw0[4 * hf] = k0.x;
            kw0[4 * hf + 1] = k0.y;
            kw0[4 * hf + 2] = k0.z;
            kw0[4 * hf + 3] = k0.w;
            kw1[4 * hf] = k1.x;
            kw1[4 * hf + 1] = k1.y;
            kw1[4 * hf + 2] = k1.z;
            kw1[4 * hf + 3] = k1.w;
        }
    }
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int w = 0; w < kWords; w++) {
        uint32_t ya[4], yb[4];
        unpack_codes(kw0[w], ya);
        unpack_codes(kw1[w], yb);
        const uint32_t a0[4] = {ya[0], yb[0], ya[1], yb[1]};
        const uint32_t a1[4] = {ya[2], yb[2], ya[3], yb[3]};
        mma_16816(acc, a0, bq[2 * w][0], bq[2 * w][1]);
        mma_16816(acc, a1, bq[2 * w + 1][0], bq[2 * w + 1][1]);
    }

    const float2 ksz0 = h2_to_f2(lds32(sbase + 4 * g));
    const float2 ksz1 = h2_to_f2(lds32(sbase + 4 * (g + 8)));
    const float ks0 = ksz0.x * kLowNibble, ks1 = ksz1.x * kLowNibble;
    s[0] = fmaf(ks0, acc[0], ksz0.y * sq[0]);
    s[1] = fmaf(ks0, acc[1], ksz0.y * sq[1]);
    s[2] = fmaf(ks1, acc[2], ksz1.y * sq[0]);
    s[3] = fmaf(ks1, acc[3], ksz1.y * sq[1]);
    if (kMask) {
        if (g >= mask.col[0])
            s[0] = -INFINITY;
        if (g >= mask.col[1])
            s[1] = -INFINITY;
        if (g + 8 >= mask.col[0])
            s[2] = -INFINITY;
        if (g + 8 >= mask.col[1])
            s[3] = -INFINITY;
    }
}

// O^T += V^T . P'^T for one page with weights pr (tokens g, g + 8 of columns 2t, 2t + 1), and the
// running sums l (weights) and z (weights times the V zero points).  kMask: tokens past
// mask.valid were never written; their V scale and zero are replaced by 0, so they contribute
// exactly 0 whatever bits their rows hold.
template <bool kMask, int kD>
__device__ __forceinline__ void page_pv(uint32_t cbase, uint32_t sbase, const PageMask &mask,
                                        const float pr[4], int lane, WarpState<kD / 16> &st)
{
    const int g = lane >> 2;
    const bool v0 = !kMask || g < mask.valid, v1 = !kMask || g + 8 < mask.valid;
    float2 vsz0 = h2_to_f2(lds32(sbase + 64 + 4 * g));
    float2 vsz1 = h2_to_f2(lds32(sbase + 64 + 4 * (g + 8)));
    if (kMask) {
        if (!v0)
            vsz0 = make_float2(0.0f, 0.0f);
        if (!v1)
            vsz1 = make_float2(0.0f, 0.0f);
    }
    st.l[0] += pr[0] + pr[2];
    st.l[1] += pr[1] + pr[3];
    st.z[0] = fmaf(pr[0], vsz0.y, fmaf(pr[2], vsz1.y, st.z[0]));
    st.z[1] = fmaf(pr[1], vsz0.y, fmaf(pr[3], vsz1.y, st.z[1]));
    const uint32_t p01 = half2_as_u32(__floats2half2_rn(pr[0] * vsz0.x, pr[1] * vsz0.x));
    const uint32_t p23 = half2_as_u32(__floats2half2_rn(pr[2] * vsz1.x, pr[3] * vsz1.x));
    const uint32_t pb0 = movmatrix_trans(p01);   // B fragment: tokens 2t, 2t+1 of head g
    const uint32_t pb1 = movmatrix_trans(p23);   // tokens 2t + 8, 2t + 9

    // ldmatrix.trans: lane L addresses row (L & 7) of matrix L >> 3; matrices are
    // (tokens 0-7 | 8-15) x (16-byte chunk 2j | 2j + 1) of the V rows (rows 16..31).
    const int vrow = 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
#pragma unroll
    for (int j = 0; j < kD / 64; j++) {
        const int chunk = 2 * j + (lane >> 4);
        uint32_t r[4];
        ldsm_x4_trans(cbase + code_offset<kD>(vrow, chunk), r[0], r[1], r[2], r[3]);
        // r[0]: tokens 0-7, chunk 2j; r[1]: tokens 8-15, chunk 2j; r[2], r[3]: chunk 2j + 1
#pragma unroll
        for (int cc = 0; cc < 2; cc++) {
            uint32_t ylo[4], yhi[4];
            unpack_codes(r[2 * cc], ylo);
            unpack_codes(r[2 * cc + 1], yhi);
            const int c = 2 * j + cc;
#pragma unroll
            for (int h2 = 0; h2 < 2; h2++) {
                const uint32_t a[4] = {ylo[2 * h2], ylo[2 * h2 + 1], yhi[2 * h2], yhi[2 * h2 + 1]};
                mma_16816(st.o[2 * c + h2], a, pb0, pb1);
            }
        }
    }
}

// One page of one warp: QK^T, online softmax, PV.
template <bool kMask, int kD>
__device__ __forceinline__ void process_page(uint32_t cbase, uint32_t sbase, const PageMask &mask,
                                             const uint32_t bq[kD / 16][2], const float sq[2],
                                             int lane, WarpState<kD / 16> &st)
{
    float s[4], pr[4];
    page_logits<kMask, kD>(cbase, sbase, mask, bq, sq, lane, s);
    softmax_update<kMask, kD / 16, 4>(s, st, pr);
    page_pv<kMask, kD>(cbase, sbase, mask, pr, lane, st);
}

// Two whole pages of one warp as one step: both pages' logits (two independent tensor-core
// chains), one online-softmax update over their 32 tokens, then PV for both.
template <int kD>
__device__ __forceinline__ void process_pages2(uint32_t cbase0, uint32_t sbase0, uint32_t cbase1,
                                               uint32_t sbase1, const uint32_t bq[kD / 16][2],
                                               const float sq[2], int lane, WarpState<kD / 16> &st)
{
    const PageMask whole = {kPageSize, {kPageSize, kPageSize}};
    float s[8], pr[8];
    page_logits<false, kD>(cbase0, sbase0, whole, bq, sq, lane, s);
    page_logits<false, kD>(cbase1, sbase1, whole, bq, sq, lane, s + 4);
    softmax_update<false, kD / 16, 8>(s, st, pr);
    page_pv<false, kD>(cbase0, sbase0, whole, pr, lane, st);
    page_pv<false, kD>(cbase1, sbase1, whole, pr + 4, lane, st);
}

// o_r = o / l, out = H o_r (o_r itself for the plain INT4 cache) for the block rows 2t, 2t + 1
// this thread holds; H acts on each block of min(kD, 128) elements of d.  As the quantized part
// of a windowed decode, out instead becomes the softmax-weighted merge of this result and the
// window part's row already in out: weights 2^lse / (2^lse_q + 2^lse_w), lse_q = m + log2 l.
template <bool kRotate, int kD, bool kMerge, class Seg>
__device__ __forceinline__ void finalize(const DecodeParams &p, const Seg &sg, int lane,
                                         float o[kD / 16][4], const float m[2], const float l[2])
{
    constexpr int kC = kD / 32;   // 32-element chunks of d
    const int g = lane >> 2, t = lane & 3;
    const float inv[2] = {1.0f / l[0], 1.0f / l[1]};
    // v[e][c][j]: head 2t + e, d = 32c + 4g + j
    float v[2][kC][4];
#pragma unroll
    for (int c = 0; c < kC; c++)
#pragma unroll
        for (int e = 0; e < 2; e++) {
            v[e][c][0] = o[2 * c][e] * inv[e];
            v[e][c][1] = o[2 * c][2 + e] * inv[e];
            v[e][c][2] = o[2 * c + 1][e] * inv[e];
            v[e][c][3] = o[2 * c + 1][2 + e] * inv[e];
        }
#pragma unroll
    for (int e = 0; kRotate && e < 2; e++) {
        // d bits 0, 1 (j) and 5, 6 (low bits of c; bit 5 only for kD = 64) in registers; bit 7
        // (kD = 256) selects the 128-block and is not transformed
#pragma unroll
        for (int c = 0; c < kC; c++)
#pragma unroll
            for (int jb = 1; jb <= 2; jb <<= 1)
#pragma unroll
                for (int j = 0; j < 4; j++)
                    if ((j & jb) == 0) {
                        const float a = v[e][c][j], b = v[e][c][j + jb];
                        v[e][c][j] = a + b;
                        v[e][c][j + jb] = a - b;
                    }
#pragma unroll
        for (int cb = 1; cb <= 2 && cb < kC; cb <<= 1)
#pragma unroll
            for (int c = 0; c < kC; c++)
                if ((c & cb) == 0)
#pragma unroll
                    for (int j = 0; j < 4; j++) {
                        const float a = v[e][c][j], b = v[e][c + cb][j];
                        v[e][c][j] = a + b;
                        v[e][c + cb][j] = a - b;
                    }
        // d bits 2..4 (g) across lanes 4, 8, 16
#pragma unroll
        for (int gb = 1; gb <= 4; gb <<= 1) {
            const bool high = (g & gb) != 0;
#pragma unroll
            for (int c = 0; c < kC; c++)
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    const float other = __shfl_xor_sync(0xFFFFFFFFu, v[e][c][j], 4 * gb);
                    v[e][c][j] = high ? other - v[e][c][j] : v[e][c][j] + other;
                }
        }
    }
#pragma unroll
    for (int e = 0; e < 2; e++) {
        const int head = 2 * t + e;
        if (head < sg.nrows) {
            const int64_t off = sg.row_offset(p, head, kD);
            float *dst = p.out + off;
            float f = kRotate ? hadamard_c(kD) : 1.0f, fw = 0.0f;
            if (kMerge) {
                const float lq = m[e] + log2f(l[e]), lw = p.lse[off / kD];
                const float mx = fmaxf(lq, lw);
                const float aq = exp2f(lq - mx), aw = exp2f(lw - mx);
                const float inv = 1.0f / (aq + aw);
                f *= aq * inv;
                fw = aw * inv;
            }
#pragma unroll
            for (int c = 0; c < kC; c++) {
                float4 val = make_float4(v[e][c][0] * f, v[e][c][1] * f, v[e][c][2] * f,
                                         v[e][c][3] * f);
                float4 *d4 = reinterpret_cast<float4 *>(dst + 32 * c + 4 * g);
                if (kMerge) {
                    const float4 w = *d4;
                    val = make_float4(fmaf(fw, w.x, val.x), fmaf(fw, w.y, val.y),
                                      fmaf(fw, w.z, val.z), fmaf(fw, w.w, val.w));
                }
                *d4 = val;
            }
        }
    }
}


// One elected lane of the (converged) warp arms the stage's mbarrier with the page's bytes and
// queues the 2-D tensor copy of its code rows and the 1-D bulk copy of its scales; no branch.
template <int kD>
__device__ __forceinline__ void copy_page_elected(uint32_t bar, uint32_t dst_codes, const void *tmap,
                                                  int32_t row, uint32_t dst_scales,
                                                  const void *src_scales)
{
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "elect.sync _|p, 0xffffffff;\n\t"
                 "@p mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %6;\n\t"
                 "@p cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
                 " [%1], [%2, {%7, %3}], [%0];\n\t"
                 "@p cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%4], [%5], %8, [%0];\n\t"
                 "}"
                 ::"r"(bar), "r"(dst_codes), "l"(tmap), "r"(row), "r"(dst_scales), "l"(src_scales),
                 "r"(static_cast<uint32_t>(code_bytes(kD) + kScaleBytes)), "r"(0), "r"(static_cast<uint32_t>(kScaleBytes))
                 : "memory");
}



// The INT4 page format for the generic decode kernel (decode_common.cuh), head dimension kD:
// 4 warps per CTA and a ring per warp whose stages hold the codes of one (page, kv head) (32
// tensor-map rows of kD / 2 bytes: 1 KiB with the 32B swizzle for kD = 64, 2 KiB with the 64B
// swizzle for kD = 128, 4 KiB with the 128B swizzle for kD = 256), codes of all stages first,
// then the scales (128 B each).  kD = 128: 4 stages, 4 CTAs per SM; kD = 256 (twice the
// accumulators): 2 stages, 3 CTAs per SM, which keeps about as many bytes in flight per SM;
// kD = 64 (half the registers, half the bytes per page): 4 stages, 5 CTAs per SM, since a warp
// completes its page copies one after another and more warps keep more copies in flight.
// kMerge: the quantized part of a windowed decode, whose finalize merges into the window part's
// output rows (a separate instantiation, so the plain decode carries none of it).
template <bool kRotate, int kD, bool kMerge = false>
struct Int4Format {
    static_assert(kD == 64 || kD == 128 || kD == 256, "head dimension");
    static constexpr int kDim = kD;
    static constexpr int kTiles = kD / 16;
    static constexpr int kWarps = 4;
    static constexpr int kStages = kD == 256 ? 2 : 4;
    static constexpr int kMinBlocks = kD == 64 ? 5 : kD == 128 ? 4 : 3;
    static constexpr int kRowsPerPage = 32;
    static constexpr int kCodeBytes = code_bytes(kD);
    static constexpr int kRingBytes = kWarps * kStages * (kCodeBytes + kScaleBytes);
    struct Ring {
        uint32_t code0, scale0;
    };
    struct Query {
        uint32_t bq[kD / 16][2];
        float sq[2];
    };
    __device__ static Ring ring(uint32_t base, int warp)
    {
        return {base + warp * kStages * kCodeBytes,
                base + kWarps * kStages * kCodeBytes + warp * kStages * kScaleBytes};
    }
    __device__ static void issue(const Ring &r, int stg, uint32_t bar, const CUtensorMap *tmap,
                                 int32_t row, const DecodeParams &p)
    {
        copy_page_elected<kD>(bar, r.code0 + stg * kCodeBytes, tmap, row,
                              r.scale0 + stg * kScaleBytes, p.scales + static_cast<int64_t>(row) * 4);
    }
    __device__ static void load_query(const DecodeParams &p, uint32_t qbuf, int nheads, int lane,
                                      Query &q)
    {
        saw::load_query<kRotate, kD>(p, qbuf, nheads, lane >> 2, lane & 3, q.bq, q.sq);
    }
    template <bool kMask>
    __device__ static void page(const Ring &r, int stg, const PageMask &mask, const Query &q,
                                int lane, WarpState<kTiles> &st)
    {
        process_page<kMask, kD>(r.code0 + stg * kCodeBytes, r.scale0 + stg * kScaleBytes, mask,
                                q.bq, q.sq, lane, st);
    }
    static constexpr bool kPairs = kD != 256;   // two whole pages as one step (page2)
    __device__ static void page2(const Ring &r, int stg0, int stg1, const Query &q, int lane,
                                 WarpState<kTiles> &st)
    {
        process_pages2<kD>(r.code0 + stg0 * kCodeBytes, r.scale0 + stg0 * kScaleBytes,
                           r.code0 + stg1 * kCodeBytes, r.scale0 + stg1 * kScaleBytes, q.bq, q.sq,
                           lane, st);
    }
    __device__ static void piece_end(WarpState<kTiles> &st)
    {
        // reduce l and z over the 8 token rows (lanes differing in g)
#pragma unroll
        for (int e = 0; e < 2; e++) {
#pragma unroll
            for (int d = 4; d <= 16; d <<= 1) {
                st.l[e] += __shfl_xor_sync(0xFFFFFFFFu, st.l[e], d);
                st.z[e] += __shfl_xor_sync(0xFFFFFFFFu, st.z[e], d);
            }
        }
        // undo the subnormal code scales (value rows g: low nibbles, g + 8: high nibbles)
        // and add the zero-point term
#pragma unroll
        for (int i2 = 0; i2 < kTiles; i2++) {
            st.o[i2][0] = fmaf(st.o[i2][0], kLowNibble, st.z[0]);
            st.o[i2][1] = fmaf(st.o[i2][1], kLowNibble, st.z[1]);
            st.o[i2][2] = fmaf(st.o[i2][2], kHighNibble, st.z[0]);
            st.o[i2][3] = fmaf(st.o[i2][3], kHighNibble, st.z[1]);
        }
    }
    template <class Seg>
    __device__ static void finalize(const DecodeParams &p, const Seg &sg, int lane,
                                    float o[kTiles][4], const float m[2], const float l[2])
    {
        saw::finalize<kRotate, kD, kMerge>(p, sg, lane, o, m, l);
    }
};

// Multiprocessor count and decode-kernel occupancy on the current device for head dimension kD
// (see decode::launch_shape).
template <int kD>
cudaError_t launch_shape(size_t smem, size_t merge_smem, LaunchShape &out)
{
    static ShapeCache shapes;
    static const void *const decode_kernels[kShapeVariants] = {
        reinterpret_cast<const void *>(paged_decode_kernel<Int4Format<true, kD>, false>),
        reinterpret_cast<const void *>(paged_decode_kernel<Int4Format<false, kD>, false>),
        reinterpret_cast<const void *>(paged_decode_kernel<Int4Format<true, kD>, true>),
        reinterpret_cast<const void *>(paged_decode_kernel<Int4Format<false, kD>, true>)};
    static const void *const merge_kernels[kShapeVariants] = {
        reinterpret_cast<const void *>(paged_decode_merge_kernel<Int4Format<true, kD>, false>),
        reinterpret_cast<const void *>(paged_decode_merge_kernel<Int4Format<false, kD>, false>),
        reinterpret_cast<const void *>(paged_decode_merge_kernel<Int4Format<true, kD>, true>),
        reinterpret_cast<const void *>(paged_decode_merge_kernel<Int4Format<false, kD>, true>)};
    return decode::launch_shape(shapes, decode_kernels, merge_kernels,
                                32 * Int4Format<true, kD>::kWarps, smem, merge_smem, out);
}

// The windowed decode's quantized part (rotated, decode, head_dim 128): only the shared-memory
// attributes are set here; its grid is the plain family's (same layout and launch bounds), which
// the workspace is sized for.
cudaError_t set_window_merge_attributes(size_t smem, size_t merge_smem)
{
    static ShapeCache shapes;
    using W = Int4Format<true, 128, true>;
    static const void *const decode_kernels[kShapeVariants] = {
        reinterpret_cast<const void *>(paged_decode_kernel<W, false>),
        reinterpret_cast<const void *>(paged_decode_kernel<W, false>),
        reinterpret_cast<const void *>(paged_decode_kernel<W, false>),
        reinterpret_cast<const void *>(paged_decode_kernel<W, false>)};
    static const void *const merge_kernels[kShapeVariants] = {
        reinterpret_cast<const void *>(paged_decode_merge_kernel<W, false>),
        reinterpret_cast<const void *>(paged_decode_merge_kernel<W, false>),
        reinterpret_cast<const void *>(paged_decode_merge_kernel<W, false>),
        reinterpret_cast<const void *>(paged_decode_merge_kernel<W, false>)};
    LaunchShape unused;
    return decode::launch_shape(shapes, decode_kernels, merge_kernels, 32 * W::kWarps, smem,
                                merge_smem, unused);
}

template <int kD>
size_t workspace_bytes(int32_t num_kv_heads, int32_t num_q_heads, int32_t num_seqs, int64_t total_q)
{
    using Fmt = Int4Format<true, kD>;
    const bool prefill = total_q >= 0;
    LaunchShape ls;
    if (launch_shape<kD>(decode_smem_bytes<Fmt>(num_seqs, query_rows(num_kv_heads, num_q_heads, prefill)),
                         merge_smem_bytes<Fmt::kTiles>(num_seqs), ls) != cudaSuccess)
        return 0;
    return workspace_bytes_for<Fmt::kTiles>(static_cast<size_t>(ls.sms) * ls.occ * Fmt::kWarps,
                                            max_segments(num_kv_heads, num_q_heads, num_seqs,
                                                         total_q, prefill));
}

// Tensor map of the code rows: [num_pages * Hkv * 32 rows][kD / 2 bytes], box = one (page, kv
// head), cached per thread for the last cache seen.
template <int kD>
const CUtensorMap *code_tensor_map(const uint8_t *kv_pages, int64_t rows)
{
    static thread_local struct {
        const void *base = nullptr;
        int64_t rows = 0;
        CUtensorMap map;
    } cache;
    if (cache.base != kv_pages || cache.rows != rows) {
        auto encode = tensor_map_encoder();
        if (encode == nullptr)
            return nullptr;
        const cuuint64_t dims[2] = {kD / 2, static_cast<cuuint64_t>(rows)};
        const cuuint64_t strides[1] = {kD / 2};
        const cuuint32_t box[2] = {kD / 2, 32};
        const cuuint32_t estr[2] = {1, 1};
        CUresult r = encode(&cache.map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                            const_cast<uint8_t *>(kv_pages), dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE,
                            kD == 64 ? CU_TENSOR_MAP_SWIZZLE_32B
                            : kD == 128 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) {
            cache.base = nullptr;
            return nullptr;
        }
        cache.base = kv_pages;
        cache.rows = rows;
    }
    return &cache.map;
}

template <int kD>
cudaError_t launch(const DecodeArgs &a, cudaStream_t stream, bool programmatic)
{
    // Chunked prefill whose chunks average at least half a 128-row tile per sequence runs on the
    // tensor cores (prefill_tc.cu); shorter chunks keep this kernel's split-K work split, which
    // spreads a few long rows over every SM.
    if (kD == 128 && a.q_start != nullptr && a.win_part == 0 &&
        a.total_q * (a.num_q_heads / a.num_kv_heads) >= 64 * static_cast<int64_t>(a.num_seqs))
        return launch_prefill_tc(a, stream, programmatic);
    const CUtensorMap *map = code_tensor_map<kD>(a.kv_pages, a.num_pages * a.num_kv_heads * 32);
    if (map == nullptr)
        return cudaErrorInvalidValue;

    using Fmt = Int4Format<true, kD>;   // the layout is the same for both variants
    const bool prefill = a.q_start != nullptr;
    const int32_t qrows = query_rows(a.num_kv_heads, a.num_q_heads, prefill);
    const size_t smem = decode_smem_bytes<Fmt>(a.num_seqs, qrows);
    const size_t msmem = merge_smem_bytes<Fmt::kTiles>(a.num_seqs);
    LaunchShape ls;
    cudaError_t e = launch_shape<kD>(smem, msmem, ls);
    if (e != cudaSuccess)
        return e;

    DecodeParams p;
    p.q = static_cast<const uint16_t *>(a.q);
    p.q_start = a.q_start;
    p.scales = static_cast<const uint8_t *>(a.scales);
    p.block_table = a.block_table;
    p.seq_lens = a.seq_lens;
    p.out = a.out;
    p.partials = static_cast<float *>(a.workspace);
    p.status = a.status;
    p.num_pages = a.num_pages;
    p.max_blocks = a.max_blocks;
    p.num_seqs = a.num_seqs;
    p.hq = a.num_q_heads;
    p.hkv = a.num_kv_heads;
    p.group = a.num_q_heads / a.num_kv_heads;
    p.qrows = qrows;
    p.lse = a.lse;
    p.win_part = a.win_part;
    p.win_sink = a.win_sink;
    p.win_recent = a.win_recent;
    p.max_segments = max_segments(a.num_kv_heads, a.num_q_heads, a.num_seqs, a.total_q, prefill);
    p.total_warps = ls.sms * ls.occ * Fmt::kWarps;
    // q carries sm_scale * log2(e), and 1/sqrt(B) of the (unnormalised) query butterfly
    p.q_mult = static_cast<float>((a.rotate ? static_cast<double>(hadamard_c(kD)) : 1.0) * a.sm_scale *
                                  1.4426950408889634);

    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(ls.sms * ls.occ));
    cfg.blockDim = dim3(32 * Fmt::kWarps);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = programmatic ? 1 : 0;
    const bool window_merge = a.win_part == 2;
    if (window_merge && (kD != 128 || prefill || !a.rotate))
        return cudaErrorInvalidValue;
    if (window_merge && (e = set_window_merge_attributes(smem, msmem)) != cudaSuccess)
        return e;
    auto *kernel = window_merge ? paged_decode_kernel<Int4Format<true, kD, true>, false>
                   : a.rotate   ? (prefill ? paged_decode_kernel<Int4Format<true, kD>, true>
                                           : paged_decode_kernel<Int4Format<true, kD>, false>)
                                : (prefill ? paged_decode_kernel<Int4Format<false, kD>, true>
                                           : paged_decode_kernel<Int4Format<false, kD>, false>);
    e = cudaLaunchKernelEx(&cfg, kernel, *map, p);
    if (e != cudaSuccess)
        return e;

    const int64_t segs = p.max_segments;
    cudaLaunchConfig_t mcfg = cfg;
    mcfg.gridDim = dim3(static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>(segs, 8 * ls.sms))));
    mcfg.blockDim = dim3(kMergeThreads);
    mcfg.dynamicSmemBytes = msmem;
    mcfg.numAttrs = 1;
    // at most one segment per SM: every segment is split over tens of warps, whose partials the
    // wider merge folds in fewer rounds (its shared memory stays below the default 48 KiB)
    // (the chunked prefill on this kernel takes the same choice from the same count, the decode's
    // segments, so that a one-token chunk stays bit-identical to the decode)
    const int64_t decode_segs = max_segments(a.num_kv_heads, a.num_q_heads, a.num_seqs, 0, false);
    if (kD <= 128 && !window_merge && decode_segs <= ls.sms) {
        constexpr int kW = kMergeWarpsWide;
        mcfg.blockDim = dim3(32 * kW);
        mcfg.dynamicSmemBytes = merge_smem_bytes<Fmt::kTiles, kW>(a.num_seqs);
        e = cudaLaunchKernelEx(&mcfg, a.rotate ? (prefill ? paged_decode_merge_kernel<Int4Format<true, kD>, true, kW>
                                                          : paged_decode_merge_kernel<Int4Format<true, kD>, false, kW>)
                                               : (prefill ? paged_decode_merge_kernel<Int4Format<false, kD>, true, kW>
                                                          : paged_decode_merge_kernel<Int4Format<false, kD>, false, kW>),
                               p);
        if (e != cudaSuccess)
            return e;
        return cudaGetLastError();
    }
    // many short segments (more than 4 per SM, each split over one or two warps): fewer warps per
    // segment, and enough CTAs for one wave over them
    if (kD <= 128 && !window_merge && decode_segs > 4 * static_cast<int64_t>(ls.sms)) {
        constexpr int kW = kMergeWarpsNarrow;
        mcfg.gridDim = dim3(static_cast<unsigned>(std::min<int64_t>(segs, (32 / kW) * ls.sms)));
        mcfg.blockDim = dim3(32 * kW);
        mcfg.dynamicSmemBytes = merge_smem_bytes<Fmt::kTiles, kW>(a.num_seqs);
        e = cudaLaunchKernelEx(&mcfg, a.rotate ? (prefill ? paged_decode_merge_kernel<Int4Format<true, kD>, true, kW>
                                                          : paged_decode_merge_kernel<Int4Format<true, kD>, false, kW>)
                                               : (prefill ? paged_decode_merge_kernel<Int4Format<false, kD>, true, kW>
                                                          : paged_decode_merge_kernel<Int4Format<false, kD>, false, kW>),
                               p);
        if (e != cudaSuccess)
            return e;
        return cudaGetLastError();
    }
    auto *merge = window_merge ? paged_decode_merge_kernel<Int4Format<true, kD, true>, false>
                  : a.rotate   ? (prefill ? paged_decode_merge_kernel<Int4Format<true, kD>, true>
                                          : paged_decode_merge_kernel<Int4Format<true, kD>, false>)
                               : (prefill ? paged_decode_merge_kernel<Int4Format<false, kD>, true>
                                          : paged_decode_merge_kernel<Int4Format<false, kD>, false>);
    e = cudaLaunchKernelEx(&mcfg, merge, p);
    if (e != cudaSuccess)
        return e;
    return cudaGetLastError();
}

}  // namespace

size_t decode_workspace_bytes(int32_t num_kv_heads, int32_t num_q_heads, int32_t num_seqs,
                              int64_t total_q, int32_t head_dim)
{
    if (num_kv_heads <= 0 || num_q_heads <= 0 || num_seqs < 0 || num_q_heads % num_kv_heads)
        return 0;
    if (head_dim == 128)
        return workspace_bytes<128>(num_kv_heads, num_q_heads, num_seqs, total_q);
    if (head_dim == 256)
        return workspace_bytes<256>(num_kv_heads, num_q_heads, num_seqs, total_q);
    if (head_dim == 64)
        return workspace_bytes<64>(num_kv_heads, num_q_heads, num_seqs, total_q);
    return 0;
}

cudaError_t launch_paged_decode(const DecodeArgs &a, cudaStream_t stream, bool programmatic)
{
    if (a.head_dim == 128)
        return launch<128>(a, stream, programmatic);
    if (a.head_dim == 256)
        return launch<256>(a, stream, programmatic);
    if (a.head_dim == 64)
        return launch<64>(a, stream, programmatic);
    return cudaErrorInvalidValue;
}

}  // namespace saw
