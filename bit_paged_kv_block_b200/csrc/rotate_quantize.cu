// rotate_quantize.cu -- fused Hadamard rotation + token-wise INT4 quantization + paged scatter.
//
// Implements the fused rotation-quantization kernel of "SAW-INT4: System-Aware 4-Bit KV-Cache
// Quantization for Real-World LLM Serving" (Research Findings): every new key and value head
// vector is rotated by the normalised 128-point Hadamard transform (per 128-element block; a
// 64-element head vector by the 64-point transform), quantized token-wise to
// asymmetric INT4 and written straight into its page of the paged KV cache.
//
// Results are bit-identical to the definition in saw.h:
//   * the butterfly performs exactly the IEEE fp32 adds/subtracts of the natural-order
//     Sylvester transform, stage h = 1, 2, ..., 64 in that order, then one multiply by
//     fp32(1/sqrt(128)); two fp32 operations are issued per packed f32x2 instruction, each
//     individually rounded, so the register layout does not change any result;
//   * scale = (max - min) / 15 is the IEEE quotient (computed by a three-operation sequence
//     checked against the IEEE divide for every non-negative fp32 dividend, below); each code is
//     read off one fused multiply-add on a 2^-16 grid, which is provably the IEEE-divide code
//     except where the grid value is exactly half-way between two codes; those rare elements
//     are settled by an exact remainder test (note above code_at_half()).
// This translation unit is compiled with -fmad=false as a second guard against contraction.
//
// Data movement: every warp streams its own tiles of 16 rows of 128 bytes (64 bf16 elements) of K
// and the same 16 rows of V into a private 3-stage shared-memory ring with tensor copies (TMA,
// 128-byte swizzle) completing on mbarriers, so warps never wait for each other.  The warps of the
// persistent grid take tiles round-robin.
//
// Thread layout: one thread per 64-element row; lanes 0-15 take the tile's K rows and lanes 16-31
// its V rows.  A thread keeps its row as packed pairs X[m] = (x[m], x[m + 32]), so butterfly
// stages h = 1 .. 16 of its 64 elements run on packed f32x2 instructions and stage h = 32 pairs the
// two halves of each register.  D = 64: that is the whole transform.  D = 128 and 256: a row is half
// of a 128-point block and stage h = 64 pairs lane r with lane r ^ 1; the two lanes swap their 64
// values by shuffles and each forms its own half of the stage's outputs: x + partner (lower row) or
// partner - x = fma(x, -1, partner), one IEEE rounding either way.  min / max combine over the
// vector's lanes by shuffles.
#include <cfloat>
#include <algorithm>

#include "saw_device.cuh"
#include "saw_internal.h"

namespace saw {
namespace {

constexpr float kHadamardC = 0.0883883461356163f;   // fp32(1/sqrt(128)) = 0x3DB504F3
constexpr float kHadamardC64 = 0.125f;               // 1/sqrt(64), exact
constexpr float kInv15 = 1.0f / 15.0f;               // RN(1/15)
// Codes are read off t = RN(d * 2^16 / s + kGridMagic): t lies in [2^23, 2^24), where the fp32
// spacing is 1, so t = 2^23 + 2^15 + N with N = rint(d * 2^16 / s) (the 2^-16 grid value of the
// quotient) and bits 16..19 of t hold floor(grid + 1/2).
constexpr float kGridMagic = 8421376.0f;             // 2^23 + 2^15
constexpr float kFastScaleMin = 0x1p-100f;           // scales outside [2^-100, 2^100] divide
constexpr float kFastScaleMax = 0x1p100f;
constexpr uint64_t kRqWaitLimitNs = 1000000000ull;

// Head dimension D = 64 (the 64-point transform: no 128-point block fits), 128, or 256 (two
// independent 128-point rotation blocks).  A thread holds one 64-element row (kN = 32 packed pairs);
// a vector is kThreadsPerVec rows; a warp tile is 16 rows of K and the same 16 rows of V.
template <int kD>
struct RqDims {
    static_assert(kD == 64 || kD == 128 || kD == 256, "head dimension");
    static constexpr int kN = 32;                              // packed registers per thread
    static constexpr int kThreadsPerVec = kD / 64;             // 1, 2 or 4
    static constexpr int kTileVecs = 16 / kThreadsPerVec;      // 16, 8 or 4
    static constexpr int kHalfBytes = 2048;                    // K (or V) bytes of one tile
    static constexpr int kStageBytes = 2 * kHalfBytes;
    static constexpr int kCodeBytes = kD / 2;                  // packed codes per vector
};
constexpr int kRqStages = 3;
constexpr int kRqWarps = 4;
constexpr int kRqThreads = 32 * kRqWarps;
template <int kD>
__host__ __device__ constexpr size_t rq_smem_bytes()
{
    return 1024 + size_t(kRqWarps) * kRqStages * RqDims<kD>::kStageBytes + kRqWarps * kRqStages * 8;
}

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(__byte_perm(u, 0, 0x1044)); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

// Packed pairs X[8 c .. 8 c + 7] of one block from 16-byte chunk c of its elements 0 .. kN - 1
// (`lo`) and of its elements kN .. 2 kN - 1 (`hi`): X[m] = (x[m], x[m + kN]).
__device__ __forceinline__ void pairs_from_chunk(uint4 lo, uint4 hi, uint64_t X[8])
{
    const uint32_t a[4] = {lo.x, lo.y, lo.z, lo.w};
    const uint32_t b[4] = {hi.x, hi.y, hi.z, hi.w};
#pragma unroll
    for (int k = 0; k < 4; k++) {
        X[2 * k] = f2_pack(bf16_lo(a[k]), bf16_lo(b[k]));
        X[2 * k + 1] = f2_pack(bf16_hi(a[k]), bf16_hi(b[k]));
    }
}

// The butterfly stages of the 2 kN elements one thread holds: stages h = 1 .. kN / 2 pair
// registers m and m + h (packed, two IEEE operations per instruction), stage h = kN pairs the two
// halves of each register.  Stages run in ascending h; low index gets a + b, high index a - b.
template <int kN>
__device__ __forceinline__ void fwht_stages(uint64_t X[kN])
{
#pragma unroll
    for (int hb = 1; hb < kN; hb <<= 1) {
#pragma unroll
        for (int i = 0; i < kN; i++) {
            if ((i & hb) == 0) {
                const uint64_t lo = X[i], hi = X[i + hb];
                X[i] = f2_add(lo, hi);
                X[i + hb] = f2_sub(lo, hi);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < kN; i++) {
        float lo, hi;
        f2_unpack(X[i], lo, hi);
        X[i] = f2_pack(__fadd_rn(lo, hi), __fsub_rn(lo, hi));
    }
}

template <int kN>
__device__ __forceinline__ void scale_all(uint64_t X[kN], float c)
{
    const uint64_t cc = f2_pack(c, c);
#pragma unroll
    for (int i = 0; i < kN; i++)
        X[i] = f2_mul(X[i], cc);
}

// Stage h = 64 of a 128-point block split over lanes L (elements 0..63, b = 0) and L ^ 1 (elements
// 64..127, b = 1): each lane takes its partner's 64 values by shuffles and forms its own half of the
// stage's outputs: x + partner (lower lane) or partner - x = fma(x, -1, partner) (upper lane).  The
// product is exact, so either is one IEEE rounding of the stage's sum or difference.
__device__ __forceinline__ void exchange_stage64(uint64_t X[32], int b)
{
    const float sg = b ? -1.0f : 1.0f;
    const uint64_t sgn = f2_pack(sg, sg);
#pragma unroll
    for (int i = 0; i < 32; i++) {
        float lo, hi;
        f2_unpack(X[i], lo, hi);
        const uint64_t other = f2_pack(__shfl_xor_sync(0xFFFFFFFFu, lo, 1),
                                       __shfl_xor_sync(0xFFFFFFFFu, hi, 1));
        X[i] = f2_fma(X[i], sgn, other);
    }
}

// min / max over the thread's elements (4 independent chains of three-input min / max)
template <int kN>
__device__ __forceinline__ void block_min_max(const uint64_t X[kN], float &mn, float &mx)
{
    float mns[4], mxs[4];
#pragma unroll
    for (int i = 0; i < 4; i++) {
        float lo, hi;
        f2_unpack(X[i], lo, hi);
        mns[i] = fminf(lo, hi);
        mxs[i] = fmaxf(lo, hi);
    }
#pragma unroll
    for (int i = 4; i < kN; i++) {
        float lo, hi;
        f2_unpack(X[i], lo, hi);
        mns[i & 3] = fmin3(mns[i & 3], lo, hi);
        mxs[i & 3] = fmax3(mxs[i & 3], lo, hi);
    }
    mn = fmin3(mns[0], mns[1], fminf(mns[2], mns[3]));
    mx = fmax3(mxs[0], mxs[1], fmaxf(mxs[2], mxs[3]));
}

// RN(x / 15) for x >= 0: q0 = RN(x c), e = x - 15 q0 (exact in one fma), q1 = RN(q0 + e c) with
// c = RN(1/15) -- the correction step of P. Markstein, "Computation of elementary functions on the
// IBM RISC System/6000 processor" (IBM J. Res. Dev. 34(1), 1990).  Checked exhaustively on the
// host: q1 equals the IEEE quotient for all 2^31 - 2^23 non-negative finite fp32 x.
__device__ __forceinline__ float div15(float x)
{
    const float q0 = __fmul_rn(x, kInv15);
    const float e = __fmaf_rn(-q0, 15.0f, x);
    return __fmaf_rn(e, kInv15, q0);
}

// 2^16 / s with relative error below 2^-23, for 2^-100 <= s <= 2^100: the hardware reciprocal
// (max error 1 ulp) refined by one Newton-Raphson step, scaled by 2^16 exactly.
__device__ __forceinline__ float recip_2p16(float s)
{
    float r0;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r0) : "f"(s));
    const float e = __fmaf_rn(-s, r0, 1.0f);
    const float r0s = __fmul_rn(r0, 65536.0f);
    return __fmaf_rn(r0s, e, r0s);
}

// Codes from grid values.  With Q = d / s (exact), r16 = (2^16 / s)(1 + e),
// |e| < 2^-23, and t = RN(d r16 + 2^23 + 2^15) = 2^23 + 2^15 + N, N = rint(d r16):
//   |N / 2^16 - Q| <= 2^-17 + 15.0001 * 2^-23 < 0.65 * 2^-16, and |RN(Q) - Q| <= 2^-21 (Q < 16),
// so the grid value g = N / 2^16 lies within 2^-16 of RN(Q).  g + 1/2 is a multiple of 2^-16: if
// it is not an integer it is at least 2^-16 from every integer, RN(Q) + 1/2 lies strictly between
// the same two integers, and rint(RN(Q)) = floor(g + 1/2) = bits 16..19 of t (never more than
// 15).  If it is an integer K (the low 16 bits of t are 0), m = K - 1/2 is the half-integer next
// to Q (0.5 <= m <= 14.5) and the code follows from the sign of one exact remainder: let
// E = d - m s; RN(Q) = m exactly when |Q - m| <= ulp(m) / 2 (m has an even last mantissa bit, so a
// tie also rounds to m), i.e. when |E| <= T = s ulp(m) / 2, and then the code is rint(m) (ties to
// even); otherwise RN(Q) lies on the same side of m as Q and the code is m + sign(E) / 2.  E is a
// multiple of ulp(s) / 4 (d and m s both are), and where |E| <= 2 T it has at most 7 significant
// bits, so RN(E) = fma(-m, s, d) is E itself; where |E| > 2 T, |RN(E)| >= 2 T.  The test
// |RN(E)| <= T is therefore exact, as are T (a power-of-two multiple of s) and the sign, for
// s >= 2^-100.  code_at_half() returns the code of element value y (d = y - min) whose t has zero
// low bits.
__device__ __noinline__ uint32_t code_at_half(float y, float mn, float s, uint32_t t_bits)
{
    const uint32_t cand = (t_bits >> 16) & 15u;
    const float d = __fsub_rn(y, mn);
    const float m = __fsub_rn(static_cast<float>(cand), 0.5f);
    const float e = __fmaf_rn(-m, s, d);
    const float half_ulp = __int_as_float((__float_as_int(m) & 0x7F800000) - (24 << 23));
    const float code = fabsf(e) <= __fmul_rn(s, half_ulp) ? rintf(m) : __fadd_rn(m, copysignf(0.5f, e));
    return static_cast<uint32_t>(code);
}

// The IEEE-divide code (scales outside [2^-100, 2^100]).
__device__ __noinline__ uint32_t code_by_divide(float y, float mn, float s)
{
    const float q = rintf(__fdiv_rn(__fsub_rn(y, mn), s));
    return static_cast<uint32_t>(fminf(fmaxf(q, 0.0f), 15.0f));
}

// Gather byte 2 of t_0..t_7 (the codes of elements e = 0..7) into one word, element e at bits
// 4e: bytes are [k0 | k1 << 4, k2 | k3 << 4, ...] (even index in the low nibble).
__device__ __forceinline__ uint32_t pack8_b2(const uint32_t tt[8])
{
    const uint32_t e01 = __byte_perm(tt[0], tt[2], 0x0062);
    const uint32_t e23 = __byte_perm(tt[4], tt[6], 0x0062);
    const uint32_t even = __byte_perm(e01, e23, 0x5410);   // [k0, k2, k4, k6]
    const uint32_t o01 = __byte_perm(tt[1], tt[3], 0x0062);
    const uint32_t o23 = __byte_perm(tt[5], tt[7], 0x0062);
    const uint32_t odd = __byte_perm(o01, o23, 0x5410);    // [k1, k3, k5, k7]
    return even | (odd << 4);
}

// Unsigned 16-bit minimum of three packed pairs.
__device__ __forceinline__ uint32_t vmin3_u16x2(uint32_t a, uint32_t b, uint32_t c)
{
    return __vimin3_u16x2(a, b, c);
}

// Codes of one thread's elements (held rotated, or raw for the plain INT4 cache, in X) and the
// vector's fp32 scale and zero point, given the vector's min and max.  words[g] (g < kN / 8) holds
// the codes of elements 8 g .. 8 g + 7 and words[kN / 8 + g] those of elements kN + 8 g .. (low
// halves, then high halves of the registers).  Groups of 8 registers are finished one after
// another (the rare exactly half-way elements inside the group), so each group's registers are
// free once its two words exist; scales outside [2^-100, 2^100] take the IEEE divide throughout.
template <int kN>
__device__ __forceinline__ void quantize_block(const uint64_t X[kN], float mn, float mx,
                                               uint32_t words[kN / 4], float &scale_out,
                                               float &zero_out)
{
    float scale = div15(__fsub_rn(mx, mn));
    const bool degenerate = !(scale != 0.0f);
    if (degenerate)
        scale = 0.0f;                               // canonical +0
    zero_out = __fadd_rn(mn, 0.0f);                 // a zero minimum is stored as +0
    scale_out = scale;
    const bool fast = scale >= kFastScaleMin && scale <= kFastScaleMax;
    const bool divide = !fast && !degenerate;       // scales outside [2^-100, 2^100]
    // a degenerate block gets r16 = 0: every t is the magic, code 0, and never flagged
    const float r16 = fast ? recip_2p16(scale) : 0.0f;
    const uint64_t nmn2 = f2_pack(-mn, -mn), r2 = f2_pack(r16, r16);
    const uint64_t m2 = f2_pack(kGridMagic, kGridMagic);

    if (divide) {
        // scales outside [2^-100, 2^100] (rare): every element by the IEEE divide
#pragma unroll
        for (int g = 0; g < kN / 8; g++) {
            uint32_t wl = 0, wh = 0;
#pragma unroll
            for (int e = 0; e < 8; e++) {
                float a, b;
                f2_unpack(X[8 * g + e], a, b);
                wl |= code_by_divide(a, mn, scale) << (4 * e);
                wh |= code_by_divide(b, mn, scale) << (4 * e);
            }
            words[g] = wl;
            words[kN / 8 + g] = wh;
        }
        return;
    }
#pragma unroll
    for (int g = 0; g < kN / 8; g++) {
        uint32_t tlo[8], thi[8];
        // the low 16 bits of a t are 0 only at an exactly half-way grid value: f collects the
        // smallest low half (its high half is never 0: bits 16..31 of t hold 0x4B00 | code)
        uint32_t f = 0xFFFFFFFFu;
#pragma unroll
        for (int e = 0; e < 8; e++) {
            const uint64_t d = f2_add(X[8 * g + e], nmn2);   // y - min, one rounding
            const uint64_t t = f2_fma(d, r2, m2);
            float a, b;
            f2_unpack(t, a, b);
            tlo[e] = __float_as_uint(a);
            thi[e] = __float_as_uint(b);
            f = vmin3_u16x2(f, tlo[e], thi[e]);
        }
        if ((f & 0xFFFFu) == 0) {
            // rare: settle each exactly half-way element by the remainder test
#pragma unroll
            for (int e = 0; e < 8; e++) {
                float a, b;
                f2_unpack(X[8 * g + e], a, b);
                if ((tlo[e] & 0xFFFFu) == 0)
                    tlo[e] = code_at_half(a, mn, scale, tlo[e]) << 16;
                if ((thi[e] & 0xFFFFu) == 0)
                    thi[e] = code_at_half(b, mn, scale, thi[e]) << 16;
            }
        }
        words[g] = pack8_b2(tlo);
        words[kN / 8 + g] = pack8_b2(thi);
    }
}

// Store one block's codes (two runs of kN / 2 bytes: low halves, then high halves) and, from the
// vector's first block, its fp16 (scale, zero); flag scales or zero points past fp16's range.
template <int kN>
__device__ __forceinline__ void store_block(uint8_t *dst, const uint32_t words[kN / 4], bool scale_here,
                                            float scale, float zero, uint32_t *scale_dst,
                                            uint32_t *status)
{
#pragma unroll
    for (int h = 0; h < 2; h++)
#pragma unroll
        for (int q = 0; q < kN / 32; q++)
            *reinterpret_cast<uint4 *>(dst + h * (kN / 2) + 16 * q) =
                make_uint4(words[h * (kN / 8) + 4 * q], words[h * (kN / 8) + 4 * q + 1],
                           words[h * (kN / 8) + 4 * q + 2], words[h * (kN / 8) + 4 * q + 3]);
    if (scale_here) {
        const __half2 sz = __halves2half2(__float2half_rn(scale), __float2half_rn(zero));
        *scale_dst = half2_as_u32(sz);
        // fp16 holds magnitudes below 65520: beyond, the stored value is infinite (as the
        // definition's round-to-nearest conversion gives), which the read side cannot use
        if (!(fabsf(scale) < 65520.0f) || !(fabsf(zero) < 65520.0f))
            set_status(status, SAW_DEV_RANGE);
    }
}

struct RqParams {
    const int64_t *slot_mapping;
    int64_t num_vecs;        // T * Hkv
    int64_t num_tiles;
    int32_t hkv;
    int64_t num_slots;       // num_pages * 16
    uint8_t *kv_pages;
    uint32_t *scales;        // fp16x2 (scale, zero) per row
    uint32_t *status;
    int32_t strided;         // k / v through 3-D tensor maps with a token stride
    uint32_t hkv_mul;        // vec / hkv by multiply and shift (div_hkv)
    uint32_t hkv_shift;
};

// vec / hkv without a divide (T. Granlund, P. Montgomery, "Division by invariant integers using
// multiplication", PLDI 1994, with a 33-bit multiplier): with s = ceil(log2 hkv) and
// m' = ceil(2^(32 + s) / hkv), floor(vec m' / 2^(32 + s)) = floor(vec / hkv) for every vec < 2^32;
// m' = 2^32 + hkv_mul, so vec m' / 2^32 = umulhi(vec, hkv_mul) + vec (no overflow for vec < 2^31).
__device__ __forceinline__ uint32_t div_hkv(uint32_t vec, const RqParams &p)
{
    return (__umulhi(vec, p.hkv_mul) + vec) >> p.hkv_shift;
}

// A vector's row of the cache: (page * Hkv + h) * 2 + K/V, times 16, plus the offset in the page.
__device__ __forceinline__ int64_t cache_row(int64_t slot, uint32_t h, int half, int64_t hkv)
{
    return ((((slot >> 4) * hkv + h) * 2 + half) << 4) + (slot & 15);
}

template <bool kRotate, int kD>
__global__ void __launch_bounds__(kRqThreads, 4)
    rotate_quantize_kernel(const __grid_constant__ CUtensorMap tk,
                           const __grid_constant__ CUtensorMap tv, const RqParams p)
{
    using Dims = RqDims<kD>;
    constexpr int kN = Dims::kN;
    constexpr int kStageBytes = Dims::kStageBytes;
    constexpr int kTpv = Dims::kThreadsPerVec;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_launch_dependents();
    // all indices below fit in 32 bits: the host limits the rows to 2^29
    const uint32_t W = gridDim.x * kRqWarps;
    const uint32_t wg = blockIdx.x * kRqWarps + warp;
    const uint32_t num_tiles = static_cast<uint32_t>(p.num_tiles);
    if (wg >= num_tiles)
        return;
    const int n = static_cast<int>((num_tiles - wg + W - 1) / W);   // this warp's tiles: wg + i W
    const uint32_t ring = smem_u32(smem) + warp * kRqStages * kStageBytes;
    const uint32_t bar0 = smem_u32(smem + kRqWarps * kRqStages * kStageBytes) + warp * kRqStages * 8;
    if (lane == 0)
        for (int i = 0; i < kRqStages; i++)
            mbar_init(bar0 + 8 * i, 1);
    mbar_init_fence();
    __syncwarp();

    int issued = 0, istg = 0;
    uint32_t itile = wg;
    // queue tile `itile` (16 rows of K and of V) into stage istg
    auto issue = [&]() {
        if (issued < n) {
            if (lane == 0) {
                const uint32_t dst = ring + istg * kStageBytes;
                const uint32_t bar = bar0 + 8 * istg;
                mbar_arrive_expect_tx(bar, kStageBytes);
                if (p.strided) {
                    // the tile's first vector: token and head (the box spans whole tiles)
                    const uint32_t v0 = itile * Dims::kTileVecs;
                    const int32_t tok = static_cast<int32_t>(div_hkv(v0, p));
                    const int32_t row = static_cast<int32_t>(kTpv * (v0 - tok * static_cast<uint32_t>(p.hkv)));
                    tma_load_3d(dst, &tk, 0, row, tok, bar);
                    tma_load_3d(dst + Dims::kHalfBytes, &tv, 0, row, tok, bar);
                } else {
                    const int32_t y = static_cast<int32_t>(itile * 16);
                    tma_load_2d(dst, &tk, 0, y, bar);
                    tma_load_2d(dst + Dims::kHalfBytes, &tv, 0, y, bar);
                }
            }
            issued++;
            itile += W;
            if (++istg == kRqStages)
                istg = 0;
        }
    };
    for (int k = 0; k < kRqStages - 1; k++)
        issue();

    const int half = lane >> 4;                     // 0: K, 1: V
    const int r = lane & 15;                        // row of the tile
    const int part = r % kTpv;                      // row of the vector (64 elements each)
    const int vt = r / kTpv;                        // vector of the tile
    const uint32_t num_vecs = static_cast<uint32_t>(p.num_vecs);
    const uint32_t hkv = static_cast<uint32_t>(p.hkv);
    uint32_t tile = wg;
    // slot of this thread's vector in the tile (prefetched one tile ahead)
    auto slot_of = [&](uint32_t t, uint32_t &vec) -> int64_t {
        const uint32_t vec_raw = t * Dims::kTileVecs + vt;
        vec = vec_raw < num_vecs ? vec_raw : num_vecs - 1;
        return p.slot_mapping[div_hkv(vec, p)];
    };
    uint32_t vec_next;
    int64_t slot_next = slot_of(tile, vec_next);
    int cstg = 0;
    uint32_t cphase = 0;
    int i = 0;
    for (; i < n; i++, tile += W) {
        issue();
        const uint32_t vec = vec_next;
        const bool in_range = tile * Dims::kTileVecs + vt < num_vecs;
        const int64_t slot = slot_next;
        if (i + 1 < n)
            slot_next = slot_of(tile + W, vec_next);
        const int stg = cstg;
        const bool ok = mbar_wait_bounded(bar0 + 8 * stg, cphase, kRqWaitLimitNs);
        if (++cstg == kRqStages) {
            cstg = 0;
            cphase ^= 1;
        }
        if (!__all_sync(0xFFFFFFFFu, ok)) {
            if (lane == 0)
                set_status(p.status, SAW_DEV_WAIT_TIMEOUT);
            break;
        }
        const uint32_t tok = div_hkv(vec, p);
        const uint32_t h = vec - tok * hkv;
        bool store = in_range && slot >= 0;
        if (store && slot >= p.num_slots) {
            if (part == 0 && half == 0)
                set_status(p.status, SAW_DEV_BAD_SLOT);
            store = false;
        }

        // this thread's row r of the stage's K or V half; the 16-byte chunk c of a row sits at
        // chunk c ^ (r & 7) under the 128-byte swizzle: X[m] = (x[m], x[m + 32])
        const uint32_t stage = ring + stg * kStageBytes;
        const uint32_t row = stage + half * Dims::kHalfBytes + r * 128;
        uint64_t X[kN];
#pragma unroll
        for (int c = 0; c < 4; c++)
            pairs_from_chunk(lds128(row + ((c ^ (r & 7)) << 4)),
                             lds128(row + (((c + 4) ^ (r & 7)) << 4)), X + 8 * c);
        __syncwarp();   // every lane has read the stage
        if constexpr (kRotate) {
            fwht_stages<kN>(X);
            if constexpr (kD == 64) {
                scale_all<kN>(X, kHadamardC64);
            } else {
                exchange_stage64(X, part & 1);
                scale_all<kN>(X, kHadamardC);
            }
        }
        float mn, mx;
        block_min_max<kN>(X, mn, mx);
#pragma unroll
        for (int d = 1; d < kTpv; d <<= 1) {
            mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, d));
            mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, d));
        }
        uint32_t words[kN / 4];
        float scale, zero;
        quantize_block<kN>(X, mn, mx, words, scale, zero);
        if (store) {
            const int64_t crow = cache_row(slot, h, half, p.hkv);
            store_block<kN>(p.kv_pages + crow * Dims::kCodeBytes + 32 * part, words, part == 0, scale,
                            zero, p.scales + crow, p.status);
        }
    }
    if (i < n) {
        // a wait gave up: let every queued copy land before the shared memory is released
        for (int k = i; k < issued; k++)
            mbar_wait_bounded(bar0 + 8 * (k % kRqStages), (k / kRqStages) & 1, kRqWaitLimitNs / 10);
    }
}

// ---- the full-precision window beside the INT4 cache: one serving step ----------------------
//
// "InnerQ: Hardware-Aware Tuning-Free Quantization of KV Cache for Large Language Models",
// Abstract and Figure 2: a small bf16 window of sink and recent tokens stays beside the quantized
// cache.  Sequence s's new token sits at position p = seq_lens[s] - 1: a sink (p < w_sink) takes
// window slot p; otherwise its slot in the recent ring is w_sink + (p - w_sink) mod w_recent, and
// the token it displaces (position p - w_recent, when that is not a sink) is rotated, quantized
// and scattered into the INT4 pages at quantized index p - w_recent - w_sink, bit-identically to
// the rotate+quantize kernel (same device code).  With w_recent = 0 the new token itself is
// quantized.  Window slot i lives in bf16 page win_table[s][i / 16] at offset i mod 16.
//
// Lanes as in the rotate+quantize kernel at D = 128: a warp takes 8 (sequence, kv head) pairs,
// lanes 0-15 their K vectors and lanes 16-31 their V vectors, two lanes per vector (lane 2 i + b
// holds elements 64 b .. 64 b + 63 of pair i; stage h = 64 is the shuffle exchange).  Each thread
// reads exactly the 128 bytes of the displaced vector that it later overwrites with the new
// token, so the read and the write of those bytes are ordered within one thread.
struct WinAppendParams {
    const uint16_t *k, *v;
    const int32_t *seq_lens;
    int32_t num_seqs, hkv, w_sink, w_recent;
    uint16_t *win_kv;
    const int32_t *win_table;
    int32_t win_blocks;
    int64_t num_win_pages;
    const int32_t *block_table;
    int32_t max_blocks;
    int64_t num_pages;
    uint8_t *kv_pages;
    uint32_t *scales;
    uint32_t *status;
};

template <bool kRotate>
__global__ void __launch_bounds__(kRqThreads)
    window_append_kernel(const WinAppendParams p)
{
    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int half = lane >> 4;
    const int part = lane & 1;
    const int64_t pair = (static_cast<int64_t>(blockIdx.x) * kRqWarps + warp) * 8 + ((lane & 15) >> 1);
    const bool live = pair < static_cast<int64_t>(p.num_seqs) * p.hkv;
    const int s = live ? static_cast<int>(pair / p.hkv) : 0;
    const int h = live ? static_cast<int>(pair - static_cast<int64_t>(s) * p.hkv) : 0;
    const int L = live ? p.seq_lens[s] : 0;
    const bool report = half == 0 && part == 0;
    // this thread's 64 elements of the new token, loaded now: nothing below depends on them, so
    // their latency overlaps the table lookups instead of following the quantization
    const uint16_t *src = (half ? p.v : p.k) + (static_cast<int64_t>(s) * p.hkv + h) * 128 + 64 * part;
    uint4 fresh[8];
    if (live) {
#pragma unroll
        for (int c = 0; c < 8; c++)
            fresh[c] = *reinterpret_cast<const uint4 *>(src + 8 * c);
    }

    // where the new token goes and which token is quantized
    bool to_win = false, quant = false, from_win = false;
    int slot = 0, j = 0;
    if (L > 0) {
        const int pos = L - 1;
        if (pos < p.w_sink) {
            to_win = true;
            slot = pos;
        } else if (p.w_recent == 0) {
            quant = true;
            j = pos - p.w_sink;
        } else {
            to_win = true;
            slot = p.w_sink + (pos - p.w_sink) % p.w_recent;
            if (pos - p.w_recent >= p.w_sink) {
                quant = from_win = true;
                j = pos - p.w_recent - p.w_sink;
            }
        }
    } else if (L < 0 && report) {
        set_status(p.status, SAW_DEV_BAD_SEQ_LEN);
    }
    // both table lookups depend only on the length: issue them together
    const bool q_in_table = j / kPageSize < p.max_blocks;
    const int32_t wpage = to_win ? p.win_table[static_cast<int64_t>(s) * p.win_blocks + slot / 16] : 0;
    const int32_t qpage = quant && q_in_table
                              ? p.block_table[static_cast<int64_t>(s) * p.max_blocks + j / kPageSize]
                              : -1;
    uint16_t *win = nullptr;   // this thread's 64 elements of the window slot
    if (to_win) {
        const int32_t page = wpage;
        if (page < 0 || page >= p.num_win_pages) {
            if (report)
                set_status(p.status, SAW_DEV_BAD_PAGE);
            to_win = quant = false;   // the displaced token cannot be read: leave the pair
        } else {
            win = p.win_kv + ((((static_cast<int64_t>(page) * p.hkv + h) * 2 + half) * kPageSize) +
                              slot % kPageSize) * 128 + 64 * part;
        }
    }
    int64_t row = 0;
    if (quant) {
        const int32_t page = qpage;
        if (page < 0 || page >= p.num_pages) {
            if (report)
                set_status(p.status, q_in_table ? SAW_DEV_BAD_PAGE : SAW_DEV_BAD_SEQ_LEN);
            to_win = quant = false;   // keep the displaced token where it is
        } else {
            row = ((static_cast<int64_t>(page) * p.hkv + h) * 2 + half) * kPageSize + j % kPageSize;
        }
    }

    // the vector to quantize (the displaced window token, or the new token itself when there is
    // no recent ring); both lanes of a vector decide alike, and every lane runs the transform
    // (its stage h = 64 pairs lanes 2 i and 2 i + 1): lanes with nothing to quantize run it on
    // zeros and store nothing
    uint64_t X[32];
    if (quant) {
        const uint16_t *qsrc = from_win ? win : src;
#pragma unroll
        for (int c = 0; c < 4; c++)
            pairs_from_chunk(*reinterpret_cast<const uint4 *>(qsrc + 8 * c),
                             *reinterpret_cast<const uint4 *>(qsrc + 32 + 8 * c), X + 8 * c);
    } else {
#pragma unroll
        for (int i = 0; i < 32; i++)
            X[i] = 0;
    }
    if constexpr (kRotate) {
        fwht_stages<32>(X);
        exchange_stage64(X, part);
        scale_all<32>(X, kHadamardC);
    }
    float mn, mx;
    block_min_max<32>(X, mn, mx);
    mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 1));
    uint32_t words[8];
    float scale, zero;
    quantize_block<32>(X, mn, mx, words, scale, zero);
    if (quant)
        store_block<32>(p.kv_pages + row * 64 + 32 * part, words, part == 0, scale, zero, p.scales + row,
                        p.status);
    // then the new token takes the slot (after this thread's own read of these bytes)
    if (to_win) {
#pragma unroll
        for (int c = 0; c < 8; c++)
            *reinterpret_cast<uint4 *>(win + 8 * c) = fresh[c];
    }
}

}  // namespace

cudaError_t launch_window_append(const WindowAppendArgs &a, cudaStream_t stream)
{
    const int64_t pairs = static_cast<int64_t>(a.num_seqs) * a.num_kv_heads;
    if (pairs == 0)
        return cudaSuccess;
    WinAppendParams p;
    p.k = static_cast<const uint16_t *>(a.k);
    p.v = static_cast<const uint16_t *>(a.v);
    p.seq_lens = a.seq_lens;
    p.num_seqs = a.num_seqs;
    p.hkv = a.num_kv_heads;
    p.w_sink = a.w_sink;
    p.w_recent = a.w_recent;
    p.win_kv = static_cast<uint16_t *>(a.win_kv);
    p.win_table = a.win_table;
    p.win_blocks = a.win_blocks;
    p.num_win_pages = a.num_win_pages;
    p.block_table = a.block_table;
    p.max_blocks = a.max_blocks;
    p.num_pages = a.num_pages;
    p.kv_pages = a.kv_pages;
    p.scales = static_cast<uint32_t *>(a.scales);
    p.status = a.status;
    const int64_t grid = (pairs + 8 * kRqWarps - 1) / (8 * kRqWarps);
    window_append_kernel<true><<<static_cast<unsigned>(grid), kRqThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_rotate_quantize(const RotateQuantizeArgs &a, cudaStream_t stream,
                                   bool trigger_dependents)
{
    (void)trigger_dependents;   // the kernel always releases dependents at its start
    const int64_t num_vecs = a.num_tokens * a.num_kv_heads;
    if (num_vecs == 0)
        return cudaSuccess;
    if (a.head_dim != 64 && a.head_dim != 128 && a.head_dim != 256)
        return cudaErrorInvalidValue;
    const int64_t rows_per_vec = a.head_dim / 64;   // 128-byte rows (64 elements) per vector
    const int64_t tile_vecs = 16 / rows_per_vec;
    if (num_vecs * rows_per_vec > (int64_t(1) << 29))
        return cudaErrorInvalidValue;       // tensor-map rows and tile indices fit in int32

    // k / v: contiguous [T][Hkv][D] (k_stride = v_stride = 0) through a 2-D map of 128-byte
    // rows whose box is one warp tile (16 rows), or with a token stride through 3-D maps (row,
    // row within the token, token) whose box is also one whole tile: 16 rows of one token (rows
    // per token a multiple of 16) or 16 / R whole tokens of R rows (R dividing 16).  Every copy
    // lands on a 1024-byte aligned stage.
    const bool strided = a.k_stride != 0 || a.v_stride != 0;
    const int64_t rows_per_token = a.num_kv_heads * rows_per_vec;
    static thread_local struct {
        const void *k = nullptr, *v = nullptr;
        int64_t num_vecs = 0, k_stride = -1, v_stride = -1;
        int32_t hkv = 0, head_dim = 0;
        CUtensorMap mk, mv;
    } cache;
    if (cache.k != a.k || cache.v != a.v || cache.num_vecs != num_vecs || cache.hkv != a.num_kv_heads ||
        cache.k_stride != a.k_stride || cache.v_stride != a.v_stride || cache.head_dim != a.head_dim) {
        auto encode = tensor_map_encoder();
        if (encode == nullptr)
            return cudaErrorNotSupported;
        if (strided && rows_per_token % 16 != 0 && 16 % rows_per_token != 0)
            return cudaErrorInvalidValue;
        const cuuint32_t estr[3] = {1, 1, 1};
        for (int which = 0; which < 2; which++) {
            CUresult r;
            void *base = const_cast<void *>(which ? a.v : a.k);
            if (!strided) {
                const cuuint64_t dims[2] = {128, static_cast<cuuint64_t>(rows_per_vec * num_vecs)};
                const cuuint64_t strides[1] = {128};
                const cuuint32_t box[2] = {128, 16};
                r = encode(which ? &cache.mv : &cache.mk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base,
                           dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
            } else {
                const int64_t stride = which ? a.v_stride : a.k_stride;   // bf16 elements
                const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(rows_per_token),
                                            static_cast<cuuint64_t>(a.num_tokens)};
                const cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(stride * 2)};
                const cuuint32_t box[3] = {128, static_cast<cuuint32_t>(std::min<int64_t>(rows_per_token, 16)),
                                           static_cast<cuuint32_t>(std::max<int64_t>(1, 16 / rows_per_token))};
                r = encode(which ? &cache.mv : &cache.mk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, base,
                           dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
            }
            if (r != CUDA_SUCCESS) {
                cache.k = nullptr;
                return cudaErrorInvalidValue;
            }
        }
        cache.k = a.k;
        cache.v = a.v;
        cache.num_vecs = num_vecs;
        cache.hkv = a.num_kv_heads;
        cache.head_dim = a.head_dim;
        cache.k_stride = a.k_stride;
        cache.v_stride = a.v_stride;
    }

    RqParams p;
    p.slot_mapping = a.slot_mapping;
    p.num_vecs = num_vecs;
    p.num_tiles = (num_vecs + tile_vecs - 1) / tile_vecs;
    p.hkv = a.num_kv_heads;
    p.num_slots = a.num_pages * kPageSize;
    p.kv_pages = a.kv_pages;
    p.scales = static_cast<uint32_t *>(a.scales);
    p.status = a.status;
    p.strided = strided ? 1 : 0;
    {
        uint32_t sh = 0;
        while ((int64_t(1) << sh) < a.num_kv_heads)
            sh++;
        const uint64_t d = static_cast<uint64_t>(a.num_kv_heads);
        p.hkv_shift = sh;
        p.hkv_mul = static_cast<uint32_t>(((uint64_t(1) << (32 + sh)) + d - 1) / d - (uint64_t(1) << 32));
    }

    // per device and kernel: multiprocessor count, the shared-memory attribute and occupancy
    constexpr int kMaxDevices = 64;
    constexpr int kVariants = 6;
    static int sms_of[kMaxDevices] = {}, occ_of[kMaxDevices][kVariants] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= kMaxDevices)
        return cudaErrorInvalidDevice;
    using KernelFn = void (*)(CUtensorMap, CUtensorMap, RqParams);
    static const KernelFn kernels[kVariants] = {
        rotate_quantize_kernel<true, 128>, rotate_quantize_kernel<false, 128>,
        rotate_quantize_kernel<true, 256>, rotate_quantize_kernel<false, 256>,
        rotate_quantize_kernel<true, 64>, rotate_quantize_kernel<false, 64>};
    static const size_t smem_of[kVariants] = {rq_smem_bytes<128>(), rq_smem_bytes<128>(),
                                              rq_smem_bytes<256>(), rq_smem_bytes<256>(),
                                              rq_smem_bytes<64>(), rq_smem_bytes<64>()};
    const int which = (a.head_dim == 128 ? 0 : a.head_dim == 256 ? 2 : 4) + (a.rotate ? 0 : 1);
    if (sms_of[dev] == 0) {
        int sms = 0;
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        for (int r = 0; r < kVariants && e == cudaSuccess; r++) {
            e = cudaFuncSetAttribute(reinterpret_cast<const void *>(kernels[r]),
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(smem_of[r]));
            int occ = 0;
            if (e == cudaSuccess)
                e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                    &occ, reinterpret_cast<const void *>(kernels[r]), kRqThreads, smem_of[r]);
            if (e == cudaSuccess && occ <= 0)
                e = cudaErrorInvalidConfiguration;
            occ_of[dev][r] = occ;
        }
        if (e != cudaSuccess)
            return e;
        sms_of[dev] = sms;
    }
    const int64_t grid = std::min<int64_t>((p.num_tiles + kRqWarps - 1) / kRqWarps,
                                           static_cast<int64_t>(sms_of[dev]) * occ_of[dev][which]);
    kernels[which]<<<static_cast<unsigned>(grid), kRqThreads, smem_of[which], stream>>>(cache.mk, cache.mv, p);
    return cudaGetLastError();
}

}  // namespace saw
