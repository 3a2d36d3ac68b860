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
//     individually rounded, so the lane layout does not change any result;
//   * scale = (max - min) / 15 uses the IEEE divide; the codes use a reciprocal (the note
//     above code_bits_tie() shows why that gives the IEEE-divide code) and fall back to the
//     IEEE divide where it might not.
// This translation unit is compiled with -fmad=false as a second guard against contraction.
//
// Data movement: every warp streams its own tiles of 8 consecutive (token, kv head) vectors of K
// and of V (2 KiB each) into a private 3-stage shared-memory ring with 2-D tensor copies (TMA,
// 128-byte swizzle) completing on mbarriers, so warps never wait for each other.  The warps of
// the persistent grid take tiles round-robin.
//
// Thread layout (D = 128; D = 256 uses two such pairs per vector, one per 128-block, and D = 64
// one thread per whole vector, 16 vectors of K and 16 of V per tile, the butterfly entirely in
// registers): two threads per head vector; a warp's tile has its 8 K vectors in lanes 0-15
// and its 8 V vectors in lanes 16-31.  Thread half b of a vector holds the 64 elements
// j = 16a + 8b + r (a, r in 0..7), read as eight 16-byte shared-memory loads that the 128-byte
// swizzle spreads over all banks.  Stage h = 8 is the only one that crosses the pair (one
// shuffle); the 64 elements are kept as 32 packed pairs X[8a + r] = (x[a][r], x[a + 4][r]).
#include <cfloat>
#include <algorithm>

#include "saw_device.cuh"
#include "saw_internal.h"

namespace saw {
namespace {

constexpr int kTileBytes = 2048;                       // K (or V) bytes of one warp tile: 16 rows
// Head dimension D = 64 (the 64-point transform: no 128-point block fits), 128, or 256 (two
// independent 128-point rotation blocks): a warp tile holds 2048 / (2 D) vectors of K and as
// many of V, D / 64 threads per vector, each thread 64 elements of one rotation block; a vector
// is D / 64 tensor-map rows of 128 bytes.
template <int kD>
struct RqDims {
    static_assert(kD == 64 || kD == 128 || kD == 256, "head dimension");
    static constexpr int kTileVecs = kTileBytes / (2 * kD);   // 16, 8 or 4
    static constexpr int kThreadsPerVec = kD / 64;             // 1, 2 or 4
    static constexpr int kRowsPerVec = kD / 64;                // 128-byte rows per vector
    static constexpr int kCodeBytes = kD / 2;                  // packed codes per vector
};
constexpr int kRqStages = 3;
constexpr int kRqWarps = 4;
constexpr int kRqThreads = 32 * kRqWarps;
constexpr int kRqStageBytes = 2 * kTileBytes;
constexpr int kRqSmemBars = kRqWarps * kRqStages * kRqStageBytes;
constexpr size_t kRqSmemBytes = 1024 + kRqSmemBars + kRqWarps * kRqStages * 8;
constexpr uint64_t kRqWaitLimitNs = 1000000000ull;
constexpr float kHadamardC = 0.0883883461356163f;   // fp32(1/sqrt(128)) = 0x3DB504F3
constexpr float kHadamardC64 = 0.125f;               // 1/sqrt(64), exact
constexpr float kRoundMagic = 12582912.0f;           // 1.5 * 2^23
// A code computed from the reciprocal is provably the IEEE-divide code unless the remainder
// is within 2^-18 of one half (derivation above code_bits_tie()).
constexpr float kNearHalf = 0.5f - 1.0f / 262144.0f;

__device__ __forceinline__ uint64_t shfl_xor_u64(uint32_t mask, uint64_t v, int delta)
{
    uint32_t lo = static_cast<uint32_t>(v), hi = static_cast<uint32_t>(v >> 32);
    lo = __shfl_xor_sync(mask, lo, delta);
    hi = __shfl_xor_sync(mask, hi, delta);
    return (static_cast<uint64_t>(hi) << 32) | lo;
}

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }


// This thread's 64 bf16 elements of 128-block blk of tile vector vt (rows (D / 64) vt + 2 blk
// and the next of 128 bytes; the 16-byte chunk c of row r sits at chunk c ^ (r & 7) under the
// 128-byte swizzle).
template <int kD>
__device__ __forceinline__ void load_half_vec(uint32_t tile, int vt, int blk, int b, uint4 raw[8])
{
#pragma unroll
    for (int a = 0; a < 8; a++) {
        const int row = RqDims<kD>::kRowsPerVec * vt + 2 * blk + (a >> 2);
        const int chunk = (2 * (a & 3) + b) ^ (row & 7);
        raw[a] = lds128(tile + row * 128 + chunk * 16);
    }
}

// D = 64: this thread's whole vector vt of the tile, one 128-byte row (chunk a = elements
// 8a .. 8a + 7 at chunk a ^ (vt & 7) under the 128-byte swizzle).
__device__ __forceinline__ void load_vec64(uint32_t tile, int vt, uint4 raw[8])
{
#pragma unroll
    for (int a = 0; a < 8; a++)
        raw[a] = lds128(tile + vt * 128 + ((a ^ (vt & 7)) << 4));
}

__device__ __forceinline__ void to_pairs(const uint4 raw[8], uint64_t X[32])
{
#pragma unroll
    for (int a = 0; a < 4; a++) {
        const uint32_t lo[4] = {raw[a].x, raw[a].y, raw[a].z, raw[a].w};
        const uint32_t hi[4] = {raw[a + 4].x, raw[a + 4].y, raw[a + 4].z, raw[a + 4].w};
#pragma unroll
        for (int q = 0; q < 4; q++) {
            X[8 * a + 2 * q] = f2_pack(bf16_lo(lo[q]), bf16_lo(hi[q]));
            X[8 * a + 2 * q + 1] = f2_pack(bf16_hi(lo[q]), bf16_hi(hi[q]));
        }
    }
}

// Normalised 128-point Hadamard transform of the vector held by a thread pair.
// `mask` names the lanes executing this call (the full warp, or just this pair).
__device__ __forceinline__ void fwht128(uint64_t X[32], int b, uint32_t mask)
{
    // h = 1, 2, 4: element bits r0..r2 = index bits 0..2 of X.
#pragma unroll
    for (int hb = 1; hb <= 4; hb <<= 1) {
#pragma unroll
        for (int i = 0; i < 32; i++) {
            if ((i & hb) == 0) {
                const uint64_t lo = X[i], hi = X[i + hb];
                X[i] = f2_add(lo, hi);
                X[i + hb] = f2_sub(lo, hi);
            }
        }
    }
    // h = 8: element bit 3 = the pair half b.  Low half: x + partner; high half:
    // partner - x, computed as fma(x, -1, partner): the product is exact, so the single
    // rounding gives exactly the IEEE difference.
    {
        const float sg = b ? -1.0f : 1.0f;
        const uint64_t sgn = f2_pack(sg, sg);
#pragma unroll
        for (int i = 0; i < 32; i++) {
            const uint64_t other = shfl_xor_u64(mask, X[i], 1);
            X[i] = f2_fma(X[i], sgn, other);
        }
    }
    // h = 16, 32: element bits a0, a1 = index bits 3, 4 of X.
#pragma unroll
    for (int hb = 8; hb <= 16; hb <<= 1) {
#pragma unroll
        for (int i = 0; i < 32; i++) {
            if ((i & hb) == 0) {
                const uint64_t lo = X[i], hi = X[i + hb];
                X[i] = f2_add(lo, hi);
                X[i + hb] = f2_sub(lo, hi);
            }
        }
    }
    // h = 64: element bit a2 = the two halves of each packed pair.
#pragma unroll
    for (int i = 0; i < 32; i++) {
        float lo, hi;
        f2_unpack(X[i], lo, hi);
        X[i] = f2_pack(__fadd_rn(lo, hi), __fsub_rn(lo, hi));
    }
    const uint64_t cc = f2_pack(kHadamardC, kHadamardC);
#pragma unroll
    for (int i = 0; i < 32; i++)
        X[i] = f2_mul(X[i], cc);
}

// Normalised 64-point Hadamard transform of the vector one thread holds as X[8 a + r] =
// (x[8 a + r], x[8 (a + 4) + r]) (a < 4, r < 8): element bits 0-2 are index bits 0-2 of X
// (h = 1, 2, 4), bits 3-4 index bits 3-4 (h = 8, 16), bit 5 the halves of each pair (h = 32);
// then the multiply by 1/8.  The stages run in ascending h, every operation one IEEE fp32 op.
__device__ __forceinline__ void fwht64(uint64_t X[32])
{
#pragma unroll
    for (int hb = 1; hb <= 16; hb <<= 1) {
#pragma unroll
        for (int i = 0; i < 32; i++) {
            if ((i & hb) == 0) {
                const uint64_t lo = X[i], hi = X[i + hb];
                X[i] = f2_add(lo, hi);
                X[i + hb] = f2_sub(lo, hi);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < 32; i++) {
        float lo, hi;
        f2_unpack(X[i], lo, hi);
        X[i] = f2_pack(__fadd_rn(lo, hi), __fsub_rn(lo, hi));
    }
    const uint64_t cc = f2_pack(kHadamardC64, kHadamardC64);
#pragma unroll
    for (int i = 0; i < 32; i++)
        X[i] = f2_mul(X[i], cc);
}

// Codes via the reciprocal.  With s = scale (a normal fp32 > 0), r = RN(1/s), d = RN(y - min)
// and Q = d / s exactly (0 <= Q < 15 (1 + 2^-23)):
//   t = RN(d r + M), M = 1.5 * 2^23: d r < 2^22, so t = M + k with k = rint(d r) (ties to even,
//   since M is even) and k sits in the low mantissa bits of t;
//   res = RN(d r - k) is the remainder to within 2^-26.
// |d r - Q| <= Q 2^-24 < 2^-20 and |RN(Q) - Q| <= 2^-21, so if |res| < 0.5 - 2^-18 then
// |RN(Q) - k| < 0.5 and rint(RN(d / s)) = k, which is the code the IEEE divide gives (no
// clamp is needed: k <= 15).  Otherwise the code is decided as follows.
//
// Near a half-way quotient the code follows from the sign of one exact remainder instead of a
// divide.  Let m = k +- 1/2 be the half-integer next to Q (0.5 <= m <= 14.5, since 0 <= Q <=
// 15 (1 + 2^-23)) and E = d - m s.  RN(Q) = m exactly when |Q - m| <= ulp(m) / 2 (m has an even
// last mantissa bit, so a tie also rounds to m), i.e. when |E| <= T = s ulp(m) / 2; then the
// code is rint(m), the even neighbour.  Otherwise RN(Q) lies on the same side of m as Q and the
// code is m + sign(E) / 2.  E is a multiple of ulp(s) / 4 (d and m s both are), and where
// |E| <= 2 T it has at most 7 significant bits, so RN(E) = fma(-m, s, d) is E itself; where
// |E| > 2 T, |RN(E)| >= 2 T.  The test |RN(E)| <= T is therefore exact, as are T (a power-of-two
// multiple of s) and the sign, for s >= 2^-100; smaller scales divide.
constexpr float kRemainderMinScale = 0x1p-100f;

// Bits of M + code for an element whose reciprocal remainder `res` lies near one half (or any
// element, for a subnormal scale: `fast` false), by the remainder test above, or by the IEEE
// divide for scales below 2^-100.  Out of line: it runs for about one element in a thousand
// of unrotated bf16 data and almost never for rotated data, and the many inlined call sites
// stay small.
__device__ __noinline__ uint32_t code_bits_tie(float d, float k, float res, float s, bool fast)
{
    float code;
    if (fast && s >= kRemainderMinScale) {
        const float m = __fadd_rn(k, copysignf(0.5f, res));
        const float e = __fmaf_rn(-m, s, d);
        const float half_ulp = __int_as_float((__float_as_int(m) & 0x7F800000) - (24 << 23));
        code = fabsf(e) <= __fmul_rn(s, half_ulp) ? m : __fadd_rn(m, copysignf(0.5f, e));
    } else {
        code = fminf(fmaxf(rintf(__fdiv_rn(d, s)), 0.0f), 15.0f);
    }
    return __float_as_uint(__fadd_rn(code, kRoundMagic));   // m + M: a tie goes to even
}

// Bits of M + code for element value y, given the reciprocal result t_bits (M + k).
__device__ __forceinline__ uint32_t code_bits_exact(float y, uint32_t t_bits, float mn, float s,
                                                    float r, bool fast)
{
    const float d = __fsub_rn(y, mn);
    const float k = __fsub_rn(__uint_as_float(t_bits), kRoundMagic);
    const float res = __fmaf_rn(d, r, -k);
    if (fast && fabsf(res) < kNearHalf)
        return t_bits;
    return code_bits_tie(d, k, res, s, fast);
}

// Gather the low nibbles of t_0..t_7 (codes of elements r = 0..7) into one word, element r at
// bits 4r: bytes are [k0 | k1 << 4, k2 | k3 << 4, ...] (even index in the low nibble).
__device__ __forceinline__ uint32_t pack8(const uint32_t tt[8])
{
    const uint32_t e01 = __byte_perm(tt[0], tt[2], 0x0040);
    const uint32_t e23 = __byte_perm(tt[4], tt[6], 0x0040);
    const uint32_t even = __byte_perm(e01, e23, 0x5410);   // [k0, k2, k4, k6]
    const uint32_t o01 = __byte_perm(tt[1], tt[3], 0x0040);
    const uint32_t o23 = __byte_perm(tt[5], tt[7], 0x0040);
    const uint32_t odd = __byte_perm(o01, o23, 0x5410);    // [k1, k3, k5, k7]
    return even | (odd << 4);
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
    bool strided;            // k / v through 3-D tensor maps with a token stride
};

// Quantize the vector (held rotated in X) and store codes + scale into cache row `row`.
// kRotate = false is the plain INT4 quantizer (H = I) used as the unrotated baseline.
template <bool kRotate, int kD>
__device__ __forceinline__ void quantize_store(const uint64_t X[32], int blk, int b, bool store,
                                               int64_t row, const RqParams &p)
{
    // min / max over the vector's D elements (its D / 64 threads)
    float mns[8], mxs[8];
#pragma unroll
    for (int i = 0; i < 32; i++) {
        float lo, hi;
        f2_unpack(X[i], lo, hi);
        mns[i & 7] = (i < 8) ? fminf(lo, hi) : fmin3(mns[i & 7], lo, hi);
        mxs[i & 7] = (i < 8) ? fmaxf(lo, hi) : fmax3(mxs[i & 7], lo, hi);
    }
    float mn = fminf(fmin3(mns[0], mns[1], mns[2]), fmin3(fmin3(mns[3], mns[4], mns[5]), mns[6], mns[7]));
    float mx = fmaxf(fmax3(mxs[0], mxs[1], mxs[2]), fmax3(fmax3(mxs[3], mxs[4], mxs[5]), mxs[6], mxs[7]));
#pragma unroll
    for (int d = 1; d < RqDims<kD>::kThreadsPerVec; d <<= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, d));
        mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, d));
    }

    float scale = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
    const bool degenerate = !(scale != 0.0f);
    if (degenerate)
        scale = 0.0f;                               // canonical +0
    const float zero = __fadd_rn(mn, 0.0f);         // a zero minimum is stored as +0

    const bool fast = !degenerate && !(scale < FLT_MIN);
    const float r = fast ? __frcp_rn(scale) : 0.0f;
    const uint64_t mn2 = f2_pack(mn, mn), r2 = f2_pack(r, r);
    const uint64_t m2 = f2_pack(kRoundMagic, kRoundMagic);

    // Codes and stores, two output words at a time: words a4 and a4 + 4 take the low and high
    // halves of the packed pairs X[8 a4 + r].  Each code comes from the reciprocal (see the
    // note above code_bits_tie()); the 16 elements of the two words go through
    // code_bits_exact() when one of them lies near a half-way quotient, or for a subnormal
    // scale.
    uint8_t *dst = p.kv_pages + row * RqDims<kD>::kCodeBytes + 64 * blk;
#pragma unroll
    for (int a4 = 0; a4 < 4; a4++) {
        uint32_t tlo[8], thi[8];
        float worst = 0.0f;
#pragma unroll
        for (int rr = 0; rr < 8; rr++) {
            const uint64_t d = f2_sub(X[8 * a4 + rr], mn2);
            const uint64_t t = f2_fma(d, r2, m2);
            const uint64_t nk = f2_sub(m2, t);          // -k, exact
            const uint64_t res = f2_fma(d, r2, nk);     // d r - k, one rounding
            float tl, th, el, eh;
            f2_unpack(t, tl, th);
            f2_unpack(res, el, eh);
            worst = fmax3(worst, fabsf(el), fabsf(eh));
            tlo[rr] = __float_as_uint(tl);
            thi[rr] = __float_as_uint(th);
        }
        if (degenerate) {
#pragma unroll
            for (int rr = 0; rr < 8; rr++)
                tlo[rr] = thi[rr] = __float_as_uint(kRoundMagic);   // every code 0
        } else if (!fast || !(worst < kNearHalf)) {
#pragma unroll
            for (int rr = 0; rr < 8; rr++) {
                float lo, hi;
                f2_unpack(X[8 * a4 + rr], lo, hi);
                tlo[rr] = code_bits_exact(lo, tlo[rr], mn, scale, r, fast);
                thi[rr] = code_bits_exact(hi, thi[rr], mn, scale, r, fast);
            }
        }
        if (store) {
            // D = 64: elements 8 a + r of one thread, word a at byte 4 a; otherwise elements
            // 16 a + 8 b + r of thread half b, word (a, b) at byte 8 a + 4 b of the block
            const int w_lo = kD == 64 ? 4 * a4 : 8 * a4 + 4 * b;
            const int w_hi = kD == 64 ? 4 * (a4 + 4) : 8 * (a4 + 4) + 4 * b;
            *reinterpret_cast<uint32_t *>(dst + w_lo) = pack8(tlo);
            *reinterpret_cast<uint32_t *>(dst + w_hi) = pack8(thi);
        }
    }
    if (store && b == 0 && blk == 0) {
        const __half2 sz = __halves2half2(__float2half_rn(scale), __float2half_rn(zero));
        p.scales[row] = half2_as_u32(sz);
    }
}

template <bool kRotate, int kD>
__global__ void __launch_bounds__(kRqThreads, 4)
    rotate_quantize_kernel(const __grid_constant__ CUtensorMap tk,
                           const __grid_constant__ CUtensorMap tv, const RqParams p)
{
    using Dims = RqDims<kD>;
    constexpr int kTileVecs = Dims::kTileVecs;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_launch_dependents();
    // all indices below fit in 32 bits: the host limits num_vecs to 2^29
    const uint32_t W = gridDim.x * kRqWarps;
    const uint32_t wg = blockIdx.x * kRqWarps + warp;
    const uint32_t num_tiles = static_cast<uint32_t>(p.num_tiles);
    if (wg >= num_tiles)
        return;
    const int n = static_cast<int>((num_tiles - wg + W - 1) / W);   // this warp's tiles: wg + i W
    const uint32_t ring = smem_u32(smem) + warp * kRqStages * kRqStageBytes;
    const uint32_t bar0 = smem_u32(smem + kRqSmemBars) + warp * kRqStages * 8;
    if (lane == 0)
        for (int i = 0; i < kRqStages; i++)
            mbar_init(bar0 + 8 * i, 1);
    mbar_init_fence();
    __syncwarp();

    int issued = 0, istg = 0;
    uint32_t itile = wg;
    const uint32_t hkv_u = static_cast<uint32_t>(p.hkv);
    auto issue = [&]() {
        if (issued < n) {
            if (lane == 0) {
                const uint32_t dst = ring + istg * kRqStageBytes;
                const uint32_t bar = bar0 + 8 * istg;
                mbar_arrive_expect_tx(bar, kRqStageBytes);
                if (p.strided) {
                    // the tile's first vector: token and head (the box spans whole tiles)
                    const uint32_t v0 = itile * kTileVecs;
                    const int32_t tok = static_cast<int32_t>(v0 / hkv_u);
                    const int32_t row = static_cast<int32_t>(Dims::kRowsPerVec * (v0 - tok * hkv_u));
                    tma_load_3d(dst, &tk, 0, row, tok, bar);
                    tma_load_3d(dst + kTileBytes, &tv, 0, row, tok, bar);
                } else {
                    const int32_t y = static_cast<int32_t>(itile * (Dims::kRowsPerVec * kTileVecs));
                    tma_load_2d(dst, &tk, 0, y, bar);
                    tma_load_2d(dst + kTileBytes, &tv, 0, y, bar);
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

    const int half = lane >> 4;          // 0: K, 1: V
    // half of a 128-block, 128-block of the vector, vector of the tile (D = 64: one thread
    // holds a whole vector)
    const int b = kD == 64 ? 0 : lane & 1;
    const int blk = kD == 64 ? 0 : (lane >> 1) & (Dims::kThreadsPerVec / 2 - 1);
    const int vt = (lane & 15) / Dims::kThreadsPerVec;
    const uint32_t num_vecs = static_cast<uint32_t>(p.num_vecs);
    const uint32_t hkv = static_cast<uint32_t>(p.hkv);
    uint32_t tile = wg;
    // slot of this thread's vector in the tile (prefetched one tile ahead)
    auto slot_of = [&](uint32_t t, uint32_t &vec) -> int64_t {
        const uint32_t vec_raw = t * kTileVecs + vt;
        vec = vec_raw < num_vecs ? vec_raw : num_vecs - 1;
        return p.slot_mapping[vec / hkv];
    };
    uint32_t vec_next;
    int64_t slot_next = slot_of(tile, vec_next);
    int cstg = 0;
    uint32_t cphase = 0;
    int i = 0;
    for (; i < n; i++, tile += W) {
        issue();
        const uint32_t vec = vec_next;
        const bool in_range = tile * kTileVecs + vt < num_vecs;
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
        const uint32_t tok = vec / hkv;
        const uint32_t h = vec - tok * hkv;
        bool store = in_range && slot >= 0;
        if (store && slot >= p.num_slots) {
            if (b == 0 && half == 0)
                set_status(p.status, SAW_DEV_BAD_SLOT);
            store = false;
        }
        const int64_t page = store ? slot >> 4 : 0;    // slot / 16
        const int64_t off = store ? slot & 15 : 0;
        const int64_t row = ((page * p.hkv + h) * 2 + half) * kPageSize + off;

        const uint32_t tile_smem = ring + stg * kRqStageBytes + half * kTileBytes;
        uint4 raw[8];
        if constexpr (kD == 64)
            load_vec64(tile_smem, vt, raw);
        else
            load_half_vec<kD>(tile_smem, vt, blk, b, raw);
        uint64_t X[32];
        to_pairs(raw, X);
        if constexpr (kRotate) {
            if constexpr (kD == 64)
                fwht64(X);
            else
                fwht128(X, b, 0xFFFFFFFFu);
        }
        quantize_store<kRotate, kD>(X, blk, b, store, row, p);
        __syncwarp();
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
// lanes 0-15 their K vectors and lanes 16-31 their V vectors, two threads per vector.  Each
// thread reads exactly the 128 bytes of the displaced vector it later overwrites with the new
// token, so the read and the write of a slot are ordered within one thread.
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
    RqParams q;        // kv_pages and scales for quantize_store; status
};

template <bool kRotate>
__global__ void __launch_bounds__(kRqThreads)
    window_append_kernel(const WinAppendParams p)
{
    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int half = lane >> 4, b = lane & 1, vt = (lane & 15) >> 1;
    const int64_t pair = (static_cast<int64_t>(blockIdx.x) * kRqWarps + warp) * 8 + vt;
    const bool live = pair < static_cast<int64_t>(p.num_seqs) * p.hkv;
    const int s = live ? static_cast<int>(pair / p.hkv) : 0;
    const int h = live ? static_cast<int>(pair - static_cast<int64_t>(s) * p.hkv) : 0;
    const int L = live ? p.seq_lens[s] : 0;
    const bool report = b == 0 && half == 0;

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
        set_status(p.q.status, SAW_DEV_BAD_SEQ_LEN);
    }
    uint16_t *win = nullptr;
    if (to_win) {
        const int32_t page = p.win_table[static_cast<int64_t>(s) * p.win_blocks + slot / 16];
        if (page < 0 || page >= p.num_win_pages) {
            if (report)
                set_status(p.q.status, SAW_DEV_BAD_PAGE);
            to_win = quant = false;   // the displaced token cannot be read: leave the pair
        } else {
            win = p.win_kv + ((((static_cast<int64_t>(page) * p.hkv + h) * 2 + half) * kPageSize) +
                              slot % kPageSize) * 128;
        }
    }
    int64_t row = 0;
    if (quant) {
        const int32_t page = j / kPageSize < p.max_blocks
                                 ? p.block_table[static_cast<int64_t>(s) * p.max_blocks + j / kPageSize]
                                 : -1;
        if (page < 0 || page >= p.num_pages) {
            if (report)
                set_status(p.q.status, j / kPageSize < p.max_blocks ? SAW_DEV_BAD_PAGE : SAW_DEV_BAD_SEQ_LEN);
            to_win = quant = false;   // keep the displaced token where it is
        } else {
            row = ((static_cast<int64_t>(page) * p.hkv + h) * 2 + half) * kPageSize + j % kPageSize;
        }
    }

    // this thread's 64 elements (16 a + 8 b + r) of the new vector and of the displaced one
    uint4 fresh[8], raw[8];
    const uint16_t *src = (half ? p.v : p.k) + (static_cast<int64_t>(s) * p.hkv + h) * 128;
#pragma unroll
    for (int a = 0; a < 8; a++) {
        fresh[a] = L > 0 ? *reinterpret_cast<const uint4 *>(src + 16 * a + 8 * b) : make_uint4(0, 0, 0, 0);
        raw[a] = from_win && quant ? *reinterpret_cast<const uint4 *>(win + 16 * a + 8 * b) : fresh[a];
    }
    uint64_t X[32];
    to_pairs(raw, X);
    if constexpr (kRotate)
        fwht128(X, b, 0xFFFFFFFFu);
    quantize_store<kRotate, 128>(X, 0, b, quant, row, p.q);
    if (to_win) {
#pragma unroll
        for (int a = 0; a < 8; a++)
            *reinterpret_cast<uint4 *>(win + 16 * a + 8 * b) = fresh[a];
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
    p.q = RqParams{};
    p.q.kv_pages = a.kv_pages;
    p.q.scales = static_cast<uint32_t *>(a.scales);
    p.q.status = a.status;
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
    const int64_t rows_per_vec = a.head_dim / 64;
    const int64_t tile_vecs = kTileBytes / (2 * a.head_dim);
    if (num_vecs * rows_per_vec > (int64_t(1) << 30))
        return cudaErrorInvalidValue;       // tensor-map rows must fit in int32

    // k / v: contiguous [T][Hkv][D] (k_stride = v_stride = 0) through a 2-D map of 128-byte
    // rows, or with a token stride through 3-D maps whose box is one whole tile of V vectors
    // (V = 16 for D = 64, 8 for D = 128, 4 for D = 256; Hkv a multiple of V: V heads of one token; Hkv dividing
    // V: V / Hkv tokens), so every copy lands on a 1024-byte aligned stage.
    const bool strided = a.k_stride != 0 || a.v_stride != 0;
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
        const int64_t hkv = a.num_kv_heads;
        if (strided && hkv % tile_vecs != 0 && tile_vecs % hkv != 0)
            return cudaErrorInvalidValue;
        const cuuint32_t estr[3] = {1, 1, 1};
        for (int which = 0; which < 2; which++) {
            CUresult r;
            void *base = const_cast<void *>(which ? a.v : a.k);
            if (!strided) {
                const cuuint64_t dims[2] = {128, static_cast<cuuint64_t>(rows_per_vec * num_vecs)};
                const cuuint64_t strides[1] = {128};
                const cuuint32_t box[2] = {128, kTileBytes / 128};   // one warp tile: 16 rows
                r = encode(which ? &cache.mv : &cache.mk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base,
                           dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
            } else {
                const int64_t stride = which ? a.v_stride : a.k_stride;   // bf16 elements
                const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(rows_per_vec * hkv),
                                            static_cast<cuuint64_t>(a.num_tokens)};
                const cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(stride * 2)};
                const cuuint32_t box[3] = {128, static_cast<cuuint32_t>(rows_per_vec * std::min<int64_t>(hkv, tile_vecs)),
                                           static_cast<cuuint32_t>(std::max<int64_t>(1, tile_vecs / hkv))};
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
    p.strided = strided;

    // per device: multiprocessor count, the shared-memory attribute and the occupancy
    constexpr int kMaxDevices = 64;
    static int sms_of[kMaxDevices] = {}, occ_of[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= kMaxDevices)
        return cudaErrorInvalidDevice;
    static const void *const kernels[6] = {
        reinterpret_cast<const void *>(rotate_quantize_kernel<true, 128>),
        reinterpret_cast<const void *>(rotate_quantize_kernel<false, 128>),
        reinterpret_cast<const void *>(rotate_quantize_kernel<true, 256>),
        reinterpret_cast<const void *>(rotate_quantize_kernel<false, 256>),
        reinterpret_cast<const void *>(rotate_quantize_kernel<true, 64>),
        reinterpret_cast<const void *>(rotate_quantize_kernel<false, 64>)};
    auto kernel = a.head_dim == 128
                      ? (a.rotate ? rotate_quantize_kernel<true, 128> : rotate_quantize_kernel<false, 128>)
                  : a.head_dim == 256
                      ? (a.rotate ? rotate_quantize_kernel<true, 256> : rotate_quantize_kernel<false, 256>)
                      : (a.rotate ? rotate_quantize_kernel<true, 64> : rotate_quantize_kernel<false, 64>);
    if (sms_of[dev] == 0) {
        int sms = 0, occ = 0;
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        for (int r = 0; r < 6 && e == cudaSuccess; r++)
            e = cudaFuncSetAttribute(kernels[r], cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(kRqSmemBytes));
        if (e == cudaSuccess)
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernels[0], kRqThreads,
                                                              kRqSmemBytes);
        if (e != cudaSuccess)
            return e;
        if (occ <= 0)
            return cudaErrorInvalidConfiguration;
        occ_of[dev] = occ;
        sms_of[dev] = sms;
    }
    const int64_t grid = std::min<int64_t>((p.num_tiles + kRqWarps - 1) / kRqWarps,
                                           static_cast<int64_t>(sms_of[dev]) * occ_of[dev]);
    kernel<<<static_cast<unsigned>(grid), kRqThreads, kRqSmemBytes, stream>>>(cache.mk, cache.mv, p);
    return cudaGetLastError();
}

}  // namespace saw
