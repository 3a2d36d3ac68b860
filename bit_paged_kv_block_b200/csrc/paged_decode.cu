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
// The query of the next segment is bulk-copied into a per-warp buffer while the current one is
// processed.  The query dimension d of QK and the value dimension of PV are consumed in a
// permuted order (both sides permuted alike), which lets every thread unpack whole 32-bit code
// words; the final inverse rotation undoes it.
#include <cfloat>
#include <cudaTypedefs.h>

#include <mutex>
#include <type_traits>

#include "saw_device.cuh"
#include "saw_internal.h"

namespace saw {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;
constexpr int kStages = 4;                              // power of two
constexpr int kCodeBytes = 2 * kPageSize * kRowBytes;   // K + V codes of one (page, kv head)
constexpr int kScaleBytes = 2 * kPageSize * 4;          // K + V (scale, zero) fp16 pairs
constexpr uint32_t kTxBytes = kCodeBytes + kScaleBytes;
constexpr int kSlotFloats = 32 * 32 + 16;               // O (lane layout) + m[8] + l[8]
constexpr int64_t kKappa = 2;                           // per-segment cost, in pages
constexpr uint64_t kWaitLimitNs = 1000000000ull;        // give up a copy wait after 1 s
constexpr float kHadamardC = 0.0883883461356163f;
constexpr int kMergeWarps = 4;
constexpr int kMergeThreads = 32 * kMergeWarps;

// shared memory carve-up of the decode kernel (bytes, from a 1024-aligned base); the query
// buffers (G * 256 bytes per warp) and the sequence prefix follow at run-time offsets
constexpr int kSmemCodes = 0;
constexpr int kSmemScales = kSmemCodes + kWarps * kStages * kCodeBytes;
constexpr int kSmemBars = kSmemScales + kWarps * kStages * kScaleBytes;
constexpr int kSmemFlags = kSmemBars + kWarps * (kStages + 1) * 8;
constexpr int kSmemQ = kSmemFlags + 64;
__host__ __device__ constexpr int q_bytes(int group) { return group * kHeadDim * 2; }
__host__ __device__ constexpr int smem_prefix_offset(int group) { return kSmemQ + kWarps * q_bytes(group); }
// merge kernel: per-warp partials, then the prefix
constexpr int kMergeSmemSlots = 0;
constexpr int kMergeSmemFlags = kMergeSmemSlots + (kMergeWarps - 1) * kSlotFloats * 4;
constexpr int kMergeSmemPrefix = kMergeSmemFlags + 64;

size_t decode_smem_bytes(int32_t num_seqs, int32_t group)
{
    return 1024 + smem_prefix_offset(group) + 4 * (static_cast<size_t>(num_seqs) + 1);
}
size_t merge_smem_bytes(int32_t num_seqs)
{
    return kMergeSmemPrefix + 4 * (static_cast<size_t>(num_seqs) + 1);
}

struct DecodeParams {
    const uint16_t *q;
    const uint8_t *scales;       // bytes; 128 B per (page, kv head)
    const int32_t *block_table;
    const int32_t *seq_lens;
    float *out;
    float *partials;             // workspace: (total warps + segments) slots
    uint32_t *status;
    int64_t num_pages;
    int32_t max_blocks;
    int32_t num_seqs;
    int32_t hq;
    int32_t hkv;
    int32_t group;
    int32_t total_warps;         // warps of the decode grid (the plan's slice count bound)
    float q_mult;                // fp32(1/sqrt(128)) * sm_scale * log2(e)
};

// ---- work plan ------------------------------------------------------------------------------

// Largest s in [0, S) with hkv * pre[s] <= pos (pos < hkv * pre[S]).
__device__ __forceinline__ int find_seq(const int32_t *pre, int S, int64_t pos, int64_t hkv)
{
    int lo = 0, hi = S;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (hkv * pre[mid] <= pos)
            lo = mid;
        else
            hi = mid;
    }
    return lo;
}

// Pages per sequence (0 for an invalid length, which is flagged) and their exclusive prefix
// pre[0..S] in shared memory; every thread of the block takes part.
__device__ void scan_pages(const DecodeParams &p, int32_t *pre, volatile int32_t *flags,
                           bool report)
{
    const int S = p.num_seqs, nthreads = blockDim.x, tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    const int per = (S + nthreads - 1) / nthreads;
    const int s0 = tid * per, s1 = min(S, s0 + per);
    int local = 0;
    for (int s = s0; s < s1; s++) {
        const int len = p.seq_lens[s];
        const bool ok = len >= 0 && len <= p.max_blocks * kPageSize;
        if (!ok && report)
            set_status(p.status, SAW_DEV_BAD_SEQ_LEN);
        local += ok ? (len + kPageSize - 1) / kPageSize : 0;
    }
    int incl = local;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int o = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        if (lane >= d)
            incl += o;
    }
    if (lane == 31)
        flags[warp] = incl;
    __syncthreads();
    int base = 0;
    for (int w = 0; w < warp; w++)
        base += flags[w];
    int run = base + incl - local;
    for (int s = s0; s < s1; s++) {
        pre[s] = run;
        const int len = p.seq_lens[s];
        const bool ok = len >= 0 && len <= p.max_blocks * kPageSize;
        run += ok ? (len + kPageSize - 1) / kPageSize : 0;
    }
    if (tid == nthreads - 1)
        pre[S] = base + incl;
    __syncthreads();
}

// The cost-space split of the flat page range into warp runs.  Segment (s, h) spans the cost
// range [seq_cost(s) + h (n_s + kKappa), + n_s + kKappa); its page i sits at cost
// seq_cost(s) + h (n_s + kKappa) + kKappa + i.  Warp u owns the cost range
// [b(u), b(u + 1)) with b(u) = u q + min(u, r), q = PT / W, r = PT % W (slices of q or q + 1,
// never empty because W <= PT), i.e. the pages whose cost falls in it.
struct Plan {
    const int32_t *pre;
    int S;
    int64_t hkv;
    int64_t P;    // pages
    int64_t PT;   // cost
    int64_t W;    // warps with a slice
    int64_t q, r;

    __device__ void init(const int32_t *pre_, int S_, int hkv_, int total_warps)
    {
        pre = pre_;
        S = S_;
        hkv = hkv_;
        P = hkv * pre[S];
        PT = hkv * (static_cast<int64_t>(pre[S]) + kKappa * S);
        W = max(int64_t(1), min(static_cast<int64_t>(total_warps), PT));
        q = PT / W;
        r = PT - q * W;
    }
    __device__ int64_t seq_cost(int s) const
    {
        return hkv * (static_cast<int64_t>(pre[s]) + kKappa * s);
    }
    __device__ int64_t slice_begin(int64_t u) const { return u * q + min(u, r); }
    // the warp whose cost slice holds cost position x (0 <= x < PT)
    __device__ int64_t warp_of_cost(int64_t x) const
    {
        const int64_t big = r * (q + 1);
        return x < big ? x / (q + 1) : r + (x - big) / q;
    }
    // cost position of page i of segment (s, h)
    __device__ int64_t page_cost(int s, int h, int64_t i) const
    {
        return seq_cost(s) + static_cast<int64_t>(h) * (pre[s + 1] - pre[s] + kKappa) + kKappa + i;
    }
    // first flat page whose cost position is >= x
    __device__ int64_t flat_of_cost(int64_t x) const
    {
        if (x >= PT)
            return P;
        int lo = 0, hi = S;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (seq_cost(mid) <= x)
                lo = mid;
            else
                hi = mid;
        }
        const int64_t n = pre[lo + 1] - pre[lo];
        const int64_t within = x - seq_cost(lo);
        const int64_t h = within / (n + kKappa);
        const int64_t rr = within - h * (n + kKappa);
        return hkv * pre[lo] + h * n + (rr < kKappa ? 0 : rr - kKappa);
    }
    // first flat page of warp u's run (u in [0, W]; the run of u is [begin(u), begin(u + 1)))
    __device__ int64_t begin(int64_t u) const { return flat_of_cost(slice_begin(u)); }
};

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

// Per-warp running state of one piece, in mma accumulator layout: thread (g, t) holds heads
// 2t and 2t + 1 and, for m-tile i = 2c + h2, the value rows d = 32c + 4g + 2h2 (+1).
struct WarpState {
    float o[8][4];
    float m[2];
    float l[2];
    float z[2];
};

__device__ __forceinline__ void state_reset(WarpState &st)
{
#pragma unroll
    for (int i = 0; i < 8; i++)
#pragma unroll
        for (int k = 0; k < 4; k++)
            st.o[i][k] = 0.0f;
#pragma unroll
    for (int e = 0; e < 2; e++) {
        st.m[e] = -INFINITY;
        st.l[e] = 0.0f;
        st.z[e] = 0.0f;
    }
}

// Rotated, scaled query of (seq s, kv head h) as fp16 mma B fragments, from the raw bf16
// queries of the group in shared memory ([G][128] at qbuf).
// Thread (g, t) owns query head g of the group and d in [32t, 32t + 32).
template <bool kRotate>
__device__ __forceinline__ void load_query(const DecodeParams &p, uint32_t qbuf, int g, int t,
                                           uint32_t bq[8][2], float sq_out[2])
{
    float x[32];
    if (g < p.group) {
#pragma unroll
        for (int c = 0; c < 4; c++) {
            const uint4 u = lds128(qbuf + g * (kHeadDim * 2) + 64 * t + 16 * c);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int k = 0; k < 4; k++) {
                x[8 * c + 2 * k] = __uint_as_float(w[k] << 16);
                x[8 * c + 2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
            }
        }
    } else {
#pragma unroll
        for (int l = 0; l < 32; l++)
            x[l] = 0.0f;
    }
    // Hadamard butterfly: d bits 0..4 in registers, bits 5, 6 across lanes t ^ 1, t ^ 2
    // (skipped for the plain INT4 cache).
#pragma unroll
    for (int hb = 1; kRotate && hb < 32; hb <<= 1)
#pragma unroll
        for (int l = 0; l < 32; l++)
            if ((l & hb) == 0) {
                const float a = x[l], b = x[l + hb];
                x[l] = a + b;
                x[l + hb] = a - b;
            }
#pragma unroll
    for (int lb = 1; kRotate && lb <= 2; lb <<= 1) {
        const bool high = (t & lb) != 0;
#pragma unroll
        for (int l = 0; l < 32; l++) {
            const float o = __shfl_xor_sync(0xFFFFFFFFu, x[l], lb);
            x[l] = high ? o - x[l] : x[l] + o;
        }
    }
    // Even d pair with low nibbles (weight 2^-24), odd d with high nibbles (weight 2^-20): odd
    // entries carry q / 16 so that every product is q_d * code_d * 2^-24.
    float sq = 0.0f;
    __half hq[32];
#pragma unroll
    for (int l = 0; l < 32; l++) {
        const float qv = x[l] * p.q_mult;
        hq[l] = __float2half_rn((l & 1) ? qv * 0.0625f : qv);
        sq += (l & 1) ? 16.0f * __half2float(hq[l]) : __half2float(hq[l]);
    }
    sq += __shfl_xor_sync(0xFFFFFFFFu, sq, 1);
    sq += __shfl_xor_sync(0xFFFFFFFFu, sq, 2);
    // k-step (i, e): k slots (2t, 2t+1 | 2t+8, 2t+9) <-> d = 32t + 8i + 2e + (0, 4 | 1, 5)
#pragma unroll
    for (int i = 0; i < 4; i++)
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

// One page of one warp: QK^T, online softmax, PV.  kMask: the page is the last of its
// segment and only its first `valid` tokens exist.
template <bool kMask>
__device__ __forceinline__ void process_page(uint32_t cbase, uint32_t sbase, int valid,
                                             const uint32_t bq[8][2], const float sq[2],
                                             int lane, WarpState &st)
{
    const int g = lane >> 2, t = lane & 3;

    // ---- S^T = K . Q^T over 16 tokens (rows g, g + 8) -----------------------------------
    const uint4 k0 = lds128(cbase + g * 64 + ((t ^ ((g >> 1) & 3)) << 4));
    const uint4 k1 = lds128(cbase + (g + 8) * 64 + ((t ^ (((g + 8) >> 1) & 3)) << 4));
    const uint32_t kw0[4] = {k0.x, k0.y, k0.z, k0.w};
    const uint32_t kw1[4] = {k1.x, k1.y, k1.z, k1.w};
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int i = 0; i < 4; i++) {
        uint32_t ya[4], yb[4];
        unpack_codes(kw0[i], ya);
        unpack_codes(kw1[i], yb);
        const uint32_t a0[4] = {ya[0], yb[0], ya[1], yb[1]};
        const uint32_t a1[4] = {ya[2], yb[2], ya[3], yb[3]};
        mma_16816(acc, a0, bq[2 * i][0], bq[2 * i][1]);
        mma_16816(acc, a1, bq[2 * i + 1][0], bq[2 * i + 1][1]);
    }

    // ---- logits (log2 domain) ---------------------------------------------------------------
    const bool v0 = !kMask || g < valid, v1 = !kMask || g + 8 < valid;
    const float2 ksz0 = h2_to_f2(lds32(sbase + 4 * g));
    const float2 ksz1 = h2_to_f2(lds32(sbase + 4 * (g + 8)));
    const float ks0 = ksz0.x * kLowNibble, ks1 = ksz1.x * kLowNibble;
    float s[4];
    s[0] = fmaf(ks0, acc[0], ksz0.y * sq[0]);
    s[1] = fmaf(ks0, acc[1], ksz0.y * sq[1]);
    s[2] = fmaf(ks1, acc[2], ksz1.y * sq[0]);
    s[3] = fmaf(ks1, acc[3], ksz1.y * sq[1]);
    if (kMask) {
        if (!v0)
            s[0] = s[1] = -INFINITY;
        if (!v1)
            s[2] = s[3] = -INFINITY;
    }

    // The running max only changes when some logit of the page exceeds it, so the cross-lane
    // reduction is needed only then (rare once a piece is a few pages long).
    const bool grow = fmaxf(s[0], s[2]) > st.m[0] || fmaxf(s[1], s[3]) > st.m[1];
    if (__any_sync(0xFFFFFFFFu, grow)) {
        float mx[2] = {fmaxf(s[0], s[2]), fmaxf(s[1], s[3])};
#pragma unroll
        for (int e = 0; e < 2; e++) {
            mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xFFFFFFFFu, mx[e], 4));
            mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xFFFFFFFFu, mx[e], 8));
            mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xFFFFFFFFu, mx[e], 16));
        }
        float alpha[2];
#pragma unroll
        for (int e = 0; e < 2; e++) {
            const float mn = fmaxf(st.m[e], mx[e]);
            alpha[e] = ex2_approx(st.m[e] - mn);
            st.m[e] = mn;
            st.l[e] *= alpha[e];
            st.z[e] *= alpha[e];
        }
#pragma unroll
        for (int i = 0; i < 8; i++) {
            st.o[i][0] *= alpha[0];
            st.o[i][1] *= alpha[1];
            st.o[i][2] *= alpha[0];
            st.o[i][3] *= alpha[1];
        }
    }
    float pr[4];
    pr[0] = ex2_approx(s[0] - st.m[0]);
    pr[1] = ex2_approx(s[1] - st.m[1]);
    pr[2] = ex2_approx(s[2] - st.m[0]);
    pr[3] = ex2_approx(s[3] - st.m[1]);

    // V-side scale / zero of tokens g, g + 8 (masked tokens contribute exactly 0)
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

    // ---- O^T += V^T . P'^T -----------------------------------------------------------------
    // ldmatrix.trans: lane L addresses row (L & 7) of matrix L >> 3; matrices are
    // (tokens 0-7 | 8-15) x (16-byte chunk 2j | 2j + 1) of the V rows (rows 16..31).
    const int vtok = ((lane >> 3) & 1) * 8 + (lane & 7);
    const int vrow = 16 + vtok;
    const uint32_t vrow_base = cbase + vrow * 64;
    const int vsw = (vrow >> 1) & 3;
#pragma unroll
    for (int j = 0; j < 2; j++) {
        const int chunk = 2 * j + (lane >> 4);
        uint32_t r[4];
        ldsm_x4_trans(vrow_base + ((chunk ^ vsw) << 4), r[0], r[1], r[2], r[3]);
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

// Fold (m, l, o) partial b (scaled by its own max) into the running partial a.
__device__ __forceinline__ void merge_into(float am[2], float al[2], float ao[8][4],
                                           const float bm[2], const float bl[2],
                                           const float4 bo[8])
{
    float fa[2], fb[2];
#pragma unroll
    for (int e = 0; e < 2; e++) {
        const float mn = fmaxf(am[e], bm[e]);
        fa[e] = (mn == -INFINITY) ? 0.0f : ex2_approx(am[e] - mn);
        fb[e] = (mn == -INFINITY) ? 0.0f : ex2_approx(bm[e] - mn);
        am[e] = mn;
        al[e] = al[e] * fa[e] + bl[e] * fb[e];
    }
#pragma unroll
    for (int i = 0; i < 8; i++) {
        ao[i][0] = ao[i][0] * fa[0] + bo[i].x * fb[0];
        ao[i][1] = ao[i][1] * fa[1] + bo[i].y * fb[1];
        ao[i][2] = ao[i][2] * fa[0] + bo[i].z * fb[0];
        ao[i][3] = ao[i][3] * fa[1] + bo[i].w * fb[1];
    }
}

// o_r = o / l, out = H o_r (o_r itself for the plain INT4 cache) for the heads this thread
// holds; written to out[s][h G + 2t + e].
template <bool kRotate>
__device__ __forceinline__ void finalize(const DecodeParams &p, int s, int h, int lane,
                                         float o[8][4], const float l[2])
{
    const int g = lane >> 2, t = lane & 3;
    const float inv[2] = {1.0f / l[0], 1.0f / l[1]};
    // v[e][c][j]: head 2t + e, d = 32c + 4g + j
    float v[2][4][4];
#pragma unroll
    for (int c = 0; c < 4; c++)
#pragma unroll
        for (int e = 0; e < 2; e++) {
            v[e][c][0] = o[2 * c][e] * inv[e];
            v[e][c][1] = o[2 * c][2 + e] * inv[e];
            v[e][c][2] = o[2 * c + 1][e] * inv[e];
            v[e][c][3] = o[2 * c + 1][2 + e] * inv[e];
        }
#pragma unroll
    for (int e = 0; kRotate && e < 2; e++) {
        // d bits 0, 1 (j) and 5, 6 (c) in registers
#pragma unroll
        for (int c = 0; c < 4; c++)
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
        for (int cb = 1; cb <= 2; cb <<= 1)
#pragma unroll
            for (int c = 0; c < 4; c++)
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
            for (int c = 0; c < 4; c++)
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
        if (head < p.group) {
            float *dst = p.out + ((static_cast<int64_t>(s) * p.hq + h * p.group + head) * kHeadDim);
#pragma unroll
            for (int c = 0; c < 4; c++) {
                const float f = kRotate ? kHadamardC : 1.0f;
                const float4 val = make_float4(v[e][c][0] * f, v[e][c][1] * f, v[e][c][2] * f,
                                               v[e][c][3] * f);
                *reinterpret_cast<float4 *>(dst + 32 * c + 4 * g) = val;
            }
        }
    }
}


// Store this warp's (m, l, o) for one piece into workspace slot `slot`.
__device__ __forceinline__ void store_partial(float *slot, int lane, const WarpState &st)
{
    const int g = lane >> 2, t = lane & 3;
    float4 *so = reinterpret_cast<float4 *>(slot);
#pragma unroll
    for (int i = 0; i < 8; i++)
        so[i * 32 + lane] = make_float4(st.o[i][0], st.o[i][1], st.o[i][2], st.o[i][3]);
    if (g == 0) {
        slot[1024 + 2 * t] = st.m[0];
        slot[1024 + 2 * t + 1] = st.m[1];
        slot[1032 + 2 * t] = st.l[0];
        slot[1032 + 2 * t + 1] = st.l[1];
    }
}

__device__ __forceinline__ void load_partial(const float *slot, int lane, float bm[2], float bl[2],
                                             float4 bo[8])
{
    const int t = lane & 3;
    const float4 *so = reinterpret_cast<const float4 *>(slot);
#pragma unroll
    for (int i = 0; i < 8; i++)
        bo[i] = so[i * 32 + lane];
    bm[0] = slot[1024 + 2 * t];
    bm[1] = slot[1024 + 2 * t + 1];
    bl[0] = slot[1032 + 2 * t];
    bl[1] = slot[1032 + 2 * t + 1];
}

// One elected lane of the (converged) warp arms the stage's mbarrier with the page's bytes and
// queues the 2-D tensor copy of its code rows and the 1-D bulk copy of its scales; no branch.
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
                 "r"(kTxBytes), "r"(0), "r"(static_cast<uint32_t>(kScaleBytes))
                 : "memory");
}

template <bool kRotate>
__global__ void __launch_bounds__(kThreads, 4)
    paged_decode_kernel(const __grid_constant__ CUtensorMap tmap, const DecodeParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int S = p.num_seqs;
    int32_t *pre = reinterpret_cast<int32_t *>(smem + smem_prefix_offset(p.group));
    volatile int32_t *flags = reinterpret_cast<volatile int32_t *>(smem + kSmemFlags);

    // ---- 1. pages per sequence, the plan, zero outputs of empty sequences ------------------
    scan_pages(p, pre, flags, blockIdx.x == 0);
    pdl_launch_dependents();   // the merge kernel may start its own prologue
    for (int s = blockIdx.x; s < S; s += gridDim.x) {
        if (pre[s + 1] == pre[s]) {
            float4 *dst = reinterpret_cast<float4 *>(p.out + static_cast<int64_t>(s) * p.hq * kHeadDim);
            for (int i = tid; i < p.hq * kHeadDim / 4; i += kThreads)
                dst[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        }
    }
    Plan plan;
    plan.init(pre, S, p.hkv, p.total_warps);
    const int64_t u = static_cast<int64_t>(blockIdx.x) * kWarps + warp;
    if (plan.P == 0 || u >= plan.W)
        return;
    const int64_t F0 = plan.begin(u), F1 = plan.begin(u + 1);
    if (F0 >= F1)
        return;
    const int n_w = static_cast<int>(F1 - F0);
    const int64_t hkv = p.hkv;

    // ---- 2. this warp's copy ring ---------------------------------------------------------------
    const uint32_t code0 = smem_u32(smem + kSmemCodes) + warp * kStages * kCodeBytes;
    const uint32_t scale0 = smem_u32(smem + kSmemScales) + warp * kStages * kScaleBytes;
    const uint32_t qbuf = smem_u32(smem + kSmemQ) + warp * q_bytes(p.group);
    const uint32_t bar0 = smem_u32(smem + kSmemBars) + warp * (kStages + 1) * 8;
    const uint32_t qbar = bar0 + kStages * 8;
    if (lane == 0)
        for (int i = 0; i <= kStages; i++)
            mbar_init(bar0 + 8 * i, 1);
    mbar_init_fence();
    __syncwarp();

    // tensor-map row (page * Hkv + h) * 32 of page m of this warp's run
    auto lookup = [&](int m) -> int32_t {
        if (m >= n_w)
            return 0;
        const int64_t pos = F0 + m;
        const int s = find_seq(pre, S, pos, hkv);
        const int32_t n_s = pre[s + 1] - pre[s];
        const int64_t rel = pos - hkv * pre[s];
        const int h = static_cast<int>(rel / n_s);
        const int i = static_cast<int>(rel - static_cast<int64_t>(h) * n_s);
        int32_t page = p.block_table[static_cast<int64_t>(s) * p.max_blocks + i];
        if (page < 0 || page >= p.num_pages) {
            set_status(p.status, SAW_DEV_BAD_PAGE);
            page = 0;
        }
        return (page * p.hkv + h) * 32;
    };
    // queue the raw queries of (s, h) into the warp's query buffer
    auto issue_query = [&](int s, int h) {
        if (lane == 0) {
            const uint32_t bytes = static_cast<uint32_t>(p.group) * kHeadDim * 2;
            mbar_arrive_expect_tx(qbar, bytes);
            bulk_g2s(qbuf, p.q + (static_cast<int64_t>(s) * p.hq + static_cast<int64_t>(h) * p.group) * kHeadDim,
                     bytes, qbar);
        }
    };

    pdl_wait();   // the cache may be written by the kernel this one depends on

    // Lanes hold the tensor-map rows of pages [look_base, look_base + 32) of the run in look_a
    // and of the 32 after them in look_b, whose block-table reads are thus in flight 32 pages
    // ahead of their use.
    int32_t look_a = lookup(lane), look_b = lookup(32 + lane);
    int look_base = 0;
    int issued = 0;        // pages queued so far (pages are queued in order)
    bool aborted = false;  // a wait gave up: stop queueing and computing
    int drain_from = 0;    // first page whose copy may still be in flight after an abort
    // queue page `issued` of the run into ring stage issued % kStages (warp-uniform call)
    auto issue_next = [&]() {
        const int j = issued++;
        if (j >= look_base + 32) {
            look_base += 32;
            look_a = look_b;
            look_b = lookup(look_base + 32 + lane);
        }
        const int32_t row = __shfl_sync(0xFFFFFFFFu, look_a, j & 31);
        const int stg = j & (kStages - 1);
        copy_page_elected(bar0 + 8 * stg, code0 + stg * kCodeBytes, &tmap, row,
                          scale0 + stg * kScaleBytes, p.scales + static_cast<int64_t>(row) * 4);
    };

    // first piece's segment and its query
    int s = find_seq(pre, S, F0, hkv);
    int h = static_cast<int>((F0 - hkv * pre[s]) / (pre[s + 1] - pre[s]));
    issue_query(s, h);
    while (issued < kStages - 1 && issued < n_w)
        issue_next();

    WarpState st;
    uint32_t bq[8][2];
    float sq[2];
    // Page m of the run: queue the page kStages - 1 ahead into the stage page m - 1 used, wait
    // for page m and attend over its first `valid` tokens (kMask) or all of them.
    auto step = [&](auto mask_tag, int m, int valid) {
        if (issued < n_w && !aborted)
            issue_next();
        const int stg = m & (kStages - 1);
        const uint32_t phase = (static_cast<uint32_t>(m) / kStages) & 1u;
        const bool ok = !aborted && mbar_wait_bounded(bar0 + 8 * stg, phase, kWaitLimitNs);
        if (__all_sync(0xFFFFFFFFu, ok)) {
            process_page<decltype(mask_tag)::value>(code0 + stg * kCodeBytes, scale0 + stg * kScaleBytes,
                                                    valid, bq, sq, lane, st);
        } else if (!aborted) {
            if (lane == 0)
                set_status(p.status, SAW_DEV_WAIT_TIMEOUT);
            drain_from = m;
            aborted = true;
        }
        __syncwarp();
    };

    // ---- 3. pieces ------------------------------------------------------------------------------
    int m = 0;
    uint32_t qphase = 0;
    int64_t pos = F0;
    while (pos < F1) {
        const int32_t n_s = pre[s + 1] - pre[s];
        const int64_t seg_start = hkv * pre[s] + static_cast<int64_t>(h) * n_s;
        const int64_t seg_end = seg_start + n_s;
        const bool ends_segment = seg_end <= F1;
        const int m_end = static_cast<int>((ends_segment ? seg_end : F1) - F0);

        // this piece's query: wait for its copy, build the fragments, then queue the next one
        const bool qok = !aborted && mbar_wait_bounded(qbar, qphase, kWaitLimitNs);
        if (!__all_sync(0xFFFFFFFFu, qok) && !aborted) {
            if (lane == 0)
                set_status(p.status, SAW_DEV_WAIT_TIMEOUT);
            drain_from = m;
            aborted = true;
        }
        qphase ^= 1;
        load_query<kRotate>(p, qbuf, g, t, bq, sq);
        __syncwarp();
        int s_next = s, h_next = h;
        if (m_end < n_w) {
            if (++h_next == p.hkv) {
                h_next = 0;
                do {
                    s_next++;
                } while (pre[s_next + 1] == pre[s_next]);
            }
            if (!aborted)
                issue_query(s_next, h_next);
        }

        // all pages but a segment's last are full
        state_reset(st);
        const int m_full = ends_segment ? m_end - 1 : m_end;
        for (; m < m_full; m++)
            step(std::false_type(), m, kPageSize);
        if (ends_segment) {
            step(std::true_type(), m, p.seq_lens[s] - kPageSize * (n_s - 1));
            m++;
        }

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
        for (int i2 = 0; i2 < 8; i2++) {
            st.o[i2][0] = fmaf(st.o[i2][0], kLowNibble, st.z[0]);
            st.o[i2][1] = fmaf(st.o[i2][1], kLowNibble, st.z[1]);
            st.o[i2][2] = fmaf(st.o[i2][2], kHighNibble, st.z[0]);
            st.o[i2][3] = fmaf(st.o[i2][3], kHighNibble, st.z[1]);
        }
        if (seg_start >= F0 && ends_segment) {
            finalize<kRotate>(p, s, h, lane, st.o, st.l);
        } else {
            const int64_t seg = static_cast<int64_t>(s) * hkv + h;
            store_partial(p.partials + (seg + u) * kSlotFloats, lane, st);
        }
        pos = F0 + m_end;
        s = s_next;
        h = h_next;
    }

    // ---- 4. after an abort, let queued copies land before the shared memory is released ----
    if (aborted) {
        for (int k = drain_from; k < issued; k++)
            mbar_wait_bounded(bar0 + 8 * (k & (kStages - 1)), (static_cast<uint32_t>(k) / kStages) & 1u,
                              kWaitLimitNs / 10);
        mbar_wait_bounded(qbar, qphase, kWaitLimitNs / 10);
    }
}

// Combine the pieces of every segment that was split across warps: slot segment + u holds
// warp u's (m, l, o); the warps of a block fold disjoint subsets in a fixed order, then warp 0
// folds the other warps' results in warp order and writes the rotated-back output, so the
// result does not depend on timing.
template <bool kRotate>
__global__ void __launch_bounds__(kMergeThreads)
    paged_decode_merge_kernel(const DecodeParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 15) & ~uintptr_t(15));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int32_t *pre = reinterpret_cast<int32_t *>(smem + kMergeSmemPrefix);
    volatile int32_t *flags = reinterpret_cast<volatile int32_t *>(smem + kMergeSmemFlags);
    float *slots = reinterpret_cast<float *>(smem + kMergeSmemSlots);

    scan_pages(p, pre, flags, false);
    Plan plan;
    plan.init(pre, p.num_seqs, p.hkv, p.total_warps);
    pdl_wait();   // the decode kernel's partials
    if (plan.P == 0)
        return;
    const int64_t hkv = p.hkv;
    const int64_t J = static_cast<int64_t>(p.num_seqs) * hkv;
    for (int64_t seg = blockIdx.x; seg < J; seg += gridDim.x) {
        const int s = static_cast<int>(seg / hkv), h = static_cast<int>(seg - s * hkv);
        const int32_t n_s = pre[s + 1] - pre[s];
        if (n_s == 0)
            continue;
        const int64_t u_lo = plan.warp_of_cost(plan.page_cost(s, h, 0));
        const int64_t u_hi = plan.warp_of_cost(plan.page_cost(s, h, n_s - 1));
        if (u_lo == u_hi)
            continue;
        WarpState st;
        state_reset(st);
        // each warp folds every kMergeWarps-th partial; two loads in flight per step
        int64_t uu = u_lo + warp;
        for (; uu + kMergeWarps <= u_hi; uu += 2 * kMergeWarps) {
            float bm0[2], bl0[2], bm1[2], bl1[2];
            float4 bo0[8], bo1[8];
            load_partial(p.partials + (seg + uu) * kSlotFloats, lane, bm0, bl0, bo0);
            load_partial(p.partials + (seg + uu + kMergeWarps) * kSlotFloats, lane, bm1, bl1, bo1);
            merge_into(st.m, st.l, st.o, bm0, bl0, bo0);
            merge_into(st.m, st.l, st.o, bm1, bl1, bo1);
        }
        if (uu <= u_hi) {
            float bm[2], bl[2];
            float4 bo[8];
            load_partial(p.partials + (seg + uu) * kSlotFloats, lane, bm, bl, bo);
            merge_into(st.m, st.l, st.o, bm, bl, bo);
        }
        if (warp > 0)
            store_partial(slots + (warp - 1) * kSlotFloats, lane, st);
        __syncthreads();
        if (warp == 0) {
            for (int w = 1; w < kMergeWarps; w++) {
                float bm[2], bl[2];
                float4 bo[8];
                load_partial(slots + (w - 1) * kSlotFloats, lane, bm, bl, bo);
                merge_into(st.m, st.l, st.o, bm, bl, bo);
            }
            finalize<kRotate>(p, s, h, lane, st.o, st.l);
        }
        __syncthreads();
    }
}

}  // namespace

namespace {

struct LaunchShape {
    int sms = 0;
    int occ = 0;
};

// Multiprocessor count and decode-kernel occupancy for the current device and smem size.  The
// dynamic shared-memory attributes of both kernels (both variants) are raised per device as
// needed; everything is cached per device.
cudaError_t launch_shape(size_t smem, size_t merge_smem, LaunchShape &out)
{
    constexpr int kMaxDevices = 64;
    struct DevState {
        int sms = 0;
        size_t decode_attr = 0, merge_attr = 0;
        size_t occ_smem = 0;
        int occ = 0;
    };
    static std::mutex mu;
    static DevState st[kMaxDevices];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= kMaxDevices)
        return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    DevState &d = st[dev];
    if (d.sms == 0 && (e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    if (smem > d.decode_attr) {
        for (int r = 0; r < 2 && e == cudaSuccess; r++)
            e = cudaFuncSetAttribute(r ? paged_decode_kernel<true> : paged_decode_kernel<false>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess)
            return e;
        d.decode_attr = smem;
    }
    if (merge_smem > d.merge_attr) {
        for (int r = 0; r < 2 && e == cudaSuccess; r++)
            e = cudaFuncSetAttribute(r ? paged_decode_merge_kernel<true> : paged_decode_merge_kernel<false>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(merge_smem));
        if (e != cudaSuccess)
            return e;
        d.merge_attr = merge_smem;
    }
    if (smem != d.occ_smem) {
        int occ = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, paged_decode_kernel<true>, kThreads, smem);
        if (e != cudaSuccess)
            return e;
        if (occ <= 0)
            return cudaErrorInvalidConfiguration;
        d.occ = occ;
        d.occ_smem = smem;
    }
    out.sms = d.sms;
    out.occ = d.occ;
    return cudaSuccess;
}

}  // namespace

size_t decode_workspace_bytes(int32_t num_kv_heads, int32_t num_q_heads, int32_t num_seqs)
{
    if (num_kv_heads <= 0 || num_q_heads <= 0 || num_seqs < 0 || num_q_heads % num_kv_heads)
        return 0;
    LaunchShape ls;
    if (launch_shape(decode_smem_bytes(num_seqs, num_q_heads / num_kv_heads), merge_smem_bytes(num_seqs), ls) != cudaSuccess)
        return 0;
    const size_t warps = static_cast<size_t>(ls.sms) * ls.occ * kWarps;
    const size_t segs = static_cast<size_t>(num_seqs) * num_kv_heads;
    return (warps + segs) * kSlotFloats * sizeof(float);
}

cudaError_t launch_paged_decode(const DecodeArgs &a, cudaStream_t stream, bool programmatic)
{
    static thread_local struct {
        const void *base = nullptr;
        int64_t rows = 0;
        CUtensorMap map;
    } cache;
    const int64_t rows = a.num_pages * a.num_kv_heads * 32;
    if (cache.base != a.kv_pages || cache.rows != rows) {
        auto encode = tensor_map_encoder();
        if (encode == nullptr)
            return cudaErrorNotSupported;
        const cuuint64_t dims[2] = {64, static_cast<cuuint64_t>(rows)};
        const cuuint64_t strides[1] = {64};
        const cuuint32_t box[2] = {64, 32};
        const cuuint32_t estr[2] = {1, 1};
        CUresult r = encode(&cache.map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                            const_cast<uint8_t *>(a.kv_pages), dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) {
            cache.base = nullptr;
            return cudaErrorInvalidValue;
        }
        cache.base = a.kv_pages;
        cache.rows = rows;
    }

    const size_t smem = decode_smem_bytes(a.num_seqs, a.num_q_heads / a.num_kv_heads);
    const size_t msmem = merge_smem_bytes(a.num_seqs);
    LaunchShape ls;
    cudaError_t e = launch_shape(smem, msmem, ls);
    if (e != cudaSuccess)
        return e;

    DecodeParams p;
    p.q = static_cast<const uint16_t *>(a.q);
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
    p.total_warps = ls.sms * ls.occ * kWarps;
    // q carries sm_scale * log2(e), and 1/sqrt(128) of the (unnormalised) query butterfly
    p.q_mult = static_cast<float>((a.rotate ? static_cast<double>(kHadamardC) : 1.0) * a.sm_scale *
                                  1.4426950408889634);

    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(ls.sms * ls.occ));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = programmatic ? 1 : 0;
    e = cudaLaunchKernelEx(&cfg, a.rotate ? paged_decode_kernel<true> : paged_decode_kernel<false>,
                           cache.map, p);
    if (e != cudaSuccess)
        return e;

    const int64_t segs = static_cast<int64_t>(a.num_seqs) * a.num_kv_heads;
    cudaLaunchConfig_t mcfg = cfg;
    mcfg.gridDim = dim3(static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>(segs, 8 * ls.sms))));
    mcfg.blockDim = dim3(kMergeThreads);
    mcfg.dynamicSmemBytes = msmem;
    mcfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&mcfg, a.rotate ? paged_decode_merge_kernel<true> : paged_decode_merge_kernel<false>, p);
    if (e != cudaSuccess)
        return e;
    return cudaGetLastError();
}

}  // namespace saw
