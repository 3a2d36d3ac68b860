// decode_common.cuh -- the parts of the paged decode kernels that do not depend on the page
// format: the cost-balanced split of all (sequence, kv head) segments into warp runs, the
// per-warp online-softmax state, split-K partial slots in the workspace and the merge kernel
// that folds a split segment's partials in a fixed order.
//
// A segment (sequence s, kv head h, query sub-group: G > 8 query heads of one kv head are split
// into ceil(G / 8) sub-groups, each its own segment reading the same pages, because the MMA
// tiles stack at most 8 heads) of n = ceil(len_s / 16) pages costs n + kKappa in a cost
// space where all segments lie end to end (sequence-major, then kv head); that range is cut
// into equal slices, one per warp of a persistent grid, and a warp owns the pages whose cost
// falls in its slice.  The pieces of a segment split across warps go to workspace slot
// segment + warp (unique, because both orders are monotone).
#pragma once

#include <cstdint>
#include <cudaTypedefs.h>
#include <mutex>
#include <type_traits>

#include "saw_device.cuh"

namespace saw {
namespace decode {

constexpr int kSlotFloats = 32 * 32 + 16;               // O (lane layout) + m[8] + l[8]
constexpr int64_t kKappa = 2;                           // per-segment cost, in pages
constexpr uint64_t kWaitLimitNs = 1000000000ull;        // give up a copy wait after 1 s
constexpr int kMergeWarps = 4;
constexpr int kMergeThreads = 32 * kMergeWarps;
// merge kernel shared memory: per-warp partials, flags, then the sequence prefix
constexpr int kMergeSmemSlots = 0;
constexpr int kMergeSmemFlags = kMergeSmemSlots + (kMergeWarps - 1) * kSlotFloats * 4;
constexpr int kMergeSmemPrefix = kMergeSmemFlags + 64;

inline size_t merge_smem_bytes(int32_t num_seqs)
{
    return kMergeSmemPrefix + 4 * (static_cast<size_t>(num_seqs) + 1);
}

// Query sub-groups of G = hq / hkv query heads per kv head (see DecodeParams).
struct SubGroups {
    int32_t nsub, gsub, hseg;
};
inline SubGroups sub_groups(int32_t num_kv_heads, int32_t num_q_heads)
{
    const int32_t G = num_q_heads / num_kv_heads;
    const int32_t nsub = (G + 7) / 8;
    return {nsub, (G + nsub - 1) / nsub, num_kv_heads * nsub};
}

// Workspace of a decode grid of `warps` warps over num_seqs * segs_per_seq segments.
inline size_t workspace_bytes_for(size_t warps, int32_t num_seqs, int32_t segs_per_seq)
{
    return (warps + static_cast<size_t>(num_seqs) * segs_per_seq) * kSlotFloats * sizeof(float);
}

struct DecodeParams {
    const uint16_t *q;
    const uint8_t *scales;       // INT4 cache: bytes, 128 B per (page, kv head); else unused
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
    int32_t group;               // G = hq / hkv
    int32_t nsub;                // query sub-groups per kv head: ceil(G / 8) (MMA tiles are 8 wide)
    int32_t gsub;                // query heads per sub-group: ceil(G / nsub) <= 8
    int32_t hseg;                // segments per sequence: hkv * nsub
    int32_t total_warps;         // warps of the decode grid (the plan's slice count bound)
    float q_mult;                // the factor the kernel applies to q (or to the logits)

    // Segment hv of a sequence is query sub-group hv % nsub of kv head hv / nsub.
    __device__ int kv_head(int hv) const { return hv / nsub; }
    __device__ int head_base(int hv) const { return (hv / nsub) * group + (hv % nsub) * gsub; }
    __device__ int head_count(int hv) const { return min(gsub, group - (hv % nsub) * gsub); }
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
__device__ inline void scan_pages(const DecodeParams &p, int32_t *pre, volatile int32_t *flags,
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

// Per-warp running state of one piece: o holds O^T (128 value rows x 8 stacked query heads) as
// eight m16n8 accumulator tiles, thread (g, t) holding heads 2t and 2t + 1 of rows g and g + 8
// of each tile (which value dimension d a row is, is up to the kernel and its finalize step);
// m, l: running max (log2 domain) and sum of the two heads; z: the kernel's zero-point sum.
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

// Online softmax over one page: s holds the logits (log2 domain) of tokens g, g + 8 for heads
// 2t, 2t + 1 (-inf for masked tokens); returns p = 2^(s - m) with m the running max after the
// page, and rescales o, l and z when m grows.  The running max only changes when some logit of
// the page exceeds it, so the cross-lane reduction runs only then (rare once a piece is a few
// pages long); the result equals reducing every page.
__device__ __forceinline__ void softmax_update(const float s[4], WarpState &st, float pr[4])
{
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
    pr[0] = ex2_approx(s[0] - st.m[0]);
    pr[1] = ex2_approx(s[1] - st.m[1]);
    pr[2] = ex2_approx(s[2] - st.m[0]);
    pr[3] = ex2_approx(s[3] - st.m[1]);
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

// Combine the pieces of every segment that was split across warps: slot segment + u holds
// warp u's (m, l, o); the warps of a block fold disjoint subsets in a fixed order, then warp 0
// folds the other warps' results in warp order and writes the output through the page format's
// finalize step, so the result does not depend on timing.
template <class Fmt>
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
    plan.init(pre, p.num_seqs, p.hseg, p.total_warps);
    pdl_wait();   // the decode kernel's partials
    if (plan.P == 0)
        return;
    const int64_t hkv = p.hseg;
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
            Fmt::finalize(p, s, h, lane, st.o, st.l);
        }
        __syncthreads();
    }
}

// ---- the decode kernel, generic over the page format ----------------------------------------
//
// A page format Fmt supplies:
//   kWarps, kStages (a power of two), kMinBlocks   warps per CTA, ring stages per warp, and the
//                                                  CTAs per SM the launch bounds ask for;
//   kRingBytes                                     the rings of all warps, from a 1024-byte
//                                                  aligned base;
//   kRowsPerPage                                   tensor-map rows of one (page, kv head);
//   Ring ring(base, warp)                          this warp's stage addresses;
//   issue(ring, stg, bar, tmap, row, p)            queue a page's copies into stage stg,
//                                                  completing on mbarrier bar (one elected lane);
//   Query; load_query(p, qbuf, n, lane, q)         per-piece query fragments from the raw bf16
//                                                  queries of the segment's n <= 8 heads in
//                                                  shared memory;
//   page<kMask>(ring, stg, valid, q, lane, st)     attend over one staged page (first `valid`
//                                                  tokens when kMask);
//   piece_end(st)                                  reductions and corrections after a piece;
//   finalize(p, s, hv, lane, o, l)                 write the output of segment hv of sequence s
//                                                  (also the merge kernel's output step).
// Shared memory: rings, then per warp (kStages + 1) mbarriers (the last for the query), 64 bytes
// of flags, the per-warp query buffers (G * 256 bytes each) and the sequence page prefix.

__host__ __device__ constexpr int query_bytes(int group) { return group * kHeadDim * 2; }
template <class Fmt>
__host__ __device__ constexpr int smem_bars_offset() { return Fmt::kRingBytes; }
template <class Fmt>
__host__ __device__ constexpr int smem_flags_offset()
{
    return Fmt::kRingBytes + Fmt::kWarps * (Fmt::kStages + 1) * 8;
}
template <class Fmt>
__host__ __device__ constexpr int smem_q_offset() { return smem_flags_offset<Fmt>() + 64; }
template <class Fmt>
__host__ __device__ constexpr int smem_prefix_offset(int group)
{
    return smem_q_offset<Fmt>() + Fmt::kWarps * query_bytes(group);
}
template <class Fmt>
inline size_t decode_smem_bytes(int32_t num_seqs, int32_t group)
{
    return 1024 + smem_prefix_offset<Fmt>(group) + 4 * (static_cast<size_t>(num_seqs) + 1);
}

template <class Fmt>
__global__ void __launch_bounds__(32 * Fmt::kWarps, Fmt::kMinBlocks)
    paged_decode_kernel(const __grid_constant__ CUtensorMap tmap, const DecodeParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int S = p.num_seqs;
    int32_t *pre = reinterpret_cast<int32_t *>(smem + smem_prefix_offset<Fmt>(p.gsub));
    volatile int32_t *flags = reinterpret_cast<volatile int32_t *>(smem + smem_flags_offset<Fmt>());

    // ---- 1. pages per sequence, the plan, zero outputs of empty sequences ------------------
    scan_pages(p, pre, flags, blockIdx.x == 0);
    pdl_launch_dependents();   // the merge kernel may start its own prologue
    for (int s = blockIdx.x; s < S; s += gridDim.x) {
        if (pre[s + 1] == pre[s]) {
            float4 *dst = reinterpret_cast<float4 *>(p.out + static_cast<int64_t>(s) * p.hq * kHeadDim);
            for (int i = tid; i < p.hq * kHeadDim / 4; i += 32 * Fmt::kWarps)
                dst[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        }
    }
    Plan plan;
    plan.init(pre, S, p.hseg, p.total_warps);
    const int64_t u = static_cast<int64_t>(blockIdx.x) * Fmt::kWarps + warp;
    if (plan.P == 0 || u >= plan.W)
        return;
    const int64_t F0 = plan.begin(u), F1 = plan.begin(u + 1);
    if (F0 >= F1)
        return;
    const int n_w = static_cast<int>(F1 - F0);
    const int64_t hkv = p.hseg;   // segments per sequence

    // ---- 2. this warp's copy ring ---------------------------------------------------------------
    constexpr int kStages = Fmt::kStages;
    const typename Fmt::Ring ring = Fmt::ring(smem_u32(smem), warp);
    const uint32_t qbuf = smem_u32(smem + smem_q_offset<Fmt>()) + warp * query_bytes(p.gsub);
    const uint32_t bar0 = smem_u32(smem + smem_bars_offset<Fmt>()) + warp * (kStages + 1) * 8;
    const uint32_t qbar = bar0 + kStages * 8;
    if (lane == 0)
        for (int i = 0; i <= kStages; i++)
            mbar_init(bar0 + 8 * i, 1);
    mbar_init_fence();
    __syncwarp();

    // tensor-map row (page * Hkv + h) * kRowsPerPage of page m of this warp's run
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
        return (page * p.hkv + p.kv_head(h)) * Fmt::kRowsPerPage;
    };
    // queue the raw queries of (s, h) into the warp's query buffer
    auto issue_query = [&](int s, int h) {
        if (lane == 0) {
            const uint32_t bytes = static_cast<uint32_t>(p.head_count(h)) * kHeadDim * 2;
            mbar_arrive_expect_tx(qbar, bytes);
            bulk_g2s(qbuf, p.q + (static_cast<int64_t>(s) * p.hq + p.head_base(h)) * kHeadDim,
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
        Fmt::issue(ring, stg, bar0 + 8 * stg, &tmap, row, p);
    };

    // first piece's segment and its query
    int s = find_seq(pre, S, F0, hkv);
    int h = static_cast<int>((F0 - hkv * pre[s]) / (pre[s + 1] - pre[s]));
    issue_query(s, h);
    while (issued < kStages - 1 && issued < n_w)
        issue_next();

    WarpState st;
    typename Fmt::Query qf;
    // Page m of the run: queue the page kStages - 1 ahead into the stage page m - 1 used, wait
    // for page m and attend over its first `valid` tokens (kMask) or all of them.
    auto step = [&](auto mask_tag, int m, int valid) {
        if (issued < n_w && !aborted)
            issue_next();
        const int stg = m & (kStages - 1);
        const uint32_t phase = (static_cast<uint32_t>(m) / kStages) & 1u;
        const bool ok = !aborted && mbar_wait_bounded(bar0 + 8 * stg, phase, kWaitLimitNs);
        if (__all_sync(0xFFFFFFFFu, ok)) {
            Fmt::template page<decltype(mask_tag)::value>(ring, stg, valid, qf, lane, st);
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
        Fmt::load_query(p, qbuf, p.head_count(h), lane, qf);
        __syncwarp();
        int s_next = s, h_next = h;
        if (m_end < n_w) {
            if (++h_next == p.hseg) {
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

        Fmt::piece_end(st);
        if (seg_start >= F0 && ends_segment) {
            Fmt::finalize(p, s, h, lane, st.o, st.l);
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

struct LaunchShape {
    int sms = 0;
    int occ = 0;
};

// Multiprocessor count and occupancy of one family of decode kernels (both variants of the
// decode and of its merge kernel) for the current device and dynamic shared-memory sizes.  The
// shared-memory attributes are raised per device as needed; everything is cached per device
// in `cache`.
struct ShapeCache {
    static constexpr int kMaxDevices = 64;
    struct Dev {
        int sms = 0;
        size_t decode_attr = 0, merge_attr = 0;
        size_t occ_smem = 0;
        int occ = 0;
    };
    std::mutex mu;
    Dev dev[kMaxDevices];
};

inline cudaError_t launch_shape(ShapeCache &cache, const void *const decode_kernels[2],
                                const void *const merge_kernels[2], int threads, size_t smem,
                                size_t merge_smem, LaunchShape &out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= ShapeCache::kMaxDevices)
        return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(cache.mu);
    ShapeCache::Dev &d = cache.dev[dev];
    if (d.sms == 0 && (e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    if (smem > d.decode_attr) {
        for (int r = 0; r < 2 && e == cudaSuccess; r++)
            e = cudaFuncSetAttribute(decode_kernels[r], cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(smem));
        if (e != cudaSuccess)
            return e;
        d.decode_attr = smem;
    }
    if (merge_smem > d.merge_attr) {
        for (int r = 0; r < 2 && e == cudaSuccess; r++)
            e = cudaFuncSetAttribute(merge_kernels[r], cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(merge_smem));
        if (e != cudaSuccess)
            return e;
        d.merge_attr = merge_smem;
    }
    if (smem != d.occ_smem) {
        int occ = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, decode_kernels[0], threads, smem);
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

}  // namespace decode
}  // namespace saw
