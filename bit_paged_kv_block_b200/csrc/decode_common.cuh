// decode_common.cuh -- the parts of the paged attention kernels that do not depend on the page
// format: the cost-balanced split of all segments into warp runs, the per-warp online-softmax
// state, split-K partial slots in the workspace, the kernel body (generic over the page format)
// and the merge kernel that folds a split segment's partials in a fixed order.
//
// Queries.  Sequence s has C_s query tokens: C_s = 1 for decode (query row s), or
// q_start[s + 1] - q_start[s] for chunked prefill (query rows q_start[s] ..), the last C_s of
// its L_s cached tokens.  Query token i sees cache tokens 0 .. L_s - C_s + i (causal; decode:
// all L_s).  A query row of kv head h is a (query token, query head of h) pair, token-major:
// row r is token r / G, head h G + r % G.
//
// Segments.  The C_s G rows of (sequence s, kv head h) are cut into blocks of at most 8 rows
// (the MMA tiles stack 8 query columns); a segment is (s, h, block) and reads all
// n_s = ceil(L_s / 16) pages of s, the rows' causal limits masking what each may not see.
// Segment j of sequence s is kv head j / nb_s, block j % nb_s.  A segment of n pages costs
// n + kKappa in a cost space where all segments lie end to end (sequence-major); that range
// is cut into equal slices, one per warp of a persistent grid, and a warp owns the pages whose
// cost falls in its slice.  The pieces of a segment split across warps go to workspace slot
// segment + warp (unique, because both orders are monotone).
#pragma once

#include <cstdint>
#include <cudaTypedefs.h>
#include <mutex>
#include <type_traits>

#include "saw_device.cuh"

namespace saw {
namespace decode {

// workspace slot of one piece's partial: O in lane layout (kTiles x 32 float4), then m[8], l[8]
template <int kTiles>
__host__ __device__ constexpr int slot_floats() { return kTiles * 128 + 16; }
constexpr int64_t kKappa = 2;                           // per-segment cost, in pages
constexpr uint64_t kWaitLimitNs = 1000000000ull;        // give up a copy wait after 1 s
constexpr int kRowsPerBlock = 8;                        // query rows (MMA columns) per segment
constexpr int kMergeWarps = 4;
constexpr int kMergeThreads = 32 * kMergeWarps;
// a launch with at most one segment per SM (few, long sequences: each split over tens of warps)
// folds each segment's partials with this many warps
constexpr int kMergeWarpsWide = 8;
// ... and a launch with more than 4 segments per SM (many short sequences) with this many
constexpr int kMergeWarpsNarrow = 1;
// per-sequence shared-memory tables (fpre int64, spre int32, npg int32, nbk int32) + ends
constexpr int kSeqTableBytes = 20;
// merge kernel shared memory: per-warp partials, flags, then the sequence tables
template <int kTiles, int kMW = kMergeWarps>
__host__ __device__ constexpr int merge_smem_flags() { return (kMW - 1) * slot_floats<kTiles>() * 4; }
// the flags hold scan_sequences' two int64 partial sums per warp
template <int kTiles, int kMW = kMergeWarps>
__host__ __device__ constexpr int merge_smem_tables() { return merge_smem_flags<kTiles, kMW>() + 16 * kMW; }

inline size_t seq_table_bytes(int32_t num_seqs)
{
    return kSeqTableBytes * (static_cast<size_t>(num_seqs) + 1);
}
template <int kTiles, int kMW = kMergeWarps>
inline size_t merge_smem_bytes(int32_t num_seqs)
{
    return merge_smem_tables<kTiles, kMW>() + seq_table_bytes(num_seqs);
}

// Segments of a launch: decode, num_seqs * hkv * ceil(G / 8); chunked prefill over total_q
// query tokens, at most hkv * (ceil(total_q G / 8) + num_seqs).
inline int64_t max_segments(int32_t num_kv_heads, int32_t num_q_heads, int32_t num_seqs,
                            int64_t total_q, bool prefill)
{
    const int64_t G = num_q_heads / num_kv_heads;
    if (!prefill)
        return static_cast<int64_t>(num_seqs) * num_kv_heads * ((G + kRowsPerBlock - 1) / kRowsPerBlock);
    return num_kv_heads * ((total_q * G + kRowsPerBlock - 1) / kRowsPerBlock + num_seqs);
}

// Rows of each warp's query buffer: a decode block holds at most G rows; a prefill block 8.
inline int32_t query_rows(int32_t num_kv_heads, int32_t num_q_heads, bool prefill)
{
    const int32_t G = num_q_heads / num_kv_heads;
    return prefill || G >= kRowsPerBlock ? kRowsPerBlock : G;
}

// Workspace of a decode grid of `warps` warps over `segments` segments (kTiles output tiles).
template <int kTiles>
inline size_t workspace_bytes_for(size_t warps, int64_t segments)
{
    return (warps + static_cast<size_t>(segments)) * slot_floats<kTiles>() * sizeof(float);
}

struct DecodeParams {
    const uint16_t *q;
    const int32_t *q_start;      // chunked prefill: [S + 1] query-row offsets; decode: null
    const uint8_t *scales;       // INT4 cache: bytes, 128 B per (page, kv head); else unused
    const int32_t *block_table;
    const int32_t *seq_lens;
    float *out;
    float *partials;             // workspace: (total warps + max_segments) slots
    uint32_t *status;
    int64_t num_pages;
    int64_t max_segments;        // segment slots the workspace holds
    int32_t max_blocks;
    int32_t num_seqs;
    int32_t hq;
    int32_t hkv;
    int32_t group;               // G = hq / hkv
    int32_t total_warps;         // warps of the decode grid (the plan's slice count bound)
    int32_t qrows;               // rows of each warp's query buffer: min(8, C G) bound
    float q_mult;                // the factor the kernel applies to q (or to the logits)
    // Full-precision window beside the quantized cache (decode only): win_part 1 attends over
    // the min(L, W) window tokens of each sequence and writes out rows and lse[row] = the log2
    // of the softmax denominator; win_part 2 attends over the max(0, L - W) quantized tokens
    // and merges its result into the out rows part 1 wrote (W = win_sink + win_recent).
    float *lse = nullptr;
    int32_t win_part = 0;
    int32_t win_sink = 0, win_recent = 0;
};

// Tokens this launch attends over in a sequence of seq_lens[s] tokens (a negative length is
// passed through, to be flagged).
__device__ __forceinline__ int attended_len(const DecodeParams &p, int s)
{
    const int L = p.seq_lens[s];
    if (p.win_part == 0 || L < 0)
        return L;
    const int W = p.win_sink + p.win_recent;
    return p.win_part == 1 ? min(L, W) : max(0, L - W);
}

// ---- per-sequence tables and the work plan -----------------------------------------------------

// Shared-memory tables over the sequences: fpre[s] flat pages (segments x pages) before s,
// spre[s] segments before s, npg[s] pages of each segment of s, nbk[s] row blocks per kv head.
struct SeqTables {
    int64_t *fpre;
    int32_t *spre, *npg, *nbk;

    __device__ void bind(uint8_t *base, int S)
    {
        fpre = reinterpret_cast<int64_t *>(base);
        spre = reinterpret_cast<int32_t *>(base + 8 * (S + 1));
        npg = spre + (S + 1);
        nbk = npg + (S + 1);
    }
};

// Query tokens of sequence s (decode: 1) and its first query row.  kPrefill: a chunked
// prefill (q_start given); the decode instantiation has none of the per-row arithmetic.
template <bool kPrefill>
__device__ __forceinline__ int query_tokens(const DecodeParams &p, int s)
{
    return kPrefill ? p.q_start[s + 1] - p.q_start[s] : 1;
}
template <bool kPrefill>
__device__ __forceinline__ int64_t query_row0(const DecodeParams &p, int s)
{
    return kPrefill ? p.q_start[s] : s;
}

// Fill the tables (every thread of the block takes part).  A sequence with an invalid length
// or query count (C > L, or C > 0 with L = 0 in prefill) is flagged and gets no segments; a
// decode sequence of length 0 gets none either (its output row is zeroed).
template <bool kPrefill>
__device__ inline void scan_sequences(const DecodeParams &p, const SeqTables &tb,
                                      volatile int64_t *flags, bool report)
{
    const int S = p.num_seqs, nthreads = blockDim.x, tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    const int per = (S + nthreads - 1) / nthreads;
    const int s0 = tid * per, s1 = min(S, s0 + per);
    int64_t local_pages = 0;
    int32_t local_segs = 0;
    for (int s = s0; s < s1; s++) {
        const int len = attended_len(p, s);
        const int c = query_tokens<kPrefill>(p, s);
        const bool len_ok = len >= 0 && len <= p.max_blocks * kPageSize;
        const bool q_ok = !kPrefill || (c >= 0 && c <= len);
        if (report && !(len_ok && q_ok))
            set_status(p.status, SAW_DEV_BAD_SEQ_LEN);
        const int n = (len_ok && q_ok) ? (len + kPageSize - 1) / kPageSize : 0;
        const int nb = n > 0 ? (c * p.group + kRowsPerBlock - 1) / kRowsPerBlock : 0;
        tb.npg[s] = n;
        tb.nbk[s] = nb;
        local_segs += p.hkv * nb;
        local_pages += static_cast<int64_t>(p.hkv) * nb * n;
    }
    int64_t ip = local_pages;
    int32_t is = local_segs;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int64_t op = __shfl_up_sync(0xFFFFFFFFu, ip, d);
        const int32_t os = __shfl_up_sync(0xFFFFFFFFu, is, d);
        if (lane >= d) {
            ip += op;
            is += os;
        }
    }
    if (lane == 31) {
        flags[2 * warp] = ip;
        flags[2 * warp + 1] = is;
    }
    __syncthreads();
    int64_t bp = 0, bs = 0;
    for (int w = 0; w < warp; w++) {
        bp += flags[2 * w];
        bs += flags[2 * w + 1];
    }
    int64_t rp = bp + ip - local_pages;
    int32_t rs = static_cast<int32_t>(bs + is - local_segs);
    for (int s = s0; s < s1; s++) {
        tb.fpre[s] = rp;
        tb.spre[s] = rs;
        rs += p.hkv * tb.nbk[s];
        rp += static_cast<int64_t>(p.hkv) * tb.nbk[s] * tb.npg[s];
    }
    if (tid == nthreads - 1) {
        tb.fpre[S] = bp + ip;
        tb.spre[S] = static_cast<int32_t>(bs + is);
    }
    __syncthreads();
}

// The cost-space split of the flat page range into warp runs.  Segment j of sequence s spans
// the cost range [cpre(s) + j (n_s + kKappa), + n_s + kKappa) with cpre(s) = fpre[s] +
// kKappa spre[s]; its page i sits at cost cpre(s) + j (n_s + kKappa) + kKappa + i.  Warp u owns
// the cost range [b(u), b(u + 1)) with b(u) = u q + min(u, r), q = PT / W, r = PT % W (slices of
// q or q + 1, never empty because W <= PT), i.e. the pages whose cost falls in it.
struct Plan {
    SeqTables tb;
    int S;
    int64_t P;    // pages
    int64_t PT;   // cost
    int64_t W;    // warps with a slice
    int64_t q, r;

    __device__ void init(const SeqTables &tb_, int S_, int total_warps)
    {
        tb = tb_;
        S = S_;
        P = tb.fpre[S];
        PT = P + kKappa * tb.spre[S];
        W = max(int64_t(1), min(static_cast<int64_t>(total_warps), PT));
        q = PT / W;
        r = PT - q * W;
    }
    __device__ int64_t seq_cost(int s) const { return tb.fpre[s] + kKappa * tb.spre[s]; }
    __device__ int64_t slice_begin(int64_t u) const { return u * q + min(u, r); }
    // the warp whose cost slice holds cost position x (0 <= x < PT)
    __device__ int64_t warp_of_cost(int64_t x) const
    {
        const int64_t big = r * (q + 1);
        return x < big ? x / (q + 1) : r + (x - big) / q;
    }
    // cost position of page i of segment j of sequence s
    __device__ int64_t page_cost(int s, int j, int64_t i) const
    {
        return seq_cost(s) + static_cast<int64_t>(j) * (tb.npg[s] + kKappa) + kKappa + i;
    }
    // the sequence holding flat page pos (0 <= pos < P): the largest s with fpre[s] <= pos
    __device__ int seq_of_flat(int64_t pos) const
    {
        int lo = 0, hi = S;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (tb.fpre[mid] <= pos)
                lo = mid;
            else
                hi = mid;
        }
        return lo;
    }
    // the sequence holding global segment g: the largest s with spre[s] <= g
    __device__ int seq_of_segment(int64_t g) const
    {
        int lo = 0, hi = S;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (tb.spre[mid] <= g)
                lo = mid;
            else
                hi = mid;
        }
        return lo;
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
        const int64_t n = tb.npg[lo];
        const int64_t within = x - seq_cost(lo);
        const int64_t j = within / (n + kKappa);
        const int64_t rr = within - j * (n + kKappa);
        return tb.fpre[lo] + j * n + (rr < kKappa ? 0 : rr - kKappa);
    }
    // first flat page of warp u's run (u in [0, W]; the run of u is [begin(u), begin(u + 1)))
    __device__ int64_t begin(int64_t u) const { return flat_of_cost(slice_begin(u)); }
};

// One segment: sequence s, its segment j = kv head h * nb + row block b.
template <bool kPrefill>
struct Segment {
    int s, j, h, b;
    int n;          // pages
    int c;          // query tokens of the sequence
    int len;        // cached tokens of the sequence
    int row0;       // first row of the block (8 b)
    int nrows;      // rows in the block (1..8)
    int64_t qrow0;  // first query row of the sequence in q / out

    __device__ void init(const DecodeParams &p, const SeqTables &tb, int s_, int j_)
    {
        s = s_;
        j = j_;
        const int nb = tb.nbk[s];
        h = nb == 1 ? j : j / nb;
        b = j - h * nb;
        n = tb.npg[s];
        c = query_tokens<kPrefill>(p, s);
        len = attended_len(p, s);
        row0 = kRowsPerBlock * b;
        nrows = min(kRowsPerBlock, c * p.group - row0);
        qrow0 = query_row0<kPrefill>(p, s);
    }
    // query token and head (within the kv head's group) of block row e; a decode has one
    // token, so no division there
    __device__ int row_token(const DecodeParams &p, int e) const
    {
        return kPrefill ? (row0 + e) / p.group : 0;
    }
    // causal limit of block row e (0..7): the last cache token it sees
    __device__ int limit(const DecodeParams &p, int e) const
    {
        return len - c + row_token(p, e);
    }
    // q / out element offset of block row e (e < nrows) for head dimension d
    __device__ int64_t row_offset(const DecodeParams &p, int e, int d) const
    {
        const int tok = row_token(p, e);
        const int head = row0 + e - tok * p.group;
        return ((qrow0 + tok) * p.hq + h * p.group + head) * d;
    }
    // pages from this index on hold a token some row of the block may not see (or past len)
    __device__ int first_masked_page(const DecodeParams &p) const
    {
        return (limit(p, 0) + 1) / kPageSize;
    }
};

// Validity of one page for the MMA columns a thread holds (block rows 2t and 2t + 1):
// tokens [0, valid) of the page exist (the rest were never written), and column e sees
// tokens [0, col[e]).
struct PageMask {
    int valid;
    int col[2];
};

// The mask of segment page `page` for a thread whose columns see tokens up to lim[0], lim[1]
// of a sequence of len tokens.
__device__ __forceinline__ PageMask page_mask(int len, const int lim[2], int page)
{
    const int base = kPageSize * page;
    PageMask m;
    m.valid = min(kPageSize, max(0, len - base));
#pragma unroll
    for (int e = 0; e < 2; e++)
        m.col[e] = min(m.valid, max(0, lim[e] - base + 1));
    return m;
}

// Per-warp running state of one piece: o holds O^T (D value rows x 8 stacked query columns) as
// kTiles = D / 16 m16n8 accumulator tiles, thread (g, t) holding columns 2t and 2t + 1 of rows g
// and g + 8 of each tile (which value dimension d a row is, is up to the kernel and its finalize
// step); m, l: running max (log2 domain) and sum of the two columns; z: the kernel's zero-point
// sum.
template <int kTiles>
struct WarpState {
    float o[kTiles][4];
    float m[2];
    float l[2];
    float z[2];
};

template <int kTiles>
__device__ __forceinline__ void state_reset(WarpState<kTiles> &st)
{
#pragma unroll
    for (int i = 0; i < kTiles; i++)
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

// Online softmax over one page (kN = 4) or two (kN = 8): s holds the logits (log2 domain) of
// tokens g, g + 8 (then g + 16, g + 24 of the second page) for columns 2t, 2t + 1 (s[k] belongs to
// column k & 1; -inf for masked tokens); returns p = 2^(s - m) with m the running max after the
// page(s), and rescales o, l and z when m grows.  The running max only changes when some logit
// exceeds it, so the cross-lane reduction runs only then (rare once a piece is a few pages long);
// the result equals reducing every page.  kMask: a column may have seen only masked tokens so far
// (m = -inf); its p stay 0 and nothing is rescaled by a NaN.
template <bool kMask, int kTiles, int kN = 4>
__device__ __forceinline__ void softmax_update(const float s[kN], WarpState<kTiles> &st, float pr[kN])
{
    float mx[2] = {fmaxf(s[0], s[2]), fmaxf(s[1], s[3])};
#pragma unroll
    for (int k = 4; k < kN; k += 2) {
        mx[0] = fmaxf(mx[0], s[k]);
        mx[1] = fmaxf(mx[1], s[k + 1]);
    }
    const bool grow = mx[0] > st.m[0] || mx[1] > st.m[1];
    if (__any_sync(0xFFFFFFFFu, grow)) {
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
            alpha[e] = mn == -INFINITY ? 1.0f : ex2_approx(st.m[e] - mn);
            st.m[e] = mn;
            st.l[e] *= alpha[e];
            st.z[e] *= alpha[e];
        }
#pragma unroll
        for (int i = 0; i < kTiles; i++) {
            st.o[i][0] *= alpha[0];
            st.o[i][1] *= alpha[1];
            st.o[i][2] *= alpha[0];
            st.o[i][3] *= alpha[1];
        }
    }
#pragma unroll
    for (int k = 0; k < kN; k++) {
        pr[k] = ex2_approx(s[k] - st.m[k & 1]);
        if (kMask)
            pr[k] = s[k] == -INFINITY ? 0.0f : pr[k];
    }
}

// Fold (m, l, o) partial b (scaled by its own max) into the running partial a.
template <int kTiles>
__device__ __forceinline__ void merge_into(float am[2], float al[2], float (&ao)[kTiles][4],
                                           const float bm[2], const float bl[2],
                                           const float4 (&bo)[kTiles])
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
    for (int i = 0; i < kTiles; i++) {
        ao[i][0] = ao[i][0] * fa[0] + bo[i].x * fb[0];
        ao[i][1] = ao[i][1] * fa[1] + bo[i].y * fb[1];
        ao[i][2] = ao[i][2] * fa[0] + bo[i].z * fb[0];
        ao[i][3] = ao[i][3] * fa[1] + bo[i].w * fb[1];
    }
}

// Store this warp's (m, l, o) for one piece into workspace slot `slot`.
template <int kTiles>
__device__ __forceinline__ void store_partial(float *slot, int lane, const WarpState<kTiles> &st)
{
    const int g = lane >> 2, t = lane & 3;
    constexpr int kM = kTiles * 128;
    float4 *so = reinterpret_cast<float4 *>(slot);
#pragma unroll
    for (int i = 0; i < kTiles; i++)
        so[i * 32 + lane] = make_float4(st.o[i][0], st.o[i][1], st.o[i][2], st.o[i][3]);
    if (g == 0) {
        slot[kM + 2 * t] = st.m[0];
        slot[kM + 2 * t + 1] = st.m[1];
        slot[kM + 8 + 2 * t] = st.l[0];
        slot[kM + 8 + 2 * t + 1] = st.l[1];
    }
}

template <int kTiles>
__device__ __forceinline__ void load_partial(const float *slot, int lane, float bm[2], float bl[2],
                                             float4 (&bo)[kTiles])
{
    const int t = lane & 3;
    constexpr int kM = kTiles * 128;
    const float4 *so = reinterpret_cast<const float4 *>(slot);
#pragma unroll
    for (int i = 0; i < kTiles; i++)
        bo[i] = so[i * 32 + lane];
    bm[0] = slot[kM + 2 * t];
    bm[1] = slot[kM + 2 * t + 1];
    bl[0] = slot[kM + 8 + 2 * t];
    bl[1] = slot[kM + 8 + 2 * t + 1];
}

// Combine the pieces of every segment that was split across warps: slot g + u holds warp u's
// (m, l, o) for global segment g; the warps of a block fold disjoint subsets in a fixed order,
// then warp 0 folds the other warps' results in warp order and writes the output through the
// page format's finalize step, so the result does not depend on timing.
template <class Fmt, bool kPrefill, int kMW = kMergeWarps>
__global__ void __launch_bounds__(32 * kMW)
    paged_decode_merge_kernel(const DecodeParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 15) & ~uintptr_t(15));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    constexpr int kTiles = Fmt::kTiles;
    constexpr int kSlot = slot_floats<kTiles>();
    SeqTables tb;
    tb.bind(smem + merge_smem_tables<kTiles, kMW>(), p.num_seqs);
    volatile int64_t *flags = reinterpret_cast<volatile int64_t *>(smem + merge_smem_flags<kTiles, kMW>());
    float *slots = reinterpret_cast<float *>(smem);

    scan_sequences<kPrefill>(p, tb, flags, false);
    Plan plan;
    plan.init(tb, p.num_seqs, p.total_warps);
    pdl_wait();   // the decode kernel's partials
    if (plan.P == 0 || tb.spre[p.num_seqs] > p.max_segments)
        return;
    const int64_t J = tb.spre[p.num_seqs];
    for (int64_t gseg = blockIdx.x; gseg < J; gseg += gridDim.x) {
        const int s = plan.seq_of_segment(gseg);
        const int j = static_cast<int>(gseg - tb.spre[s]);
        const int32_t n_s = tb.npg[s];
        const int64_t u_lo = plan.warp_of_cost(plan.page_cost(s, j, 0));
        const int64_t u_hi = plan.warp_of_cost(plan.page_cost(s, j, n_s - 1));
        if (u_lo == u_hi)
            continue;
        WarpState<kTiles> st;
        state_reset(st);
        // each warp folds every kMW-th partial; two loads in flight per step
        int64_t uu = u_lo + warp;
        for (; uu + kMW <= u_hi; uu += 2 * kMW) {
            float bm0[2], bl0[2], bm1[2], bl1[2];
            float4 bo0[kTiles], bo1[kTiles];
            load_partial(p.partials + (gseg + uu) * kSlot, lane, bm0, bl0, bo0);
            load_partial(p.partials + (gseg + uu + kMW) * kSlot, lane, bm1, bl1, bo1);
            merge_into(st.m, st.l, st.o, bm0, bl0, bo0);
            merge_into(st.m, st.l, st.o, bm1, bl1, bo1);
        }
        if (uu <= u_hi) {
            float bm[2], bl[2];
            float4 bo[kTiles];
            load_partial(p.partials + (gseg + uu) * kSlot, lane, bm, bl, bo);
            merge_into(st.m, st.l, st.o, bm, bl, bo);
        }
        if (warp > 0)
            store_partial(slots + (warp - 1) * kSlot, lane, st);
        __syncthreads();
        if (warp == 0) {
            for (int w = 1; w < kMW; w++) {
                float bm[2], bl[2];
                float4 bo[kTiles];
                load_partial(slots + (w - 1) * kSlot, lane, bm, bl, bo);
                merge_into(st.m, st.l, st.o, bm, bl, bo);
            }
            Segment<kPrefill> sg;
            sg.init(p, tb, s, j);
            Fmt::finalize(p, sg, lane, st.o, st.m, st.l);
        }
        __syncthreads();
    }
}

// ---- the attention kernel, generic over the page format --------------------------------------
//
// A page format Fmt supplies:
//   kWarps, kStages, kMinBlocks                    warps per CTA, ring stages per warp, and the
//                                                  CTAs per SM the launch bounds ask for;
//   kRingBytes                                     the rings of all warps, from a 1024-byte
//                                                  aligned base;
//   kRowsPerPage                                   tensor-map rows of one (page, kv head);
//   Ring ring(base, warp)                          this warp's stage addresses;
//   issue(ring, stg, bar, tmap, row, p)            queue a page's copies into stage stg,
//                                                  completing on mbarrier bar (one elected lane);
//   Query; load_query(p, qbuf, n, lane, q)         per-piece query fragments from the n <= 8
//                                                  raw bf16 query rows in shared memory;
//   page<kMask>(ring, stg, mask, q, lane, st)      attend over one staged page (PageMask when
//                                                  kMask: never-written tokens, causal limits);
//   kPairs; page2(ring, stg0, stg1, q, lane, st)   whether whole pages go two at a time, and
//                                                  the two-page step (one softmax update);
//   piece_end(st)                                  reductions and corrections after a piece;
//   finalize(p, segment, lane, o, m, l)            write a finished segment's output rows (a
//                                                  template on the segment type)
//                                                  (also the merge kernel's output step).
// Shared memory: rings, then per warp (kStages + 1) mbarriers (the last for the query), 128 bytes
// of flags, the per-warp query buffers (qrows * 256 bytes each) and the sequence tables.

constexpr int kSmemFlagBytes = 128;   // scan_sequences' two int64 partial sums per warp
// bytes of `rows` raw bf16 query rows of a format's head dimension
template <class Fmt>
__host__ __device__ constexpr int query_bytes(int rows) { return rows * Fmt::kDim * 2; }
template <class Fmt>
__host__ __device__ constexpr int smem_bars_offset() { return Fmt::kRingBytes; }
template <class Fmt>
__host__ __device__ constexpr int smem_flags_offset()
{
    return Fmt::kRingBytes + Fmt::kWarps * (Fmt::kStages + 1) * 8;
}
template <class Fmt>
__host__ __device__ constexpr int smem_q_offset() { return smem_flags_offset<Fmt>() + kSmemFlagBytes; }
template <class Fmt>
__host__ __device__ constexpr int smem_tables_offset(int qrows)
{
    return smem_q_offset<Fmt>() + Fmt::kWarps * query_bytes<Fmt>(qrows);
}
template <class Fmt>
inline size_t decode_smem_bytes(int32_t num_seqs, int32_t qrows)
{
    return 1024 + smem_tables_offset<Fmt>(qrows) + seq_table_bytes(num_seqs);
}

template <class Fmt, bool kPrefill>
__global__ void __launch_bounds__(32 * Fmt::kWarps, Fmt::kMinBlocks)
    paged_decode_kernel(const __grid_constant__ CUtensorMap tmap, const DecodeParams p)
{
    static_assert(16 * Fmt::kWarps <= kSmemFlagBytes, "the flags hold two int64 per warp");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int S = p.num_seqs;
    SeqTables tb;
    tb.bind(smem + smem_tables_offset<Fmt>(p.qrows), S);
    volatile int64_t *flags = reinterpret_cast<volatile int64_t *>(smem + smem_flags_offset<Fmt>());

    // ---- 1. sequence tables, the plan, zero the output rows that get no segment ----------------
    scan_sequences<kPrefill>(p, tb, flags, blockIdx.x == 0);
    // The merge kernel may start its own prologue.  The window part of a windowed decode holds
    // its dependent (the quantized part) back until the cache writes it waits for are complete
    // (below), so that the quantized part can read the cache at once.
    if (p.win_part != 1)
        pdl_launch_dependents();
    // (the quantized part of a windowed decode leaves such rows to the window part, which
    // also marks their lse empty)
    for (int s = blockIdx.x; s < S && p.win_part != 2; s += gridDim.x) {
        const int c = query_tokens<kPrefill>(p, s);
        if (tb.nbk[s] == 0 && c > 0 && (!kPrefill || c <= p.seq_lens[s])) {
            const int64_t row0 = query_row0<kPrefill>(p, s) * p.hq;
            float4 *dst = reinterpret_cast<float4 *>(p.out + row0 * Fmt::kDim);
            for (int i = tid; i < c * p.hq * Fmt::kDim / 4; i += 32 * Fmt::kWarps)
                dst[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            if (p.lse != nullptr)
                for (int i = tid; i < c * p.hq; i += 32 * Fmt::kWarps)
                    p.lse[row0 + i] = -INFINITY;
        }
    }
    // Leaving early keeps a windowed decode's order: the window part waits for the cache writes
    // before it releases the quantized part, and the quantized part completes only after the
    // window part (its merge kernel reads the window part's rows).
    auto pdl_exit = [&]() {
        if (p.win_part != 0)
            pdl_wait();
        if (p.win_part == 1)
            pdl_launch_dependents();
    };
    if (tb.spre[S] > p.max_segments) {   // more query rows than the workspace was sized for
        if (blockIdx.x == 0 && tid == 0)
            set_status(p.status, SAW_DEV_BAD_SEQ_LEN);
        pdl_exit();
        return;
    }
    Plan plan;
    plan.init(tb, S, p.total_warps);
    const int64_t u = static_cast<int64_t>(blockIdx.x) * Fmt::kWarps + warp;
    int64_t F0, F1;
    if (p.win_part == 1) {
        // the window part: warp u takes segment u whole (no split, so no partials to merge)
        if (u >= tb.spre[S]) {
            pdl_exit();
            return;
        }
        const int s = plan.seq_of_segment(u);
        F0 = tb.fpre[s] + (u - tb.spre[s]) * tb.npg[s];
        F1 = F0 + tb.npg[s];
    } else {
        if (plan.P == 0 || u >= plan.W) {
            pdl_exit();
            return;
        }
        F0 = plan.begin(u);
        F1 = plan.begin(u + 1);
    }
    if (F0 >= F1) {
        pdl_exit();
        return;
    }
    const int n_w = static_cast<int>(F1 - F0);

    // ---- 2. this warp's copy ring ---------------------------------------------------------------
    constexpr int kStages = Fmt::kStages;
    const typename Fmt::Ring ring = Fmt::ring(smem_u32(smem), warp);
    const uint32_t qbuf = smem_u32(smem + smem_q_offset<Fmt>()) + warp * query_bytes<Fmt>(p.qrows);
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
        const int s = plan.seq_of_flat(pos);
        const int32_t n_s = tb.npg[s];
        const int64_t rel = pos - tb.fpre[s];
        const int j = static_cast<int>(rel / n_s);
        const int i = static_cast<int>(rel - static_cast<int64_t>(j) * n_s);
        const int nb = tb.nbk[s];
        const int h = nb == 1 ? j : j / nb;
        int32_t page = p.block_table[static_cast<int64_t>(s) * p.max_blocks + i];
        if (page < 0 || page >= p.num_pages) {
            set_status(p.status, SAW_DEV_BAD_PAGE);
            page = 0;
        }
        return (page * p.hkv + h) * Fmt::kRowsPerPage;
    };
    // queue a segment's raw query rows into the warp's query buffer: one bulk copy per run of
    // rows of the same query token (its heads are contiguous)
    auto issue_query = [&](const Segment<kPrefill> &sg) {
        if (lane == 0) {
            mbar_arrive_expect_tx(qbar, static_cast<uint32_t>(sg.nrows) * Fmt::kDim * 2);
            for (int e = 0; e < sg.nrows;) {
                const int head = sg.row0 + e - sg.row_token(p, e) * p.group;
                const int cnt = min(p.group - head, sg.nrows - e);
                bulk_g2s(qbuf + e * Fmt::kDim * 2, p.q + sg.row_offset(p, e, Fmt::kDim),
                         static_cast<uint32_t>(cnt) * Fmt::kDim * 2, qbar);
                e += cnt;
            }
        }
    };

    // The cache may be written by the kernel this one depends on.  The quantized part of a
    // windowed decode depends on the window part, which released it only after that kernel's
    // writes were complete: it waits only where it needs the window part's rows (finalize).
    if (p.win_part != 2)
        pdl_wait();
    if (p.win_part == 1)
        pdl_launch_dependents();

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
        const int stg = j % kStages;
        Fmt::issue(ring, stg, bar0 + 8 * stg, &tmap, row, p);
    };

    // first piece's segment and its query; across pieces only (sequence, segment index) of the
    // current and next segments stay live, the rest is rebuilt where needed
    int cs = plan.seq_of_flat(F0);
    int cj = static_cast<int>((F0 - tb.fpre[cs]) / tb.npg[cs]);
    {
        Segment<kPrefill> sg;
        sg.init(p, tb, cs, cj);
        issue_query(sg);
    }
    while (issued < kStages - 1 && issued < n_w)
        issue_next();

    WarpState<Fmt::kTiles> st;
    typename Fmt::Query qf;
    // Page m of the run: queue the page kStages - 1 ahead into the stage page m - 1 used, wait
    // for page m and attend over it (through `mask` when kMask).
    auto step = [&](auto mask_tag, int m, const PageMask &mask) {
        if (issued < n_w && !aborted)
            issue_next();
        const int stg = m % kStages;
        const uint32_t phase = (static_cast<uint32_t>(m) / kStages) & 1u;
        const bool ok = !aborted && mbar_wait_bounded(bar0 + 8 * stg, phase, kWaitLimitNs);
        if (__all_sync(0xFFFFFFFFu, ok)) {
            Fmt::template page<decltype(mask_tag)::value>(ring, stg, mask, qf, lane, st);
        } else if (!aborted) {
            if (lane == 0)
                set_status(p.status, SAW_DEV_WAIT_TIMEOUT);
            drain_from = m;
            aborted = true;
        }
        __syncwarp();
    };

    // Whole pages m and m + 1 as one step (formats with kPairs): queue pages up to m + kStages - 1
    // (the stages pages m - 2 and m - 1 used), wait for both pages, attend over both.
    auto step2 = [&](int m) {
        while (issued <= m + kStages - 1 && issued < n_w && !aborted)
            issue_next();
        const int stg0 = m % kStages, stg1 = (m + 1) % kStages;
        const bool ok = !aborted &&
                        mbar_wait_bounded(bar0 + 8 * stg0, (static_cast<uint32_t>(m) / kStages) & 1u, kWaitLimitNs) &&
                        mbar_wait_bounded(bar0 + 8 * stg1, (static_cast<uint32_t>(m + 1) / kStages) & 1u, kWaitLimitNs);
        if (__all_sync(0xFFFFFFFFu, ok)) {
            if constexpr (Fmt::kPairs)
                Fmt::page2(ring, stg0, stg1, qf, lane, st);
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
    const int t4 = lane & 3;
    while (pos < F1) {
        const int n_s = tb.npg[cs];
        const int64_t seg_start = tb.fpre[cs] + static_cast<int64_t>(cj) * n_s;
        const int64_t seg_end = seg_start + n_s;
        const bool ends_segment = seg_end <= F1;
        const int m_end = static_cast<int>((ends_segment ? seg_end : F1) - F0);
        int len, lim[2], first_masked, nrows;
        {
            Segment<kPrefill> sg;
            sg.init(p, tb, cs, cj);
            len = sg.len;
            lim[0] = sg.limit(p, 2 * t4);
            lim[1] = sg.limit(p, 2 * t4 + 1);
            first_masked = sg.first_masked_page(p);
            nrows = sg.nrows;
        }

        // this piece's query: wait for its copy, build the fragments, then queue the next one
        const bool qok = !aborted && mbar_wait_bounded(qbar, qphase, kWaitLimitNs);
        if (!__all_sync(0xFFFFFFFFu, qok) && !aborted) {
            if (lane == 0)
                set_status(p.status, SAW_DEV_WAIT_TIMEOUT);
            drain_from = m;
            aborted = true;
        }
        qphase ^= 1;
        Fmt::load_query(p, qbuf, nrows, lane, qf);
        __syncwarp();
        int ns = cs, nj = cj;
        if (m_end < n_w) {
            if (cj + 1 < p.hkv * tb.nbk[cs]) {
                nj = cj + 1;
            } else {
                do {
                    ns++;
                } while (tb.spre[ns + 1] == tb.spre[ns]);
                nj = 0;
            }
            if (!aborted) {
                Segment<kPrefill> nx;
                nx.init(p, tb, ns, nj);
                issue_query(nx);
            }
        }

        // pages before the block's first limit are whole for every row; the rest are masked
        state_reset(st);
        const int i0 = static_cast<int>(pos - seg_start) - m;   // page index of run page m
        const int m_full = min(m_end, max(m, first_masked - i0));
        const PageMask whole = {kPageSize, {kPageSize, kPageSize}};
        if constexpr (Fmt::kPairs) {
            for (; m + 1 < m_full; m += 2)
                step2(m);
        }
        for (; m < m_full; m++)
            step(std::false_type(), m, whole);
        for (; m < m_end; m++)
            step(std::true_type(), m, page_mask(len, lim, i0 + m));

        Fmt::piece_end(st);
        if (seg_start >= F0 && ends_segment) {
            Segment<kPrefill> sg;
            sg.init(p, tb, cs, cj);
            if (p.win_part == 2)
                pdl_wait();   // the window part's rows and lse
            Fmt::finalize(p, sg, lane, st.o, st.m, st.l);
        } else {
            store_partial(p.partials + (tb.spre[cs] + cj + u) * slot_floats<Fmt::kTiles>(), lane, st);
        }
        pos = F0 + m_end;
        cs = ns;
        cj = nj;
    }

    // ---- 4. after an abort, let queued copies land before the shared memory is released ----
    if (aborted) {
        for (int k = drain_from; k < issued; k++)
            mbar_wait_bounded(bar0 + 8 * (k % kStages), (static_cast<uint32_t>(k) / kStages) & 1u,
                              kWaitLimitNs / 10);
        mbar_wait_bounded(qbar, qphase, kWaitLimitNs / 10);
    }
    if (p.win_part == 2)
        pdl_wait();   // complete only after the window part (the merge kernel reads its rows)
}

constexpr int kShapeVariants = 4;

struct LaunchShape {
    int sms = 0;
    int occ = 0;
};

// Multiprocessor count and occupancy of one family of decode kernels (the kShapeVariants
// instantiations of the decode and of its merge kernel: rotation x decode / prefill) for the current device and dynamic shared-memory sizes.  The
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

inline cudaError_t launch_shape(ShapeCache &cache, const void *const decode_kernels[kShapeVariants],
                                const void *const merge_kernels[kShapeVariants], int threads,
                                size_t smem, size_t merge_smem, LaunchShape &out)
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
        for (int r = 0; r < kShapeVariants && e == cudaSuccess; r++)
            e = cudaFuncSetAttribute(decode_kernels[r], cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(smem));
        if (e != cudaSuccess)
            return e;
        d.decode_attr = smem;
    }
    if (merge_smem > d.merge_attr) {
        for (int r = 0; r < kShapeVariants && e == cudaSuccess; r++)
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
