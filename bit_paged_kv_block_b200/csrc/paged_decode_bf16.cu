// paged_decode_bf16.cu -- the uncompressed BF16 paged KV cache: append (scatter) and decode.
//
// The baseline the INT4 format is measured against: "SAW-INT4: System-Aware 4-Bit KV-Cache
// Quantization for Real-World LLM Serving" (Research Findings) states its serving gains
// against a 16-bit KV cache and "BitDecoding-FP4" (abstract) its speedup over BF16 KV decoding.
// Same page geometry as the INT4 cache with 16-bit elements and no scales:
//   kv uint16 (bf16 bits) [num_pages][Hkv][2 (K, V)][16][128]: one (page, kv head) is 8 KiB.
// No rotation and no quantization: attention over exactly the stored bf16 values.
//
// The decode uses the format-generic kernel of decode_common.cuh (cost-balanced warp runs,
// split-K slots, merge kernel) with this page format:
//   * one 2-D tensor copy per page: the 8 KiB block as 64 rows of 128 B (128-byte swizzle) into
//     a 2-stage ring per warp (4 warps per CTA, 3 CTAs per SM);
//   * S^T[16 tok x 8 heads] = K[16 x 128] . Q^T with mma.m16n8k16 bf16 x bf16 -> fp32: K comes
//     straight from ldmatrix, q is the raw bf16 query (the products are exact), and the logits
//     are acc * sm_scale * log2 e in fp32;
//   * online softmax in the log2 domain (shared with the INT4 format);
//   * O^T[128 d x 8 heads] += V^T . P^T with V by ldmatrix.trans and P split into bf16 high and
//     low parts (two MMAs), so P keeps about 16 significant bits although the MMA takes bf16.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "decode_common.cuh"
#include "saw_device.cuh"
#include "saw_internal.h"

namespace saw {
namespace {

using namespace decode;

constexpr int kBf16PageBytes = 2 * kPageSize * kHeadDim * 2;   // K + V of one (page, kv head)
constexpr int kBf16RowBytes = 128;                              // tensor-map row: 64 elements

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// Byte offset, inside a staged page, of the 16-byte chunk holding elements [d0, d0 + 8) of token
// `tok` of K (sel 0) or V (sel 1): row 32 sel + 2 tok + d0 / 64, chunk (d0 % 64) / 8, the chunk
// index XOR-ed with the row's low three bits by the 128-byte swizzle.
__device__ __forceinline__ uint32_t bf16_chunk(int sel, int tok, int d0)
{
    const int row = 32 * sel + 2 * tok + (d0 >> 6);
    const int chunk = (d0 & 63) >> 3;
    return row * kBf16RowBytes + ((chunk ^ (row & 7)) << 4);
}

// kLse: the window part of a windowed decode, which also records each row's log2 softmax
// denominator (a separate instantiation, so the plain decode carries none of it).
template <bool kLse>
struct Bf16FormatT {
    static constexpr int kDim = kHeadDim;
    static constexpr int kTiles = kHeadDim / 16;
    static constexpr int kWarps = 4;
    // the window part streams a short run of pages per warp and holds the registers of two of the
    // quantized part's CTAs anyway: a third stage (same registers) shortens it (windowed step
    // 97.5 -> 95.2 us back to back; a fourth measured no better)
    static constexpr int kStages = kLse ? 3 : 2;
    static constexpr int kMinBlocks = 3;
    static constexpr bool kPairs = false;
    static constexpr int kRowsPerPage = kBf16PageBytes / kBf16RowBytes;   // 64
    static constexpr int kRingBytes = kWarps * kStages * kBf16PageBytes;
    struct Ring {
        uint32_t base;
    };
    struct Query {
        uint32_t bq[8][2];   // k-step i: q[g][16 i + 2t, +1], q[g][16 i + 2t + 8, +9]
        float mult;          // sm_scale * log2 e
    };

    __device__ static Ring ring(uint32_t base, int warp)
    {
        return {base + warp * kStages * kBf16PageBytes};
    }

    __device__ static void issue(const Ring &r, int stg, uint32_t bar, const CUtensorMap *tmap,
                                 int32_t row, const DecodeParams &)
    {
        asm volatile("{\n\t.reg .pred p;\n\t"
                     "elect.sync _|p, 0xffffffff;\n\t"
                     "@p mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %4;\n\t"
                     "@p cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
                     " [%1], [%2, {%5, %3}], [%0];\n\t"
                     "}"
                     ::"r"(bar), "r"(r.base + stg * kBf16PageBytes), "l"(tmap), "r"(row),
                     "r"(static_cast<uint32_t>(kBf16PageBytes)), "r"(0)
                     : "memory");
    }

    // Thread (g, t) holds query head g of the segment (zero for g >= nheads) as mma B fragments.
    __device__ static void load_query(const DecodeParams &p, uint32_t qbuf, int nheads, int lane,
                                      Query &q)
    {
        const int g = lane >> 2, t = lane & 3;
#pragma unroll
        for (int i = 0; i < 8; i++) {
            const uint32_t a = qbuf + g * (kHeadDim * 2) + (16 * i + 2 * t) * 2;
            q.bq[i][0] = g < nheads ? lds32(a) : 0u;
            q.bq[i][1] = g < nheads ? lds32(a + 16) : 0u;
        }
        q.mult = p.q_mult;
    }

    template <bool kMask>
    __device__ static void page(const Ring &r, int stg, const PageMask &mask, const Query &q,
                                int lane, WarpState<8> &st)
    {
        const uint32_t base = r.base + stg * kBf16PageBytes;
        const int g = lane >> 2, t = lane & 3;

        // S^T = K . Q^T: ldmatrix matrix j = lane / 8 is (tokens 8 (j & 1) .., d 8 (j >> 1) ..)
        float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        const int ktok = (lane & 7) + 8 * ((lane >> 3) & 1);
        const int kd = 8 * (lane >> 4);
#pragma unroll
        for (int i = 0; i < 8; i++) {
            uint32_t a[4];
            ldsm_x4(base + bf16_chunk(0, ktok, 16 * i + kd), a[0], a[1], a[2], a[3]);
            mma_16816_bf16(acc, a, q.bq[i][0], q.bq[i][1]);
        }
        float s[4] = {acc[0] * q.mult, acc[1] * q.mult, acc[2] * q.mult, acc[3] * q.mult};
        if (kMask) {   // column e (block row 2t + e) sees tokens [0, mask.col[e])
            if (g >= mask.col[0])
                s[0] = -INFINITY;
            if (g >= mask.col[1])
                s[1] = -INFINITY;
            if (g + 8 >= mask.col[0])
                s[2] = -INFINITY;
            if (g + 8 >= mask.col[1])
                s[3] = -INFINITY;
        }
        float pr[4];
        softmax_update<kMask, 8, 4>(s, st, pr);
        st.l[0] += pr[0] + pr[2];
        st.l[1] += pr[1] + pr[3];

        // P = hi + lo in bf16, each turned into the B fragment (tokens 2t, 2t+1 | 2t+8, 2t+9)
        float lo[4];
#pragma unroll
        for (int k = 0; k < 4; k++)
            lo[k] = pr[k] - __bfloat162float(__float2bfloat16_rn(pr[k]));
        const uint32_t ph0 = movmatrix_trans(pack_bf16x2(pr[0], pr[1]));
        const uint32_t ph1 = movmatrix_trans(pack_bf16x2(pr[2], pr[3]));
        const uint32_t pl0 = movmatrix_trans(pack_bf16x2(lo[0], lo[1]));
        const uint32_t pl1 = movmatrix_trans(pack_bf16x2(lo[2], lo[3]));

        // O^T += V^T . P^T: ldmatrix.trans matrix j is (tokens 8 (j >> 1) .., d 8 (j & 1) ..),
        // giving the A fragment of rows d = 16 c + (0..15) and columns tokens 0..15.  Tokens
        // >= mask.valid (never written: any bits) are zeroed so 0 * Inf cannot reach the output.
        const int vtok = (lane & 7) + 8 * (lane >> 4);
        const int vd = 8 * ((lane >> 3) & 1);
        uint32_t keep[2] = {0xFFFFFFFFu, 0xFFFFFFFFu};   // tokens 2t, 2t+1 | 2t+8, 2t+9
        if (kMask) {
            const int valid = mask.valid;
            keep[0] = (2 * t < valid ? 0x0000FFFFu : 0u) | (2 * t + 1 < valid ? 0xFFFF0000u : 0u);
            keep[1] = (2 * t + 8 < valid ? 0x0000FFFFu : 0u) | (2 * t + 9 < valid ? 0xFFFF0000u : 0u);
        }
#pragma unroll
        for (int c = 0; c < 8; c++) {
            uint32_t a[4];
            ldsm_x4_trans(base + bf16_chunk(1, vtok, 16 * c + vd), a[0], a[1], a[2], a[3]);
            if (kMask) {
                a[0] &= keep[0];
                a[1] &= keep[0];
                a[2] &= keep[1];
                a[3] &= keep[1];
            }
            mma_16816_bf16(st.o[c], a, ph0, ph1);
            mma_16816_bf16(st.o[c], a, pl0, pl1);
        }
    }

    __device__ static void piece_end(WarpState<8> &st)
    {
#pragma unroll
        for (int e = 0; e < 2; e++)
#pragma unroll
            for (int d = 4; d <= 16; d <<= 1)
                st.l[e] += __shfl_xor_sync(0xFFFFFFFFu, st.l[e], d);
    }

    // block row 2t + e: out[row][d] = o / l; tile c, rows g and g + 8 are d = 16 c + g (+ 8).
    // As the window part of a windowed decode it also records lse[row] = m + log2 l, the log2 of
    // the row's softmax denominator, for the quantized part to merge with.
    template <class Seg>
    __device__ static void finalize(const DecodeParams &p, const Seg &sg, int lane, float o[8][4],
                                    const float m[2], const float l[2])
    {
        const int g = lane >> 2, t = lane & 3;
#pragma unroll
        for (int e = 0; e < 2; e++) {
            const int head = 2 * t + e;
            if (head >= sg.nrows)
                continue;
            const float inv = 1.0f / l[e];
            const int64_t off = sg.row_offset(p, head, kHeadDim);
            float *dst = p.out + off;
            if (kLse && g == 0)
                p.lse[off / kHeadDim] = m[e] + log2f(l[e]);
#pragma unroll
            for (int c = 0; c < 8; c++) {
                dst[16 * c + g] = o[c][e] * inv;
                dst[16 * c + g + 8] = o[c][2 + e] * inv;
            }
        }
    }
};
using Bf16Format = Bf16FormatT<false>;

// Scatter T tokens of bf16 K and V into the bf16 pages: one warp per (token, kv head), lanes
// 0-15 moving the K vector and lanes 16-31 the V vector, 16 bytes each.
__global__ void __launch_bounds__(256)
    append_bf16_kernel(const uint8_t *k, const uint8_t *v, const int64_t *slot_mapping,
                       int64_t num_vecs, int32_t hkv, int64_t num_slots, uint8_t *kv,
                       uint32_t *status)
{
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int sel = lane >> 4;
    const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    for (int64_t vec = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
         vec < num_vecs; vec += warps) {
        const int64_t tok = vec / hkv;
        const int h = static_cast<int>(vec - tok * hkv);
        const int64_t slot = slot_mapping[tok];
        if (slot < 0)
            continue;
        if (slot >= num_slots) {
            if (lane == 0)
                set_status(status, SAW_DEV_BAD_SLOT);
            continue;
        }
        const int64_t page = slot / kPageSize, off = slot % kPageSize;
        const uint8_t *src = (sel ? v : k) + vec * (kHeadDim * 2) + 16 * (lane & 15);
        uint8_t *dst = kv + (((page * hkv + h) * 2 + sel) * kPageSize + off) * (kHeadDim * 2) +
                       16 * (lane & 15);
        *reinterpret_cast<uint4 *>(dst) = ldg_stream16(src);
    }
}

ShapeCache g_bf16_shapes;

cudaError_t bf16_launch_shape(size_t smem, size_t merge_smem, LaunchShape &out)
{
    static const void *const decode_kernels[kShapeVariants] = {
        reinterpret_cast<const void *>(paged_decode_kernel<Bf16Format, false>),
        reinterpret_cast<const void *>(paged_decode_kernel<Bf16Format, true>),
        reinterpret_cast<const void *>(paged_decode_kernel<Bf16Format, false>),
        reinterpret_cast<const void *>(paged_decode_kernel<Bf16Format, true>)};
    static const void *const merge_kernels[kShapeVariants] = {
        reinterpret_cast<const void *>(paged_decode_merge_kernel<Bf16Format, false>),
        reinterpret_cast<const void *>(paged_decode_merge_kernel<Bf16Format, true>),
        reinterpret_cast<const void *>(paged_decode_merge_kernel<Bf16Format, false>),
        reinterpret_cast<const void *>(paged_decode_merge_kernel<Bf16Format, true>)};
    return decode::launch_shape(g_bf16_shapes, decode_kernels, merge_kernels,
                                32 * Bf16Format::kWarps, smem, merge_smem, out);
}

// The window part of a windowed decode: only the shared-memory attributes are set here; its grid
// is the plain family's (same layout and launch bounds), which the workspace is sized for.
cudaError_t set_window_attributes(size_t smem, size_t merge_smem)
{
    static ShapeCache shapes;
    using W = Bf16FormatT<true>;
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

}  // namespace

cudaError_t launch_append_bf16(const AppendBf16Args &a, cudaStream_t stream)
{
    const int64_t num_vecs = a.num_tokens * a.num_kv_heads;
    if (num_vecs == 0)
        return cudaSuccess;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess)
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess)
        return e;
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>((num_vecs + 7) / 8, 8LL * sms));
    append_bf16_kernel<<<static_cast<unsigned>(grid), 256, 0, stream>>>(
        static_cast<const uint8_t *>(a.k), static_cast<const uint8_t *>(a.v), a.slot_mapping,
        num_vecs, a.num_kv_heads, a.num_pages * kPageSize, static_cast<uint8_t *>(a.kv), a.status);
    return cudaGetLastError();
}

size_t decode_bf16_workspace_bytes(int32_t num_kv_heads, int32_t num_q_heads, int32_t num_seqs,
                                   int64_t total_q)
{
    if (num_kv_heads <= 0 || num_q_heads <= 0 || num_seqs < 0 || num_q_heads % num_kv_heads)
        return 0;
    const bool prefill = total_q >= 0;
    LaunchShape ls;
    if (bf16_launch_shape(decode_smem_bytes<Bf16Format>(num_seqs, query_rows(num_kv_heads, num_q_heads, prefill)),
                          merge_smem_bytes<8>(num_seqs), ls) != cudaSuccess)
        return 0;
    return workspace_bytes_for<8>(static_cast<size_t>(ls.sms) * ls.occ * Bf16Format::kWarps,
                               max_segments(num_kv_heads, num_q_heads, num_seqs, total_q, prefill));
}

cudaError_t launch_paged_decode_bf16(const DecodeArgs &a, cudaStream_t stream, bool programmatic)
{
    static thread_local struct {
        const void *base = nullptr;
        int64_t rows = 0;
        CUtensorMap map;
    } cache;
    const int64_t rows = a.num_pages * a.num_kv_heads * Bf16Format::kRowsPerPage;
    if (cache.base != a.kv_pages || cache.rows != rows) {
        auto encode = tensor_map_encoder();
        if (encode == nullptr)
            return cudaErrorNotSupported;
        const cuuint64_t dims[2] = {kBf16RowBytes / 2, static_cast<cuuint64_t>(rows)};
        const cuuint64_t strides[1] = {kBf16RowBytes};
        const cuuint32_t box[2] = {kBf16RowBytes / 2, Bf16Format::kRowsPerPage};
        const cuuint32_t estr[2] = {1, 1};
        CUresult r = encode(&cache.map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                            const_cast<uint8_t *>(a.kv_pages), dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) {
            cache.base = nullptr;
            return cudaErrorInvalidValue;
        }
        cache.base = a.kv_pages;
        cache.rows = rows;
    }

    const bool prefill = a.q_start != nullptr;
    const int32_t qrows = query_rows(a.num_kv_heads, a.num_q_heads, prefill);
    const size_t smem = decode_smem_bytes<Bf16Format>(a.num_seqs, qrows);
    // the window part's own layout (its ring may differ from the plain format's)
    const size_t wsmem = decode_smem_bytes<Bf16FormatT<true>>(a.num_seqs, qrows);
    const size_t msmem = merge_smem_bytes<8>(a.num_seqs);
    LaunchShape ls;
    cudaError_t e = bf16_launch_shape(smem, msmem, ls);
    if (e != cudaSuccess)
        return e;

    DecodeParams p;
    p.q = static_cast<const uint16_t *>(a.q);
    p.q_start = a.q_start;
    p.scales = nullptr;
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
    p.total_warps = ls.sms * ls.occ * Bf16Format::kWarps;
    // The window part's segments are short (at most sink + recent tokens each): one warp per
    // segment, never split, so it needs no merge kernel; the quantized part follows it directly
    // and overlaps it, waiting for its rows only at finalize.
    if (a.win_part == 1)
        p.total_warps = static_cast<int32_t>(std::max<int64_t>(1, p.max_segments));
    p.q_mult = static_cast<float>(static_cast<double>(a.sm_scale) * 1.4426950408889634);

    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>((p.total_warps + Bf16Format::kWarps - 1) / Bf16Format::kWarps));
    cfg.blockDim = dim3(32 * Bf16Format::kWarps);
    const bool window = a.win_part == 1;
    cfg.dynamicSmemBytes = window ? wsmem : smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = programmatic ? 1 : 0;
    if (window && prefill)
        return cudaErrorInvalidValue;
    if (window && (e = set_window_attributes(wsmem, msmem)) != cudaSuccess)
        return e;
    e = cudaLaunchKernelEx(&cfg, window    ? paged_decode_kernel<Bf16FormatT<true>, false>
                                 : prefill ? paged_decode_kernel<Bf16Format, true>
                                           : paged_decode_kernel<Bf16Format, false>,
                           cache.map, p);
    if (e != cudaSuccess)
        return e;

    if (window)
        return cudaGetLastError();
    const int64_t segs = p.max_segments;
    cudaLaunchConfig_t mcfg = cfg;
    mcfg.gridDim = dim3(static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>(segs, 8 * ls.sms))));
    mcfg.blockDim = dim3(kMergeThreads);
    mcfg.dynamicSmemBytes = msmem;
    mcfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&mcfg, window    ? paged_decode_merge_kernel<Bf16FormatT<true>, false>
                                  : prefill ? paged_decode_merge_kernel<Bf16Format, true>
                                            : paged_decode_merge_kernel<Bf16Format, false>,
                           p);
    if (e != cudaSuccess)
        return e;
    return cudaGetLastError();
}

}  // namespace saw
