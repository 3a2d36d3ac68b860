// saw_api.cu -- the extern "C" entry points declared in include/saw.h.
//
// Argument validation, workspace sizing and kernel launches.  Nothing here allocates device
// memory; every launch is asynchronous on the caller's stream.
#include <algorithm>
#include <cmath>
#include <cstdint>

#include "saw.h"
#include "saw_internal.h"

namespace {

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int check_cache(const saw_cache_desc *c)
{
    if (c == nullptr || c->num_kv_heads <= 0 || c->num_pages < 0)
        return SAW_ERR_INVALID_ARGUMENT;
    if ((c->head_dim != 64 && c->head_dim != 128 && c->head_dim != 256) || c->page_size != 16)
        return SAW_ERR_UNSUPPORTED;
    // tensor-map rows (page * Hkv + h) * 32 must stay below 2^31
    if (c->num_pages > (int64_t(1) << 31) / (int64_t(c->num_kv_heads) * 32))
        return SAW_ERR_UNSUPPORTED;
    return SAW_OK;
}

// bf16: the uncompressed baseline cache (no scales)
int check_append(const saw_cache_desc *cache, const void *k, const void *v,
                 const int64_t *slot_mapping, int64_t num_tokens, const uint8_t *kv_pages,
                 const void *scales, bool bf16 = false)
{
    if (num_tokens < 0)
        return SAW_ERR_INVALID_ARGUMENT;
    if (num_tokens == 0)
        return SAW_OK;
    if (!k || !v || !slot_mapping || !kv_pages || (!bf16 && !scales))
        return SAW_ERR_INVALID_ARGUMENT;
    if (!aligned(k, 16) || !aligned(v, 16) || !aligned(kv_pages, 16) ||
        (!bf16 && !aligned(scales, 16)) || !aligned(slot_mapping, 8))
        return SAW_ERR_INVALID_ARGUMENT;
    if (num_tokens > INT64_MAX / (int64_t(cache->num_kv_heads) * 2 * cache->head_dim))
        return SAW_ERR_INVALID_ARGUMENT;
    return SAW_OK;
}

int check_decode(const saw_cache_desc *cache, int32_t num_q_heads, const void *q,
                 const uint8_t *kv_pages, const void *scales, const int32_t *block_table,
                 int32_t max_blocks, const int32_t *seq_lens, int32_t num_seqs, float sm_scale,
                 const float *out, const void *workspace, size_t workspace_bytes,
                 bool bf16 = false, int64_t total_q = -1)
{
    if (num_q_heads <= 0 || num_seqs < 0 || num_q_heads % cache->num_kv_heads != 0)
        return SAW_ERR_INVALID_ARGUMENT;
    if (bf16 && cache->head_dim != 128)
        return SAW_ERR_UNSUPPORTED;   // the BF16 baseline cache: D = 128
    if (num_q_heads / cache->num_kv_heads > 16)
        return SAW_ERR_UNSUPPORTED;
    if (!std::isfinite(sm_scale))
        return SAW_ERR_INVALID_ARGUMENT;
    if (num_seqs == 0)
        return SAW_OK;
    if (!q || !kv_pages || (!bf16 && !scales) || !block_table || !seq_lens || !out || max_blocks <= 0)
        return SAW_ERR_INVALID_ARGUMENT;
    if (!aligned(q, 16) || !aligned(kv_pages, 16) || (!bf16 && !aligned(scales, 16)) || !aligned(out, 16) ||
        !aligned(block_table, 4) || !aligned(seq_lens, 4))
        return SAW_ERR_INVALID_ARGUMENT;
    if (cache->num_pages == 0)
        return SAW_ERR_INVALID_ARGUMENT;
    if (int64_t(max_blocks) * 16 > INT32_MAX)
        return SAW_ERR_INVALID_ARGUMENT;
    const size_t need =
        bf16 ? saw::decode_bf16_workspace_bytes(cache->num_kv_heads, num_q_heads, num_seqs, total_q)
             : saw::decode_workspace_bytes(cache->num_kv_heads, num_q_heads, num_seqs, total_q,
                                           cache->head_dim);
    if (need == 0)
        return SAW_ERR_CUDA;
    if (workspace == nullptr || workspace_bytes < need || !aligned(workspace, 256))
        return SAW_ERR_WORKSPACE;
    return SAW_OK;
}

saw::DecodeArgs decode_args(const saw_cache_desc *cache, int32_t num_q_heads, const void *q,
                            const uint8_t *kv_pages, const void *scales,
                            const int32_t *block_table, int32_t max_blocks,
                            const int32_t *seq_lens, int32_t num_seqs, float sm_scale,
                            float *out, void *workspace, size_t workspace_bytes,
                            uint32_t *dev_status)
{
    saw::DecodeArgs a;
    a.q = q;
    a.kv_pages = kv_pages;
    a.scales = scales;
    a.block_table = block_table;
    a.max_blocks = max_blocks;
    a.seq_lens = seq_lens;
    a.num_seqs = num_seqs;
    a.num_q_heads = num_q_heads;
    a.num_kv_heads = cache->num_kv_heads;
    a.num_pages = cache->num_pages;
    a.sm_scale = sm_scale;
    a.out = out;
    a.workspace = workspace;
    a.workspace_bytes = workspace_bytes;
    a.status = dev_status;
    a.head_dim = cache->head_dim;
    return a;
}

}  // namespace

extern "C" {

int saw_version(void) { return 100; }

const char *saw_status_string(int status)
{
    switch (status) {
    case SAW_OK:
        return "ok";
    case SAW_ERR_INVALID_ARGUMENT:
        return "invalid argument (null pointer, bad size or alignment, Hq not a multiple of Hkv)";
    case SAW_ERR_UNSUPPORTED:
        return "unsupported shape (head_dim 64, 128 or 256, the BF16 cache 128; page_size 16; "
               "Hq/Hkv at most 16)";
    case SAW_ERR_CUDA:
        return "CUDA runtime error";
    case SAW_ERR_WORKSPACE:
        return "workspace missing, misaligned or too small";
    case SAW_ERR_SCRATCH_LIMIT:
        return "shape too large for the fixed scratch of saw_paged_decode_attn_static "
               "(num_seqs * num_kv_heads * ceil(Hq / Hkv / 8) must be at most 2048)";
    default:
        return "unknown status";
    }
}

}  // extern "C"

namespace {

saw::RotateQuantizeArgs append_args(const saw_cache_desc *cache, const void *k, const void *v,
                                    const int64_t *slot_mapping, int64_t num_tokens,
                                    uint8_t *kv_pages, void *scales, uint32_t *dev_status,
                                    bool rotate)
{
    saw::RotateQuantizeArgs a;
    a.k = k;
    a.v = v;
    a.slot_mapping = slot_mapping;
    a.num_tokens = num_tokens;
    a.num_kv_heads = cache->num_kv_heads;
    a.head_dim = cache->head_dim;
    a.num_pages = cache->num_pages;
    a.kv_pages = kv_pages;
    a.scales = scales;
    a.status = dev_status;
    a.rotate = rotate;
    return a;
}

// k_stride / v_stride: bf16 elements between consecutive tokens of k / v (0: contiguous)
int append_impl(const saw_cache_desc *cache, const void *k, const void *v,
                const int64_t *slot_mapping, int64_t num_tokens, uint8_t *kv_pages, void *scales,
                uint32_t *dev_status, void *stream, bool rotate, int64_t k_stride = 0,
                int64_t v_stride = 0)
{
    int rc = check_cache(cache);
    if (rc != SAW_OK)
        return rc;
    rc = check_append(cache, k, v, slot_mapping, num_tokens, kv_pages, scales);
    if (rc != SAW_OK)
        return rc;
    if (k_stride != 0 || v_stride != 0) {
        // strided rows: each token's Hkv head vectors are contiguous; tokens start every
        // *_stride elements (a multiple of 8, so every token starts on 16 bytes)
        const int64_t row = int64_t(cache->num_kv_heads) * cache->head_dim;
        const int64_t tile_vecs = 1024 / cache->head_dim;   // vectors per quantizer tile
        if (k_stride < row || v_stride < row || k_stride % 8 != 0 || v_stride % 8 != 0 ||
            k_stride > (int64_t(1) << 36) || v_stride > (int64_t(1) << 36))
            return SAW_ERR_INVALID_ARGUMENT;
        if (cache->num_kv_heads % tile_vecs != 0 && tile_vecs % cache->num_kv_heads != 0)
            return SAW_ERR_UNSUPPORTED;
        if (num_tokens > (int64_t(1) << 31) - 1)
            return SAW_ERR_INVALID_ARGUMENT;
    }
    if (num_tokens == 0)
        return SAW_OK;
    saw::RotateQuantizeArgs a =
        append_args(cache, k, v, slot_mapping, num_tokens, kv_pages, scales, dev_status, rotate);
    a.k_stride = k_stride;
    a.v_stride = v_stride;
    return saw::launch_rotate_quantize(a, static_cast<cudaStream_t>(stream), false) == cudaSuccess
               ? SAW_OK
               : SAW_ERR_CUDA;
}

int decode_impl(const saw_cache_desc *cache, int32_t num_q_heads, const void *q,
                const uint8_t *kv_pages, const void *scales, const int32_t *block_table,
                int32_t max_blocks_per_seq, const int32_t *seq_lens, int32_t num_seqs,
                float sm_scale, float *out, void *workspace, size_t workspace_bytes,
                uint32_t *dev_status, void *stream, bool rotate)
{
    int rc = check_cache(cache);
    if (rc != SAW_OK)
        return rc;
    rc = check_decode(cache, num_q_heads, q, kv_pages, scales, block_table, max_blocks_per_seq,
                      seq_lens, num_seqs, sm_scale, out, workspace, workspace_bytes);
    if (rc != SAW_OK || num_seqs == 0)
        return rc;
    saw::DecodeArgs a =
        decode_args(cache, num_q_heads, q, kv_pages, scales, block_table, max_blocks_per_seq,
                    seq_lens, num_seqs, sm_scale, out, workspace, workspace_bytes, dev_status);
    a.rotate = rotate;
    return saw::launch_paged_decode(a, static_cast<cudaStream_t>(stream), false) == cudaSuccess
               ? SAW_OK
               : SAW_ERR_CUDA;
}

int step_impl(const saw_cache_desc *cache, int32_t num_q_heads, const void *q, const void *k_new,
              const void *v_new, const int64_t *slot_mapping, int64_t num_new_tokens,
              uint8_t *kv_pages, void *scales, const int32_t *block_table,
              int32_t max_blocks_per_seq, const int32_t *seq_lens, int32_t num_seqs,
              float sm_scale, float *out, void *workspace, size_t workspace_bytes,
              uint32_t *dev_status, void *stream, bool rotate)
{
    int rc = check_cache(cache);
    if (rc != SAW_OK)
        return rc;
    rc = check_append(cache, k_new, v_new, slot_mapping, num_new_tokens, kv_pages, scales);
    if (rc != SAW_OK)
        return rc;
    rc = check_decode(cache, num_q_heads, q, kv_pages, scales, block_table, max_blocks_per_seq,
                      seq_lens, num_seqs, sm_scale, out, workspace, workspace_bytes);
    if (rc != SAW_OK)
        return rc;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool appended = num_new_tokens > 0;
    if (appended) {
        const saw::RotateQuantizeArgs a = append_args(cache, k_new, v_new, slot_mapping,
                                                      num_new_tokens, kv_pages, scales,
                                                      dev_status, rotate);
        if (saw::launch_rotate_quantize(a, s, true) != cudaSuccess)
            return SAW_ERR_CUDA;
    }
    if (num_seqs == 0)
        return SAW_OK;
    saw::DecodeArgs d =
        decode_args(cache, num_q_heads, q, kv_pages, scales, block_table, max_blocks_per_seq,
                    seq_lens, num_seqs, sm_scale, out, workspace, workspace_bytes, dev_status);
    d.rotate = rotate;
    return saw::launch_paged_decode(d, s, appended) == cudaSuccess ? SAW_OK : SAW_ERR_CUDA;
}

}  // namespace

extern "C" {

int saw_rotate_quantize_paged(const saw_cache_desc *cache, const void *k, const void *v,
                              const int64_t *slot_mapping, int64_t num_tokens,
                              uint8_t *kv_pages, void *scales, uint32_t *dev_status,
                              void *stream)
{
    return append_impl(cache, k, v, slot_mapping, num_tokens, kv_pages, scales, dev_status,
                       stream, true);
}

int saw_quantize_paged_plain(const saw_cache_desc *cache, const void *k, const void *v,
                             const int64_t *slot_mapping, int64_t num_tokens, uint8_t *kv_pages,
                             void *scales, uint32_t *dev_status, void *stream)
{
    return append_impl(cache, k, v, slot_mapping, num_tokens, kv_pages, scales, dev_status,
                       stream, false);
}

int saw_rotate_quantize_paged_strided(const saw_cache_desc *cache, const void *k, int64_t k_stride,
                                      const void *v, int64_t v_stride, const int64_t *slot_mapping,
                                      int64_t num_tokens, uint8_t *kv_pages, void *scales,
                                      uint32_t *dev_status, void *stream)
{
    if (k_stride == 0 || v_stride == 0)
        return SAW_ERR_INVALID_ARGUMENT;
    return append_impl(cache, k, v, slot_mapping, num_tokens, kv_pages, scales, dev_status,
                       stream, true, k_stride, v_stride);
}

int saw_quantize_paged_plain_strided(const saw_cache_desc *cache, const void *k, int64_t k_stride,
                                     const void *v, int64_t v_stride, const int64_t *slot_mapping,
                                     int64_t num_tokens, uint8_t *kv_pages, void *scales,
                                     uint32_t *dev_status, void *stream)
{
    if (k_stride == 0 || v_stride == 0)
        return SAW_ERR_INVALID_ARGUMENT;
    return append_impl(cache, k, v, slot_mapping, num_tokens, kv_pages, scales, dev_status,
                       stream, false, k_stride, v_stride);
}

size_t saw_paged_decode_workspace_bytes(const saw_cache_desc *cache, int32_t num_q_heads,
                                        int32_t num_seqs)
{
    if (check_cache(cache) != SAW_OK || num_q_heads <= 0 ||
        num_q_heads % cache->num_kv_heads != 0 || num_q_heads / cache->num_kv_heads > 16)
        return 0;
    return saw::decode_workspace_bytes(cache->num_kv_heads, num_q_heads, num_seqs, -1,
                                       cache->head_dim);
}

int saw_paged_decode_workspace_init(void *workspace, size_t workspace_bytes, void *stream)
{
    if (workspace == nullptr && workspace_bytes != 0)
        return SAW_ERR_INVALID_ARGUMENT;
    if (workspace_bytes == 0)
        return SAW_OK;
    return cudaMemsetAsync(workspace, 0, workspace_bytes, static_cast<cudaStream_t>(stream)) ==
                   cudaSuccess
               ? SAW_OK
               : SAW_ERR_CUDA;
}

int saw_paged_decode_attn(const saw_cache_desc *cache, int32_t num_q_heads, const void *q,
                          const uint8_t *kv_pages, const void *scales,
                          const int32_t *block_table, int32_t max_blocks_per_seq,
                          const int32_t *seq_lens, int32_t num_seqs, float sm_scale,
                          float *out, void *workspace, size_t workspace_bytes,
                          uint32_t *dev_status, void *stream)
{
    return decode_impl(cache, num_q_heads, q, kv_pages, scales, block_table, max_blocks_per_seq,
                       seq_lens, num_seqs, sm_scale, out, workspace, workspace_bytes, dev_status,
                       stream, true);
}

int saw_paged_decode_attn_plain(const saw_cache_desc *cache, int32_t num_q_heads, const void *q,
                                const uint8_t *kv_pages, const void *scales,
                                const int32_t *block_table, int32_t max_blocks_per_seq,
                                const int32_t *seq_lens, int32_t num_seqs, float sm_scale,
                                float *out, void *workspace, size_t workspace_bytes,
                                uint32_t *dev_status, void *stream)
{
    return decode_impl(cache, num_q_heads, q, kv_pages, scales, block_table, max_blocks_per_seq,
                       seq_lens, num_seqs, sm_scale, out, workspace, workspace_bytes, dev_status,
                       stream, false);
}

int saw_decode_step(const saw_cache_desc *cache, int32_t num_q_heads, const void *q,
                    const void *k_new, const void *v_new, const int64_t *slot_mapping,
                    int64_t num_new_tokens, uint8_t *kv_pages, void *scales,
                    const int32_t *block_table, int32_t max_blocks_per_seq,
                    const int32_t *seq_lens, int32_t num_seqs, float sm_scale, float *out,
                    void *workspace, size_t workspace_bytes, uint32_t *dev_status,
                    void *stream)
{
    return step_impl(cache, num_q_heads, q, k_new, v_new, slot_mapping, num_new_tokens,
                     kv_pages, scales, block_table, max_blocks_per_seq, seq_lens, num_seqs,
                     sm_scale, out, workspace, workspace_bytes, dev_status, stream, true);
}

int saw_decode_step_plain(const saw_cache_desc *cache, int32_t num_q_heads, const void *q,
                          const void *k_new, const void *v_new, const int64_t *slot_mapping,
                          int64_t num_new_tokens, uint8_t *kv_pages, void *scales,
                          const int32_t *block_table, int32_t max_blocks_per_seq,
                          const int32_t *seq_lens, int32_t num_seqs, float sm_scale, float *out,
                          void *workspace, size_t workspace_bytes, uint32_t *dev_status,
                          void *stream)
{
    return step_impl(cache, num_q_heads, q, k_new, v_new, slot_mapping, num_new_tokens,
                     kv_pages, scales, block_table, max_blocks_per_seq, seq_lens, num_seqs,
                     sm_scale, out, workspace, workspace_bytes, dev_status, stream, false);
}

// ---- the uncompressed BF16 paged cache (baseline) -------------------------------------------

static int check_bf16_cache(const saw_cache_desc *cache)
{
    const int rc = check_cache(cache);
    if (rc != SAW_OK)
        return rc;
    if (cache->head_dim != 128)
        return SAW_ERR_UNSUPPORTED;
    // tensor-map rows (page * Hkv + h) * 64 must stay below 2^31
    if (cache->num_pages > (int64_t(1) << 31) / (int64_t(cache->num_kv_heads) * 64))
        return SAW_ERR_UNSUPPORTED;
    return SAW_OK;
}

static int append_bf16_impl(const saw_cache_desc *cache, const void *k, const void *v,
                            const int64_t *slot_mapping, int64_t num_tokens, void *kv_bf16,
                            uint32_t *dev_status, cudaStream_t stream)
{
    saw::AppendBf16Args a;
    a.k = k;
    a.v = v;
    a.slot_mapping = slot_mapping;
    a.num_tokens = num_tokens;
    a.num_kv_heads = cache->num_kv_heads;
    a.num_pages = cache->num_pages;
    a.kv = kv_bf16;
    a.status = dev_status;
    return saw::launch_append_bf16(a, stream) == cudaSuccess ? SAW_OK : SAW_ERR_CUDA;
}

int saw_append_bf16_paged(const saw_cache_desc *cache, const void *k, const void *v,
                          const int64_t *slot_mapping, int64_t num_tokens, void *kv_bf16,
                          uint32_t *dev_status, void *stream)
{
    int rc = check_bf16_cache(cache);
    if (rc != SAW_OK)
        return rc;
    rc = check_append(cache, k, v, slot_mapping, num_tokens,
                      static_cast<const uint8_t *>(kv_bf16), nullptr, true);
    if (rc != SAW_OK || num_tokens == 0)
        return rc;
    return append_bf16_impl(cache, k, v, slot_mapping, num_tokens, kv_bf16, dev_status,
                            static_cast<cudaStream_t>(stream));
}

size_t saw_paged_decode_bf16_workspace_bytes(const saw_cache_desc *cache, int32_t num_q_heads,
                                             int32_t num_seqs)
{
    if (check_bf16_cache(cache) != SAW_OK)
        return 0;
    return saw::decode_bf16_workspace_bytes(cache->num_kv_heads, num_q_heads, num_seqs);
}

static int decode_bf16_impl(const saw_cache_desc *cache, int32_t num_q_heads, const void *q,
                            const void *kv_bf16, const int32_t *block_table,
                            int32_t max_blocks_per_seq, const int32_t *seq_lens,
                            int32_t num_seqs, float sm_scale, float *out, void *workspace,
                            size_t workspace_bytes, uint32_t *dev_status, cudaStream_t stream,
                            bool programmatic)
{
    saw::DecodeArgs a = decode_args(cache, num_q_heads, q, static_cast<const uint8_t *>(kv_bf16),
                                    nullptr, block_table, max_blocks_per_seq, seq_lens, num_seqs,
                                    sm_scale, out, workspace, workspace_bytes, dev_status);
    a.rotate = false;
    return saw::launch_paged_decode_bf16(a, stream, programmatic) == cudaSuccess ? SAW_OK
                                                                                 : SAW_ERR_CUDA;
}

int saw_paged_decode_attn_bf16(const saw_cache_desc *cache, int32_t num_q_heads, const void *q,
                               const void *kv_bf16, const int32_t *block_table,
                               int32_t max_blocks_per_seq, const int32_t *seq_lens,
                               int32_t num_seqs, float sm_scale, float *out, void *workspace,
                               size_t workspace_bytes, uint32_t *dev_status, void *stream)
{
    int rc = check_bf16_cache(cache);
    if (rc != SAW_OK)
        return rc;
    rc = check_decode(cache, num_q_heads, q, static_cast<const uint8_t *>(kv_bf16), nullptr,
                      block_table, max_blocks_per_seq, seq_lens, num_seqs, sm_scale, out,
                      workspace, workspace_bytes, true);
    if (rc != SAW_OK || num_seqs == 0)
        return rc;
    return decode_bf16_impl(cache, num_q_heads, q, kv_bf16, block_table, max_blocks_per_seq,
                            seq_lens, num_seqs, sm_scale, out, workspace, workspace_bytes,
                            dev_status, static_cast<cudaStream_t>(stream), false);
}

int saw_decode_step_bf16(const saw_cache_desc *cache, int32_t num_q_heads, const void *q,
                         const void *k_new, const void *v_new, const int64_t *slot_mapping,
                         int64_t num_new_tokens, void *kv_bf16, const int32_t *block_table,
                         int32_t max_blocks_per_seq, const int32_t *seq_lens, int32_t num_seqs,
                         float sm_scale, float *out, void *workspace, size_t workspace_bytes,
                         uint32_t *dev_status, void *stream)
{
    int rc = check_bf16_cache(cache);
    if (rc != SAW_OK)
        return rc;
    rc = check_append(cache, k_new, v_new, slot_mapping, num_new_tokens,
                      static_cast<const uint8_t *>(kv_bf16), nullptr, true);
    if (rc != SAW_OK)
        return rc;
    rc = check_decode(cache, num_q_heads, q, static_cast<const uint8_t *>(kv_bf16), nullptr,
                      block_table, max_blocks_per_seq, seq_lens, num_seqs, sm_scale, out,
                      workspace, workspace_bytes, true);
    if (rc != SAW_OK)
        return rc;
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool appended = num_new_tokens > 0;
    if (appended) {
        rc = append_bf16_impl(cache, k_new, v_new, slot_mapping, num_new_tokens, kv_bf16,
                              dev_status, s);
        if (rc != SAW_OK)
            return rc;
    }
    if (num_seqs == 0)
        return SAW_OK;
    return decode_bf16_impl(cache, num_q_heads, q, kv_bf16, block_table, max_blocks_per_seq,
                            seq_lens, num_seqs, sm_scale, out, workspace, workspace_bytes,
                            dev_status, s, appended);
}

// ---- chunked-prefill attention over the INT4 cache -------------------------------------------

size_t saw_paged_prefill_workspace_bytes(const saw_cache_desc *cache, int32_t num_q_heads,
                                         int32_t num_seqs, int64_t total_q)
{
    if (check_cache(cache) != SAW_OK || num_q_heads <= 0 || total_q < 0 ||
        num_q_heads % cache->num_kv_heads != 0 || num_q_heads / cache->num_kv_heads > 16)
        return 0;
    return saw::decode_workspace_bytes(cache->num_kv_heads, num_q_heads, num_seqs, total_q,
                                       cache->head_dim);
}

static int prefill_impl(const saw_cache_desc *cache, int32_t num_q_heads, const void *q,
                        const int32_t *q_start, int64_t total_q, const uint8_t *kv_pages,
                        const void *scales, const int32_t *block_table, int32_t max_blocks_per_seq,
                        const int32_t *seq_lens, int32_t num_seqs, float sm_scale, float *out,
                        void *workspace, size_t workspace_bytes, uint32_t *dev_status,
                        void *stream, bool rotate)
{
    int rc = check_cache(cache);
    if (rc != SAW_OK)
        return rc;
    if (total_q < 0 || (num_seqs > 0 && (q_start == nullptr || !aligned(q_start, 4))) ||
        total_q > (int64_t(1) << 31) - 1)
        return SAW_ERR_INVALID_ARGUMENT;
    rc = check_decode(cache, num_q_heads, q, kv_pages, scales, block_table, max_blocks_per_seq,
                      seq_lens, num_seqs, sm_scale, out, workspace, workspace_bytes, false,
                      total_q);
    if (rc != SAW_OK || num_seqs == 0 || total_q == 0)
        return rc;
    saw::DecodeArgs a =
        decode_args(cache, num_q_heads, q, kv_pages, scales, block_table, max_blocks_per_seq,
                    seq_lens, num_seqs, sm_scale, out, workspace, workspace_bytes, dev_status);
    a.rotate = rotate;
    a.q_start = q_start;
    a.total_q = total_q;
    return saw::launch_paged_decode(a, static_cast<cudaStream_t>(stream), false) == cudaSuccess
               ? SAW_OK
               : SAW_ERR_CUDA;
}

int saw_paged_prefill_attn(const saw_cache_desc *cache, int32_t num_q_heads, const void *q,
                           const int32_t *q_start, int64_t total_q, const uint8_t *kv_pages,
                           const void *scales, const int32_t *block_table,
                           int32_t max_blocks_per_seq, const int32_t *seq_lens, int32_t num_seqs,
                           float sm_scale, float *out, void *workspace, size_t workspace_bytes,
                           uint32_t *dev_status, void *stream)
{
    return prefill_impl(cache, num_q_heads, q, q_start, total_q, kv_pages, scales, block_table,
                        max_blocks_per_seq, seq_lens, num_seqs, sm_scale, out, workspace,
                        workspace_bytes, dev_status, stream, true);
}

int saw_paged_prefill_attn_plain(const saw_cache_desc *cache, int32_t num_q_heads, const void *q,
                                 const int32_t *q_start, int64_t total_q, const uint8_t *kv_pages,
                                 const void *scales, const int32_t *block_table,
                                 int32_t max_blocks_per_seq, const int32_t *seq_lens,
                                 int32_t num_seqs, float sm_scale, float *out, void *workspace,
                                 size_t workspace_bytes, uint32_t *dev_status, void *stream)
{
    return prefill_impl(cache, num_q_heads, q, q_start, total_q, kv_pages, scales, block_table,
                        max_blocks_per_seq, seq_lens, num_seqs, sm_scale, out, workspace,
                        workspace_bytes, dev_status, stream, false);
}

// ---- full-precision sink / recent window beside the INT4 cache ------------------------------

static int check_window(const saw_cache_desc *cache, const saw_window_cache *win, int32_t num_seqs)
{
    if (win == nullptr || win->sink < 0 || win->recent < 0 || win->blocks < 0)
        return SAW_ERR_INVALID_ARGUMENT;
    if (cache->head_dim != 128)
        return SAW_ERR_UNSUPPORTED;   // the window pages use the bf16 page format: D = 128
    const int64_t W = int64_t(win->sink) + win->recent;
    if (W > int64_t(16) * win->blocks || W > (int64_t(1) << 30))
        return SAW_ERR_INVALID_ARGUMENT;
    if (num_seqs > 0 && W > 0) {
        if (win->kv == nullptr || win->table == nullptr || win->num_pages <= 0 ||
            !aligned(win->kv, 16) || !aligned(win->table, 4))
            return SAW_ERR_INVALID_ARGUMENT;
        // tensor-map rows (page * Hkv + h) * 64 of the window pages must stay below 2^31
        if (win->num_pages > (int64_t(1) << 31) / (int64_t(cache->num_kv_heads) * 64))
            return SAW_ERR_UNSUPPORTED;
    }
    return SAW_OK;
}

// workspace: the split-K slots of either part (they run one after the other), then the window
// part's per-row lse
static size_t window_partials_bytes(const saw_cache_desc *cache, int32_t num_q_heads,
                                    int32_t num_seqs)
{
    const size_t a = saw::decode_bf16_workspace_bytes(cache->num_kv_heads, num_q_heads, num_seqs);
    const size_t b = saw::decode_workspace_bytes(cache->num_kv_heads, num_q_heads, num_seqs, -1, 128);
    if (a == 0 || b == 0)
        return 0;
    return (std::max(a, b) + 255) / 256 * 256;
}

size_t saw_paged_decode_window_workspace_bytes(const saw_cache_desc *cache, int32_t num_q_heads,
                                               int32_t num_seqs)
{
    if (check_cache(cache) != SAW_OK || cache->head_dim != 128 || num_q_heads <= 0 ||
        num_seqs < 0 || num_q_heads % cache->num_kv_heads != 0 ||
        num_q_heads / cache->num_kv_heads > 16)
        return 0;
    const size_t part = window_partials_bytes(cache, num_q_heads, num_seqs);
    return part == 0 ? 0 : part + size_t(num_seqs) * num_q_heads * sizeof(float);
}

static int window_append_impl(const saw_cache_desc *cache, const saw_window_cache *win,
                              const void *k, const void *v, const int32_t *seq_lens,
                              int32_t num_seqs, uint8_t *kv_pages, void *scales,
                              const int32_t *block_table, int32_t max_blocks_per_seq,
                              uint32_t *dev_status, cudaStream_t stream)
{
    saw::WindowAppendArgs a;
    a.k = k;
    a.v = v;
    a.seq_lens = seq_lens;
    a.num_seqs = num_seqs;
    a.num_kv_heads = cache->num_kv_heads;
    a.w_sink = win->sink;
    a.w_recent = win->recent;
    a.win_kv = win->kv;
    a.num_win_pages = win->num_pages;
    a.win_table = win->table;
    a.win_blocks = win->blocks;
    a.kv_pages = kv_pages;
    a.scales = scales;
    a.num_pages = cache->num_pages;
    a.block_table = block_table;
    a.max_blocks = max_blocks_per_seq;
    a.status = dev_status;
    return saw::launch_window_append(a, stream) == cudaSuccess ? SAW_OK : SAW_ERR_CUDA;
}

static int check_window_append(const saw_cache_desc *cache, const saw_window_cache *win,
                               const void *k, const void *v, const int32_t *seq_lens,
                               int32_t num_seqs, const uint8_t *kv_pages, const void *scales,
                               const int32_t *block_table, int32_t max_blocks_per_seq)
{
    int rc = check_cache(cache);
    if (rc != SAW_OK)
        return rc;
    rc = check_window(cache, win, num_seqs);
    if (rc != SAW_OK || num_seqs == 0)
        return rc;
    if (num_seqs < 0 || !k || !v || !seq_lens || !kv_pages || !scales || !block_table ||
        max_blocks_per_seq <= 0 || !aligned(k, 16) || !aligned(v, 16) || !aligned(seq_lens, 4) ||
        !aligned(kv_pages, 16) || !aligned(scales, 16) || !aligned(block_table, 4))
        return SAW_ERR_INVALID_ARGUMENT;
    if (win->sink + win->recent == 0 && win->blocks == 0)
        return SAW_OK;
    if (win->kv == nullptr || win->table == nullptr)
        return SAW_ERR_INVALID_ARGUMENT;
    return SAW_OK;
}

static int decode_window_impl(const saw_cache_desc *cache, const saw_window_cache *win,
                              int32_t num_q_heads, const void *q, const uint8_t *kv_pages,
                              const void *scales, const int32_t *block_table,
                              int32_t max_blocks_per_seq, const int32_t *seq_lens,
                              int32_t num_seqs, float sm_scale, float *out, void *workspace,
                              size_t workspace_bytes, uint32_t *dev_status, cudaStream_t stream,
                              bool programmatic)
{
    const size_t part = window_partials_bytes(cache, num_q_heads, num_seqs);
    float *lse = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + part);
    saw::DecodeArgs a =
        decode_args(cache, num_q_heads, q, kv_pages, scales, block_table, max_blocks_per_seq,
                    seq_lens, num_seqs, sm_scale, out, workspace, workspace_bytes, dev_status);
    if (win->sink + win->recent == 0)   // no window: every token is quantized
        return saw::launch_paged_decode(a, stream, programmatic) == cudaSuccess ? SAW_OK
                                                                                : SAW_ERR_CUDA;
    a.win_sink = win->sink;
    a.win_recent = win->recent;
    a.lse = lse;
    // part 1: the window tokens from the bf16 window pages (writes out and lse)
    saw::DecodeArgs w = a;
    w.kv_pages = static_cast<const uint8_t *>(win->kv);
    w.scales = nullptr;
    w.block_table = win->table;
    w.max_blocks = win->blocks;
    w.num_pages = win->num_pages;
    w.rotate = false;
    w.win_part = 1;
    if (saw::launch_paged_decode_bf16(w, stream, programmatic) != cudaSuccess)
        return SAW_ERR_CUDA;
    // part 2: the quantized tokens, merged into out by the lse of part 1
    a.win_part = 2;
    return saw::launch_paged_decode(a, stream, true) == cudaSuccess ? SAW_OK : SAW_ERR_CUDA;
}

static int check_decode_window(const saw_cache_desc *cache, const saw_window_cache *win,
                               int32_t num_q_heads, const void *q, const uint8_t *kv_pages,
                               const void *scales, const int32_t *block_table,
                               int32_t max_blocks_per_seq, const int32_t *seq_lens,
                               int32_t num_seqs, float sm_scale, const float *out,
                               const void *workspace, size_t workspace_bytes)
{
    int rc = check_cache(cache);
    if (rc != SAW_OK)
        return rc;
    rc = check_window(cache, win, num_seqs);
    if (rc != SAW_OK)
        return rc;
    const size_t need = saw_paged_decode_window_workspace_bytes(cache, num_q_heads, num_seqs);
    // the INT4 checks, against the whole workspace (its first part holds the split-K slots)
    rc = check_decode(cache, num_q_heads, q, kv_pages, scales, block_table, max_blocks_per_seq,
                      seq_lens, num_seqs, sm_scale, out, workspace, workspace_bytes);
    if (rc != SAW_OK || num_seqs == 0)
        return rc;
    if (need == 0)
        return SAW_ERR_CUDA;
    if (workspace_bytes < need)
        return SAW_ERR_WORKSPACE;
    return SAW_OK;
}

int saw_window_append(const saw_cache_desc *cache, const saw_window_cache *win, const void *k,
                      const void *v, const int32_t *seq_lens, int32_t num_seqs, uint8_t *kv_pages,
                      void *scales, const int32_t *block_table, int32_t max_blocks_per_seq,
                      uint32_t *dev_status, void *stream)
{
    const int rc = check_window_append(cache, win, k, v, seq_lens, num_seqs, kv_pages, scales,
                                       block_table, max_blocks_per_seq);
    if (rc != SAW_OK || num_seqs == 0)
        return rc;
    return window_append_impl(cache, win, k, v, seq_lens, num_seqs, kv_pages, scales, block_table,
                              max_blocks_per_seq, dev_status, static_cast<cudaStream_t>(stream));
}

int saw_paged_decode_attn_window(const saw_cache_desc *cache, const saw_window_cache *win,
                                 int32_t num_q_heads, const void *q, const uint8_t *kv_pages,
                                 const void *scales, const int32_t *block_table,
                                 int32_t max_blocks_per_seq, const int32_t *seq_lens,
                                 int32_t num_seqs, float sm_scale, float *out, void *workspace,
                                 size_t workspace_bytes, uint32_t *dev_status, void *stream)
{
    const int rc = check_decode_window(cache, win, num_q_heads, q, kv_pages, scales, block_table,
                                       max_blocks_per_seq, seq_lens, num_seqs, sm_scale, out,
                                       workspace, workspace_bytes);
    if (rc != SAW_OK || num_seqs == 0)
        return rc;
    return decode_window_impl(cache, win, num_q_heads, q, kv_pages, scales, block_table,
                              max_blocks_per_seq, seq_lens, num_seqs, sm_scale, out, workspace,
                              workspace_bytes, dev_status, static_cast<cudaStream_t>(stream), false);
}

int saw_decode_step_window(const saw_cache_desc *cache, const saw_window_cache *win,
                           int32_t num_q_heads, const void *q, const void *k_new, const void *v_new,
                           uint8_t *kv_pages, void *scales, const int32_t *block_table,
                           int32_t max_blocks_per_seq, const int32_t *seq_lens, int32_t num_seqs,
                           float sm_scale, float *out, void *workspace, size_t workspace_bytes,
                           uint32_t *dev_status, void *stream)
{
    int rc = check_window_append(cache, win, k_new, v_new, seq_lens, num_seqs, kv_pages, scales,
                                 block_table, max_blocks_per_seq);
    if (rc != SAW_OK)
        return rc;
    rc = check_decode_window(cache, win, num_q_heads, q, kv_pages, scales, block_table,
                             max_blocks_per_seq, seq_lens, num_seqs, sm_scale, out, workspace,
                             workspace_bytes);
    if (rc != SAW_OK || num_seqs == 0)
        return rc;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    rc = window_append_impl(cache, win, k_new, v_new, seq_lens, num_seqs, kv_pages, scales,
                            block_table, max_blocks_per_seq, dev_status, st);
    if (rc != SAW_OK)
        return rc;
    return decode_window_impl(cache, win, num_q_heads, q, kv_pages, scales, block_table,
                              max_blocks_per_seq, seq_lens, num_seqs, sm_scale, out, workspace,
                              workspace_bytes, dev_status, st, true);
}

}  // extern "C"
