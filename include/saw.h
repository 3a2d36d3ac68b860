/*
 * saw.h -- C ABI of libsaw: SAW-INT4 paged INT4 KV-cache compression on NVIDIA B200 (sm_100a).
 *
 * The method ("SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World LLM Serving",
 * Research Findings; restated on "Memory compression method reducing KV-cache size...", Core
 * Innovation and Summary) quantizes every new key/value head vector token-wise to INT4 after a
 * block-diagonal Hadamard rotation, inside one fused kernel that writes straight into a paged
 * KV cache, and reads that cache back with fused attention.  This library implements the two
 * halves of that path:
 *
 *   saw_rotate_quantize_paged  rotate + quantize + scatter new K/V vectors into the cache
 *   saw_paged_decode_attn      decode attention over the INT4 paged cache (split-K, GQA)
 *   saw_decode_step            one serving step: append one token per sequence, then decode
 *
 * Fixed build parameters (the pages give no numbers; these are the library's definition):
 *   head_dim D = 64, 128 or 256; Hadamard block B = min(D, 128) (a D = 256 vector is rotated
 *   as two independent 128-element blocks and keeps one (scale, zero) pair over all 256
 *   elements; a D = 64 vector holds no 128-element block and is rotated as one 64-element
 *   block); H is the Sylvester Hadamard matrix of order B in natural order,
 *   normalised by 1/sqrt(B), applied as an fp32 butterfly (stages h = 1, 2, ..., B/2,
 *   (x[j], x[j+h]) <- (x[j] + x[j+h], x[j] - x[j+h]), then a multiply by fp32(1/sqrt(B)),
 *   every step one IEEE fp32 operation); per (token, kv head) and separately for K and V:
 *   scale = (max - min) / 15 and zero = min in fp32, stored as fp16 (round to nearest even);
 *   code_i = clamp(rint((y_i - min) / scale), 0, 15) with IEEE division and ties to even;
 *   a vector whose fp32 scale is 0 stores scale +0 and all codes 0; a zero minimum is stored
 *   as +0; two codes per byte, the even index in the low nibble; pages of 16 tokens.
 *
 * Memory layout (all buffers caller-owned device memory, C-contiguous, 16-byte aligned):
 *   k, v (new tokens)   bf16   [T][Hkv][D]
 *   slot_mapping        int64  [T]        slot = page * 16 + offset; slot < 0 skips the token
 *   kv_pages            uint8  [num_pages][Hkv][2 (K, V)][16][D / 2]
 *                        so one (page, kv head) is one contiguous block of 16 D bytes (2 KiB
 *                        for D = 128): K codes then V codes, D / 2 bytes per token row
 *   scales              fp16   [num_pages][Hkv][2 (K, V)][16][2 (scale, zero)]
 *                        128 bytes per (page, kv head)
 *   q                   bf16   [S][Hq][D]      query head hq reads kv head hq / (Hq / Hkv)
 *   block_table         int32  [S][max_blocks_per_seq]  logical block -> page
 *   seq_lens            int32  [S]    tokens of each sequence in the cache (including the
 *                                     token appended by this step), 0 <= len <= 16 * max_blocks
 *   out                 fp32   [S][Hq][D]
 *
 * Ownership and threading: the library allocates no device memory.  Every call is
 * asynchronous on the given stream (a cudaStream_t passed as void*; NULL is the legacy
 * default stream) and returns as soon as its kernels are queued.  Calls on different streams
 * that share a workspace race.
 *
 * Errors: every entry point returns a saw_status.  Host-side checks (null pointers, sizes,
 * alignment, unsupported shapes) return before anything is queued.  Errors that only the
 * device can see -- a slot or page id out of range, a sequence length out of range, a bounded
 * wait that gave up -- never trap: the kernel skips the offending access, ORs a SAW_DEV_* bit
 * into *dev_status (when dev_status is not NULL) and carries on; the caller reads the word
 * after synchronising.  NaN or Inf inputs are not supported (their codes are unspecified).
 * Input range: a vector's rotated minimum and its scale must stay below fp16's largest finite
 * magnitude (65504; a value that rounds to 65520 or more is stored as infinity, as the
 * round-to-nearest conversion of the definition gives).  The rotation can grow a value by up to
 * sqrt(128) = 11.3 (a constant vector of -5800 already has a rotated minimum of -65600), so keys
 * and values beyond a few thousand in magnitude are out of range; the quantizer then still
 * stores the definition's bits but ORs SAW_DEV_RANGE into *dev_status.
 */
#ifndef SAW_H_
#define SAW_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum saw_status {
    SAW_OK = 0,
    SAW_ERR_INVALID_ARGUMENT = 1, /* null pointer, bad size, misalignment, Hq % Hkv != 0 */
    SAW_ERR_UNSUPPORTED = 2,      /* head_dim not 64 / 128 / 256 (BF16 cache: not 128), page_size
                                     != 16, Hq / Hkv > 16 */
    SAW_ERR_CUDA = 3,             /* a CUDA runtime call or kernel launch failed */
    SAW_ERR_WORKSPACE = 4,        /* workspace missing or smaller than required */
    SAW_ERR_SCRATCH_LIMIT = 5     /* shape too large for saw_paged_decode_attn_static */
} saw_status;

/* Bits ORed into *dev_status by the kernels. */
#define SAW_DEV_BAD_SLOT 0x1u     /* slot_mapping[t] >= num_pages * 16: token skipped */
#define SAW_DEV_BAD_PAGE 0x2u     /* block_table entry outside [0, num_pages): page 0 read */
#define SAW_DEV_BAD_SEQ_LEN 0x4u  /* seq_lens[s] < 0 or > 16 * max_blocks: output zeroed */
#define SAW_DEV_WAIT_TIMEOUT 0x8u /* a bounded wait on a page copy gave up */
#define SAW_DEV_RANGE 0x10u       /* a scale or zero point beyond fp16's range (|x| >= 65520) was
                                     stored as +-inf: that vector cannot be read back */

typedef struct saw_cache_desc {
    int32_t num_kv_heads; /* Hkv >= 1 */
    int32_t head_dim;     /* 64, 128 or 256 (the BF16 baseline cache: 128) */
    int32_t page_size;    /* must be 16 */
    int64_t num_pages;    /* pages in kv_pages / scales; num_pages * Hkv * 32 < 2^31 */
} saw_cache_desc;

/* Rotate, quantize and scatter T new tokens into the paged cache.
 * Follows "SAW-INT4" (Research Findings): the fused rotation-quantization kernel that writes
 * token-wise INT4 codes of Hadamard-rotated vectors directly into the paged KV cache.
 * k, v: bf16 [T][Hkv][D] device; slot_mapping: int64 [T] device; kv_pages, scales: the
 * cache (device, updated in place); dev_status: device uint32 or NULL.  T == 0 is a no-op.
 * Codes and scales are bit-identical to the definition above for every finite input. */
int saw_rotate_quantize_paged(const saw_cache_desc *cache, const void *k, const void *v,
                              const int64_t *slot_mapping, int64_t num_tokens,
                              uint8_t *kv_pages, void *scales, uint32_t *dev_status,
                              void *stream);

/* saw_rotate_quantize_paged (and its plain INT4 counterpart) for k and v that are not
 * contiguous, e.g. slices of a fused QKV projection output [T][(Hq + 2 Hkv) * D]: each
 * token's Hkv head vectors are contiguous (D bf16 each, head-major), and token t starts at
 * k + t * k_stride (v + t * v_stride) bf16 elements.  Strides are at least Hkv * D and a
 * multiple of 8 (every token starts on 16 bytes; k and v themselves 16-byte aligned).
 * Supported for Hkv a multiple or a divisor of the tile's 1024 / D vectors (16 for D = 64, 8 for
 * D = 128, 4 for D = 256; else SAW_ERR_UNSUPPORTED): the kernel copies whole tiles.  Results are bit-identical to the contiguous call on the same
 * values. */
int saw_rotate_quantize_paged_strided(const saw_cache_desc *cache, const void *k, int64_t k_stride,
                                      const void *v, int64_t v_stride, const int64_t *slot_mapping,
                                      int64_t num_tokens, uint8_t *kv_pages, void *scales,
                                      uint32_t *dev_status, void *stream);
int saw_quantize_paged_plain_strided(const saw_cache_desc *cache, const void *k, int64_t k_stride,
                                     const void *v, int64_t v_stride, const int64_t *slot_mapping,
                                     int64_t num_tokens, uint8_t *kv_pages, void *scales,
                                     uint32_t *dev_status, void *stream);

/* Bytes of workspace saw_paged_decode_attn / saw_decode_step need for this shape on the
 * current device (split-K partial results: one slot per warp of the decode grid plus one per
 * (seq, kv head)).  Returns 0 for an unsupported or invalid shape. */
size_t saw_paged_decode_workspace_bytes(const saw_cache_desc *cache, int32_t num_q_heads,
                                        int32_t num_seqs);

/* Zero a workspace (cudaMemsetAsync on the stream).  Optional: the decode never reads a
 * workspace byte it has not written in the same call. */
int saw_paged_decode_workspace_init(void *workspace, size_t workspace_bytes, void *stream);

/* Decode attention over the INT4 paged cache.
 * Follows "SAW-INT4" (Research Findings: fused attention execution over a paged cache) and
 * "BitDecoding-FP4" (abstract: stacked query heads over paged KV).  For each sequence s and
 * query head hq (kv head h = hq / G, G = Hq / Hkv <= 16; G > 8 runs as ceil(G / 8) groups of
 * query heads that each read the kv head's pages):
 *     q_r = H q,   s_t = sm_scale * <q_r, zero_t + code_t * scale_t>  for t < seq_lens[s],
 *     o_r = softmax(s) . (zero_t + code_t * scale_t) over the V side,   out = H o_r.
 * The kernel computes in fp16 x fp16 -> fp32 tensor-core tiles on raw codes with the scale
 * and zero applied in fp32 afterwards; results agree with an fp64 evaluation of the same
 * formula to about 1e-3.  A sequence with seq_lens[s] == 0 gets an all-zero output.
 * The work is cut into equal-cost runs of pages, one per warp of a persistent grid; sequences
 * split across warps are combined by a second kernel queued right after the first (as its
 * programmatic dependent), so one call queues two kernels.
 * workspace: device memory of at least saw_paged_decode_workspace_bytes() bytes, 256-byte
 * aligned; its contents need no initialisation and are scratch after the call. */
int saw_paged_decode_attn(const saw_cache_desc *cache, int32_t num_q_heads, const void *q,
                          const uint8_t *kv_pages, const void *scales,
                          const int32_t *block_table, int32_t max_blocks_per_seq,
                          const int32_t *seq_lens, int32_t num_seqs, float sm_scale,
                          float *out, void *workspace, size_t workspace_bytes,
                          uint32_t *dev_status, void *stream);

/* One serving step: saw_rotate_quantize_paged on the num_new_tokens tokens (k_new, v_new,
 * slot_mapping), then saw_paged_decode_attn, queued back to back on the stream (the decode
 * kernel is launched as a programmatic dependent of the append so that its launch and
 * prologue overlap the append; the split-K merge kernel follows the same way).  seq_lens must
 * already count the appended tokens. */
int saw_decode_step(const saw_cache_desc *cache, int32_t num_q_heads, const void *q,
                    const void *k_new, const void *v_new, const int64_t *slot_mapping,
                    int64_t num_new_tokens, uint8_t *kv_pages, void *scales,
                    const int32_t *block_table, int32_t max_blocks_per_seq,
                    const int32_t *seq_lens, int32_t num_seqs, float sm_scale, float *out,
                    void *workspace, size_t workspace_bytes, uint32_t *dev_status,
                    void *stream);

/* Plain INT4 baseline (H = I): the same token-wise asymmetric INT4 quantizer, page layout and
 * decode kernels without the Hadamard rotation -- the "naive INT4" the SAW-INT4 page compares
 * against ("SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World LLM Serving",
 * Concerns Raised: naive INT4 degrades accuracy; Research Findings: SAW-INT4 matches the
 * throughput of plain INT4 and its fused rotation adds no measurable overhead).  Arguments,
 * layouts, workspace and status codes are those of the rotated entry points; a cache written by
 * saw_quantize_paged_plain must be read by the *_plain decode (codes are not rotated, and q and
 * the output are not rotated either).  Codes and scales are bit-identical to the definition at
 * the top of this file with the rotation step removed. */
int saw_quantize_paged_plain(const saw_cache_desc *cache, const void *k, const void *v,
                             const int64_t *slot_mapping, int64_t num_tokens, uint8_t *kv_pages,
                             void *scales, uint32_t *dev_status, void *stream);
int saw_paged_decode_attn_plain(const saw_cache_desc *cache, int32_t num_q_heads, const void *q,
                                const uint8_t *kv_pages, const void *scales,
                                const int32_t *block_table, int32_t max_blocks_per_seq,
                                const int32_t *seq_lens, int32_t num_seqs, float sm_scale,
                                float *out, void *workspace, size_t workspace_bytes,
                                uint32_t *dev_status, void *stream);
int saw_decode_step_plain(const saw_cache_desc *cache, int32_t num_q_heads, const void *q,
                          const void *k_new, const void *v_new, const int64_t *slot_mapping,
                          int64_t num_new_tokens, uint8_t *kv_pages, void *scales,
                          const int32_t *block_table, int32_t max_blocks_per_seq,
                          const int32_t *seq_lens, int32_t num_seqs, float sm_scale, float *out,
                          void *workspace, size_t workspace_bytes, uint32_t *dev_status,
                          void *stream);

/* Chunked-prefill attention over the INT4 paged cache: the read step for a chunk of new tokens
 * whose K/V were already appended with saw_rotate_quantize_paged ("SAW-INT4: System-Aware
 * 4-Bit KV-Cache Quantization for Real-World LLM Serving", Research Findings: the quantized
 * cache must serve fused attention over paged memory; a prefill chunk is its multi-query case).
 * Sequence s has C_s = q_start[s + 1] - q_start[s] query tokens (rows q_start[s] .. of q and
 * out), the last C_s of its seq_lens[s] cached tokens; query i sits at position
 * seq_lens[s] - C_s + i and attends causally to cache tokens 0 .. seq_lens[s] - C_s + i, with
 * the rotation, scales and arithmetic of saw_paged_decode_attn (a decode is the case C_s = 1).
 *     q: bf16 [total_q][Hq][D]; out: fp32 [total_q][Hq][D]; q_start: int32 [num_seqs + 1],
 *     device, non-decreasing, q_start[0] = 0, q_start[num_seqs] = total_q, 0 <= C_s <= seq_lens[s]
 *     (a violating sequence is flagged SAW_DEV_BAD_SEQ_LEN and skipped).
 * Two kernels serve the call.  At D = 128, when the chunks average at least half a 128-row tile
 * per sequence (total_q G >= 64 num_seqs), a tensor-core kernel (tcgen05) takes tiles of 128 / G
 * query tokens x G heads and walks each tile's causal range of the cache once (the repeated reads
 * of a page by the tiles of one sequence come from L2).  Otherwise, and at D = 64 or 256, the
 * decode kernel runs with segments of 8 (query token, head) rows, whose K/V traffic is about
 * total_q G / 8 times that of one decode of the batch.  The tensor-core kernel's arithmetic
 * keeps its fp16 operands in fp16's normal range (queries scaled by 2^8, weights by 2^4): results
 * agree with the decode kernel's within the attention tolerance, not bit for bit.  workspace: at
 * least saw_paged_prefill_workspace_bytes() bytes, 256-byte aligned, no initialisation needed.
 * The _plain variant reads a cache written by saw_quantize_paged_plain. */
size_t saw_paged_prefill_workspace_bytes(const saw_cache_desc *cache, int32_t num_q_heads,
                                         int32_t num_seqs, int64_t total_q);
int saw_paged_prefill_attn(const saw_cache_desc *cache, int32_t num_q_heads, const void *q,
                           const int32_t *q_start, int64_t total_q, const uint8_t *kv_pages,
                           const void *scales, const int32_t *block_table,
                           int32_t max_blocks_per_seq, const int32_t *seq_lens, int32_t num_seqs,
                           float sm_scale, float *out, void *workspace, size_t workspace_bytes,
                           uint32_t *dev_status, void *stream);
int saw_paged_prefill_attn_plain(const saw_cache_desc *cache, int32_t num_q_heads, const void *q,
                                 const int32_t *q_start, int64_t total_q, const uint8_t *kv_pages,
                                 const void *scales, const int32_t *block_table,
                                 int32_t max_blocks_per_seq, const int32_t *seq_lens,
                                 int32_t num_seqs, float sm_scale, float *out, void *workspace,
                                 size_t workspace_bytes, uint32_t *dev_status, void *stream);

/* The uncompressed BF16 paged KV cache: the baseline the INT4 format is measured against
 * ("SAW-INT4: System-Aware 4-Bit KV-Cache Quantization for Real-World LLM Serving", Research
 * Findings: serving throughput against a 16-bit KV cache; "BitDecoding-FP4: Native FP4 KV
 * Cache Decoding via Algorithm-System Co-Design", abstract: speedup over BF16 KV decoding).
 * Same page geometry without quantization, scales or rotation:
 *     kv_bf16: bf16 [num_pages][Hkv][2 (K, V)][16][128], 8 KiB per (page, kv head), 16-byte
 *     aligned; num_pages * Hkv * 64 < 2^31.
 * saw_append_bf16_paged scatters T tokens exactly (the stored bits are the input bits);
 * saw_paged_decode_attn_bf16 computes, for each sequence s and query head hq (kv head
 * h = hq / G, G <= 16), softmax(sm_scale <q, k_t>) . v over t < seq_lens[s] with bf16 x bf16
 * tensor-core products accumulated in fp32 (results agree with fp64 to about 1e-3); its
 * workspace comes from saw_paged_decode_bf16_workspace_bytes (no initialisation needed).
 * saw_decode_step_bf16 is the append followed by the decode on one stream, as saw_decode_step.
 * Arguments, ownership, alignment and status codes are those of the INT4 entry points. */
int saw_append_bf16_paged(const saw_cache_desc *cache, const void *k, const void *v,
                          const int64_t *slot_mapping, int64_t num_tokens, void *kv_bf16,
                          uint32_t *dev_status, void *stream);
size_t saw_paged_decode_bf16_workspace_bytes(const saw_cache_desc *cache, int32_t num_q_heads,
                                             int32_t num_seqs);
int saw_paged_decode_attn_bf16(const saw_cache_desc *cache, int32_t num_q_heads, const void *q,
                               const void *kv_bf16, const int32_t *block_table,
                               int32_t max_blocks_per_seq, const int32_t *seq_lens,
                               int32_t num_seqs, float sm_scale, float *out, void *workspace,
                               size_t workspace_bytes, uint32_t *dev_status, void *stream);
int saw_decode_step_bf16(const saw_cache_desc *cache, int32_t num_q_heads, const void *q,
                         const void *k_new, const void *v_new, const int64_t *slot_mapping,
                         int64_t num_new_tokens, void *kv_bf16, const int32_t *block_table,
                         int32_t max_blocks_per_seq, const int32_t *seq_lens, int32_t num_seqs,
                         float sm_scale, float *out, void *workspace, size_t workspace_bytes,
                         uint32_t *dev_status, void *stream);

/* saw_paged_decode_attn for callers that cannot allocate device memory.
 * The pages have no counterpart of this entry point: it exists for callers that are not allowed
 * or not able to call cudaMalloc -- a plug-in inside a serving framework whose memory pool
 * already owns the GPU, a request path that must not allocate (cudaMalloc synchronises the
 * device), or a host library that is only ever handed input and output pointers.  It computes
 * exactly what saw_paged_decode_attn computes, but its split-K scratch lives in one fixed array
 * of 18.3 MiB inside this library's device code (present on every GPU that loads the library,
 * until the process exits) instead of a caller workspace.  It allocates nothing.
 * Limit: num_seqs * num_kv_heads * ceil(G / 8) <= 2048 and a decode grid of at most 2560 warps
 * (a B200 runs 2368), and the workspace the shape needs must fit the array (D = 256 slots are
 * twice as large: about 550 segments on a B200); larger shapes return SAW_ERR_SCRATCH_LIMIT
 * before anything is queued.
 * The first call on each device looks up the array's device address (cudaGetSymbolAddress with
 * that device current) and keeps it for the life of the process; make that first call before
 * any stream capture.  A cudaDeviceReset (or any other teardown of the device's primary
 * context) invalidates the kept address: do not call this entry point on that device after
 * one.  Nothing in the array
 * needs to start at zero.  All calls on a device share the array and it keeps the previous
 * call's contents, so calls that can overlap on the GPU (other streams, other host threads)
 * race on it: the caller must serialise them.
 * Arguments, layouts and the other status codes are those of saw_paged_decode_attn. */
int saw_paged_decode_attn_static(const saw_cache_desc *cache, int32_t num_q_heads,
                                 const void *q, const uint8_t *kv_pages, const void *scales,
                                 const int32_t *block_table, int32_t max_blocks_per_seq,
                                 const int32_t *seq_lens, int32_t num_seqs, float sm_scale,
                                 float *out, uint32_t *dev_status, void *stream);

/* Human-readable text of a saw_status (never NULL). */
const char *saw_status_string(int status);

/* Library ABI version: 100 * major + minor. */
int saw_version(void);

/* ---- full-precision sink / recent window beside the INT4 cache ----------------------------
 *
 * "InnerQ: Hardware-Aware Tuning-Free Quantization of KV Cache for Large Language Models",
 * Abstract and Figure 2: a small high-precision window of attention-sink tokens and recent
 * tokens is kept beside the quantized cache; the attention over the quantized part and over the
 * window are computed separately and merged.  Layout (the pages give none; head_dim 128):
 *   - of a sequence of L tokens, positions p < sink are sinks and positions
 *     p >= max(sink, L - recent) are recent: min(L, W) window tokens, W = sink + recent, kept in
 *     bf16.  Window slot of p: p for a sink, sink + (p - sink) mod recent for a recent token;
 *     slot i of sequence s lives in window page table[s * blocks + i / 16] at offset i mod 16 of
 *     kv, bf16 [num_pages][Hkv][2 (K, V)][16][128] (the layout of the bf16 baseline cache);
 *   - the other max(0, L - W) tokens are rotated INT4 in the ordinary paged cache (kv_pages,
 *     scales), as their own sequence: position p is quantized index j = p - sink, at page
 *     block_table[s][j / 16], offset j mod 16.
 * The decode attends over the window (bf16 arithmetic of saw_paged_decode_attn_bf16) and over the
 * quantized tokens (that of saw_paged_decode_attn), and merges the two results by their softmax
 * denominators, so the output is one softmax over all L tokens. */
typedef struct saw_window_cache {
    int32_t sink;            /* sink tokens kept in bf16, >= 0 */
    int32_t recent;          /* most recent tokens kept in bf16, >= 0 */
    void *kv;                /* device: bf16 window pages [num_pages][Hkv][2][16][128] */
    int64_t num_pages;       /* pages in kv; num_pages * Hkv * 64 < 2^31 */
    const int32_t *table;    /* device: int32 [num_seqs][blocks] window pages per sequence */
    int32_t blocks;          /* row stride of table; sink + recent <= 16 * blocks */
} saw_window_cache;

/* Workspace bytes saw_paged_decode_attn_window / saw_decode_step_window need (0 if the shape is
 * unsupported: head_dim != 128, Hq / Hkv > 16). */
size_t saw_paged_decode_window_workspace_bytes(const saw_cache_desc *cache, int32_t num_q_heads,
                                               int32_t num_seqs);

/* One serving step's write: sequence s's new token (k, v: bf16 [num_seqs][Hkv][128], device) sits
 * at position p = seq_lens[s] - 1.  A sink takes window slot p.  Otherwise it takes its slot in the
 * recent ring, and the token it displaces there (position p - recent, when that is not a sink) is
 * rotated, quantized and scattered into kv_pages / scales at quantized index p - recent - sink,
 * with the arithmetic of saw_rotate_quantize_paged (bit-identical codes and scales).  With
 * recent = 0 the new token itself is quantized at index p - sink.  A sequence with
 * seq_lens[s] <= 0 is skipped (negative: SAW_DEV_BAD_SEQ_LEN); a window or INT4 page id out of
 * range, or a quantized index past max_blocks_per_seq, leaves the pair untouched and sets
 * SAW_DEV_BAD_PAGE / SAW_DEV_BAD_SEQ_LEN. */
int saw_window_append(const saw_cache_desc *cache, const saw_window_cache *win, const void *k,
                      const void *v, const int32_t *seq_lens, int32_t num_seqs, uint8_t *kv_pages,
                      void *scales, const int32_t *block_table, int32_t max_blocks_per_seq,
                      uint32_t *dev_status, void *stream);

/* Decode attention of q (bf16 [num_seqs][Hq][128]) over the window and the quantized tokens of
 * each sequence (seq_lens[s] tokens in all, including the newest) into out (fp32
 * [num_seqs][Hq][128]).  workspace: at least saw_paged_decode_window_workspace_bytes(), 256-byte
 * aligned.  Launches the window part, then the quantized part as a programmatic dependent. */
int saw_paged_decode_attn_window(const saw_cache_desc *cache, const saw_window_cache *win,
                                 int32_t num_q_heads, const void *q, const uint8_t *kv_pages,
                                 const void *scales, const int32_t *block_table,
                                 int32_t max_blocks_per_seq, const int32_t *seq_lens,
                                 int32_t num_seqs, float sm_scale, float *out, void *workspace,
                                 size_t workspace_bytes, uint32_t *dev_status, void *stream);

/* saw_window_append then saw_paged_decode_attn_window on one stream (the decode launched as a
 * programmatic dependent of the append). */
int saw_decode_step_window(const saw_cache_desc *cache, const saw_window_cache *win,
                           int32_t num_q_heads, const void *q, const void *k_new, const void *v_new,
                           uint8_t *kv_pages, void *scales, const int32_t *block_table,
                           int32_t max_blocks_per_seq, const int32_t *seq_lens, int32_t num_seqs,
                           float sm_scale, float *out, void *workspace, size_t workspace_bytes,
                           uint32_t *dev_status, void *stream);

#ifdef __cplusplus
} /* extern "C" */
#endif

#endif /* SAW_H_ */
