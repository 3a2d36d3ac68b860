// saw_internal.h -- launchers shared between the C-ABI layer and the kernel translation units.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

namespace saw {

// cuTensorMapEncodeTiled from the driver, looked up through the runtime (no libcuda link).
inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            ptr = nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }();
    return fn;
}

struct RotateQuantizeArgs {
    const void *k;               // bf16 [T][Hkv][128]
    const void *v;               // bf16 [T][Hkv][128]
    const int64_t *slot_mapping; // [T]
    int64_t num_tokens;
    int32_t num_kv_heads;
    int32_t head_dim = 128;      // D: 128 or 256 (two 128-point rotation blocks)
    int64_t num_pages;
    uint8_t *kv_pages;           // [num_pages][Hkv][2][16][D / 2]
    void *scales;                // fp16 [num_pages][Hkv][2][16][2]
    uint32_t *status;            // nullable
    bool rotate = true;          // false: plain INT4 (no Hadamard rotation)
    int64_t k_stride = 0;        // bf16 elements between tokens of k (0: contiguous, Hkv * 128)
    int64_t v_stride = 0;        // the same for v
};

struct DecodeArgs {
    const void *q;               // bf16 [S][Hq][D]
    const uint8_t *kv_pages;
    const void *scales;
    const int32_t *block_table;  // [S][max_blocks]
    int32_t max_blocks;
    const int32_t *seq_lens;     // [S]
    int32_t num_seqs;
    int32_t num_q_heads;
    int32_t num_kv_heads;
    int64_t num_pages;
    float sm_scale;
    float *out;                  // fp32 [S][Hq][D]
    void *workspace;
    size_t workspace_bytes;
    uint32_t *status;
    bool rotate = true;          // false: plain INT4 cache (no query / output rotation)
    const int32_t *q_start = nullptr;   // chunked prefill: [S + 1] query-row offsets (else decode)
    int64_t total_q = 0;         // chunked prefill: query rows (q_start[S])
    int32_t head_dim = 128;      // D: 64, 128 or 256 (INT4 cache only)
    // windowed decode: 1 = the window part (bf16 pages), 2 = the quantized part (merged into
    // out with the window part's lse); 0 = a plain decode
    int32_t win_part = 0;
    int32_t win_sink = 0, win_recent = 0;
    float *lse = nullptr;        // [S][Hq] log2 softmax denominators of the window part
};

struct AppendBf16Args {
    const void *k;               // bf16 [T][Hkv][128]
    const void *v;               // bf16 [T][Hkv][128]
    const int64_t *slot_mapping; // [T]
    int64_t num_tokens;
    int32_t num_kv_heads;
    int64_t num_pages;
    void *kv;                    // bf16 [num_pages][Hkv][2][16][128]
    uint32_t *status;            // nullable
};

// Queue the rotate+quantize+scatter kernel.  `trigger_dependents` makes the kernel release
// a programmatic dependent launch early.  Returns a cudaError_t.
cudaError_t launch_rotate_quantize(const RotateQuantizeArgs &a, cudaStream_t stream,
                                   bool trigger_dependents);

// Workspace bytes the decode kernel needs on the current device (0 if the shape is invalid);
// total_q >= 0: a chunked prefill over total_q query rows.
size_t decode_workspace_bytes(int32_t num_kv_heads, int32_t num_q_heads, int32_t num_seqs,
                              int64_t total_q = -1, int32_t head_dim = 128);

// Queue the decode kernel; `programmatic` launches it as a programmatic dependent of the
// previous kernel on the stream.  Returns a cudaError_t.
cudaError_t launch_paged_decode(const DecodeArgs &a, cudaStream_t stream, bool programmatic);

// Chunked prefill at head_dim 128 on the tensor cores (tcgen05): one CTA per tile of up to 128
// query rows; no workspace.  prefill_tc_grid: the CTAs a launch takes (an upper bound on tiles).
cudaError_t launch_prefill_tc(const DecodeArgs &a, cudaStream_t stream, bool programmatic);
int64_t prefill_tc_grid(int32_t num_kv_heads, int32_t num_q_heads, int32_t num_seqs, int64_t total_q);

// The uncompressed BF16 paged cache (baseline): scatter, decode workspace size, decode
// (DecodeArgs::kv_pages is the bf16 cache; scales and rotate are unused).
cudaError_t launch_append_bf16(const AppendBf16Args &a, cudaStream_t stream);

struct WindowAppendArgs {
    const void *k;               // new tokens, bf16 [S][Hkv][128]: one per sequence
    const void *v;
    const int32_t *seq_lens;     // [S], including the new token
    int32_t num_seqs;
    int32_t num_kv_heads;
    int32_t w_sink, w_recent;
    void *win_kv;                // bf16 window pages [num_win_pages][Hkv][2][16][128]
    int64_t num_win_pages;
    const int32_t *win_table;    // [S][win_blocks]
    int32_t win_blocks;
    uint8_t *kv_pages;           // INT4 pages of the quantized tokens
    void *scales;
    int64_t num_pages;
    const int32_t *block_table;  // [S][max_blocks], indexed by quantized position
    int32_t max_blocks;
    uint32_t *status;            // nullable
};

// Queue the window append: per sequence and kv head, the token leaving the recent window is
// rotated, quantized and scattered into the INT4 pages, and the new token takes its slot.
cudaError_t launch_window_append(const WindowAppendArgs &a, cudaStream_t stream);
size_t decode_bf16_workspace_bytes(int32_t num_kv_heads, int32_t num_q_heads, int32_t num_seqs,
                                   int64_t total_q = -1);
cudaError_t launch_paged_decode_bf16(const DecodeArgs &a, cudaStream_t stream, bool programmatic);

}  // namespace saw
