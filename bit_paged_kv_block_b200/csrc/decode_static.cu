// decode_static.cu -- saw_paged_decode_attn_static: the decode entry point for callers that
// cannot allocate device memory.
//
// saw_paged_decode_attn needs a caller-provided workspace (split-K partial results).  Some
// callers have no way to provide one: a plug-in running inside a serving
// framework that has already reserved the whole GPU for its own memory pool, a request path
// with a no-allocation rule (cudaMalloc synchronises the device and can stall every stream),
// or a host library that only ever receives pointers to inputs and outputs.  For them this
// entry point takes its scratch from one fixed array in device memory that is part of this
// library itself: kScratchBytes (18.3 MiB) on every GPU that loads the library, held until
// the process exits.  Nothing here calls cudaMalloc, cudaFree or any allocating routine.
//
// The scratch is shared by all calls on a device and keeps whatever the last call left in it,
// so calls whose kernels can overlap on the GPU (different streams, or several host threads)
// race on it and must be serialised by the caller.  Nothing in it needs to start at zero: every
// split-K partial is written by the decode kernel before the merge kernel reads it.
#include <cuda_runtime.h>

#include <mutex>

#include "saw.h"
#include "saw_internal.h"

namespace {

// Room for num_seqs * num_kv_heads * ceil(G / 8) <= 2048 decode segments and a decode grid of up
// to 2560 warps: (2560 + 2048) partial-result slots of 4160 bytes.
constexpr int kScratchMaxSegments = 2048;
constexpr size_t kScratchBytes = (2560 + kScratchMaxSegments) * size_t(4160);

static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device, looked up once per device and kept
// for the life of the process (a device reset would invalidate it; the header says so).
// In host code the symbol is only a host-side stand-in; the real address comes from
// cudaGetSymbolAddress with that device current.
int scratch_address(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return SAW_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr)
            return SAW_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return SAW_OK;
}

}  // namespace

extern "C" int saw_paged_decode_attn_static(const saw_cache_desc *cache, int32_t num_q_heads,
                                            const void *q, const uint8_t *kv_pages,
                                            const void *scales, const int32_t *block_table,
                                            int32_t max_blocks_per_seq, const int32_t *seq_lens,
                                            int32_t num_seqs, float sm_scale, float *out,
                                            uint32_t *dev_status, void *stream)
{
    if (cache == nullptr || cache->num_kv_heads <= 0 || num_seqs < 0)
        return SAW_ERR_INVALID_ARGUMENT;
    if (num_q_heads <= 0 || num_q_heads % cache->num_kv_heads != 0)
        return SAW_ERR_INVALID_ARGUMENT;
    const int64_t group = num_q_heads / cache->num_kv_heads;
    if (int64_t(num_seqs) * cache->num_kv_heads * ((group + 7) / 8) > kScratchMaxSegments)
        return SAW_ERR_SCRATCH_LIMIT;
    const size_t need = saw_paged_decode_workspace_bytes(cache, num_q_heads, num_seqs);
    if (num_seqs > 0 && need > kScratchBytes)
        return SAW_ERR_SCRATCH_LIMIT;
    void *scratch = nullptr;
    const int rc = scratch_address(&scratch);
    if (rc != SAW_OK)
        return rc;
    return saw_paged_decode_attn(cache, num_q_heads, q, kv_pages, scales, block_table,
                                 max_blocks_per_seq, seq_lens, num_seqs, sm_scale, out, scratch,
                                 kScratchBytes, dev_status, stream);
}
