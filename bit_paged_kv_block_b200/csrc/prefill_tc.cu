// prefill_tc.cu -- chunked-prefill attention over the INT4 paged cache on the 5th-generation
// tensor cores (tcgen05.mma, accumulators in tensor memory).
//
// The read step for a chunk of new tokens whose K/V are already in the cache ("SAW-INT4:
// System-Aware 4-Bit KV-Cache Quantization for Real-World LLM Serving", Research Findings: the
// quantized cache must serve fused attention over paged memory; a prefill chunk is the
// multi-query case).  Sequence s has C query tokens, the last C of its L cached tokens; query i
// attends causally to cache tokens 0 .. L - C + i.  The arithmetic is the decode's: the query is
// rotated by the same Hadamard transform and scaled by sm_scale log2(e) and 1/sqrt(128); logits
// are s = scale_K acc + zero_K sum(q) over the raw codes; P' = p scale_V meets the raw V codes
// and sum p zero_V is added in fp32; the output is rotated back.
//
// A CTA (8 warps, 2 per SM) owns one tile of up to 128 query rows: T = 128 / G consecutive query
// tokens x the G query heads of one kv head, row r = token (r / G), head (r % G).  It walks the
// tile's causal range of the cache in blocks of 64 tokens (4 pages) with two roles:
//   - producers (warps 4-7) load each block's code words and scales straight into registers, two
//     blocks ahead (block-table ids three ahead), unpack them into fp16 tiles K and V [64 tokens x
//     128 d] (V double-buffered; token rows of 128 B per half of d, 128-byte swizzle), write the
//     block's scale table (a ring of 4), and one of them issues S = Q K^T (M 128, N 64, K 128:
//     8 x tcgen05.mma.kind::f16) into one of two S buffers in tensor memory;
//   - softmax warps (0-3) read S with tcgen05.ld.16x256b, which gives each thread 4 rows x 16
//     tokens (rows r, r + 8 of each 16-lane half, r = lane / 4; tokens 8 k + 2 (lane % 4), + 1), so
//     a scale-table entry loaded once serves 4 rows and a row's maximum is combined over the 4
//     threads of a quad by two shuffles; they apply scales, zero points and the causal limit, run
//     the online softmax one 16-lane half at a time, write P' (fp16) to a shared tile by stmatrix,
//     and thread 0 issues O += P' V (M 128, N 128, K 64: 4 MMAs, V the MN-major operand).
// The roles hand off through mbarriers: the tensor cores' commits (S and P' V done), the softmax's
// release of an S buffer, and the producers' V and scale-table arrivals; each role also meets at
// its own named barrier once per block.  So the tensor cores compute S of block kb + 1 while the
// softmax runs on block kb, and the producers unpack block kb + 2 meanwhile.  When a block's
// maximum exceeds a row's running maximum, the row's O accumulator is rescaled in tensor memory
// (a half warp's rows together; rows without a change multiply by 1).  Letting the maximum lag
// saved little time and doubled the largest error (weights kept in fp16's normal range then flush
// more of the small ones).  The epilogue reads each half of an O row (two threads per row), adds
// the zero-point term, divides by the row sum and rotates back (the last Hadamard stage pairs the
// halves through shared memory).
//
// Codes enter the tensor cores as exact fp16 integers n = (1024 + n) - 1024 (a magic OR and one
// half2 subtraction per pair).  These tensor cores flush fp16 subnormals, so the operands are kept
// normal: the query enters scaled by 2^8 (logit = (scale_K acc + zero_K sq) / 2^8, sq the sum of the
// fp16 query entries), and the weights as P' = 2^4 p scale_V with p <= 1 (O = O_acc / 2^4 +
// sum p zero_V), so only weights below about 2^-14 of a row's maximum fall under fp16's normal
// range.  A 32-bit word of 8 codes (d .. d + 7) gives the fp16 pairs (d, d+4), (d+1, d+5),
// (d+2, d+6), (d+3, d+7); Q is written in that d order, and the epilogue reads O's columns back
// through it.
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "saw_device.cuh"
#include "saw_internal.h"

namespace saw {
namespace {

constexpr int kTcThreads = 256;
constexpr int kTcRows = 128;                 // M of the MMAs: query rows per tile
constexpr int kTcBlockTokens = 64;           // N of QK, K of PV: cache tokens per block
constexpr int kTcBlockPages = kTcBlockTokens / kPageSize;
constexpr float kTcHadamardC = 0.0883883461356163f;
constexpr float kTcRescale = 0.0f;           // move the running max whenever a block exceeds it
constexpr float kTcQScale = 256.0f;          // query entries enter the MMA scaled by 2^8
constexpr float kTcPScale = 16.0f;           // weights enter the MMA scaled by 2^4
constexpr uint64_t kTcWaitLimitNs = 1000000000ull;

// shared memory (from a 1024-byte aligned base); 2 CTAs fit on an SM
constexpr int kSmQ = 0;                                  // Q tile: 2 x [128 rows][128 B]
constexpr int kSmK = kSmQ + 2 * kTcRows * 128;           // K tile: 2 x [64 tokens][128 B]
constexpr int kSmV = kSmK + 2 * kTcBlockTokens * 128;    // 2 V tiles: 2 x [64 tokens][128 B] each
constexpr int kSmVTile = 2 * kTcBlockTokens * 128;
constexpr int kSmP = kSmV + 2 * kSmVTile;                // P' tile: [128 rows][128 B]
constexpr int kSmScales = kSmP + kTcRows * 128;          // 4 x (K, V) token-pair factors
constexpr int kSmScaleSet = 2 * 2 * kTcBlockTokens * 4;
constexpr int kSmXchg = kSmScales + 4 * kSmScaleSet;     // per row: the query halves' sums, then l, z
constexpr int kSmBars = kSmXchg + 4 * kTcRows * 4;       // 12 mbarriers, tmem addr, flags
constexpr int kSmTile = kSmBars + 128;                   // tile descriptor
constexpr int kSmBytes = kSmTile + 64;
constexpr size_t kTcSmemBytes = 1024 + kSmBytes;
constexpr uint32_t kTmemCols = 256;                      // O: columns 0..127, S: 128..255 (2 x 64)

// byte offset of 16-bit element (row, k) in a tile of rows of 64 elements (128 B) per atom,
// atom stride atom_bytes, 128-byte swizzle (16-byte chunk index XOR row mod 8)
__device__ __forceinline__ uint32_t sw128_chunk(int row, int chunk16, uint32_t atom_bytes)
{
    return static_cast<uint32_t>((chunk16 >> 3) * atom_bytes + row * 128 + (((chunk16 & 7) ^ (row & 7)) << 4));
}

// tcgen05 shared-memory matrix descriptor: 128-byte swizzle, version 1 (sm_100), base offset 0
__device__ __forceinline__ uint64_t umma_desc(uint32_t addr, uint32_t lbo, uint32_t sbo)
{
    uint64_t d = static_cast<uint64_t>((addr >> 4) & 0x3FFF);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFF) << 16;
    d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFF) << 32;
    d |= static_cast<uint64_t>(1) << 46;
    d |= static_cast<uint64_t>(2) << 61;
    return d;
}

// instruction descriptor of kind::f16: fp16 A and B, fp32 accumulator, M x N, A / B K- or
// MN-major
__host__ __device__ constexpr uint32_t umma_idesc(int m, int n, int a_mn, int b_mn)
{
    return (1u << 4) | (static_cast<uint32_t>(a_mn) << 15) | (static_cast<uint32_t>(b_mn) << 16) |
           (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(m >> 4) << 24);
}

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                 ::"r"(tmem_d), "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
                 : "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void async_proxy_fence() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// 32 consecutive fp32 columns of this thread's tensor-memory lane
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float v[32])
{
    uint32_t r[32];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
                 "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
                   "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
                   "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
                   "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; i++)
        v[i] = __uint_as_float(r[i]);
}


// tcgen05.ld.16x256b.x8 of one 16-lane half (32 columns per thread's pair of rows), waited for
__device__ __forceinline__ void tmem_ld_16x256b_x8(uint32_t ta, float v[32])
{
    uint32_t *a = reinterpret_cast<uint32_t *>(v);
    asm volatile("tcgen05.ld.sync.aligned.16x256b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
                 "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
                 "tcgen05.wait::ld.sync.aligned;"
                 : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]), "=r"(a[4]), "=r"(a[5]), "=r"(a[6]), "=r"(a[7]),
                   "=r"(a[8]), "=r"(a[9]), "=r"(a[10]), "=r"(a[11]), "=r"(a[12]), "=r"(a[13]), "=r"(a[14]), "=r"(a[15]),
                   "=r"(a[16]), "=r"(a[17]), "=r"(a[18]), "=r"(a[19]), "=r"(a[20]), "=r"(a[21]), "=r"(a[22]), "=r"(a[23]),
                   "=r"(a[24]), "=r"(a[25]), "=r"(a[26]), "=r"(a[27]), "=r"(a[28]), "=r"(a[29]), "=r"(a[30]), "=r"(a[31])
                 : "r"(ta)
                 : "memory");
}

// the matching store (no wait)
__device__ __forceinline__ void tmem_st_16x256b_x8(uint32_t ta, const float v[32])
{
    const uint32_t *a = reinterpret_cast<const uint32_t *>(v);
    asm volatile("tcgen05.st.sync.aligned.16x256b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
                 "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
                 ::"r"(ta), "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(a[4]), "r"(a[5]), "r"(a[6]), "r"(a[7]),
                   "r"(a[8]), "r"(a[9]), "r"(a[10]), "r"(a[11]), "r"(a[12]), "r"(a[13]), "r"(a[14]), "r"(a[15]),
                   "r"(a[16]), "r"(a[17]), "r"(a[18]), "r"(a[19]), "r"(a[20]), "r"(a[21]), "r"(a[22]), "r"(a[23]),
                   "r"(a[24]), "r"(a[25]), "r"(a[26]), "r"(a[27]), "r"(a[28]), "r"(a[29]), "r"(a[30]), "r"(a[31])
                 : "memory");
}

// four 8x8 fp16 matrices from the fragment layout (thread t: row t / 4, columns 2 (t % 4), + 1 of
// each); thread t gives the shared address of row t % 8 of matrix t / 8
__device__ __forceinline__ void stmatrix_x4(uint32_t addr, const uint32_t r[4])
{
    asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(r[0]), "r"(r[1]),
                 "r"(r[2]), "r"(r[3])
                 : "memory");
}

// d order of the 8 entries of a 16-byte chunk: position j holds d = 8 a + kPerm[j]
__host__ __device__ constexpr int chunk_d(int j) { return (j >> 1) + ((j & 1) << 2); }

struct TcParams {
    const uint16_t *q;           // bf16 [total_q][Hq][128]
    const int32_t *q_start;      // [S + 1]
    const uint8_t *codes;        // INT4 pages [num_pages][Hkv][2][16][64]
    const uint8_t *scales;       // fp16 pairs [num_pages][Hkv][2][16][2]
    const int32_t *block_table;  // [S][max_blocks]
    const int32_t *seq_lens;     // [S]
    float *out;                  // fp32 [total_q][Hq][128]
    uint32_t *status;
    int64_t num_pages;
    int32_t max_blocks, num_seqs, hq, hkv, group, tile_tokens;
    float q_mult;
};

// Tile of CTA `cta`: sequence s, kv head h, first query token t0 of the chunk (tiles of T tokens
// in sequence order, the kv heads of one tile on consecutive CTAs).  Returns false past the last
// tile.  All threads of the CTA take part (block-wide scan over the sequences).
__device__ bool find_tile(const TcParams &p, int cta, int &s_out, int &h_out, int &t0_out,
                          int *sm_tile)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    __shared__ int warp_sums[kTcThreads / 32];
    __shared__ int carry;
    const int g_tile = cta / p.hkv;
    if (tid == 0) {
        carry = 0;
        sm_tile[0] = -1;
    }
    __syncthreads();
    for (int base = 0; base < p.num_seqs; base += kTcThreads) {
        const int s = base + tid;
        int n = 0;
        if (s < p.num_seqs) {
            const int c = p.q_start[s + 1] - p.q_start[s];
            n = c > 0 ? (c + p.tile_tokens - 1) / p.tile_tokens : 0;
        }
        int x = n;   // inclusive scan over the chunk of sequences
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int y = __shfl_up_sync(0xFFFFFFFFu, x, d);
            if (lane >= d)
                x += y;
        }
        if (lane == 31)
            warp_sums[warp] = x;
        __syncthreads();
        int before = carry;
        for (int w = 0; w < warp; w++)
            before += warp_sums[w];
        const int lo = before + x - n, hi = before + x;   // tiles [lo, hi) belong to s
        if (n > 0 && g_tile >= lo && g_tile < hi) {
            sm_tile[0] = s;
            sm_tile[1] = g_tile - lo;
        }
        __syncthreads();
        if (tid == kTcThreads - 1)
            carry = before + x;
        __syncthreads();
        if (sm_tile[0] >= 0)
            break;
    }
    if (sm_tile[0] < 0)
        return false;
    s_out = sm_tile[0];
    h_out = cta - g_tile * p.hkv;
    t0_out = sm_tile[1] * p.tile_tokens;
    return true;
}

__device__ __forceinline__ void tc_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Bounded wait on phase `parity` of an mbarrier that also gives up once the other role has
// (the shared abort flag); a timeout raises the flag.
__device__ __forceinline__ bool tc_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity))
            return true;
        if (*abort_flag != 0)
            return false;
        if (globaltimer_ns() - t0 > kTcWaitLimitNs) {
            *abort_flag = 1;
            return false;
        }
    }
}

// Named barrier of one role (128 threads: barrier 1 the producers, 2 the softmax warps) that
// also ANDs a flag over them, so that the role leaves its loop as one.
__device__ __forceinline__ bool role_bar_and(int id, bool v)
{
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
                 "bar.red.and.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
                 : "=r"(r)
                 : "r"(static_cast<uint32_t>(v)), "r"(id), "r"(kTcThreads / 2)
                 : "memory");
    return r != 0;
}

__device__ __forceinline__ uint4 ldg_nc16(const void *p)
{
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// four fp16 pairs of the 8 codes of a 32-bit word as exact integers ((0x6400 | n) - 1024), stored
// as one 16-byte chunk of an fp16 tile
__device__ __forceinline__ void unpack_word_store(uint32_t dst, uint32_t word)
{
    const __half2 k1024 = __halves2half2(__ushort_as_half(0x6400), __ushort_as_half(0x6400));
    const uint32_t y0 = half2_as_u32(__hsub2(u32_as_half2((word & 0x000F000Fu) | 0x64006400u), k1024));
    const uint32_t y1 = half2_as_u32(__hsub2(u32_as_half2(((word >> 4) & 0x000F000Fu) | 0x64006400u), k1024));
    const uint32_t y2 = half2_as_u32(__hsub2(u32_as_half2(((word >> 8) & 0x000F000Fu) | 0x64006400u), k1024));
    const uint32_t y3 = half2_as_u32(__hsub2(u32_as_half2(((word >> 12) & 0x000F000Fu) | 0x64006400u), k1024));
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(y0), "r"(y1), "r"(y2), "r"(y3)
                 : "memory");
}

// Roles: warps 0-3 run the softmax, one query row per thread (row = thread = tensor-memory lane);
// warps 4-7 are the producers: they load the pages of each block straight into registers (two
// blocks ahead), unpack K and V into the fp16 tiles and write the scale table, and one of them
// issues S = Q K^T.  Thread 0 issues O += P' V once the softmax warps have written P'.  The roles
// hand off through mbarriers (the tensor cores' commits included) and two named barriers, one per
// role, so neither waits for the other except where the data requires it.  Every wait is bounded;
// a timeout sets the status bit and a shared abort flag that ends the other role's waits too.
template <bool kRotate>
__global__ void __launch_bounds__(kTcThreads, 2)
    prefill_tc_kernel(const TcParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int hf = warp >> 2;                             // prologue / epilogue: column half
    const int row = 32 * (warp & 3) + lane;               // tile row = tensor-memory lane
    const uint32_t sbase = smem_u32(smem);
    int *sm_tile = reinterpret_cast<int *>(smem + kSmTile);
    float *xchg = reinterpret_cast<float *>(smem + kSmXchg);   // [2][128] fp32 per-row hand-overs
    const uint32_t bars = sbase + kSmBars;
    // bar_s[b]: S of blocks b, b + 2, ... done (tensor-core commit); bar_sfree[b]: the softmax has
    // read that S buffer (one arrival per softmax warp); bar_o[b]: P' V of blocks b, b + 2, ... done;
    // bar_v[b]: V of those blocks unpacked (128 producer arrivals); bar_sc[i]: the scale table of
    // blocks i, i + 4, ... written (128 producer arrivals)
    auto bar_s = [&](int b) { return bars + 8 * b; };
    auto bar_sfree = [&](int b) { return bars + 16 + 8 * b; };
    auto bar_o = [&](int b) { return bars + 32 + 8 * b; };
    auto bar_v = [&](int b) { return bars + 48 + 8 * b; };
    auto bar_sc = [&](int i) { return bars + 64 + 8 * i; };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kSmBars + 96);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kSmBars + 100);
    int *issued = reinterpret_cast<int *>(smem + kSmBars + 104);   // [0] S issued, [1] P' V issued

    pdl_launch_dependents();
    int s, h, t0;
    if (!find_tile(p, blockIdx.x, s, h, t0, sm_tile))
        return;
    const int G = p.group;
    const int C = p.q_start[s + 1] - p.q_start[s];
    const int L = p.seq_lens[s];
    if (C > L || L > p.max_blocks * kPageSize) {   // a chunk longer than its sequence: skipped
        if (tid == 0 && t0 == 0 && h == 0)
            set_status(p.status, SAW_DEV_BAD_SEQ_LEN);
        return;
    }
    const int ntok = min(p.tile_tokens, C - t0);          // query tokens of this tile
    const int nrows = ntok * G;
    const bool live = row < nrows;
    const int tq = live ? row / G : 0, hg = live ? row - tq * G : 0;
    const int n_kv = L - C + t0 + ntok;                    // cache tokens any row sees
    const int n_blocks = (n_kv + kTcBlockTokens - 1) / kTcBlockTokens;
    const int n_pages = (n_kv + kPageSize - 1) / kPageSize;

    // ---- tensor memory and barriers -----------------------------------------------------------
    if (tid == 0) {
        for (int b = 0; b < 2; b++) {
            mbar_init(bar_s(b), 1);
            mbar_init(bar_sfree(b), 4);
            mbar_init(bar_o(b), 1);
            mbar_init(bar_v(b), kTcThreads / 2);
        }
        for (int i = 0; i < 4; i++)
            mbar_init(bar_sc(i), kTcThreads / 2);
        *abort_flag = 0;
        issued[0] = issued[1] = 0;
    }
    mbar_init_fence();
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(kTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }

    pdl_wait();   // the cache may be written by the kernel this one depends on

    // ---- the query tile: rotate, scale, fp16, in the codes' d order --------------------------------
    // This thread's half of d: the cross-half Hadamard stage (d, d + 64) first, from the whole
    // row, then the 6 stages within the half (the order of the stages does not matter here: the
    // query is not required to be bit-exact, only the quantized cache is).
    {
        float x[64];
        if (live) {
            const uint4 *src = reinterpret_cast<const uint4 *>(
                p.q + ((static_cast<int64_t>(p.q_start[s]) + t0 + tq) * p.hq + h * G + hg) * 128);
#pragma unroll
            for (int c = 0; c < 8; c++) {
                const uint4 ua = src[c], ub = src[8 + c];   // d in [0, 64) and [64, 128)
                const uint32_t wa[4] = {ua.x, ua.y, ua.z, ua.w}, wb[4] = {ub.x, ub.y, ub.z, ub.w};
#pragma unroll
                for (int k = 0; k < 4; k++) {
#pragma unroll
                    for (int e = 0; e < 2; e++) {
                        const float a = __uint_as_float(e ? (wa[k] & 0xFFFF0000u) : (wa[k] << 16));
                        const float b = __uint_as_float(e ? (wb[k] & 0xFFFF0000u) : (wb[k] << 16));
                        x[8 * c + 2 * k + e] = !kRotate ? (hf ? b : a) : (hf ? a - b : a + b);
                    }
                }
            }
        } else {
#pragma unroll
            for (int i = 0; i < 64; i++)
                x[i] = 0.0f;
        }
#pragma unroll
        for (int hb = 1; kRotate && hb < 64; hb <<= 1)
#pragma unroll
            for (int i = 0; i < 64; i++)
                if ((i & hb) == 0) {
                    const float a = x[i], b = x[i + hb];
                    x[i] = a + b;
                    x[i + hb] = a - b;
                }
        float sq_half = 0.0f;
#pragma unroll
        for (int c = 0; c < 8; c++) {
            uint32_t wv[4];
#pragma unroll
            for (int k = 0; k < 4; k++) {
                __half hh[2];
#pragma unroll
                for (int e = 0; e < 2; e++) {
                    hh[e] = __float2half_rn(x[8 * c + chunk_d(2 * k + e)] * (p.q_mult * kTcQScale));
                    sq_half += __half2float(hh[e]);
                }
                wv[k] = half2_as_u32(__halves2half2(hh[0], hh[1]));
            }
            const uint32_t a = sbase + kSmQ + sw128_chunk(row, 8 * hf + c, kTcRows * 128);
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(wv[0]), "r"(wv[1]),
                         "r"(wv[2]), "r"(wv[3]) : "memory");
        }
        xchg[hf * kTcRows + row] = sq_half;
    }



    // ---- tensor-memory base; the roles split here ----------------------------------------------
    async_proxy_fence();   // the Q tile is read by the tensor cores
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
    float l_quad[4] = {0.0f, 0.0f, 0.0f, 0.0f}, z_quad[4] = {0.0f, 0.0f, 0.0f, 0.0f};   // softmax: row sums

    if (warp >= 4) {
        // ======== producers: pages -> registers (two blocks ahead) -> fp16 K / V tiles, scales ====
        // Thread pt holds, of each block, the 16-byte quarter q4 of token rk's K and V rows in
        // pages pgk and pgk + 2 (4 code words each), and the (scale, zero) pair `sel` of token tks
        // of page pgs.
        const int pt = tid - kTcThreads / 2;
        const int pgk = pt >> 6, rk = (pt & 63) >> 2, q4 = pt & 3;
        const int pgs = pt >> 5, sel = (pt >> 4) & 1, tks = pt & 15;
        const int32_t *bt = p.block_table + static_cast<int64_t>(s) * p.max_blocks;
        auto raw_id = [&](int pg) -> int32_t { return pg < n_pages ? __ldg(bt + pg) : -1; };
        auto checked = [&](int pg, int32_t id) -> int32_t {   // -1 past the tile's range
            if (pg < n_pages && (id < 0 || id >= p.num_pages)) {
                set_status(p.status, SAW_DEV_BAD_PAGE);
                return 0;
            }
            return id;
        };
        struct Words {
            uint4 k0, k1, v0, v1;   // pages pgk, pgk + 2
            uint32_t sc;
        };
        auto fetch = [&](int b, int32_t ia, int32_t ib, int32_t is) -> Words {
            Words w;
            const uint4 zero4 = make_uint4(0u, 0u, 0u, 0u);
            ia = checked(kTcBlockPages * b + pgk, ia);
            ib = checked(kTcBlockPages * b + pgk + 2, ib);
            is = checked(kTcBlockPages * b + pgs, is);
            const int off = rk * kRowBytes + q4 * 16;
            const uint8_t *a = p.codes + (static_cast<int64_t>(ia) * p.hkv + h) * (2 * kPageSize * kRowBytes) + off;
            const uint8_t *c = p.codes + (static_cast<int64_t>(ib) * p.hkv + h) * (2 * kPageSize * kRowBytes) + off;
            w.k0 = ia >= 0 ? ldg_nc16(a) : zero4;
            w.v0 = ia >= 0 ? ldg_nc16(a + kPageSize * kRowBytes) : zero4;
            w.k1 = ib >= 0 ? ldg_nc16(c) : zero4;
            w.v1 = ib >= 0 ? ldg_nc16(c + kPageSize * kRowBytes) : zero4;
            w.sc = is >= 0 ? __ldg(reinterpret_cast<const uint32_t *>(
                                 p.scales + (static_cast<int64_t>(is) * p.hkv + h) * (2 * kPageSize * 4) +
                                 sel * (kPageSize * 4) + tks * 4))
                           : 0u;
            return w;
        };
        // S = Q K^T of block kb_ into S buffer kb_ mod 2
        auto issue_qk = [&](int kb_) {
            constexpr uint32_t id_qk = umma_idesc(kTcRows, kTcBlockTokens, 0, 0);
#pragma unroll
            for (int ks = 0; ks < 8; ks++) {
                const uint32_t oq = (ks >> 2) * (kTcRows * 128) + (ks & 3) * 32;
                const uint32_t ok_ = (ks >> 2) * (kTcBlockTokens * 128) + (ks & 3) * 32;
                umma_f16(tmem + 128 + 64 * (kb_ & 1), umma_desc(sbase + kSmQ + oq, 16, 1024),
                         umma_desc(sbase + kSmK + ok_, 16, 1024), id_qk, ks > 0);
            }
            umma_commit(bar_s(kb_ & 1));
        };
        // this thread's four fp16 chunks of a token row in a K or V tile (128-byte swizzle)
        const int tk0 = pgk * kPageSize + rk, tk1 = (pgk + 2) * kPageSize + rk;
        auto unpack4 = [&](uint32_t tile, int tok, const uint4 &w) {
            unpack_word_store(tile + sw128_chunk(tok, 4 * q4 + 0, kTcBlockTokens * 128), w.x);
            unpack_word_store(tile + sw128_chunk(tok, 4 * q4 + 1, kTcBlockTokens * 128), w.y);
            unpack_word_store(tile + sw128_chunk(tok, 4 * q4 + 2, kTcBlockTokens * 128), w.z);
            unpack_word_store(tile + sw128_chunk(tok, 4 * q4 + 3, kTcBlockTokens * 128), w.w);
        };

        int32_t ra = raw_id(pgk), rb = raw_id(pgk + 2), rs = raw_id(pgs);
        Words w0 = fetch(0, ra, rb, rs);
        ra = raw_id(kTcBlockPages + pgk), rb = raw_id(kTcBlockPages + pgk + 2), rs = raw_id(kTcBlockPages + pgs);
        Words w1 = fetch(1, ra, rb, rs);
        ra = raw_id(2 * kTcBlockPages + pgk), rb = raw_id(2 * kTcBlockPages + pgk + 2);
        rs = raw_id(2 * kTcBlockPages + pgs);
        bool ok = true;
        for (int kb = 0; kb < n_blocks; kb++) {
            // the words of block kb + 2 (ids read a block ago) and the ids of block kb + 3
            Words w2 = {};
            if (kb + 2 < n_blocks)
                w2 = fetch(kb + 2, ra, rb, rs);
            const int nb = kTcBlockPages * (kb + 3);
            ra = raw_id(nb + pgk), rb = raw_id(nb + pgk + 2), rs = raw_id(nb + pgs);

            // V of block kb into V tile kb mod 2, once P' V of block kb - 2 has read it
            if (kb >= 2)
                ok = ok && tc_wait(bar_o(kb & 1), static_cast<uint32_t>((kb - 2) >> 1) & 1u, abort_flag);
            if (ok) {
                const uint32_t vt = sbase + kSmV + (kb & 1) * kSmVTile;
                unpack4(vt, tk0, w0.v0);
                unpack4(vt, tk1, w0.v1);
                async_proxy_fence();
                tc_arrive(bar_v(kb & 1));
            }
            // K of block kb and its scale table, once S of block kb - 1 has read the K tile
            if (kb >= 1)
                ok = ok && tc_wait(bar_s((kb - 1) & 1), static_cast<uint32_t>((kb - 1) >> 1) & 1u, abort_flag);
            if (ok) {
                unpack4(sbase + kSmK, tk0, w0.k0);
                unpack4(sbase + kSmK, tk1, w0.k1);
                const int tk = pgs * kPageSize + tks;
                float2 sz = __half22float2(u32_as_half2(w0.sc));
                if (kb * kTcBlockTokens + tk >= n_kv)
                    sz = make_float2(0.0f, 0.0f);   // past the tile's range: no weight, no NaN
                float *par = reinterpret_cast<float *>(smem + kSmScales + (kb & 3) * kSmScaleSet) +
                             sel * 2 * kTcBlockTokens + 4 * (tk >> 1) + (tk & 1);
                // K: logit = (scale acc + zero sq) / 2^8; V: P' = 2^4 p scale, zero point
                par[0] = sel == 0 ? sz.x * (1.0f / kTcQScale) : sz.x * kTcPScale;
                par[2] = sel == 0 ? sz.y * (1.0f / kTcQScale) : sz.y;
                async_proxy_fence();
                tc_arrive(bar_sc(kb & 3));
            }
            ok = role_bar_and(1, ok);
            if (!ok)
                break;
            if (pt == 0) {
                // the S buffer of block kb - 2 has been read by the softmax
                ok = kb < 2 || tc_wait(bar_sfree(kb & 1), static_cast<uint32_t>((kb - 2) >> 1) & 1u, abort_flag);
                if (ok) {
                    tc_fence_after();
                    issue_qk(kb);
                    issued[0] = kb + 1;
                }
            }
            w0 = w1;
            w1 = w2;
        }
    } else {
        // ======== softmax: fragment layout ===========================================================
        // S is read with tcgen05.ld.16x256b: in each 16-lane half of its quarter, thread (r = lane / 4,
        // c = lane % 4) gets rows r and r + 8 at columns 8 k + 2 c, 8 k + 2 c + 1 (k = 0 .. 7).  So a
        // thread holds 4 rows (slots i: row 32 w + r + 8 i) x 16 tokens.  The halves are processed
        // one after the other (32 live S values); each scale-table entry a thread loads (8 for K and
        // 8 for V per half) serves the half's 2 rows, the row maximum is combined over the 4 threads
        // of a quad by shuffles, and the sums l, z stay per thread until the end.
        const int fr = lane >> 2, fc = lane & 3;
        float sq[4], m_ref[4];
        uint64_t l2[4], z2[4];   // this thread's share of the row sums (two lanes each)
        bool live_i[4];
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const int ri = 32 * warp + fr + 8 * i;
            sq[i] = xchg[ri] + xchg[kTcRows + ri];
            m_ref[i] = -INFINITY;
            l2[i] = f2_pack(0.0f, 0.0f);
            z2[i] = l2[i];
            live_i[i] = ri < nrows;
        }
        const uint32_t quarter = tmem + (static_cast<uint32_t>(32 * warp) << 16);
        bool ok = true;
        for (int kb = 0; kb < n_blocks; kb++) {
            // S of block kb and its scale table
            ok = ok && tc_wait(bar_s(kb & 1), static_cast<uint32_t>(kb >> 1) & 1u, abort_flag);
            ok = ok && tc_wait(bar_sc(kb & 3), static_cast<uint32_t>(kb >> 2) & 1u, abort_flag);
            ok = __all_sync(0xFFFFFFFFu, ok);   // tensor-memory loads are warp-wide
            const float4 *kp4 = reinterpret_cast<const float4 *>(smem + kSmScales + (kb & 3) * kSmScaleSet);
            const float4 *vp4 = kp4 + kTcBlockTokens / 2;
            const uint32_t cb = 128 + 64 * (kb & 1);
            // the two 16-lane halves of the quarter are independent rows: one at a time
#pragma unroll
            for (int h = 0; h < 2; h++) {
                float s[32];   // s[4 k + e]: row slot 2 h + e / 2, token 8 k + 2 c + e % 2
                bool grow = false;
                float alpha[2] = {1.0f, 1.0f};
                if (ok) {
                    tc_fence_after();
                    tmem_ld_16x256b_x8(quarter + (static_cast<uint32_t>(16 * h) << 16) + cb, s);
                    if (h == 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0)
                            tc_arrive(bar_sfree(kb & 1));   // the S buffer may be overwritten
                    }
#pragma unroll
                    for (int k = 0; k < 8; k++) {
                        const float4 kp = kp4[4 * k + fc];   // tokens 8 k + 2 c, + 1
                        const uint64_t sk2 = f2_pack(kp.x, kp.y), zk2 = f2_pack(kp.z, kp.w);
#pragma unroll
                        for (int j = 0; j < 2; j++) {
                            float &a = s[4 * k + 2 * j], &b = s[4 * k + 2 * j + 1];
                            const float q = sq[2 * h + j];
                            const uint64_t t = f2_fma(sk2, f2_pack(a, b), f2_mul(zk2, f2_pack(q, q)));
                            f2_unpack(t, a, b);
                        }
                    }
                    // the causal limit (and the end of the cache) only reaches the last blocks of a tile
                    if (kb * kTcBlockTokens + kTcBlockTokens - 1 > L - C + t0) {
                        const int tok0 = kb * kTcBlockTokens + 2 * fc;
#pragma unroll
                        for (int j = 0; j < 2; j++) {
                            const int ri = 32 * warp + fr + 8 * (2 * h + j);
                            const int lim = L - C + t0 + (live_i[2 * h + j] ? ri / G : 0);
#pragma unroll
                            for (int k = 0; k < 8; k++)
#pragma unroll
                                for (int e = 0; e < 2; e++)
                                    if (tok0 + 8 * k + e > lim)
                                        s[4 * k + 2 * j + e] = -INFINITY;
                        }
                    }
#pragma unroll
                    for (int j = 0; j < 2; j++) {
                        const int i = 2 * h + j;
                        float m = -INFINITY;
#pragma unroll
                        for (int k = 0; k < 8; k++)
                            m = fmax3(m, s[4 * k + 2 * j], s[4 * k + 2 * j + 1]);
                        m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
                        m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
                        if (!live_i[i])
                            m = -INFINITY;
                        if (m > m_ref[i] + kTcRescale) {
                            alpha[j] = ex2_approx(m_ref[i] - m);   // 0 on the first block a row sees
                            const uint64_t a2 = f2_pack(alpha[j], alpha[j]);
                            l2[i] = f2_mul(l2[i], a2);
                            z2[i] = f2_mul(z2[i], a2);
                            m_ref[i] = m;
                            grow |= alpha[j] != 0.0f;
                        }
                    }
                }
                if (h == 0) {
                    // P' V of block kb - 1 has finished with the P' tile and the O accumulator
                    if (kb >= 1)
                        ok = ok && tc_wait(bar_o((kb - 1) & 1), static_cast<uint32_t>((kb - 1) >> 1) & 1u, abort_flag);
                    ok = __all_sync(0xFFFFFFFFu, ok);
                }
                if (ok) {
                    tc_fence_after();
                    // the weights of the half's two rows, two 8-token chunks per stmatrix (matrices:
                    // (row slot 2 h, chunk k), (2 h + 1, k), (2 h, k + 1), (2 h + 1, k + 1))
#pragma unroll
                    for (int k = 0; k < 8; k += 2) {
                        uint32_t pw[4];
#pragma unroll
                        for (int kk = 0; kk < 2; kk++) {
                            const float4 vp = vp4[4 * (k + kk) + fc];
                            const uint64_t sv2 = f2_pack(vp.x, vp.y), zv2 = f2_pack(vp.z, vp.w);
#pragma unroll
                            for (int j = 0; j < 2; j++) {
                                const int i = 2 * h + j;
                                const float mr = live_i[i] ? m_ref[i] : INFINITY;   // rows past the tile: 0
                                float d0, d1;
                                f2_unpack(f2_sub(f2_pack(s[4 * (k + kk) + 2 * j], s[4 * (k + kk) + 2 * j + 1]),
                                                 f2_pack(mr, mr)),
                                          d0, d1);
                                const uint64_t p2 = f2_pack(ex2_approx(d0), ex2_approx(d1));
                                l2[i] = f2_add(l2[i], p2);
                                z2[i] = f2_fma(p2, zv2, z2[i]);
                                float q0, q1;
                                f2_unpack(f2_mul(p2, sv2), q0, q1);
                                pw[2 * kk + j] = half2_as_u32(__floats2half2_rn(q0, q1));
                            }
                        }
                        // thread t: row 32 w + 16 h + t % 16 of chunk k + t / 16
                        stmatrix_x4(sbase + kSmP + sw128_chunk(32 * warp + 16 * h + (lane & 15), k + (lane >> 4),
                                                                kTcRows * 128),
                                    pw);
                    }
                    // rescale the half's O rows in tensor memory (warp-wide; alpha 1 where no change)
                    if (kb > 0 && __any_sync(0xFFFFFFFFu, grow)) {
#pragma unroll 1
                        for (int c = 0; c < 2; c++) {   // 64 columns at a time
                            const uint32_t ta = quarter + (static_cast<uint32_t>(16 * h) << 16) + 64 * c;
                            float ov[32];
                            tmem_ld_16x256b_x8(ta, ov);
#pragma unroll
                            for (int j = 0; j < 32; j += 4) {
                                ov[j] *= alpha[0];
                                ov[j + 1] *= alpha[0];
                                ov[j + 2] *= alpha[1];
                                ov[j + 3] *= alpha[1];
                            }
                            tmem_st_16x256b_x8(ta, ov);
                        }
                        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
                    }
                }
            }
            if (ok) {
                async_proxy_fence();
                tc_fence_before();
            }
            ok = role_bar_and(2, ok);
            if (!ok)
                break;
            if (tid == 0) {
                // O += P' V of block kb, once the producers have written V of block kb
                ok = tc_wait(bar_v(kb & 1), static_cast<uint32_t>(kb >> 1) & 1u, abort_flag);
                if (ok) {
                    tc_fence_after();
                    constexpr uint32_t id_pv = umma_idesc(kTcRows, 128, 0, 1);
#pragma unroll
                    for (int ks = 0; ks < 4; ks++)
                        umma_f16(tmem, umma_desc(sbase + kSmP + ks * 32, 16, 1024),
                                 umma_desc(sbase + kSmV + (kb & 1) * kSmVTile + ks * 2048,
                                           kTcBlockTokens * 128, 1024),
                                 id_pv, kb > 0 || ks > 0);
                    umma_commit(bar_o(kb & 1));
                    issued[1] = kb + 1;
                }
            }
        }
        // the row sums over the quad, for the epilogue
#pragma unroll
        for (int i = 0; i < 4; i++) {
            float la, lb, za, zb;
            f2_unpack(l2[i], la, lb);
            f2_unpack(z2[i], za, zb);
            float lt = la + lb, zt = za + zb;
            lt += __shfl_xor_sync(0xFFFFFFFFu, lt, 1);
            zt += __shfl_xor_sync(0xFFFFFFFFu, zt, 1);
            lt += __shfl_xor_sync(0xFFFFFFFFu, lt, 2);
            zt += __shfl_xor_sync(0xFFFFFFFFu, zt, 2);
            l_quad[i] = lt;
            z_quad[i] = zt;
        }
    }

    // ---- epilogue: O row -> zero term, 1 / l, the weights' scale, inverse rotation ----------------
    __syncthreads();
    bool fine = *abort_flag == 0;
    if (fine) {
        const int last = n_blocks - 1;
        const bool ok = tc_wait(bar_o(last & 1), static_cast<uint32_t>(last >> 1) & 1u, abort_flag);
        fine = __syncthreads_and(ok);
    }
    if (!fine) {
        if (tid == 0) {
            set_status(p.status, SAW_DEV_WAIT_TIMEOUT);
            // let the MMAs that may still be in flight finish before the tensor memory is released
            for (int b = max(0, issued[0] - 2); b < issued[0]; b++)
                mbar_wait_bounded(bar_s(b & 1), static_cast<uint32_t>(b >> 1) & 1u, kTcWaitLimitNs / 10);
            for (int b = max(0, issued[1] - 2); b < issued[1]; b++)
                mbar_wait_bounded(bar_o(b & 1), static_cast<uint32_t>(b >> 1) & 1u, kTcWaitLimitNs / 10);
        }
    } else {
        tc_fence_after();
        // this half's 64 O columns = d in [64 hf, 64 hf + 64) (the d order permutes within 8)
        float o[64];
        tmem_ld32(lane_base + 64 * hf, o);
        tmem_ld32(lane_base + 64 * hf + 32, o + 32);
        if (warp < 4 && (lane & 3) == 0) {
#pragma unroll
            for (int i = 0; i < 4; i++) {
                xchg[32 * warp + (lane >> 2) + 8 * i] = l_quad[i];
                xchg[kTcRows + 32 * warp + (lane >> 2) + 8 * i] = z_quad[i];
            }
        }
        __syncthreads();
        const float lt = xchg[row];
        const float zt = xchg[kTcRows + row];
        const float inv = live ? 1.0f / lt : 0.0f;
        float v[64];
#pragma unroll
        for (int n = 0; n < 64; n++) {
            const int d = (n & ~7) + chunk_d(n & 7);
            v[d] = fmaf(o[n], 1.0f / kTcPScale, zt) * inv;
        }
        // inverse rotation: the 6 stages within the half, then (d, d + 64) through shared memory
        // (all tiles are free now: the exchange uses the Q, K and V tiles' 64 KB)
#pragma unroll
        for (int hb = 1; kRotate && hb < 64; hb <<= 1)
#pragma unroll
            for (int i = 0; i < 64; i++)
                if ((i & hb) == 0) {
                    const float a = v[i], b = v[i + hb];
                    v[i] = a + b;
                    v[i + hb] = a - b;
                }
        if (kRotate) {
            float4 *mine = reinterpret_cast<float4 *>(smem + kSmQ) + (hf * kTcRows + row) * 16;
            const float4 *other = reinterpret_cast<const float4 *>(smem + kSmQ) + ((1 - hf) * kTcRows + row) * 16;
#pragma unroll
            for (int c = 0; c < 16; c++)
                mine[c] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
            __syncthreads();
#pragma unroll
            for (int c = 0; c < 16; c++) {
                const float4 w = other[c];
                const float b4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int k = 0; k < 4; k++)   // low half: a + b; high half: a - b (a the low value)
                    v[4 * c + k] = hf ? b4[k] - v[4 * c + k] : v[4 * c + k] + b4[k];
            }
        }
        if (live) {
            const float f = kRotate ? kTcHadamardC : 1.0f;
            float4 *dst = reinterpret_cast<float4 *>(
                p.out + ((static_cast<int64_t>(p.q_start[s]) + t0 + tq) * p.hq + h * G + hg) * 128 + 64 * hf);
#pragma unroll
            for (int c = 0; c < 16; c++)
                dst[c] = make_float4(v[4 * c] * f, v[4 * c + 1] * f, v[4 * c + 2] * f, v[4 * c + 3] * f);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                     : "memory");
}

}  // namespace

// Tiles of T = 128 / G query tokens; the grid covers the most tiles any chunk split can give.
int64_t prefill_tc_grid(int32_t num_kv_heads, int32_t num_q_heads, int32_t num_seqs, int64_t total_q)
{
    const int32_t G = num_q_heads / num_kv_heads;
    const int32_t T = std::max(1, kTcRows / G);
    return static_cast<int64_t>(num_kv_heads) * ((total_q + T - 1) / T + num_seqs);
}

cudaError_t launch_prefill_tc(const DecodeArgs &a, cudaStream_t stream, bool programmatic)
{
    TcParams p;
    p.q = static_cast<const uint16_t *>(a.q);
    p.q_start = a.q_start;
    p.codes = a.kv_pages;
    p.scales = static_cast<const uint8_t *>(a.scales);
    p.block_table = a.block_table;
    p.seq_lens = a.seq_lens;
    p.out = a.out;
    p.status = a.status;
    p.num_pages = a.num_pages;
    p.max_blocks = a.max_blocks;
    p.num_seqs = a.num_seqs;
    p.hq = a.num_q_heads;
    p.hkv = a.num_kv_heads;
    p.group = a.num_q_heads / a.num_kv_heads;
    p.tile_tokens = std::max(1, kTcRows / p.group);
    // q carries sm_scale * log2(e) and 1/sqrt(128) of the unnormalised butterfly
    p.q_mult = static_cast<float>((a.rotate ? static_cast<double>(kTcHadamardC) : 1.0) * a.sm_scale *
                                  1.4426950408889634);
    static bool attr_set[2] = {false, false};
    auto *kernel = a.rotate ? prefill_tc_kernel<true> : prefill_tc_kernel<false>;
    if (!attr_set[a.rotate ? 1 : 0]) {
        const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   static_cast<int>(kTcSmemBytes));
        if (e != cudaSuccess)
            return e;
        attr_set[a.rotate ? 1 : 0] = true;
    }
    const int64_t grid = prefill_tc_grid(a.num_kv_heads, a.num_q_heads, a.num_seqs, a.total_q);
    if (grid <= 0)
        return cudaSuccess;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = kTcSmemBytes;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = programmatic ? 1 : 0;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, p);
    if (e != cudaSuccess)
        return e;
    return cudaGetLastError();
}

}  // namespace saw
