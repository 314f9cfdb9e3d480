/*
 * pagedkv.h — C ABI of the B200 (sm_100a) paged KV-cache library.
 *
 * Two operations on a paged KV cache, as described in "vLLM 推理引擎源码级拆解：
 * PagedAttention 显存虚拟化、Continuous Batching 调度与量化落地全指南"
 * (chenxutan.com/d/5333):
 *   - paged_kv_append: each new token's K/V row is written into the slot the
 *     caller assigned it in a shared pool of fixed-size blocks (§2.1-§2.2: the
 *     token fills the last block's next slot, or the first slot of a block just
 *     taken from the free pool);
 *   - paged_attention_decode: one query token per sequence attends over that
 *     sequence's cached tokens, walking its block table from logical to
 *     physical block (§2.3), with grouped-query heads (GQA/MQA, §2.3), blocks
 *     shared between sequences (§2.1), an optional split of long sequences into
 *     partitions merged by log-sum-exp, and an FP8-E4M3 cache with per-tensor
 *     scales ("vLLM 0.5 深度拆解", chenxutan.com/d/4924, §4.2).
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers owned by the caller, C-contiguous,
 *     and 16-byte aligned. The library allocates nothing and keeps no state
 *     between calls.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream). Calls only
 *     enqueue work and return; they never synchronise and never read device
 *     memory on the host.
 *   - Arguments are checked on the host before anything is enqueued; a negative
 *     pkv_status is returned and nothing runs. PKV_ERR_CUDA reports a launch
 *     failure; faults inside a kernel surface at the caller's next
 *     synchronisation, as with any CUDA call.
 *   - Pool layout: k_cache and v_cache are [num_blocks, block_size,
 *     num_kv_heads, head_dim] in cache_dtype. Token t of sequence i lives in
 *     physical block block_table[i][t / block_size] at offset t % block_size;
 *     its flat slot is physical_block * block_size + offset.
 */
#ifndef PAGEDKV_H
#define PAGEDKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Element types. PKV_FP8_E4M3 is the OCP E4M3 format: bias 7, 3 mantissa bits,
 * subnormals, largest finite 448, no infinities, S.1111.111 = NaN. */
typedef enum {
  PKV_F32 = 0,
  PKV_F16 = 1,
  PKV_BF16 = 2,
  PKV_FP8_E4M3 = 3
} pkv_dtype;

typedef enum {
  PKV_OK = 0,
  PKV_ERR_NULL = -1,        /* a required pointer is NULL */
  PKV_ERR_SHAPE = -2,       /* a size is out of range or inconsistent */
  PKV_ERR_DTYPE = -3,       /* an unknown dtype or an unsupported dtype pair */
  PKV_ERR_UNSUPPORTED = -4, /* head_dim or block_size outside the supported set */
  PKV_ERR_WORKSPACE = -5,   /* workspace missing or smaller than required */
  PKV_ERR_CUDA = -6,        /* a CUDA runtime call or kernel launch failed */
  PKV_ERR_ALIGN = -7,       /* a pointer is not 16-byte aligned */
  PKV_ERR_NO_BLOCKS = -8,   /* not enough free blocks (block manager) */
  PKV_ERR_SEQ = -9,         /* unknown, duplicate or swapped-out sequence id */
  PKV_ERR_MEMORY = -10      /* a pool is neither device memory nor pinned host memory */
} pkv_status;

/* Flags for paged_attention_decode. */
#define PKV_DECODE_FORCE_SIMT 1u  /* use the CUDA-core kernel even where the
                                     tensor-core kernel applies */
/* The workspace's split counters are zero on entry, as every decode call
 * leaves them (or as the caller zeroed them): the call skips the memset that
 * zeroes them. Do not set it on a fresh workspace, on one used for anything
 * else since, or after pkv_device_status reported an expired wait. */
#define PKV_DECODE_ZEROED_WORKSPACE 2u
/* Start the tensor-core kernel while the previous kernel in the stream is still
 * running (programmatic dependent launch); it sets up its schedule and reads
 * the block table, and waits for that kernel to finish only before its first
 * read of the caches. Allowed only when the previous kernel writes nothing the
 * call reads except the K/V caches (e.g. paged_kv_append of this step's
 * tokens) and does not touch `out` or the workspace. Without a preceding
 * kernel, or on the CUDA-core path, it changes nothing. */
#define PKV_DECODE_EARLY_START 4u
/* Where the TMA-fed decode kernel (16-bit caches, head_dim 64/128) runs its
 * Q K^T and P V products. By default every group size uses the tensor cores
 * (mma.sync, tokens on M): measured on B200, even one query head per KV head
 * runs faster there than with fp32 FMA on the CUDA cores, since the CUDA-core
 * form needs several times the instructions. CUDA_CORES selects the CUDA-core
 * form for groups of up to 4 heads (wider groups stay on the tensor cores);
 * TENSOR_CORES states the default. Both set is an error. Comparison and testing
 * knobs. */
#define PKV_DECODE_TENSOR_CORES 8u
#define PKV_DECODE_CUDA_CORES 16u

/*
 * paged_kv_append — write new tokens' K/V into their slots ("reshape and cache").
 *
 *   key, value    [num_tokens, num_kv_heads, head_dim], src_dtype (F32/F16/BF16)
 *   k_cache,
 *   v_cache       [num_blocks, block_size, num_kv_heads, head_dim], cache_dtype;
 *                 cache_dtype is src_dtype (bytes are copied) or PKV_FP8_E4M3
 *   slot_mapping  [num_tokens] int64, device: flat slot of each token. A slot
 *                 < 0 (padding) or >= num_blocks * block_size writes nothing.
 *   k_scale,
 *   v_scale       device fp32 scalars, read only for an FP8 cache: the stored
 *                 code is E4M3(x / scale), x widened to fp32, the division in
 *                 IEEE fp32, rounded to nearest-even, saturated to +-448.
 *
 * Slots within one call must be distinct, and must belong to blocks no other
 * sequence shares (copy-on-write of shared blocks is the caller's job). Every
 * other byte of the pool is left untouched.
 * Requirements: num_tokens >= 0, num_kv_heads > 0, head_dim a positive
 * multiple of 8, block_size > 0, num_blocks > 0.
 */
int paged_kv_append(const void* key, const void* value, void* k_cache, void* v_cache,
                    const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                    int head_dim, int block_size, int64_t num_blocks, int src_dtype,
                    int cache_dtype, const float* k_scale, const float* v_scale,
                    void* stream);

/*
 * Bytes of workspace paged_attention_decode needs for these sizes: zero when no
 * sequence can be split (partition_size 0, or max_seq_len <= partition_size);
 * otherwise room for the partial results of at most two pieces per CTA (up to
 * 1024 CTAs), each num_heads / num_kv_heads fp32 rows of head_dim plus as many
 * log-sum-exp values, and one int32 counter per (sequence, KV head). It does
 * not grow with max_seq_len.
 * Returns 0 for invalid sizes.
 */
size_t paged_attention_workspace_size(int num_seqs, int num_heads, int num_kv_heads,
                                      int head_dim, int max_seq_len, int partition_size);

/*
 * paged_attention_decode — one-token attention per sequence over a paged cache.
 *
 * For sequence i and query head j (KV head h = j / (num_heads / num_kv_heads)):
 *   K[t] = k_cache[block_table[i][t / block_size], t % block_size, h, :]
 *          (times *k_scale for an FP8 cache), t = 0 .. seq_lens[i]-1; V alike
 *   s_t  = scale * <query[i, j, :], K[t]>
 *   out[i, j, :] = sum_t softmax(s)_t V[t]
 *
 *   out          [num_seqs, num_heads, head_dim], q_dtype; written for every
 *                (i, j); a sequence of length 0 gets zeros
 *   query        [num_seqs, num_heads, head_dim], q_dtype (F32/F16/BF16)
 *   k_cache,
 *   v_cache      pool as above, cache_dtype = q_dtype or PKV_FP8_E4M3
 *   block_table  [num_seqs, max_blocks_per_seq] int32, device. Entries past a
 *                sequence's last block are never read. An entry outside
 *                [0, num_blocks) reads as a block of zeros.
 *   seq_lens     [num_seqs] int32, device: tokens per sequence, including the
 *                token appended this step. Values are clamped to
 *                [0, min(max_seq_len, max_blocks_per_seq * block_size)].
 *   max_seq_len  host upper bound on seq_lens (sizes the split and workspace)
 *   scale        softmax scale (usually 1/sqrt(head_dim))
 *   k_scale,
 *   v_scale      device fp32 scalars, read only for an FP8 cache
 *   partition_size  0: a sequence is never split. > 0 (a multiple of
 *                block_size): a sequence may be split at multiples of this many
 *                tokens; each piece yields a partial (output, log-sum-exp) in the
 *                workspace, and the CTA that finishes a sequence's last piece
 *                merges the pieces by log-sum-exp. The split points are chosen
 *                on the device to balance work across the GPU. The call then
 *                enqueues a small memset of the workspace's counters and one
 *                kernel; with partition_size 0, just the kernel.
 *   max_ctas     0: one resident wave of CTAs; > 0: at most this many CTAs (a
 *                tuning and testing knob)
 *   flags        PKV_DECODE_* bits
 *   workspace    device scratch of at least paged_attention_workspace_size()
 *                bytes (may be NULL when that is 0); the caller owns it, need not
 *                initialise it, and must not use it concurrently for another call
 *
 * Requirements: num_seqs >= 0, num_heads > 0, num_kv_heads > 0,
 * num_heads % num_kv_heads == 0, head_dim in {64, 128}, block_size in
 * {8, 16, 32}, max_blocks_per_seq > 0, num_blocks > 0, max_seq_len >= 0.
 */
int paged_attention_decode(void* out, const void* query, const void* k_cache,
                           const void* v_cache, const int32_t* block_table,
                           const int32_t* seq_lens, int num_seqs, int num_heads,
                           int num_kv_heads, int head_dim, int block_size,
                           int max_blocks_per_seq, int64_t num_blocks, int max_seq_len,
                           float scale, int q_dtype, int cache_dtype, const float* k_scale,
                           const float* v_scale, int partition_size, int max_ctas,
                           unsigned flags, void* workspace, size_t workspace_bytes,
                           void* stream);

/*
 * paged_attention_decode_static — paged_attention_decode without a caller
 * workspace, for callers that cannot allocate device memory (code inside a
 * framework that owns all device allocations, loops where cudaMalloc's implicit
 * synchronisation is not acceptable, bindings with no device-memory API). The
 * pages have no counterpart: it is a packaging of the same decode.
 *
 * Arguments and results are those of paged_attention_decode without
 * `workspace` and `workspace_bytes`. The split-sequence scratch is a fixed
 * 16 MiB array of device memory inside this library, present on every device
 * where the library's device code is loaded until the process exits. Sizes whose
 * paged_attention_workspace_size() exceeds 16 MiB are rejected with
 * PKV_ERR_WORKSPACE before anything is enqueued. The call allocates nothing.
 * Its first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make it before any stream
 * capture. Every call shares the array, and each call clears what must start at
 * zero (a memset on `stream`; PKV_DECODE_ZEROED_WORKSPACE in `flags` is ignored,
 * since the array may hold another call's data); calls whose work overlaps on
 * the GPU (several streams or host threads) race on the array and must be
 * serialised by the caller.
 */
int paged_attention_decode_static(void* out, const void* query, const void* k_cache,
                                  const void* v_cache, const int32_t* block_table,
                                  const int32_t* seq_lens, int num_seqs, int num_heads,
                                  int num_kv_heads, int head_dim, int block_size,
                                  int max_blocks_per_seq, int64_t num_blocks, int max_seq_len,
                                  float scale, int q_dtype, int cache_dtype,
                                  const float* k_scale, const float* v_scale, int partition_size,
                                  int max_ctas, unsigned flags, void* stream);

/*
 * paged_attention_prefill — multi-token queries over the paged cache, causal.
 *
 * "vLLM 0.5 深度拆解" (chenxutan.com/d/4924) §2.3: a long prompt is filled in
 * chunks, each chunk's tokens attending over everything before them and over
 * the chunk itself; "vLLM 推理引擎源码级拆解" (chenxutan.com/d/5333) §4.2: a
 * request whose leading blocks are cached computes only the rest. Both are:
 *
 *   query        [num_q_tokens, num_heads, head_dim], q_dtype (BF16/F16)
 *   query_start  [num_seqs + 1] int32, device: rows query_start[i] ..
 *                query_start[i+1]-1 are the last q_i tokens of sequence i
 *   seq_lens     [num_seqs] int32, device: sequence i's cached tokens, the q_i
 *                chunk tokens included (their K/V appended beforehand with
 *                paged_kv_append)
 *   k_cache,
 *   v_cache      the pool, cache_dtype = q_dtype or PKV_FP8_E4M3
 *   k_scale,
 *   v_scale      device fp32 scalars, read only for an FP8 cache (K = code *
 *                k_scale, V = code * v_scale, as in paged_attention_decode)
 *   out          [num_q_tokens, num_heads, head_dim], q_dtype
 *
 * Row r of sequence i sits at position p = seq_lens[i] - q_i + (r -
 * query_start[i]) and gets softmax(scale * q . K[t]) over t = 0..p applied to V
 * (GQA: query head j reads KV head j / (num_heads / num_kv_heads)); a row with
 * p < 0 gets zeros. max_q_len must be >= every q_i: a longer chunk has only its
 * last max_q_len rows computed. Lengths are clamped to max_blocks_per_seq *
 * block_size and query_start to [0, num_q_tokens]. head_dim 64 or 128,
 * block_size 8/16/32. The default kernel (16-bit and FP8-E4M3 caches) runs on
 * the tcgen05 tensor cores with tensor-memory accumulators: a persistent kernel,
 * one CTA per SM taking items of 256 query rows (two tiles) from a work counter
 * in device memory. Each call takes the next of 64 such counters (the call's
 * last CTA resets it), so up to 64 prefill calls may be in flight at once, on
 * any streams; a CUDA graph that holds a call keeps that call's counter, so
 * replays of one graph must not overlap each other. flags PKV_PREFILL_MMA_SYNC
 * selects the mma.sync kernel (64 rows per CTA, no counter) instead; other flag
 * bits are an error. With an FP8-E4M3 cache the codes are widened exactly to
 * f16 (in shared memory on the tcgen05 kernel, in registers on the mma.sync
 * one), the query is rounded to f16, k_scale is folded into the score scale
 * and v_scale into the output.
 * Errors: PKV_ERR_SHAPE, PKV_ERR_UNSUPPORTED, PKV_ERR_DTYPE, PKV_ERR_NULL,
 * PKV_ERR_ALIGN, PKV_ERR_CUDA.
 */
#define PKV_PREFILL_MMA_SYNC 1u  /* use the mma.sync kernel instead of the tcgen05 one */
int paged_attention_prefill(void* out, const void* query, const void* k_cache,
                            const void* v_cache, const int32_t* block_table,
                            const int32_t* seq_lens, const int32_t* query_start, int num_seqs,
                            int num_q_tokens, int max_q_len, int num_heads, int num_kv_heads,
                            int head_dim, int block_size, int max_blocks_per_seq,
                            int64_t num_blocks, float scale, int q_dtype, int cache_dtype,
                            const float* k_scale, const float* v_scale, unsigned flags,
                            void* stream);

/*
 * Health word of the device kernels, a bitmask since the last clear:
 *   1  a bounded wait inside a kernel expired (every wait is bounded, about one
 *      second; the CTA skips the rest of its work, so a wrong result is
 *      reported instead of a hung GPU);
 *   2  a kernel read a block-table entry outside [0, num_blocks) (a corrupt
 *      table; those rows read as zeros).
 * Returns 0 when healthy, the bitmask, or PKV_ERR_CUDA. Synchronises the
 * current device; clear != 0 resets the word.
 */
int pkv_device_status(int clear);

/*
 * Self-test of the health word above, with no fault: enqueues one tiny kernel
 * on `stream` that, if note_out_of_pool != 0, records an out-of-pool block id
 * (value 2) as the kernels do, then waits, through the same bounded wait the
 * kernels use, on a barrier nothing completes, for at most limit_cycles SM
 * clock cycles (0 .. 2^31, about one second at 2 GHz). The wait expires and
 * records value 1 without clearing value 2; the kernel returns and the context
 * stays usable. pkv_device_status() then reads 1 | (note_out_of_pool ? 2 : 0),
 * plus whatever was set before. Errors: PKV_ERR_SHAPE (limit out of range),
 * PKV_ERR_CUDA.
 */
int pkv_selftest_expired_wait(int64_t limit_cycles, int note_out_of_pool, void* stream);

/* Static, NUL-terminated description of a pkv_status value. */
const char* pkv_status_string(int status);

/* Library version, major * 10000 + minor * 100 + patch. */
int pkv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H */
