// C ABI entry points: argument checks, workspace layout, kernel dispatch.
#include <math.h>

#include "pagedkv.h"
#include "schedule.cuh"

namespace pkv {
cudaError_t launch_append(const void* key, const void* value, void* k_cache, void* v_cache,
                          const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                          int head_dim, int64_t num_slots, int src_dtype, bool fp8,
                          const float* k_scale, const float* v_scale, cudaStream_t stream);
cudaError_t launch_decode_simt(const DecodeParams& prm, int q_dtype, int cache_dtype,
                               int max_ctas, int num_sms, cudaStream_t stream);
bool tc_supported(int q_dtype, int cache_dtype, int head_dim, int group);
cudaError_t launch_decode_tc(const DecodeParams& prm, int q_dtype, int cache_dtype,
                             int max_ctas, int num_sms, bool early_start, int products,
                             cudaStream_t stream);
int tc_timeout_flag(bool clear, int* value);
int pf_timeout_flag(bool clear, int* value);
int simt_status_flag(bool clear, int* value);
int pf5_status_flag(bool clear, int* value);
int launch_status_selftest(long long limit_cycles, int note_out_of_pool, cudaStream_t stream);

static bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

static int num_sms_of_current_device(int* out) {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PKV_ERR_CUDA;
  if (dev < 0 || dev >= 64) return PKV_ERR_CUDA;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
      return PKV_ERR_CUDA;
    cache[dev] = n;
  }
  *out = cache[dev];
  return PKV_OK;
}

struct WsLayout {
  size_t o, lse, done, total;
};

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Partials: two slots per range, up to kMaxRanges ranges, each g rows of D
// floats plus g log-sum-exp values; one counter per (sequence, KV head) and the
// dynamic-range counter.
static WsLayout workspace_layout(int64_t S, int64_t Hq, int64_t Hkv, int64_t D, int64_t parts) {
  WsLayout w;
  const int64_t g = Hq / Hkv, slots = 2 * (int64_t)kMaxRanges;
  w.o = 0;
  w.lse = align256(w.o + sizeof(float) * slots * g * D);
  w.done = align256(w.lse + sizeof(float) * slots * g);
  w.total = align256(w.done + sizeof(int32_t) * (S * Hkv + 1));
  if (parts <= 1) w.total = 0;  // no sequence can be cut
  return w;
}

static int64_t parts_for(int max_seq_len, int partition_size) {
  if (partition_size <= 0 || max_seq_len <= 0) return 0;
  return ((int64_t)max_seq_len + partition_size - 1) / partition_size;
}

}  // namespace pkv

using namespace pkv;

extern "C" {

int pkv_version(void) { return 100; }

int pkv_device_status(int clear) {
  int v = 0, w = 0, x = 0, y = 0;
  if (tc_timeout_flag(clear != 0, &v) != 0 || pf_timeout_flag(clear != 0, &w) != 0 ||
      simt_status_flag(clear != 0, &x) != 0 || pf5_status_flag(clear != 0, &y) != 0)
    return PKV_ERR_CUDA;
  return v | w | x | y;
}

int pkv_selftest_expired_wait(int64_t limit_cycles, int note_out_of_pool, void* stream) {
  if (limit_cycles < 0 || limit_cycles > (int64_t(1) << 31)) return PKV_ERR_SHAPE;
  return launch_status_selftest(limit_cycles, note_out_of_pool, (cudaStream_t)stream) == 0
             ? PKV_OK
             : PKV_ERR_CUDA;
}

const char* pkv_status_string(int status) {
  switch (status) {
    case PKV_OK: return "ok";
    case PKV_ERR_NULL: return "a required pointer is NULL";
    case PKV_ERR_SHAPE: return "a size is out of range or inconsistent";
    case PKV_ERR_DTYPE: return "unknown dtype or unsupported dtype pair";
    case PKV_ERR_UNSUPPORTED: return "head_dim or block_size outside the supported set";
    case PKV_ERR_WORKSPACE: return "workspace missing or too small";
    case PKV_ERR_CUDA: return "CUDA runtime call or kernel launch failed";
    case PKV_ERR_ALIGN: return "pointer not 16-byte aligned";
    case PKV_ERR_NO_BLOCKS: return "not enough free blocks";
    case PKV_ERR_SEQ: return "unknown, duplicate or swapped-out sequence id";
    case PKV_ERR_MEMORY: return "pool is neither device memory nor pinned host memory";
    default: return "unknown status";
  }
}

int paged_kv_append(const void* key, const void* value, void* k_cache, void* v_cache,
                    const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                    int head_dim, int block_size, int64_t num_blocks, int src_dtype,
                    int cache_dtype, const float* k_scale, const float* v_scale,
                    void* stream) {
  if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || head_dim % 8 != 0 ||
      block_size <= 0 || num_blocks <= 0)
    return PKV_ERR_SHAPE;
  if (src_dtype != PKV_F32 && src_dtype != PKV_F16 && src_dtype != PKV_BF16) return PKV_ERR_DTYPE;
  if (cache_dtype != src_dtype && cache_dtype != PKV_FP8_E4M3) return PKV_ERR_DTYPE;
  const bool fp8 = cache_dtype == PKV_FP8_E4M3;
  if (num_tokens == 0) return PKV_OK;
  if (!key || !value || !k_cache || !v_cache || !slot_mapping) return PKV_ERR_NULL;
  if (fp8 && (!k_scale || !v_scale)) return PKV_ERR_NULL;
  if (!aligned16(key) || !aligned16(value) || !aligned16(k_cache) || !aligned16(v_cache) ||
      ((uintptr_t)slot_mapping & 7u))
    return PKV_ERR_ALIGN;
  cudaError_t e = launch_append(key, value, k_cache, v_cache, slot_mapping, num_tokens,
                                num_kv_heads, head_dim, num_blocks * (int64_t)block_size,
                                src_dtype, fp8, k_scale, v_scale, (cudaStream_t)stream);
  return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

size_t paged_attention_workspace_size(int num_seqs, int num_heads, int num_kv_heads,
                                      int head_dim, int max_seq_len, int partition_size) {
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
      max_seq_len < 0 || partition_size < 0)
    return 0;
  return workspace_layout(num_seqs, num_heads, num_kv_heads, head_dim,
                          parts_for(max_seq_len, partition_size)).total;
}

int paged_attention_decode(void* out, const void* query, const void* k_cache,
                           const void* v_cache, const int32_t* block_table,
                           const int32_t* seq_lens, int num_seqs, int num_heads,
                           int num_kv_heads, int head_dim, int block_size,
                           int max_blocks_per_seq, int64_t num_blocks, int max_seq_len,
                           float scale, int q_dtype, int cache_dtype, const float* k_scale,
                           const float* v_scale, int partition_size, int max_ctas,
                           unsigned flags, void* workspace, size_t workspace_bytes,
                           void* stream) {
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0 ||
      max_blocks_per_seq <= 0 || num_blocks <= 0 || max_seq_len < 0 || partition_size < 0 ||
      max_ctas < 0 || !isfinite(scale) ||
      (flags & ~(PKV_DECODE_FORCE_SIMT | PKV_DECODE_ZEROED_WORKSPACE | PKV_DECODE_EARLY_START |
                 PKV_DECODE_TENSOR_CORES | PKV_DECODE_CUDA_CORES)) ||
      ((flags & PKV_DECODE_TENSOR_CORES) && (flags & PKV_DECODE_CUDA_CORES)))
    return PKV_ERR_SHAPE;
  if (head_dim != 64 && head_dim != 128) return PKV_ERR_UNSUPPORTED;
  if (block_size != 8 && block_size != 16 && block_size != 32) return PKV_ERR_UNSUPPORTED;
  if (partition_size > 0 && partition_size % block_size != 0) return PKV_ERR_SHAPE;
  if (q_dtype != PKV_F32 && q_dtype != PKV_F16 && q_dtype != PKV_BF16) return PKV_ERR_DTYPE;
  if (cache_dtype != q_dtype && cache_dtype != PKV_FP8_E4M3) return PKV_ERR_DTYPE;
  const bool fp8 = cache_dtype == PKV_FP8_E4M3;
  if (num_seqs == 0) return PKV_OK;
  if (!out || !query || !k_cache || !v_cache || !block_table || !seq_lens) return PKV_ERR_NULL;
  if (fp8 && (!k_scale || !v_scale)) return PKV_ERR_NULL;
  if (!aligned16(out) || !aligned16(query) || !aligned16(k_cache) || !aligned16(v_cache) ||
      ((uintptr_t)block_table & 3u) || ((uintptr_t)seq_lens & 3u))
    return PKV_ERR_ALIGN;
  const int64_t parts = parts_for(max_seq_len, partition_size);
  const WsLayout ws = workspace_layout(num_seqs, num_heads, num_kv_heads, head_dim, parts);
  if (ws.total > 0) {
    if (!workspace || workspace_bytes < ws.total) return PKV_ERR_WORKSPACE;
    if (((uintptr_t)workspace & 255u) != 0) return PKV_ERR_ALIGN;
  }
  int sms = 0;
  if (num_sms_of_current_device(&sms) != PKV_OK) return PKV_ERR_CUDA;

  DecodeParams prm;
  prm.out = out;
  prm.query = query;
  prm.k_cache = k_cache;
  prm.v_cache = v_cache;
  prm.block_table = block_table;
  prm.seq_lens = seq_lens;
  prm.num_seqs = num_seqs;
  prm.num_heads = num_heads;
  prm.num_kv_heads = num_kv_heads;
  prm.head_dim = head_dim;
  prm.block_size = block_size;
  prm.max_blocks_per_seq = max_blocks_per_seq;
  prm.num_blocks = num_blocks;
  const int64_t cap = (int64_t)max_blocks_per_seq * block_size;
  prm.len_cap = (int)(cap < max_seq_len ? cap : max_seq_len);
  prm.part = parts > 1 ? partition_size : 0;
  prm.unit_cost = 24;  // a segment's set-up and hand-off, in tokens (measured)
  prm.unit_round = 64;  // the tensor-core kernel streams 64-token chunks
  prm.dyn_ranges = 0;  // the tensor-core launcher enables dynamic ranges
  prm.static_share = 1024;
  prm.score_scale = scale * kLog2e;
  prm.k_scale = k_scale;
  prm.v_scale = v_scale;
  char* wsb = static_cast<char*>(workspace);
  prm.ws_o = ws.total ? reinterpret_cast<float*>(wsb + ws.o) : nullptr;
  prm.ws_lse = ws.total ? reinterpret_cast<float*>(wsb + ws.lse) : nullptr;
  prm.ws_done = ws.total ? reinterpret_cast<int*>(wsb + ws.done) : nullptr;

  cudaStream_t st = (cudaStream_t)stream;
  const int group = num_heads / num_kv_heads;
  cudaError_t e;
  if (ws.total > 0 && !(flags & PKV_DECODE_ZEROED_WORKSPACE)) {
    // Per-unit counters of finished split tokens and the dynamic-range counter
    // start at zero (each call also leaves them at zero).
    e = cudaMemsetAsync(prm.ws_done, 0, sizeof(int32_t) * ((size_t)num_seqs * num_kv_heads + 1),
                        st);
    if (e != cudaSuccess) return PKV_ERR_CUDA;
  }
  if (!(flags & PKV_DECODE_FORCE_SIMT) && tc_supported(q_dtype, cache_dtype, head_dim, group))
    e = launch_decode_tc(prm, q_dtype, cache_dtype, max_ctas, sms,
                         (flags & PKV_DECODE_EARLY_START) != 0,
                         (flags & PKV_DECODE_CUDA_CORES) ? 1 : (flags & PKV_DECODE_TENSOR_CORES) ? -1 : 0,
                         st);
  else
    e = launch_decode_simt(prm, q_dtype, cache_dtype, max_ctas, sms, st);
  if (e != cudaSuccess) return PKV_ERR_CUDA;
  return PKV_OK;
}

}  // extern "C"
