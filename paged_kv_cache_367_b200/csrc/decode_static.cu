// paged_attention_decode_static: paged_attention_decode for callers that cannot
// allocate device memory.
//
// Some callers have no way to obtain scratch memory on the device: code that
// runs inside another framework which owns every device allocation through its
// own pool and forbids outside cudaMalloc calls, latency-critical decode loops
// where cudaMalloc's implicit device synchronisation is not acceptable, and
// bindings from environments that have no device-memory API at all. This entry
// point gives them the same decode with its split-sequence scratch held in a
// fixed array of device memory that belongs to this library.
//
// The array is a file-scope static __device__ object of kStaticScratchBytes
// (16 MiB). It occupies that much memory on every device where this file's
// device code is loaded, until the process exits. Host code may not use the
// array's name as an address (on the host it is only a stand-in for the device
// object), so the first call on each device looks the address up with
// cudaGetSymbolAddress while that device is current and keeps it; make that
// first call before any stream capture. All calls share the array and it keeps
// the contents of the last call: the counters that must start at zero are
// cleared by every call (a memset on the caller's stream, whatever the flags
// say), and two calls whose
// work overlaps on the GPU (different streams, or different host threads) race
// on the array and must be serialised by the caller.
#include <mutex>

#include "pagedkv.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_address[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once).
int static_scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PKV_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_address[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr)
      return PKV_ERR_CUDA;
    g_scratch_address[dev] = p;
  }
  *out = g_scratch_address[dev];
  return PKV_OK;
}

}  // namespace

extern "C" int paged_attention_decode_static(
    void* out, const void* query, const void* k_cache, const void* v_cache,
    const int32_t* block_table, const int32_t* seq_lens, int num_seqs, int num_heads,
    int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq, int64_t num_blocks,
    int max_seq_len, float scale, int q_dtype, int cache_dtype, const float* k_scale,
    const float* v_scale, int partition_size, int max_ctas, unsigned flags, void* stream) {
  const size_t need = paged_attention_workspace_size(num_seqs, num_heads, num_kv_heads,
                                                     head_dim, max_seq_len, partition_size);
  if (need > kStaticScratchBytes) return PKV_ERR_WORKSPACE;  // beyond the fixed scratch
  void* scratch = nullptr;
  if (need > 0) {
    const int st = static_scratch_address(&scratch);
    if (st != PKV_OK) return st;
  }
  // The shared array may hold another call's data where this call keeps its
  // counters (their place depends on the group size and head_dim), so the
  // counters are always cleared: a caller's PKV_DECODE_ZEROED_WORKSPACE is
  // ignored here.
  flags &= ~PKV_DECODE_ZEROED_WORKSPACE;
  return paged_attention_decode(out, query, k_cache, v_cache, block_table, seq_lens, num_seqs,
                                num_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                                num_blocks, max_seq_len, scale, q_dtype, cache_dtype, k_scale,
                                v_scale, partition_size, max_ctas, flags, scratch,
                                need > 0 ? kStaticScratchBytes : 0, stream);
}
