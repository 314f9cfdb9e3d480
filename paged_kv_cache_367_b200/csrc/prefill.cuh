// Arguments of the multi-token (causal) paged attention kernels, shared by the
// mma.sync kernel (prefill_tc.cu) and the tcgen05 kernel (prefill_tc5.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace pkv {
namespace pf {

struct PrefillParams {
  void* out;
  const void* query;
  const int32_t* block_table;
  const int32_t* seq_lens;
  const int32_t* query_start;
  int num_heads, num_kv_heads, block_size, max_blocks_per_seq;
  int num_q_tokens, max_q_len;
  int num_blocks;
  float score_scale;  // softmax scale * log2(e)
  const float* k_scale;  // device scalars of an E4M3 cache (unused otherwise)
  const float* v_scale;
};

// Launch of the tcgen05 kernel (prefill_tc5.cu); mk / mv are per-plane pool maps.
cudaError_t launch_prefill_tc5(const PrefillParams& p, const CUtensorMap& mk, const CUtensorMap& mv,
                               int head_dim, bool bf16, bool f8, int num_seqs, cudaStream_t stream);
bool prefill_tc5_supported(int head_dim);

}  // namespace pf

int pf5_status_flag(bool clear, int* value);

}  // namespace pkv
