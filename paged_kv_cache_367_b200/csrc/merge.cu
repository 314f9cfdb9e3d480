// Log-sum-exp merge of the partial results of split sequences.
//
// A sequence cut into segments (see schedule.cuh) leaves, per query head and
// segment, a normalised partial output o_p and its base-2 log-sum-exp lse_p.
// The exact softmax over the whole sequence is recovered as
//   M = max_p lse_p,  w_p = 2^(lse_p - M),  out = sum_p w_p o_p / sum_p w_p,
// the blockwise form of the online softmax that "vLLM 推理引擎源码级拆解"
// (chenxutan.com/d/5333) §2.3 names. Segments are found by following the link
// array from partition 0; a unit whose first link reaches its last partition
// was finished by the decode kernel and is skipped.
#include "schedule.cuh"

namespace pkv {

template <typename OT>
__global__ void __launch_bounds__(128) merge_kernel(const DecodeParams prm) {
  const int Hq = prm.num_heads, Hkv = prm.num_kv_heads, g = Hq / Hkv, D = prm.head_dim;
  const int MP = prm.max_parts, P = prm.part;
  for (int64_t u = blockIdx.x; u < (int64_t)prm.num_seqs * Hkv; u += gridDim.x) {
    const int i = (int)(u / Hkv), h = (int)(u % Hkv);
    const int L = clamp_len(__ldg(prm.seq_lens + i), prm.len_cap);
    if (L == 0) continue;
    const int nparts = (L + P - 1) / P;
    const int* link = prm.ws_link + u * MP;
    if (__ldg(link) >= nparts) continue;  // finished whole by the decode kernel
    for (int e = threadIdx.x; e < g * D; e += blockDim.x) {
      const int j = e / D, d = e % D;
      const int64_t row = ((int64_t)i * Hq + h * g + j) * MP;
      float M = -INFINITY;
      int p = 0;
      for (int guard = 0; guard < nparts && p < nparts; ++guard) {
        M = fmaxf(M, prm.ws_lse[row + p]);
        const int nx = __ldg(link + p);
        if (nx <= p) break;
        p = nx;
      }
      float num = 0.f, den = 0.f;
      p = 0;
      for (int guard = 0; guard < nparts && p < nparts; ++guard) {
        const float w = fast_exp2(prm.ws_lse[row + p] - M);
        num = fmaf(w, prm.ws_o[(row + p) * D + d], num);
        den += w;
        const int nx = __ldg(link + p);
        if (nx <= p) break;
        p = nx;
      }
      static_cast<OT*>(prm.out)[((int64_t)i * Hq + h * g + j) * D + d] = from_f32<OT>(num / den);
    }
  }
}

cudaError_t launch_merge(const DecodeParams& prm, int q_dtype, int num_sms, cudaStream_t stream) {
  const int64_t units = (int64_t)prm.num_seqs * prm.num_kv_heads;
  if (units == 0 || prm.part == 0) return cudaSuccess;
  int grid = (int)(units < (int64_t)num_sms * 16 ? units : (int64_t)num_sms * 16);
  switch (q_dtype) {
    case PKV_F32: merge_kernel<float><<<grid, 128, 0, stream>>>(prm); break;
    case PKV_F16: merge_kernel<__half><<<grid, 128, 0, stream>>>(prm); break;
    case PKV_BF16: merge_kernel<__nv_bfloat16><<<grid, 128, 0, stream>>>(prm); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace pkv
