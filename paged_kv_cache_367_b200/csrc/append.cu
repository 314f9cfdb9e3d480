// paged_kv_append: write each new token's K/V row into its slot of the block pool.
//
// "vLLM 推理引擎源码级拆解" (chenxutan.com/d/5333) §2.2: the token generated in a
// step goes into the next free slot of the sequence's last block (a fresh block
// from the free pool when the last one is full). The caller has already chosen
// that slot; this kernel only moves the bytes, converting to E4M3 for an FP8
// cache ("vLLM 0.5 深度拆解", chenxutan.com/d/4924, §4.2).
//
// One thread moves one 8-element vector of one (token, KV head) row: a 16-byte
// load (32 for fp32 sources) and a 16-, 32- or 8-byte store. Launch-bound for a
// decode step (one token per sequence), so the grid is just large enough.
#include "common.cuh"

namespace pkv {

template <typename ST>
__device__ __forceinline__ void load8(const ST* p, float (&x)[8]) {
  load_row<ST, 8>(p, x);
}

// Same-dtype copy: move raw bytes.
template <typename ST>
__device__ __forceinline__ void copy8(const ST* __restrict__ src, ST* __restrict__ dst) {
  constexpr int kVec = 8 * (int)sizeof(ST) / 16;
#pragma unroll
  for (int k = 0; k < kVec; ++k)
    reinterpret_cast<uint4*>(dst)[k] = __ldg(reinterpret_cast<const uint4*>(src) + k);
}

__device__ __forceinline__ void quant8(const float (&x)[8], float scale, uint8_t* __restrict__ dst) {
  uint32_t w[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t acc = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      // IEEE fp32 division, then round-to-nearest-even E4M3 with saturation.
      float v = __fdiv_rn(x[4 * h + k], scale);
      uint32_t code = (uint32_t)__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
      acc |= code << (8 * k);
    }
    w[h] = acc;
  }
  *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
}

template <typename ST, bool kFp8>
__global__ void __launch_bounds__(256) append_kernel(
    const ST* __restrict__ key, const ST* __restrict__ value, void* __restrict__ k_cache,
    void* __restrict__ v_cache, const int64_t* __restrict__ slot_mapping, int num_tokens,
    int num_kv_heads, int head_dim, int64_t num_slots, const float* __restrict__ k_scale,
    const float* __restrict__ v_scale) {
  // A kernel launched after this one with programmatic stream serialization
  // (the decode's early start) may begin now; it waits for this grid to finish
  // before it reads the caches.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int vec_per_row = head_dim / 8;
  const int64_t row = (int64_t)num_kv_heads * head_dim;
  const int64_t total = (int64_t)num_tokens * num_kv_heads * vec_per_row;
  float ks = 1.f, vs = 1.f;
  if constexpr (kFp8) {
    ks = __ldg(k_scale);
    vs = __ldg(v_scale);
  }
  for (int64_t n = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; n < total;
       n += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = n / ((int64_t)num_kv_heads * vec_per_row);
    const int64_t rem = n - t * num_kv_heads * vec_per_row;  // head * vec_per_row + c
    const int64_t slot = __ldg(slot_mapping + t);
    if (slot < 0 || slot >= num_slots) continue;
    const int64_t src = t * row + rem * 8;
    const int64_t dst = slot * row + rem * 8;
    if constexpr (kFp8) {
      float x[8];
      load8(key + src, x);
      quant8(x, ks, static_cast<uint8_t*>(k_cache) + dst);
      load8(value + src, x);
      quant8(x, vs, static_cast<uint8_t*>(v_cache) + dst);
    } else {
      copy8(key + src, static_cast<ST*>(k_cache) + dst);
      copy8(value + src, static_cast<ST*>(v_cache) + dst);
    }
  }
}

template <typename ST, bool kFp8>
static cudaError_t launch_append_t(const void* key, const void* value, void* k_cache,
                                   void* v_cache, const int64_t* slot_mapping, int num_tokens,
                                   int num_kv_heads, int head_dim, int64_t num_slots,
                                   const float* k_scale, const float* v_scale,
                                   cudaStream_t stream) {
  const int64_t total = (int64_t)num_tokens * num_kv_heads * (head_dim / 8);
  if (total == 0) return cudaSuccess;
  const int threads = 256;
  int64_t blocks = (total + threads - 1) / threads;
  if (blocks > 148 * 16) blocks = 148 * 16;
  append_kernel<ST, kFp8><<<(unsigned)blocks, threads, 0, stream>>>(
      static_cast<const ST*>(key), static_cast<const ST*>(value), k_cache, v_cache,
      slot_mapping, num_tokens, num_kv_heads, head_dim, num_slots, k_scale, v_scale);
  return cudaGetLastError();
}

cudaError_t launch_append(const void* key, const void* value, void* k_cache, void* v_cache,
                          const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                          int head_dim, int64_t num_slots, int src_dtype, bool fp8,
                          const float* k_scale, const float* v_scale, cudaStream_t stream) {
#define PKV_APPEND_CASE(CODE, T)                                                              \
  case CODE:                                                                                 \
    return fp8 ? launch_append_t<T, true>(key, value, k_cache, v_cache, slot_mapping,       \
                                          num_tokens, num_kv_heads, head_dim, num_slots,     \
                                          k_scale, v_scale, stream)                          \
               : launch_append_t<T, false>(key, value, k_cache, v_cache, slot_mapping,      \
                                           num_tokens, num_kv_heads, head_dim, num_slots,    \
                                           k_scale, v_scale, stream);
  switch (src_dtype) {
    PKV_APPEND_CASE(PKV_F32, float)
    PKV_APPEND_CASE(PKV_F16, __half)
    PKV_APPEND_CASE(PKV_BF16, __nv_bfloat16)
    default:
      return cudaErrorInvalidValue;
  }
#undef PKV_APPEND_CASE
}

}  // namespace pkv
