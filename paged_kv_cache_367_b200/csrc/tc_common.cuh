// Device and host helpers shared by the tensor-core attention kernels
// (decode_tc.cu, prefill_tc.cu): mbarriers with bounded waits, TMA tile and
// bulk copies, ldmatrix, mma.sync m16n8k16 for bf16/f16, and the 5-D tensor
// map that describes a paged pool [num_blocks, bs, Hkv, D] so that one copy
// moves a (block, KV head) tile as 128-byte rows with the 128B swizzle.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace pkv {
namespace tcx {

constexpr long long kWaitCycles = 1ll << 31;  // ~1 s at 2 GHz

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase of `bar` with the given parity. Returns false if
// the CTA is aborting or the wait expired, which starts the abort and sets the
// device error word *timeout.
__device__ __forceinline__ bool mbar_wait_or_abort(uint64_t* bar, uint32_t parity,
                                                   volatile int* abort, int* timeout,
                                                   long long limit = kWaitCycles) {
  if (*abort) return false;
  const long long t0 = clock64();
  for (int it = 1;; ++it) {
    if (mbar_try(bar, parity)) return true;
    if ((it & 31) == 0) {
      if (*abort) return false;
      if (clock64() - t0 > limit) {
        *abort = 1;
        atomicOr(timeout, 1);
        return false;
      }
    }
  }
}

__device__ __forceinline__ void tma_load_5d(void* dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            int c3, int c4, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4),
      "r"(smem_u32(bar))
      : "memory");
}

// The same copy with an L2 cache-policy hint (createpolicy).
__device__ __forceinline__ void tma_load_5d_hint(void* dst, const CUtensorMap* map, int c0, int c1,
                                                 int c2, int c3, int c4, uint64_t* bar,
                                                 uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3, %4, %5, %6}], [%7], %8;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4),
      "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// L2 policy that evicts the lines it marks first: for data read once.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// Two E4M3 codes (low byte first) to an f16x2 pair.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_codes) {
  uint32_t d;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(d) : "h"((unsigned short)(two_codes & 0xffffu)));
  return d;
}

// bf16x2 or f16x2 bits to f16x2 bits.
template <typename T> __device__ __forceinline__ uint32_t to_f16x2(uint32_t v);
template <> __device__ __forceinline__ uint32_t to_f16x2<__half>(uint32_t v) { return v; }
template <> __device__ __forceinline__ uint32_t to_f16x2<__nv_bfloat16>(uint32_t v) {
  const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v));
  __half2 h = __floats2half2_rn(f.x, f.y);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint32_t movmatrix_t(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
  return d;
}

template <typename T> struct Mma;
template <> struct Mma<__nv_bfloat16> {
  static __device__ __forceinline__ void run(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                             uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
  static __device__ __forceinline__ uint32_t pack(float lo, float hi, float& rlo, float& rhi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    rlo = __low2float(v);
    rhi = __high2float(v);
    return *reinterpret_cast<uint32_t*>(&v);
  }
};
template <> struct Mma<__half> {
  static __device__ __forceinline__ void run(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                             uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
  static __device__ __forceinline__ uint32_t pack(float lo, float hi, float& rlo, float& rhi) {
    __half2 v = __floats2half2_rn(lo, hi);
    rlo = __low2float(v);
    rhi = __high2float(v);
    return *reinterpret_cast<uint32_t*>(&v);
  }
};


// ---------------------------------------------------------------- host ----

inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 5-D view of a [num_blocks, bs, Hkv, D] pool of e-byte elements: (d_lo, token
// bs, d_hi, head Hkv, block num_blocks), d_lo spanning a row piece of
// min(D * e, 128) bytes; one box is a whole (block, head) tile, landing as
// 128-byte rows with the 128B swizzle (64-byte rows with the 64B swizzle when a
// token's whole row is 64 bytes, as for E4M3 at head_dim 64).
// per_plane: the box covers one piece of head_dim (d_hi extent 1) instead of
// all of them, for copies that place each piece in its own region.
inline bool encode_pool_map(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int e,
                            int D, int bs, int Hkv, int64_t nb, bool per_plane = false) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const int row_bytes = D * e >= 128 ? 128 : D * e;
  if (row_bytes != 128 && row_bytes != 64) return false;
  const cuuint64_t row = (cuuint64_t)(row_bytes / e);  // elements per row piece
  cuuint64_t dims[5] = {row, (cuuint64_t)bs, (cuuint64_t)(D / row), (cuuint64_t)Hkv, (cuuint64_t)nb};
  cuuint64_t strides[4] = {(cuuint64_t)Hkv * D * e, (cuuint64_t)row_bytes, (cuuint64_t)D * e,
                           (cuuint64_t)bs * Hkv * D * e};
  cuuint32_t box[5] = {(cuuint32_t)row, (cuuint32_t)bs, per_plane ? 1u : (cuuint32_t)(D / row), 1, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = enc(map, dt, 5, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE,
                   row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace tcx
}  // namespace pkv
