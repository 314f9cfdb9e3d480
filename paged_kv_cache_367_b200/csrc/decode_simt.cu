// PagedAttention decode on CUDA cores (fp32/fp16/bf16 queries, any cache type).
//
// "vLLM 推理引擎源码级拆解" (chenxutan.com/d/5333) §2.3: for each token of a
// sequence, logical block = tok / block_size, offset = tok % block_size,
// physical block = block_table[logical block]; score = dot(q, k) * scale; an
// online softmax accumulates V; the result is written back. GQA: the g query
// heads that share a KV head are served from one read of its K/V rows.
//
// Layout of the work: a 128-thread CTA walks its segments (see schedule.cuh).
// Each half-warp takes one token at a time; its 16 lanes each own D/16
// consecutive dimensions, so one K row is one coalesced 16-lane read. Up to 8
// query heads are handled per pass over the K/V rows (more passes when g > 8).
// The 8 half-warps keep separate softmax states, merged through shared memory
// at the end of each segment; pieces of split units are finished as in
// schedule.cuh (finish_piece). This kernel is the general path (fp32, mixed
// dtypes, wide groups); 16-bit caches at head_dim 64/128 use the tensor-core
// kernel.
#include "schedule.cuh"

namespace pkv {

__device__ int g_simt_status = 0;  // bit 1: a block id outside the pool was read

constexpr int kSimtThreads = 128;
constexpr int kSimtHeads = 8;    // query heads per pass

template <int D>
struct SimtShared {
  SchedShared sched;
  float m[8][kSimtHeads];
  float l[8][kSimtHeads];
  float acc[8][kSimtHeads][D];
  int flag;
};

template <typename QT, typename KT, int D>
__global__ void __launch_bounds__(kSimtThreads) decode_simt_kernel(const DecodeParams prm) {
  constexpr int DPL = D / 16;  // dimensions per lane
  constexpr int kSimtUnroll = D == 64 ? 4 : 2;  // tokens per half-warp per step
  __shared__ SimtShared<D> sm;

  SegmentWalker walker;
  init_walker<QT>(prm, sm.sched, walker);

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int half = lane >> 4, l16 = lane & 15;
  const int hw = warp * 2 + half;  // half-warp index 0..7
  const int Hq = prm.num_heads, Hkv = prm.num_kv_heads, g = Hq / Hkv;
  const int bs = prm.block_size;
  constexpr bool kFp8 = sizeof(KT) == 1;
  const float kscale = kFp8 ? __ldg(prm.k_scale) : 1.f;
  const float vscale = kFp8 ? __ldg(prm.v_scale) : 1.f;
  const float qmul = prm.score_scale * kscale;
  const KT* kc = static_cast<const KT*>(prm.k_cache);
  const KT* vc = static_cast<const KT*>(prm.v_cache);
  const QT* qp = static_cast<const QT*>(prm.query);
  const int64_t row_stride = (int64_t)Hkv * D;  // elements between consecutive tokens

  Segment seg;
  while (walker.next(seg)) {
    const int i = seg.seq, h = seg.head;
    const int32_t* bt = prm.block_table + (int64_t)i * prm.max_blocks_per_seq;
    for (int hg = 0; hg < g; hg += kSimtHeads) {
      const int gcnt = min(kSimtHeads, g - hg);
      float q[kSimtHeads][DPL];
#pragma unroll
      for (int j = 0; j < kSimtHeads; ++j) {
        if (j < gcnt) {
          load_row<QT, DPL>(qp + ((int64_t)i * Hq + h * g + hg + j) * D + l16 * DPL, q[j]);
#pragma unroll
          for (int k = 0; k < DPL; ++k) q[j][k] *= qmul;
        } else {
#pragma unroll
          for (int k = 0; k < DPL; ++k) q[j][k] = 0.f;
        }
      }
      float m[kSimtHeads], l[kSimtHeads], acc[kSimtHeads][DPL];
#pragma unroll
      for (int j = 0; j < kSimtHeads; ++j) {
        m[j] = -INFINITY;
        l[j] = 0.f;
#pragma unroll
        for (int k = 0; k < DPL; ++k) acc[j][k] = 0.f;
      }
      // Warp-uniform loop: each step covers 2 * kSimtUnroll tokens per warp.
      for (int tb = seg.t0 + warp * 2 * kSimtUnroll; tb < seg.t1; tb += 8 * kSimtUnroll) {
        float kv[kSimtUnroll][DPL], vv[kSimtUnroll][DPL];
        bool act[kSimtUnroll];
#pragma unroll
        for (int u = 0; u < kSimtUnroll; ++u) {
          const int t = tb + 2 * u + half;
          act[u] = t < seg.t1;
          int64_t phys = -1;
          if (act[u]) phys = __ldg(bt + t / bs);
          if (act[u] && (phys < 0 || phys >= prm.num_blocks)) atomicOr(&g_simt_status, 2);
          if (act[u] && phys >= 0 && phys < prm.num_blocks) {
            const int64_t off = ((phys * bs + t % bs) * row_stride) + (int64_t)h * D + l16 * DPL;
            load_row<KT, DPL>(kc + off, kv[u]);
            load_row<KT, DPL>(vc + off, vv[u]);
          } else {
#pragma unroll
            for (int k = 0; k < DPL; ++k) kv[u][k] = vv[u][k] = 0.f;
          }
        }
        float s[kSimtUnroll][kSimtHeads];
#pragma unroll
        for (int u = 0; u < kSimtUnroll; ++u) {
#pragma unroll
          for (int j = 0; j < kSimtHeads; ++j) {
            float d = 0.f;
#pragma unroll
            for (int k = 0; k < DPL; ++k) d = fmaf(q[j][k], kv[u][k], d);
#pragma unroll
            for (int o = 8; o >= 1; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
            s[u][j] = act[u] ? d : -INFINITY;
          }
        }
#pragma unroll
        for (int j = 0; j < kSimtHeads; ++j) {
          float mx = m[j];
#pragma unroll
          for (int u = 0; u < kSimtUnroll; ++u) mx = fmaxf(mx, s[u][j]);
          const float mu = mx == -INFINITY ? 0.f : mx;
          const float a = fast_exp2(m[j] - mu);
          m[j] = mx;
          l[j] *= a;
#pragma unroll
          for (int k = 0; k < DPL; ++k) acc[j][k] *= a;
#pragma unroll
          for (int u = 0; u < kSimtUnroll; ++u) {
            const float p = fast_exp2(s[u][j] - mu);
            l[j] += p;
#pragma unroll
            for (int k = 0; k < DPL; ++k) acc[j][k] = fmaf(p, vv[u][k], acc[j][k]);
          }
        }
      }
      // Merge the 8 half-warp states of this head group.
      if (l16 == 0) {
#pragma unroll
        for (int j = 0; j < kSimtHeads; ++j) {
          sm.m[hw][j] = m[j];
          sm.l[hw][j] = l[j];
        }
      }
#pragma unroll
      for (int j = 0; j < kSimtHeads; ++j)
#pragma unroll
        for (int k = 0; k < DPL; ++k) sm.acc[hw][j][l16 * DPL + k] = acc[j][k];
      __syncthreads();
      const bool whole = seg.t0 == 0 && seg.t1 == seg.len;
      for (int e = threadIdx.x; e < gcnt * D; e += kSimtThreads) {
        const int j = e / D, d = e % D;
        float M = -INFINITY;
#pragma unroll
        for (int x = 0; x < 8; ++x) M = fmaxf(M, sm.m[x][j]);
        float L = 0.f, O = 0.f;
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          const float w = fast_exp2(sm.m[x][j] - M);
          L = fmaf(w, sm.l[x][j], L);
          O = fmaf(w, sm.acc[x][j][d], O);
        }
        const int qh = h * g + hg + j;
        const float o = O / L * vscale;
        if (whole) {
          static_cast<QT*>(prm.out)[((int64_t)i * Hq + qh) * D + d] = from_f32<QT>(o);
        } else {
          const int64_t rowp = (int64_t)own_piece_slot(blockIdx.x, seg) * g + hg + j;
          prm.ws_o[rowp * D + d] = o;
          if (d == 0) prm.ws_lse[rowp] = M + fast_log2(L);
        }
      }
      __syncthreads();
    }
    if (!(seg.t0 == 0 && seg.t1 == seg.len)) {
      finish_piece<QT>(prm, walker.cuts, walker.P, seg, threadIdx.x, kSimtThreads, &sm.flag,
                       [] { __syncthreads(); });
      __syncthreads();
    }
  }
}

// CTAs per SM of one kernel instance, queried once.
template <typename K>
static int resident_ctas(K kernel, int threads, size_t smem) {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem) != cudaSuccess ||
      n < 1)
    n = 1;
  return n;
}

template <typename QT, typename KT>
static cudaError_t launch_simt_t(const DecodeParams& prm, int max_ctas, int num_sms,
                                 cudaStream_t stream) {
  auto kernel = prm.head_dim == 64 ? decode_simt_kernel<QT, KT, 64>
                                   : decode_simt_kernel<QT, KT, 128>;
  static int occ64 = 0, occ128 = 0;
  int& occ = prm.head_dim == 64 ? occ64 : occ128;
  if (occ == 0) occ = resident_ctas(kernel, kSimtThreads, 0);
  int grid = occ * num_sms;
  if (grid > kMaxRanges) grid = kMaxRanges;
  if (max_ctas > 0 && max_ctas < grid) grid = max_ctas;
  kernel<<<grid, kSimtThreads, 0, stream>>>(prm);
  return cudaGetLastError();
}

cudaError_t launch_decode_simt(const DecodeParams& prm_in, int q_dtype, int cache_dtype,
                               int max_ctas, int num_sms, cudaStream_t stream) {
  DecodeParams prm = prm_in;
  prm.dyn_ranges = 0;  // static ranges only: one per CTA
  const bool fp8 = cache_dtype == PKV_FP8_E4M3;
  switch (q_dtype) {
    case PKV_F32:
      return fp8 ? launch_simt_t<float, __nv_fp8_storage_t>(prm, max_ctas, num_sms, stream)
                 : launch_simt_t<float, float>(prm, max_ctas, num_sms, stream);
    case PKV_F16:
      return fp8 ? launch_simt_t<__half, __nv_fp8_storage_t>(prm, max_ctas, num_sms, stream)
                 : launch_simt_t<__half, __half>(prm, max_ctas, num_sms, stream);
    case PKV_BF16:
      return fp8 ? launch_simt_t<__nv_bfloat16, __nv_fp8_storage_t>(prm, max_ctas, num_sms, stream)
                 : launch_simt_t<__nv_bfloat16, __nv_bfloat16>(prm, max_ctas, num_sms, stream);
    default:
      return cudaErrorInvalidValue;
  }
}

int simt_status_flag(bool clear, int* value) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_simt_status, sizeof(int)) != cudaSuccess) return -1;
  if (clear && v) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_simt_status, &zero, sizeof(int)) != cudaSuccess) return -1;
  }
  *value = v;
  return 0;
}

}  // namespace pkv
