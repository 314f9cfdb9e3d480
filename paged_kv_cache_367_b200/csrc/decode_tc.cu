// PagedAttention decode on tensor cores, K/V tiles staged by TMA (sm_100a).
//
// What it computes is the per-sequence walk of "vLLM 推理引擎源码级拆解"
// (chenxutan.com/d/5333) §2.3: logical block = tok / block_size, physical
// block = block_table[logical block], score = dot(q, k) * scale, online
// softmax, accumulate V, write back; with GQA (§2.3), the g query heads of one
// KV head are served by a single read of its K/V.
//
// How, on B200:
//  * One CTA per SM (persistent) takes a balanced, contiguous share of the
//    (sequence, KV head) work (schedule.cuh).
//  * A producer warp walks the same segments and streams 64-token chunks of K
//    and V into a ring of shared-memory stages (marked evict-first in L2: each
//    tile is read once). Each physical block is one TMA
//    tensor copy: the pool [num_blocks, bs, Hkv, D] is described as a 5-D tensor
//    (d_lo 64, token, d_hi, head, block) so a (block, head) tile lands as
//    128-byte rows with the 128B swizzle; a block id outside the pool is out of
//    the tensor's bounds and lands as zeros. The query rows of a segment come
//    with its first chunk by a bulk copy. Stages are handed over with mbarriers.
//  * Four consumer warps each take 16 tokens of a chunk. The dense part is
//    small (g <= 16 query heads, head_dim 64/128) but it is a real contraction,
//    so it runs on the tensor pipe with mma.sync m16n8k16 in the transposed form
//    S^T = K Q^T (tokens on M, query heads on N = 8), keeping the CUDA cores free
//    and avoiding per-element conversions and cross-lane dot-product reductions.
//    P is rounded to the cache dtype, transposed in registers (movmatrix) into
//    the B operand of O^T += V^T P^T, with V^T fed by ldmatrix.trans.
//  * At the end of a segment each consumer warp drops its softmax state
//    (running max, sum, O^T) into one of two shared hand-off buffers and moves
//    on to the next segment. An epilogue warp combines the four states, writes
//    the output rows of a whole unit or the partial (output row, base-2
//    log-sum-exp) of a piece of a split unit, and merges a split unit when its
//    piece is the last to finish (a per-unit counter of finished tokens; no
//    CTA waits for another). The epilogue is thus off the streaming path.
//  * Every mbarrier wait is bounded (about a second); on expiry the CTA sets an
//    error word, skips the rest of its work and still waits, bounded, for its
//    own copies in flight before it exits.
#include <cuda.h>
#include <atomic>
#include <type_traits>
#include <cudaTypedefs.h>

#include "schedule.cuh"
#include "tc_common.cuh"

namespace pkv {

using namespace tcx;

__device__ int g_tc_timeout = 0;  // bit 0: a wait expired; bit 1: a block id outside the pool

namespace tc {

constexpr int kChunk = 64;                           // tokens per stage
constexpr int kConsumerWarps = 4;                    // 16 tokens of a chunk each
constexpr int kProducerWarp = kConsumerWarps;        // TMA issue
constexpr int kEpilogueWarp = kConsumerWarps + 1;    // combine, store, merge
constexpr int kThreads = (kConsumerWarps + 2) * 32;

template <int D, int NT, int NS, int EKV>
struct Cfg {
  static constexpr int kKV = kChunk * D * EKV;       // bytes of K (or V) per stage
  static constexpr int kQ = 8 * NT * D * 2;          // query rows of one KV head group
  static constexpr int kStage = (2 * kKV + kQ + 1023) / 1024 * 1024;
  static constexpr int kHeads = 8 * NT;
  static constexpr int kRedO = kConsumerWarps * kHeads * D;   // floats per hand-off buffer
  static constexpr int kRed = (kRedO + 2 * kConsumerWarps * kHeads) * 4;
  static constexpr int kBar = (2 * NS + 4) * 8 + (NS + 2) * 48;  // barriers, descriptors
  static constexpr int kSmem = 1024 + NS * kStage + 2 * kRed + kBar +
                               (int)sizeof(SchedShared) + (32 * 16 + 16) * 4 + 32 * 4 + 32;
  static_assert(kSmem <= 227 * 1024, "shared memory per CTA exceeds 227 KB");
};

// Bounded wait that reports expiry in this kernel's error word.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  return mbar_wait_or_abort(bar, parity, abort, &g_tc_timeout);
}

__device__ __forceinline__ void named_sync_consumers() {
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
}

// 16-byte copy global -> shared that completes asynchronously (cp.async).
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem)
               : "memory");
}
// Waits for this thread's cp.async copies.
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// Merge of all pieces of a split unit by one warp. The pieces are listed 32
// ranges at a time (a lane per range; a ballot numbers the non-empty ones, in
// token order) into `wslot`, and taken 32 at a time, one per lane: each lane
// reads its piece's log-sum-exp values, the warp reduces the per-head maxima,
// and the maxima and the pieces' weights go to shared scratch (`msc`, 16
// floats; `wsc`, 32 x 16 floats). The pieces' partial rows are then brought
// into `stage` (stage_floats floats of shared memory the warp owns meanwhile)
// as many pieces at a time as fit, by asynchronous 16-byte copies that are all
// in flight together, and each lane accumulates its D/32 columns of every head
// from there: a merge costs one memory latency per staging round rather than
// one per piece and head.
template <typename T, int D, int NT>
__device__ void warp_merge_unit(const DecodeParams& prm, const Cuts& cu, int64_t P,
                                const Segment& s, int lane, float* wsc, float* msc, int* wslot,
                                float* stage, int stage_floats) {
  constexpr int V = D / 32, H = 8 * NT;
  static_assert(V == 2 || V == 4, "rows are read as float2 or float4");
  const int Hq = prm.num_heads, g = Hq / prm.num_kv_heads;
  const int rowf = g * D;                 // floats of one piece's partial rows
  const int B = stage_floats / rowf;      // pieces per staging round (>= 4)
  const int64_t nparts = div_nn(s.len + P - 1, P);
  const int64_t r0 = cu.owner(s.first);
  const int64_t r1 = cu.owner(s.first + (nparts - 1) * P);
  // Writes the slots of pieces [b0, b0 + 32) to wslot; returns the piece count.
  auto list = [&](int b0) {
    int k = 0;
    for (int64_t rb = r0; rb <= r1; rb += 32) {
      const int64_t r = rb + lane;
      bool has = false;
      if (r <= r1) {
        const int64_t s0 = r == r0 ? 0 : range_first_part(cu, r, s.first, P);
        const int64_t s1 = r == r1 ? nparts : range_first_part(cu, r + 1, s.first, P);
        has = s0 < s1;
      }
      const unsigned m = __ballot_sync(0xffffffffu, has);
      const int idx = k + __popc(m & ((1u << lane) - 1u)) - b0;
      if (has && idx >= 0 && idx < 32) wslot[idx] = piece_slot(r, r0);
      k += __popc(m);
    }
    __syncwarp();
    return k;
  };
  auto load_lse = [&](int b0, int n, float (&lk)[H]) {
#pragma unroll
    for (int j = 0; j < H; ++j) lk[j] = -INFINITY;
    if (b0 + lane < n) {
      const float* src = prm.ws_lse + (int64_t)wslot[lane] * g;
#pragma unroll
      for (int j = 0; j < H; ++j)
        if (j < g) lk[j] = __ldcg(src + j);
    }
  };
  // Copies the partial rows of pieces [q, q + nq) of the listed batch into the
  // stage (not waited for).
  auto stage_rows = [&](int q, int nq) {
    for (int p = 0; p < nq; ++p) {
      const float* src = prm.ws_o + (int64_t)wslot[q + p] * rowf;
      for (int e = lane * 4; e < rowf; e += 128) cp_async16(stage + p * rowf + e, src + e);
    }
  };
  const int n = list(0);
  // The first staging round's copies are issued before the log-sum-exp loads,
  // so both wait out one memory latency together.
  const int B0 = min(B, min(32, n));
  stage_rows(0, B0);
  float lk[H], M[H];
#pragma unroll
  for (int j = 0; j < H; ++j) M[j] = -INFINITY;
  for (int b0 = 0; b0 < n; b0 += 32) {
    if (b0 > 0) {
      __syncwarp();
      list(b0);
    }
    load_lse(b0, n, lk);
#pragma unroll
    for (int j = 0; j < H; ++j) M[j] = fmaxf(M[j], lk[j]);
  }
#pragma unroll
  for (int j = 0; j < H; ++j)
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) M[j] = fmaxf(M[j], __shfl_xor_sync(0xffffffffu, M[j], o));
  if (lane == 0) {
#pragma unroll
    for (int j = 0; j < H; ++j) msc[j] = M[j];
  }
  float num[H][V], den[H];
#pragma unroll
  for (int j = 0; j < H; ++j) {
    den[j] = 0.f;
#pragma unroll
    for (int v = 0; v < V; ++v) num[j][v] = 0.f;
  }
  for (int b0 = 0; b0 < n; b0 += 32) {
    __syncwarp();
    if (n > 32) {  // the list and log-sum-exp values held another batch
      list(b0);
      load_lse(b0, n, lk);
    }
    if (b0 + lane < n) {
#pragma unroll
      for (int j = 0; j < H; ++j) wsc[lane * H + j] = j < g ? fast_exp2(lk[j] - msc[j]) : 0.f;
    }
    __syncwarp();
    const int nb = min(32, n - b0);
    for (int q = 0; q < nb; q += B) {
      const int nq = min(B, nb - q);
      if (b0 > 0 || q > 0) stage_rows(q, nq);  // the first round is in flight already
      cp_async_wait_all();
      __syncwarp();
      for (int p = 0; p < nq; ++p) {
#pragma unroll
        for (int j = 0; j < H; ++j) {
          if (j < g) {
            const float wt = wsc[(q + p) * H + j];
            const float* x = stage + p * rowf + j * D + lane * V;
            den[j] += wt;
            if constexpr (V == 4) {
              const float4 t = *reinterpret_cast<const float4*>(x);
              num[j][0] = fmaf(wt, t.x, num[j][0]);
              num[j][1] = fmaf(wt, t.y, num[j][1]);
              num[j][2] = fmaf(wt, t.z, num[j][2]);
              num[j][3] = fmaf(wt, t.w, num[j][3]);
            } else {
              const float2 t = *reinterpret_cast<const float2*>(x);
              num[j][0] = fmaf(wt, t.x, num[j][0]);
              num[j][1] = fmaf(wt, t.y, num[j][1]);
            }
          }
        }
      }
      __syncwarp();  // the stage is refilled next round
    }
  }
#pragma unroll
  for (int j = 0; j < H; ++j) {
    if (j < g) {
      const float inv = 1.f / den[j];
      float a, b;
      T* dst = static_cast<T*>(prm.out) + ((int64_t)s.seq * Hq + s.head * g + j) * D + lane * V;
      if constexpr (V == 4) {
        uint2 w;
        w.x = Mma<T>::pack(num[j][0] * inv, num[j][1] * inv, a, b);
        w.y = Mma<T>::pack(num[j][2] * inv, num[j][3] * inv, a, b);
        *reinterpret_cast<uint2*>(dst) = w;
      } else {
        *reinterpret_cast<uint32_t*>(dst) = Mma<T>::pack(num[j][0] * inv, num[j][1] * inv, a, b);
      }
    }
  }
}

// What the producer tells the other warps about the chunk in a stage (and the
// consumers tell the epilogue warp about a finished segment).
struct ChunkDesc {
  int64_t first;             // work offset of the unit's partition 0
  int seq, head, t0, t1, len;  // the segment
  int c0;                    // first token of the chunk
  int range;                 // range the segment belongs to
  int flags;
};
constexpr int kFirst = 1, kLast = 2, kEnd = 4;

// 16-bit pair (bf16 or f16, low element first) to two floats.
template <typename T> __device__ __forceinline__ float2 pair_to_f32(uint32_t v);
template <> __device__ __forceinline__ float2 pair_to_f32<__nv_bfloat16>(uint32_t v) {
  return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
}
template <> __device__ __forceinline__ float2 pair_to_f32<__half>(uint32_t v) {
  return __half22float2(*reinterpret_cast<const __half2*>(&v));
}

// Consumer warps on the CUDA cores, for narrow groups (g <= G query heads per
// KV head, where Q K^T is a matrix-vector product rather than a dense
// contraction). Warp w takes tokens [16 w, 16 w + 16) of each chunk, as the
// tensor-core consumers do; inside the warp, LPT = D / 8 lanes hold one token's
// row, eight dimensions (one 16-byte unit of the 128B-swizzled tile) each, so
// TPS = 32 / LPT tokens are read per step with conflict-free 16-byte shared
// loads. A token's score is the LPT-lane sum of the lanes' partial dot
// products (xor shuffles); the online softmax runs per 16-token slice in fp32
// (P is not rounded); each lane accumulates P V for its eight dimensions over
// its tokens, and the TPS lane groups are summed at the end of a segment.
// Slots past the segment's end are neither read nor counted.
template <typename T, int D, int G, int NS, int H>
__device__ void consumer_cuda_cores(const DecodeParams& prm, uint8_t* ring, int stage_bytes,
                                    int kv_bytes, const ChunkDesc* desc, uint64_t* full,
                                    uint64_t* empty, float* red, int red_floats, int red_o,
                                    ChunkDesc* hdesc, uint64_t* rfull, uint64_t* rempty,
                                    volatile int* abort, int w, int lane) {
  constexpr int LPT = D / 8, TPS = 32 / LPT, STEPS = 16 / TPS;
  const int grp = lane / LPT, ln = lane % LPT;
  const int bs = prm.block_size, g = prm.num_heads / prm.num_kv_heads;
  const int tile = bs * D * 2;                // bytes of one (block, head) tile
  const int plane = ln >> 3, unit = ln & 7;   // 128-byte piece of the row, 16-byte unit in it
  const float sscale = prm.score_scale;
  uint32_t kc = 0;
  int sidx = 0;
  float q[G][8], acc[G][8], m[G], l[G];
  for (;;) {
    const int stage = (int)(kc % NS);
    const uint32_t phase = (kc / NS) & 1u;
    ++kc;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(full + stage, phase, abort));
    if (!ok) break;
    const ChunkDesc d = desc[stage];
    if (d.flags & kEnd) break;
    const uint8_t* st = ring + stage * stage_bytes;
    if (d.flags & kFirst) {
      // This lane's eight dimensions of each query row, pre-scaled.
      const uint8_t* qs = st + 2 * kv_bytes;
#pragma unroll
      for (int j = 0; j < G; ++j) {
        m[j] = -INFINITY;
        l[j] = 0.f;
        uint4 raw = make_uint4(0, 0, 0, 0);
        if (j < g) raw = *reinterpret_cast<const uint4*>(qs + (j * D + 8 * ln) * 2);
        const uint32_t u[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 f = pair_to_f32<T>(u[k]);
          q[j][2 * k] = f.x * sscale;
          q[j][2 * k + 1] = f.y * sscale;
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[j][k] = 0.f;
      }
    }
    const int nv = min(16, max(0, d.t1 - (d.c0 + 16 * w)));
    if (nv > 0) {
      // Scores of this lane group's tokens (base-2 domain).
      float sc[G][STEPS];
#pragma unroll
      for (int s = 0; s < STEPS; ++s) {
        const int tw = s * TPS + grp, t = 16 * w + tw;
        const int tt = t % bs;
        const uint32_t off = (uint32_t)((t / bs) * tile + plane * (bs * 128) + tt * 128 +
                                        ((unit ^ (tt & 7)) << 4));
        uint4 raw = make_uint4(0, 0, 0, 0);
        if (tw < nv) raw = *reinterpret_cast<const uint4*>(st + off);
        const uint32_t u[4] = {raw.x, raw.y, raw.z, raw.w};
        float kf[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 f = pair_to_f32<T>(u[k]);
          kf[2 * k] = f.x;
          kf[2 * k + 1] = f.y;
        }
#pragma unroll
        for (int j = 0; j < G; ++j) {
          float dot = 0.f;
#pragma unroll
          for (int k = 0; k < 8; ++k) dot = fmaf(q[j][k], kf[k], dot);
#pragma unroll
          for (int o = LPT / 2; o >= 1; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
          sc[j][s] = tw < nv ? dot : -INFINITY;
        }
      }
      // Online softmax over the warp's slice of the chunk.
      float p[G][STEPS];
#pragma unroll
      for (int j = 0; j < G; ++j) {
        float mx = sc[j][0];
#pragma unroll
        for (int s = 1; s < STEPS; ++s) mx = fmaxf(mx, sc[j][s]);
#pragma unroll
        for (int o = LPT; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        const float mn = fmaxf(m[j], mx);
        const float mu = mn == -INFINITY ? 0.f : mn;
        const float alpha = fast_exp2(m[j] - mu);
        m[j] = mn;
        float ls = 0.f;
#pragma unroll
        for (int s = 0; s < STEPS; ++s) {
          p[j][s] = fast_exp2(sc[j][s] - mu);
          ls += p[j][s];
        }
        l[j] = l[j] * alpha + ls;
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[j][k] *= alpha;
      }
      // P V for this lane's eight dimensions.
#pragma unroll
      for (int s = 0; s < STEPS; ++s) {
        const int tw = s * TPS + grp, t = 16 * w + tw;
        const int tt = t % bs;
        const uint32_t off = (uint32_t)((t / bs) * tile + plane * (bs * 128) + tt * 128 +
                                        ((unit ^ (tt & 7)) << 4));
        if (tw < nv) {
          const uint4 raw = *reinterpret_cast<const uint4*>(st + kv_bytes + off);
          const uint32_t u[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 f = pair_to_f32<T>(u[k]);
#pragma unroll
            for (int j = 0; j < G; ++j) {
              acc[j][2 * k] = fmaf(p[j][s], f.x, acc[j][2 * k]);
              acc[j][2 * k + 1] = fmaf(p[j][s], f.y, acc[j][2 * k + 1]);
            }
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty + stage);
    if (d.flags & kLast) {
      // ---- hand the warp's state to the epilogue warp ----
#pragma unroll
      for (int j = 0; j < G; ++j) {
#pragma unroll
        for (int o = LPT; o < 32; o <<= 1) {
          l[j] += __shfl_xor_sync(0xffffffffu, l[j], o);
#pragma unroll
          for (int k = 0; k < 8; ++k) acc[j][k] += __shfl_xor_sync(0xffffffffu, acc[j][k], o);
        }
      }
      const int rb = sidx & 1;
      const uint32_t use = (uint32_t)(sidx >> 1);
      ++sidx;
      mbar_wait(rempty + rb, (use & 1u) ^ 1u, abort);  // read two segments ago
      if (w == 0 && lane == 0) hdesc[rb] = d;
      float* ro = red + rb * red_floats + (w * H) * D;
      float* rm = red + rb * red_floats + red_o;
      float* rl = rm + 4 * H;
#pragma unroll
      for (int j = 0; j < G; ++j) {
        if (j < g && grp == 0) {
          *reinterpret_cast<float4*>(ro + j * D + 8 * ln) =
              make_float4(acc[j][0], acc[j][1], acc[j][2], acc[j][3]);
          *reinterpret_cast<float4*>(ro + j * D + 8 * ln + 4) =
              make_float4(acc[j][4], acc[j][5], acc[j][6], acc[j][7]);
        }
        if (j < g && lane == 0) {
          rm[w * H + j] = m[j];
          rl[w * H + j] = l[j];
        }
      }
      mbar_arrive(rfull + rb);
    }
  }
  // Tell the epilogue warp there is nothing more.
  const int rb = sidx & 1;
  const uint32_t use = (uint32_t)(sidx >> 1);
  mbar_wait(rempty + rb, (use & 1u) ^ 1u, abort);
  if (w == 0 && lane == 0) hdesc[rb].flags = kEnd;
  mbar_arrive(rfull + rb);
}

// T: query/output type (bf16 or f16). F8: the cache holds E4M3 codes; the
// products then run in f16 (exact for E4M3 values) with k_scale folded into the
// score scale and v_scale applied to the output.
// CC > 0: the products run on the CUDA cores (consumer_cuda_cores) for groups
// of at most CC query heads; 16-bit caches only.
template <typename T, int D, int NT, int NS, int MINB, bool F8, int CC>
__global__ void __launch_bounds__(kThreads, MINB)
    decode_tc_kernel(const DecodeParams prm, const __grid_constant__ CUtensorMap tmap_k,
                     const __grid_constant__ CUtensorMap tmap_v) {
  constexpr int EKV = F8 ? 1 : 2;  // cache element bytes
  using C = Cfg<D, NT, NS, EKV>;
  using M = typename std::conditional<F8, __half, T>::type;  // MMA operand type
  constexpr int H = C::kHeads;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* ring = smem;
  float* red = reinterpret_cast<float*>(smem + NS * C::kStage);  // 2 hand-off buffers
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + NS * C::kStage + 2 * C::kRed);
  uint64_t* empty = full + NS;
  uint64_t* rfull = empty + NS;    // consumers -> epilogue warp, per hand-off buffer
  uint64_t* rempty = rfull + 2;    // epilogue warp -> consumers
  ChunkDesc* desc = reinterpret_cast<ChunkDesc*>(rempty + 2);  // per stage
  ChunkDesc* hdesc = desc + NS;                                 // per hand-off buffer
  SchedShared* sched = reinterpret_cast<SchedShared*>(hdesc + 2);
  float* merge_scratch = reinterpret_cast<float*>(sched + 1);  // 32 x 16 floats, epilogue warp
  float* merge_max = merge_scratch + 32 * 16;                         // 16, epilogue warp
  int* merge_slots = reinterpret_cast<int*>(merge_max + 16);          // 32, epilogue warp
  volatile int* abort = reinterpret_cast<volatile int*>(merge_slots + 32);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, kConsumerWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(rfull + b, kConsumerWarps * 32);
      mbar_init(rempty + b, 32);
    }
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  SegmentWalker walker;
  init_walker<T>(prm, *sched, walker);  // ends with __syncthreads

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Hq = prm.num_heads, Hkv = prm.num_kv_heads, g = Hq / Hkv, bs = prm.block_size;
  const int tile = bs * D * EKV;  // bytes of one (block, head) tile
  const Cuts cuts = sched->cuts;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer ----
    // Streams the chunks of every segment of this CTA's static range, then of
    // each dynamic range it takes, in order, into the ring, with a descriptor
    // per chunk. The next segment is found, and its block ids loaded, once the
    // current segment's first chunk is issued; the lane holding a block's id
    // issues that block's K and V tile copies. A final descriptor marks the end.
    uint32_t kc = 0;  // chunk counter: stage kc % NS, phase (kc / NS) & 1
    uint32_t armed = 0, last_parity = 0;
    bool ok = true, waited = false;
    const T* qbase = static_cast<const T*>(prm.query);
    int64_t r = blockIdx.x;
    int ci = sched->d_i;            // forward cursor for dynamic ranges
    int64_t cbase = sched->d_base;
    int* const dyn_counter = prm.ws_done + (int64_t)prm.num_seqs * Hkv;
    // K/V tiles are read once: evicted from L2 first, so the lengths, block
    // tables, query rows and split partials stay there.
    const uint64_t kv_policy = l2_evict_first_policy();
    for (;;) {
      Segment seg, nseg;
      bool have = walker.next(seg);
      int cur = 0;
      if (have) {
        const int32_t* bt = prm.block_table + (int64_t)seg.seq * prm.max_blocks_per_seq;
        const int lb0 = seg.t0 / bs, nlb = (seg.t1 + bs - 1) / bs - lb0;
        cur = lane < nlb ? __ldg(bt + lb0 + lane) : 0;
      }
      while (have && ok) {
        const int32_t* bt = prm.block_table + (int64_t)seg.seq * prm.max_blocks_per_seq;
        const int lb0 = seg.t0 / bs;
        const int nlb = (seg.t1 + bs - 1) / bs - lb0;
        int nxt = lane + 32 < nlb ? __ldg(bt + lb0 + 32 + lane) : 0;
        bool have_next = false;
        int ncur = 0;
        int batch = 0;
        for (int c0 = seg.t0; c0 < seg.t1; c0 += kChunk, ++kc) {
          const int stage = (int)(kc % NS);
          const uint32_t phase = (kc / NS) & 1u;
          const int rel = (c0 - seg.t0) / bs;
          if (rel >= batch + 32) {
            cur = nxt;
            batch += 32;
            nxt = lane + batch + 32 < nlb ? __ldg(bt + lb0 + batch + 32 + lane) : 0;
          }
          const int ntok = min(kChunk, seg.t1 - c0);
          const int nblk = (ntok + bs - 1) / bs;
          const bool first = c0 == seg.t0;
          if (lane == 0 && ok) ok = mbar_wait(empty + stage, phase ^ 1u, abort);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          uint8_t* st = ring + stage * C::kStage;
          if (ok && lane == 0) {
            ChunkDesc& dd = desc[stage];
            dd.first = seg.first;
            dd.seq = seg.seq;
            dd.head = seg.head;
            dd.t0 = seg.t0;
            dd.t1 = seg.t1;
            dd.len = seg.len;
            dd.c0 = c0;
            dd.range = (int)r;
            dd.flags = (first ? kFirst : 0) | (c0 + kChunk >= seg.t1 ? kLast : 0);
            const uint32_t qbytes = first ? (uint32_t)(g * D * 2) : 0u;
            mbar_expect_tx(full + stage, (uint32_t)(2 * nblk * tile) + qbytes);  // releases dd
            if (first)
              bulk_load(st + 2 * C::kKV, qbase + ((int64_t)seg.seq * Hq + seg.head * g) * D,
                        qbytes, full + stage);
          }
          __syncwarp();
          if (!waited) {
            // Launched early (programmatic dependent launch): the previous
            // kernel may still be writing the caches. A no-op otherwise.
            asm volatile("griddepcontrol.wait;" ::: "memory");
            waited = true;
          }
          const int b = lane - (rel - batch);
          if (ok && b >= 0 && b < nblk) {
            // An id outside the pool reads as zeros (the copy's bounds fill);
            // it is also reported in the status word (bit 1).
            if (cur < 0 || (int64_t)cur >= prm.num_blocks) atomicOr(&g_tc_timeout, 2);
            tma_load_5d_hint(st + b * tile, &tmap_k, 0, 0, 0, seg.head, cur, full + stage, kv_policy);
            tma_load_5d_hint(st + C::kKV + b * tile, &tmap_v, 0, 0, 0, seg.head, cur, full + stage,
                             kv_policy);
          }
          if (ok) {
            armed |= 1u << stage;
            last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          }
          if (first) {
            have_next = walker.next(nseg);
            if (have_next) {
              const int32_t* nbt = prm.block_table + (int64_t)nseg.seq * prm.max_blocks_per_seq;
              const int nlb0 = nseg.t0 / bs, nnlb = (nseg.t1 + bs - 1) / bs - nlb0;
              ncur = lane < nnlb ? __ldg(nbt + nlb0 + lane) : 0;
            }
          }
        }
        seg = nseg;
        cur = ncur;
        have = have_next;
      }
      if (!ok || cuts.Rd == 0) break;
      int64_t nr = 0;
      if (lane == 0) {
        const int64_t taken = atomicAdd(dyn_counter, 1);
        // Every CTA asks until it is refused once, so the counter ends at Rd + G:
        // the last refusal (no other CTA asks after it) leaves it at zero for
        // the next call on this workspace.
        if (taken == cuts.Rd + cuts.G - 1) atomicExch(dyn_counter, 0);
        nr = cuts.G + taken;
      }
      nr = __shfl_sync(0xffffffffu, nr, 0);
      if (nr >= cuts.R()) break;
      r = nr;
      warp_start_range(prm, walker, r, ci, cbase);  // an empty range leaves the walker done
    }
    // Wait, bounded, for this CTA's copies in flight (before the end marker,
    // which moves a stage's barrier on to another phase).
    if (lane == 0) {
      for (int s = 0; s < NS; ++s) {
        if (!(armed >> s & 1u)) continue;
        const long long t0 = clock64();
        while (!mbar_try(full + s, (last_parity >> s) & 1u)) {
          if (clock64() - t0 > kWaitCycles) {
            atomicOr(&g_tc_timeout, 1);
            break;
          }
        }
      }
    }
    // End marker.
    {
      const int stage = (int)(kc % NS);
      const uint32_t phase = (kc / NS) & 1u;
      if (lane == 0 && ok) ok = mbar_wait(empty + stage, phase ^ 1u, abort);
      if (lane == 0 && ok) {
        desc[stage].flags = kEnd;
        mbar_arrive(full + stage);
      }
    }
    return;
  }

  if (warp == kEpilogueWarp) {
    // ------------------------------------------------------------ epilogue ----
    // For every segment: combine the four consumer warps' softmax states from
    // the hand-off buffer, write the output rows (whole unit) or the partial
    // (piece of a split unit), release the buffer, and merge the unit if this
    // piece completed it.
    constexpr int V = D / 32;
    const float vscale = F8 ? __ldg(prm.v_scale) : 1.f;
    int sidx = 0;
    for (;;) {
      const int rb = sidx & 1;
      const uint32_t use = (uint32_t)(sidx >> 1);
      ++sidx;
      const bool ok = __all_sync(0xffffffffu, mbar_wait(rfull + rb, use & 1u, abort));
      const ChunkDesc d = hdesc[rb];
      if (!ok || (d.flags & kEnd)) break;
      Segment seg;
      seg.seq = d.seq;
      seg.head = d.head;
      seg.t0 = d.t0;
      seg.t1 = d.t1;
      seg.len = d.len;
      seg.first = d.first;
      const float* ro = red + rb * (C::kRed / 4);
      const float* rm = ro + C::kRedO;
      const float* rl = rm + kConsumerWarps * H;
      const bool whole = seg.t0 == 0 && seg.t1 == seg.len;
      const int i = seg.seq, h = seg.head;
      {
        // Lanes j < g: per-head maximum, warp weights and 1/denominator, into
        // the shared scratch (each head: 4 weights, the reciprocal, the lse).
        if (lane < g) {
          float mx = -INFINITY;
#pragma unroll
          for (int x = 0; x < kConsumerWarps; ++x) mx = fmaxf(mx, rm[x * H + lane]);
          float lsum = 0.f;
#pragma unroll
          for (int x = 0; x < kConsumerWarps; ++x) {
            const float wt = fast_exp2(rm[x * H + lane] - mx);
            merge_scratch[lane * 8 + x] = wt;
            lsum = fmaf(wt, rl[x * H + lane], lsum);
          }
          merge_scratch[lane * 8 + 4] = vscale / lsum;
          if (!whole) {
            const int64_t rowp = (int64_t)own_piece_slot(d.range, seg) * g + lane;
            prm.ws_lse[rowp] = mx + fast_log2(lsum);
          }
        }
        __syncwarp();
#pragma unroll
        for (int j = 0; j < H; ++j) {
          if (j < g) {
            const float* sc = merge_scratch + j * 8;
            float o[V];
#pragma unroll
            for (int v = 0; v < V; ++v) o[v] = 0.f;
#pragma unroll
            for (int x = 0; x < kConsumerWarps; ++x) {
              const float wt = sc[x];
              const float* src = ro + (x * H + j) * D + lane * V;
              if constexpr (V == 4) {
                const float4 r = *reinterpret_cast<const float4*>(src);
                o[0] = fmaf(wt, r.x, o[0]);
                o[1] = fmaf(wt, r.y, o[1]);
                o[2] = fmaf(wt, r.z, o[2]);
                o[3] = fmaf(wt, r.w, o[3]);
              } else {
#pragma unroll
                for (int v = 0; v < V; ++v) o[v] = fmaf(wt, src[v], o[v]);
              }
            }
            const float inv = sc[4];
#pragma unroll
            for (int v = 0; v < V; ++v) o[v] *= inv;
            const int qh = h * g + j;
            if (whole) {
              T* dst = static_cast<T*>(prm.out) + ((int64_t)i * Hq + qh) * D + lane * V;
              if constexpr (V == 4) {
                uint2 pk;
                float r0, r1;
                pk.x = Mma<T>::pack(o[0], o[1], r0, r1);
                pk.y = Mma<T>::pack(o[2], o[3], r0, r1);
                *reinterpret_cast<uint2*>(dst) = pk;
              } else {
#pragma unroll
                for (int v = 0; v < V; ++v) dst[v] = from_f32<T>(o[v]);
              }
            } else {
              const int64_t rowp = (int64_t)own_piece_slot(d.range, seg) * g + j;
              float* dst = prm.ws_o + rowp * D + lane * V;
              if constexpr (V == 4) {
                *reinterpret_cast<float4*>(dst) = make_float4(o[0], o[1], o[2], o[3]);
              } else {
#pragma unroll
                for (int v = 0; v < V; ++v) dst[v] = o[v];
              }
            }
          }
        }
        __syncwarp();  // the scratch is rewritten by the next segment
      }
      __syncwarp();  // also orders the lanes' partial stores before lane 0's release
      if (!whole) {
        const int last = lane == 0 ? (int)complete_piece(prm, seg) : 0;
        if (__shfl_sync(0xffffffffu, last, 0))  // lane 0 acquired the other pieces
          warp_merge_unit<T, D, NT>(prm, cuts, walker.P, seg, lane, merge_scratch, merge_max,
                                    merge_slots, red + rb * (C::kRed / 4), C::kRed / 4);
      }
      mbar_arrive(rempty + rb);  // the hand-off buffer (the merge's stage) may be refilled
    }
    return;
  }

  // -------------------------------------------------------------- consumers ----
  // Warp w takes tokens [16 w, 16 w + 16) of every 64-token chunk.
  if constexpr (CC > 0) {
    static_assert(!F8, "CUDA-core products: 16-bit caches");
    consumer_cuda_cores<T, D, CC, NS, H>(prm, ring, C::kStage, C::kKV, desc, full, empty, red,
                                         C::kRed / 4, C::kRedO, hdesc, rfull, rempty, abort, warp,
                                         lane);
    return;
  }
  const int w = warp;
  const int g0 = lane >> 2, cq = lane & 3, x7 = lane & 7;
  const int kt = 16 * w + ((lane >> 3) & 1) * 8 + x7;  // token row this lane addresses for K
  const int vt = 16 * w + ((lane >> 4) & 1) * 8 + x7;  // ... and for V
  const int kj = (lane >> 4) & 1, vj = (lane >> 3) & 1;
  const uint32_t krow = (uint32_t)((kt / bs) * tile + (kt % bs) * 128);
  const uint32_t vrow = (uint32_t)((vt / bs) * tile + (vt % bs) * 128);
  const uint32_t dh_stride = (uint32_t)(bs * 128);
  const uint32_t ring_u32 = smem_u32(ring);
  const float sscale = prm.score_scale * (F8 ? __ldg(prm.k_scale) : 1.f);
  constexpr int MT = D / 16;

  uint32_t kc = 0;
  int sidx = 0;
  float m[2 * NT], l[2 * NT];
  float o[MT][NT][4];
  uint32_t bq[MT][NT][2];
  for (;;) {
    const int stage = (int)(kc % NS);
    const uint32_t phase = (kc / NS) & 1u;
    ++kc;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(full + stage, phase, abort));
    if (!ok) break;
    const ChunkDesc d = desc[stage];
    if (d.flags & kEnd) break;
    const uint32_t st = ring_u32 + stage * C::kStage;
    if (d.flags & kFirst) {
#pragma unroll
      for (int x = 0; x < 2 * NT; ++x) {
        m[x] = -INFINITY;
        l[x] = 0.f;
      }
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) o[mt][nt][e] = 0.f;
    }
      if (d.flags & kFirst) {
        // Q^T fragments: b0b1 = Q[head g0][16ks + 2cq, +1], b2b3 = the same + 8 dims.
        const uint8_t* qs = ring + stage * C::kStage + 2 * C::kKV;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int head = nt * 8 + g0;
#pragma unroll
          for (int ks = 0; ks < MT; ++ks) {
            uint32_t b0 = 0, b1 = 0;
            if (head < g) {
              const uint32_t* row = reinterpret_cast<const uint32_t*>(qs + head * D * 2);
              if constexpr (F8) {
                // E4M3 K rows give each lane 4 consecutive dimensions of a
                // 16-wide step; the contraction index is permuted to match:
                // logical (2cq, 2cq+1) <- dims 4cq, 4cq+1; (2cq+8, +9) <- 4cq+2, +3.
                b0 = to_f16x2<T>(row[(16 * ks + 4 * cq) / 2]);
                b1 = to_f16x2<T>(row[(16 * ks + 4 * cq + 2) / 2]);
              } else {
                b0 = row[(16 * ks + 2 * cq) / 2];
                b1 = row[(16 * ks + 8 + 2 * cq) / 2];
              }
            }
            bq[ks][nt][0] = b0;
            bq[ks][nt][1] = b1;
          }
        }
      }
      const int nv = min(16, max(0, d.t1 - (d.c0 + 16 * w)));
      if (ok && nv > 0) {
        // S^T = K Q^T for this warp's 16 tokens; two accumulator chains.
        float s[NT][4], s2[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) s[nt][e] = s2[nt][e] = 0.f;
        if constexpr (F8) {
          // One ldmatrix.x4 brings 16 tokens x 32 dimensions (two 16-wide steps).
#pragma unroll
          for (int q2 = 0; q2 < MT / 2; ++q2) {
            uint32_t r[4];
            const int j = 2 * q2 + kj;
            ldsm_x4(r, st + krow + ((j ^ x7) << 4));
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              const int ks = 2 * q2 + half;
              const uint32_t a[4] = {e4m3x2_to_f16x2(r[2 * half]), e4m3x2_to_f16x2(r[2 * half + 1]),
                                     e4m3x2_to_f16x2(r[2 * half] >> 16),
                                     e4m3x2_to_f16x2(r[2 * half + 1] >> 16)};
#pragma unroll
              for (int nt = 0; nt < NT; ++nt) {
                if (half)
                  Mma<M>::run(s2[nt], a, bq[ks][nt][0], bq[ks][nt][1]);
                else
                  Mma<M>::run(s[nt], a, bq[ks][nt][0], bq[ks][nt][1]);
              }
            }
          }
        } else {
#pragma unroll
          for (int ks = 0; ks < MT; ++ks) {
            uint32_t a[4];
            const int dh = ks >> 2, j = ((ks & 3) << 1) + kj;
            ldsm_x4(a, st + krow + dh * dh_stride + ((j ^ x7) << 4));
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              if (ks & 1)
                Mma<M>::run(s2[nt], a, bq[ks][nt][0], bq[ks][nt][1]);
              else
                Mma<M>::run(s[nt], a, bq[ks][nt][0], bq[ks][nt][1]);
            }
          }
        }
        const bool v0 = g0 < nv, v1 = g0 + 8 < nv;
        uint32_t bp[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          float alpha[2], p[2][2];
#pragma unroll
          for (int hi = 0; hi < 2; ++hi) {
            const float s0 = v0 ? (s[nt][hi] + s2[nt][hi]) * sscale : -INFINITY;
            const float s1 = v1 ? (s[nt][2 + hi] + s2[nt][2 + hi]) * sscale : -INFINITY;
            float mx = fmaxf(s0, s1);
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            const int x = nt * 2 + hi;
            const float mn = fmaxf(m[x], mx);
            const float mu = mn == -INFINITY ? 0.f : mn;
            alpha[hi] = fast_exp2(m[x] - mu);
            m[x] = mn;
            p[hi][0] = fast_exp2(s0 - mu);
            p[hi][1] = fast_exp2(s1 - mu);
          }
          float r00, r01, r10, r11;
          const uint32_t P0 = Mma<M>::pack(p[0][0], p[1][0], r00, r01);  // token g0, heads 2cq, 2cq+1
          const uint32_t P1 = Mma<M>::pack(p[0][1], p[1][1], r10, r11);  // token g0 + 8
          l[nt * 2 + 0] = l[nt * 2 + 0] * alpha[0] + (r00 + r10);
          l[nt * 2 + 1] = l[nt * 2 + 1] * alpha[1] + (r01 + r11);
          if (alpha[0] != 1.f || alpha[1] != 1.f) {
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
              o[mt][nt][0] *= alpha[0];
              o[mt][nt][1] *= alpha[1];
              o[mt][nt][2] *= alpha[0];
              o[mt][nt][3] *= alpha[1];
            }
          }
          bp[nt][0] = movmatrix_t(P0);
          bp[nt][1] = movmatrix_t(P1);
        }
        // Tokens past the end of the segment hold stale or poisoned rows: zero
        // their V operands (their P is already 0, and 0 * NaN would be NaN).
        uint32_t mlo = 0xffffffffu, mhi = 0xffffffffu;
        if (nv < 16) {
          mlo = (2 * cq < nv ? 0x0000ffffu : 0u) | (2 * cq + 1 < nv ? 0xffff0000u : 0u);
          mhi = (2 * cq + 8 < nv ? 0x0000ffffu : 0u) | (2 * cq + 9 < nv ? 0xffff0000u : 0u);
        }
        if constexpr (F8) {
          // ldmatrix.trans on E4M3 rows gives each lane, per 8x16-byte matrix,
          // dims (2g0, 2g0+1) of tokens (2cq, 2cq+1). One byte permute splits
          // them into an even-dimension and an odd-dimension pair of tokens, so
          // M-row g0 of the product is dim 16mt + 2g0 and row g0+8 is dim
          // 16mt + 2g0 + 1.
#pragma unroll
          for (int q2 = 0; q2 < MT / 2; ++q2) {
            uint32_t r[4];
            const int j = 2 * q2 + kj;
            ldsm_x4_t(r, st + C::kKV + krow + ((j ^ x7) << 4));
            r[0] &= mlo;
            r[1] &= mhi;
            r[2] &= mlo;
            r[3] &= mhi;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              const uint32_t lo = __byte_perm(r[2 * half], 0, 0x3120);      // tokens 2cq, 2cq+1
              const uint32_t hi8 = __byte_perm(r[2 * half + 1], 0, 0x3120); // tokens 8+2cq, +1
              const uint32_t a[4] = {e4m3x2_to_f16x2(lo), e4m3x2_to_f16x2(lo >> 16),
                                     e4m3x2_to_f16x2(hi8), e4m3x2_to_f16x2(hi8 >> 16)};
#pragma unroll
              for (int nt = 0; nt < NT; ++nt)
                Mma<M>::run(o[2 * q2 + half][nt], a, bp[nt][0], bp[nt][1]);
            }
          }
        } else {
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            uint32_t a[4];
            const int dh = mt >> 2, j = ((mt & 3) << 1) + vj;
            ldsm_x4_t(a, st + C::kKV + vrow + dh * dh_stride + ((j ^ x7) << 4));
            a[0] &= mlo;
            a[1] &= mlo;
            a[2] &= mhi;
            a[3] &= mhi;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) Mma<M>::run(o[mt][nt], a, bp[nt][0], bp[nt][1]);
          }
        }
      }
      __syncwarp();
    if (lane == 0) mbar_arrive(empty + stage);
    if (d.flags & kLast) {
      // ---- hand the warp's state to the epilogue warp ----
  #pragma unroll
      for (int x = 0; x < 2 * NT; ++x) {
        l[x] += __shfl_xor_sync(0xffffffffu, l[x], 4);
        l[x] += __shfl_xor_sync(0xffffffffu, l[x], 8);
        l[x] += __shfl_xor_sync(0xffffffffu, l[x], 16);
      }
      const int rb = sidx & 1;
      const uint32_t use = (uint32_t)(sidx >> 1);
      ++sidx;
      // The buffer's previous contents (two segments ago) must have been read.
      mbar_wait(rempty + rb, (use & 1u) ^ 1u, abort);
      if (w == 0 && lane == 0) hdesc[rb] = d;
      float* ro = red + rb * (C::kRed / 4) + (w * H) * D;
      float* rm = red + rb * (C::kRed / 4) + C::kRedO;
      float* rl = rm + kConsumerWarps * H;
      if (g0 == 0) {
  #pragma unroll
        for (int nt = 0; nt < NT; ++nt)
  #pragma unroll
          for (int hi = 0; hi < 2; ++hi) {
            const int head = nt * 8 + 2 * cq + hi;
            rm[w * H + head] = m[nt * 2 + hi];
            rl[w * H + head] = l[nt * 2 + hi];
          }
      }
  #pragma unroll
      for (int mt = 0; mt < MT; ++mt)
  #pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          // Rows g0 and g0 + 8 of m-tile mt: dims (16mt + g0, + 8), or for E4M3
          // caches (16mt + 2g0, + 1).
          const int h0 = nt * 8 + 2 * cq;
          const int d0 = F8 ? mt * 16 + 2 * g0 : mt * 16 + g0, d1 = F8 ? d0 + 1 : d0 + 8;
          ro[h0 * D + d0] = o[mt][nt][0];
          ro[(h0 + 1) * D + d0] = o[mt][nt][1];
          ro[h0 * D + d1] = o[mt][nt][2];
          ro[(h0 + 1) * D + d1] = o[mt][nt][3];
        }
    mbar_arrive(rfull + rb);
    }
  }
  // Tell the epilogue warp there is nothing more.
  {
    const int rb = sidx & 1;
    const uint32_t use = (uint32_t)(sidx >> 1);
    mbar_wait(rempty + rb, (use & 1u) ^ 1u, abort);
    if (w == 0 && lane == 0) hdesc[rb].flags = kEnd;
    mbar_arrive(rfull + rb);
  }
}

// The status word's self-test: one thread notes an out-of-pool block id (bit
// 1) as the producer does, then waits on an mbarrier that nothing completes,
// with a short limit, through the kernels' own bounded wait. The wait must
// expire, add bit 0 without erasing bit 1, and return.
__global__ void status_selftest_kernel(long long limit_cycles, int note_out_of_pool) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  abort_flag = 0;
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  if (note_out_of_pool) atomicOr(&g_tc_timeout, 2);
  mbar_wait_or_abort(&bar, 0, &abort_flag, &g_tc_timeout, limit_cycles);
}

}  // namespace tc

// ---------------------------------------------------------------- host side ----

int launch_status_selftest(long long limit_cycles, int note_out_of_pool, cudaStream_t stream) {
  tc::status_selftest_kernel<<<1, 32, 0, stream>>>(limit_cycles, note_out_of_pool);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

int tc_timeout_flag(bool clear, int* value) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_tc_timeout, sizeof(int)) != cudaSuccess) return -1;
  if (clear && v) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_tc_timeout, &zero, sizeof(int)) != cudaSuccess) return -1;
  }
  *value = v;
  return 0;
}

// Largest group whose products run on the CUDA cores by default (see
// launch_decode_tc): none. Measured on B200 with the same TMA pipeline, the
// CUDA-core products take 2.8x the instructions of mma.sync at one query head
// per KV head (the dot products need per-element conversions and cross-lane
// sums), hold each stage longer, and run the MHA decode 1.46x slower (DRAM
// throughput 52% against 76%); at four heads per KV head 2.2x slower.
constexpr int kCudaCoreMaxGroup = 0;

bool tc_supported(int q_dtype, int cache_dtype, int head_dim, int group) {
  if (q_dtype != PKV_BF16 && q_dtype != PKV_F16) return false;
  if (group < 1 || group > 16) return false;
  if (cache_dtype == q_dtype) return head_dim == 64 || head_dim == 128;
  return cache_dtype == PKV_FP8_E4M3 && head_dim == 128;
}

template <typename T, int D, int NT, int NS, int MINB, bool F8, int CC>
static cudaError_t launch_tc_t(const DecodeParams& prm, const CUtensorMap& mk,
                               const CUtensorMap& mv, int max_ctas, int num_sms,
                               bool early_start, cudaStream_t stream) {
  using C = tc::Cfg<D, NT, NS, F8 ? 1 : 2>;
  auto kernel = tc::decode_tc_kernel<T, D, NT, NS, MINB, F8, CC>;
  // The shared-memory opt-in is a per-device setting: done, and the residency
  // queried, once per device.
  static std::atomic<int> occ_of[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  int occ = occ_of[dev].load(std::memory_order_relaxed);
  if (occ == 0) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::kSmem);
    if (e != cudaSuccess) return e;
    int n = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, tc::kThreads, C::kSmem);
    if (e != cudaSuccess) return e;
    occ = n > 0 ? n : 1;
    occ_of[dev].store(occ, std::memory_order_relaxed);
  }
  int grid = occ * num_sms;
  if (grid > kMaxRanges) grid = kMaxRanges;
  if (max_ctas > 0 && max_ctas < grid) grid = max_ctas;
  // Dynamic ranges: the last (1024 - kStaticShare) / 1024 of the work cut into
  // kDynPerCta4 / 4 ranges per CTA, handed out at run time to whichever CTA is
  // free; only where units may be split (a workspace exists). Off: CTAs do
  // stream at unequal rates (with static ranges the last one finishes about
  // 7 us after the median on the 70B-class workload), but measured on B200 the
  // dynamic ranges cost more than that: each starts with a search of the
  // lengths and a fresh block-table read, and they cut long units into many
  // small pieces whose merges land at the end (116 against 110 us there, 333
  // against 317 us on the long-context workload).
  constexpr int kDynPerCta4 = 0, kStaticShare = 870;
  DecodeParams p = prm;
  const int dyn = grid * kDynPerCta4 / 4;
  p.dyn_ranges = prm.ws_done ? (dyn < kMaxRanges - grid ? dyn : kMaxRanges - grid) : 0;
  p.static_share = kStaticShare;
  if (early_start) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(tc::kThreads);
    cfg.dynamicSmemBytes = C::kSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, p, mk, mv);
  }
  kernel<<<grid, tc::kThreads, C::kSmem, stream>>>(p, mk, mv);
  return cudaGetLastError();
}

// cc > 0: products on the CUDA cores for a group of at most cc heads (1, 2, 4).
template <typename T, int D, bool F8>
static cudaError_t launch_tc_d(const DecodeParams& prm, const CUtensorMap& mk,
                               const CUtensorMap& mv, int max_ctas, int num_sms,
                               bool early_start, int cc, cudaStream_t stream) {
  // Two CTAs per SM (two producers keep more copies in flight than one) where
  // shared memory allows; head_dim 128 with more than 8 heads per group runs one.
  const int g = prm.num_heads / prm.num_kv_heads;
  // E4M3 stages are half the size: four of them per CTA.
  constexpr int kNS = F8 ? 4 : (D == 128 ? 2 : 4);
  if constexpr (!F8) {
    if (cc == 1)
      return launch_tc_t<T, D, 1, kNS, 2, F8, 1>(prm, mk, mv, max_ctas, num_sms, early_start, stream);
    if (cc == 2)
      return launch_tc_t<T, D, 1, kNS, 2, F8, 2>(prm, mk, mv, max_ctas, num_sms, early_start, stream);
    if (cc == 4)
      return launch_tc_t<T, D, 1, kNS, 2, F8, 4>(prm, mk, mv, max_ctas, num_sms, early_start, stream);
  }
  if (g <= 8) return launch_tc_t<T, D, 1, kNS, 2, F8, 0>(prm, mk, mv, max_ctas, num_sms, early_start, stream);
  if (D == 64 || F8) return launch_tc_t<T, D, 2, 4, 2, F8, 0>(prm, mk, mv, max_ctas, num_sms, early_start, stream);
  return launch_tc_t<T, D, 2, 4, 1, F8, 0>(prm, mk, mv, max_ctas, num_sms, early_start, stream);
}

cudaError_t launch_decode_tc(const DecodeParams& prm, int q_dtype, int cache_dtype, int max_ctas,
                             int num_sms, bool early_start, int products, cudaStream_t stream) {
  const bool f8 = cache_dtype == PKV_FP8_E4M3;
  // Where the products run: the CUDA cores for narrow groups of a 16-bit cache
  // (by default up to kCudaCoreMaxGroup heads; products > 0 forces them up to
  // 4), else the tensor cores (products < 0 forces them).
  const int g = prm.num_heads / prm.num_kv_heads;
  const int cc_max = products > 0 ? 4 : products < 0 ? 0 : kCudaCoreMaxGroup;
  const int cc = f8 || g > cc_max ? 0 : (g == 1 ? 1 : g == 2 ? 2 : 4);
  const CUtensorMapDataType dt = f8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                 : q_dtype == PKV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                       : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const int e = f8 ? 1 : 2;
  CUtensorMap mk, mv;
  if (!encode_pool_map(&mk, prm.k_cache, dt, e, prm.head_dim, prm.block_size, prm.num_kv_heads,
                       prm.num_blocks) ||
      !encode_pool_map(&mv, prm.v_cache, dt, e, prm.head_dim, prm.block_size, prm.num_kv_heads,
                       prm.num_blocks))
    return cudaErrorInvalidValue;
  if (f8) {
    return q_dtype == PKV_BF16
               ? launch_tc_d<__nv_bfloat16, 128, true>(prm, mk, mv, max_ctas, num_sms, early_start, cc, stream)
               : launch_tc_d<__half, 128, true>(prm, mk, mv, max_ctas, num_sms, early_start, cc, stream);
  }
  if (q_dtype == PKV_BF16) {
    return prm.head_dim == 128
               ? launch_tc_d<__nv_bfloat16, 128, false>(prm, mk, mv, max_ctas, num_sms, early_start, cc, stream)
               : launch_tc_d<__nv_bfloat16, 64, false>(prm, mk, mv, max_ctas, num_sms, early_start, cc, stream);
  }
  return prm.head_dim == 128 ? launch_tc_d<__half, 128, false>(prm, mk, mv, max_ctas, num_sms, early_start, cc, stream)
                             : launch_tc_d<__half, 64, false>(prm, mk, mv, max_ctas, num_sms, early_start, cc, stream);
}

}  // namespace pkv
