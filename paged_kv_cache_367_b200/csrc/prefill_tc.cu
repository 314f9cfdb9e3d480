// Multi-token paged attention with a causal mask, on tensor cores (sm_100a).
//
// What it computes: "vLLM 0.5 深度拆解" (chenxutan.com/d/4924) §2.3 fills a long
// prompt in chunks, so the tokens of a chunk attend over everything cached
// before them and over the chunk itself; "vLLM 推理引擎源码级拆解"
// (chenxutan.com/d/5333) §4.2 lets a request whose leading blocks are cached
// compute only the rest, which is the same operation. Query rows
// query_start[i] .. query_start[i+1]-1 are the last q_i tokens of sequence i,
// whose seq_lens[i] tokens are all in the paged cache already (the chunk's own
// K/V appended first); the row at position p attends over tokens 0..p, read
// through the block table as in §2.3 of the second page.
//
// How, on B200: this is the first paged operation with real arithmetic
// intensity (64 query rows share every K/V tile), so it is written as a
// flash-attention tile on the tensor pipe.
//  * A CTA takes 64 query rows of one (sequence, KV head): rows are (token,
//    query head of the group) pairs, so with GQA the g heads of a token share
//    the K/V reads. Tiles are spread as grid (row tile, sequence, KV head),
//    the row-tile index reversed so the tiles with the longest causal range
//    start first.
//  * A producer warp streams the causal range [0, last position + 1) in
//    64-token chunks of K and V through a ring of shared-memory stages, one TMA
//    tensor copy per (block, KV head) tile of the paged pool (the 5-D map of
//    tc_common.cuh; ids outside the pool land as zeros), with mbarriers.
//  * Four consumer warps own 16 rows each: S = Q K^T with mma.sync m16n8k16
//    (Q fragments held in registers for the whole tile, K by ldmatrix from the
//    swizzled tiles), the causal mask and an online base-2 softmax on the score
//    fragments, P re-packed in registers as the A operand of O += P V (V by
//    ldmatrix.trans). Slots past the causal range are masked in the scores and
//    zeroed in V, so stale or poisoned memory never reaches the output.
//  * FP8-E4M3 caches ("vLLM 0.5 深度拆解" §4.2): the tiles land as codes and are
//    widened in registers, exactly, to f16 pairs (cvt.rn.f16x2.e4m3x2) right
//    after ldmatrix; the products run in f16 (the query rounded to f16 once, P
//    in f16), k_scale is folded into the score scale and v_scale into the final
//    division. A K row then gives each lane four consecutive dimensions of a
//    16-dimension step, so the query fragments take the contraction index in
//    the same permuted order; a transposed V load gives each lane two
//    dimensions of two tokens, split by one byte permute into an even- and an
//    odd-dimension operand, so each thread's output columns come out as four
//    consecutive dimensions.
//  * Every mbarrier wait is bounded; expiry sets an error word, the CTA stops
//    and still waits, bounded, for its own copies in flight.
#include <atomic>
#include <type_traits>

#include "common.cuh"
#include "prefill.cuh"
#include "tc_common.cuh"

namespace pkv {

__device__ int g_pf_timeout = 0;  // bit 0: a wait expired; bit 1: a block id outside the pool

namespace pf {

using namespace tcx;

constexpr int kChunk = 64;          // K/V tokens per stage
constexpr int kRows = 64;           // query rows per CTA
constexpr int kConsumerWarps = 4;   // 16 rows each
constexpr int kThreads = (kConsumerWarps + 1) * 32;

template <int D, int NS, int EKV>
struct Cfg {
  static constexpr int kRowB = D * EKV;                       // bytes of one token's K (or V) row
  static constexpr int kPieceB = kRowB >= 128 ? 128 : kRowB;  // swizzled row piece (128B or 64B)
  static constexpr int kKV = kChunk * kRowB;                  // bytes of K (or V) per stage
  static constexpr int kStage = 2 * kKV;
  static constexpr int kQRow = D * 2 + 16;                    // padded Q staging row
  static constexpr int kQ = kConsumerWarps * 16 * kQRow;
  static constexpr int kSmem = 1024 + NS * kStage + kQ + (2 * NS) * 8 + 16;
  static_assert(kSmem <= 227 * 1024, "shared memory per CTA exceeds 227 KB");
};

__device__ __forceinline__ bool wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  return mbar_wait_or_abort(bar, parity, abort, &g_pf_timeout);
}

// Shared-memory byte offset of 16-byte unit u of token t in a stage's K (or V)
// half: t / bs selects the block tile, whose rows are PB-byte pieces of the
// token's RB-byte row (RB / PB pieces, bs * PB bytes apart) in the PB-byte
// swizzle (128B: unit j of row r at j ^ (r % 8); 64B: at j ^ (r / 2 % 4)).
template <int RB, int PB>
__device__ __forceinline__ uint32_t kv_offset(int t, int u, int bs) {
  constexpr int kUnits = PB / 16;
  const int tt = t % bs, dh = u / kUnits, uu = u % kUnits;
  const int x = PB == 128 ? (tt & 7) : ((tt >> 1) & 3);
  return (uint32_t)((t / bs) * (bs * RB) + dh * (bs * PB) + tt * PB + ((uu ^ x) << 4));
}

// T: query/output type (bf16 or f16). F8: the cache holds E4M3 codes.
template <typename T, int D, int NS, bool F8>
__global__ void __launch_bounds__(kThreads, 2)
    prefill_tc_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap tmap_k,
                      const __grid_constant__ CUtensorMap tmap_v) {
  constexpr int EKV = F8 ? 1 : 2;
  using C = Cfg<D, NS, EKV>;
  using M = typename std::conditional<F8, __half, T>::type;  // MMA operand type
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint8_t* qstage = smem + NS * C::kStage;
  uint64_t* full = reinterpret_cast<uint64_t*>(qstage + C::kQ);
  uint64_t* empty = full + NS;
  volatile int* abort = reinterpret_cast<volatile int*>(empty + NS);

  const int Hq = p.num_heads, Hkv = p.num_kv_heads, g = Hq / Hkv, bs = p.block_size;
  const int seq = blockIdx.y, h = blockIdx.z;
  // Rows stay inside the query tensor, a chunk longer than max_q_len keeps its
  // last max_q_len tokens, and lengths are clamped to the block table.
  const int q1 = min(max(__ldg(p.query_start + seq + 1), 0), p.num_q_tokens);
  const int q0 = max(min(max(__ldg(p.query_start + seq), 0), q1), q1 - p.max_q_len);
  const int qn = q1 - q0;
  const int L = min(__ldg(p.seq_lens + seq), p.max_blocks_per_seq * p.block_size);
  const int rows = qn * g;
  const int rb = (int)(gridDim.x - 1 - blockIdx.x);  // longest causal ranges first
  const int row0 = rb * kRows;
  if (qn <= 0 || row0 >= rows || L <= 0) return;
  const int base_pos = L - qn;                       // position of the chunk's first token
  const int last_row = min(rows, row0 + kRows) - 1;
  const int kv_end = min(L, base_pos + last_row / g + 1);  // causal range of the tile
  if (kv_end <= 0) return;
  const int nchunks = (kv_end + kChunk - 1) / kChunk;
  const int tile = bs * C::kRowB;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, kConsumerWarps);
    }
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer ----
    const int32_t* bt = p.block_table + (int64_t)seq * p.max_blocks_per_seq;
    uint32_t armed = 0, last_parity = 0;
    bool ok = true;
    for (int c = 0; c < nchunks && ok; ++c) {
      const int stage = c % NS;
      const uint32_t phase = (uint32_t)(c / NS) & 1u;
      const int c0 = c * kChunk;
      const int nblk = (min(kChunk, kv_end - c0) + bs - 1) / bs;
      const int blk = lane < nblk ? __ldg(bt + c0 / bs + lane) : 0;
      if (lane == 0) ok = wait(empty + stage, phase ^ 1u, abort);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      uint8_t* st = ring + stage * C::kStage;
      if (lane == 0) mbar_expect_tx(full + stage, (uint32_t)(2 * nblk * tile));
      __syncwarp();
      if (lane < nblk) {
        if (blk < 0 || blk >= p.num_blocks) atomicOr(&g_pf_timeout, 2);  // reads as zeros
        tma_load_5d(st + lane * tile, &tmap_k, 0, 0, 0, h, blk, full + stage);
        tma_load_5d(st + C::kKV + lane * tile, &tmap_v, 0, 0, 0, h, blk, full + stage);
      }
      armed |= 1u << stage;
      last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
    }
    // On abort, wait (bounded) for this CTA's copies in flight before exiting.
    if (!ok && lane == 0) {
      for (int s = 0; s < NS; ++s) {
        if (!(armed >> s & 1u)) continue;
        const long long t0 = clock64();
        while (!mbar_try(full + s, (last_parity >> s) & 1u))
          if (clock64() - t0 > kWaitCycles) break;
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers ----
  const int w = warp;
  const int g0 = lane >> 2, cq = lane & 3;
  // This thread's two rows (g0 and g0 + 8 of the warp's 16) and their positions.
  int pos[2];
#pragma unroll
  for (int x = 0; x < 2; ++x) {
    const int r = row0 + 16 * w + g0 + 8 * x;
    pos[x] = r < rows ? base_pos + r / g : -1;
  }
  // Stage the warp's 16 query rows (zeros past the chunk) and take the A
  // fragments of S = Q K^T for the whole tile.
  uint8_t* qs = qstage + w * 16 * C::kQRow;
  for (int e = lane; e < 16 * (D / 8); e += 32) {
    const int rr = e / (D / 8), u = e % (D / 8);
    const int r = row0 + 16 * w + rr;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < rows) {
      const int tok = r / g, j = r - tok * g;
      v = __ldg(reinterpret_cast<const uint4*>(static_cast<const T*>(p.query) +
                                               ((int64_t)(q0 + tok) * Hq + h * g + j) * D) + u);
    }
    *reinterpret_cast<uint4*>(qs + rr * C::kQRow + u * 16) = v;
  }
  __syncwarp();
  constexpr int KS = D / 16;  // k-steps over head_dim
  uint32_t qa[KS][4];
  if constexpr (F8) {
    // Contraction index permuted as the E4M3 K fragments hold it: logical
    // (2cq, 2cq+1) <- dims 4cq, 4cq+1 and (2cq+8, +9) <- dims 4cq+2, +3 of
    // each 16-dimension step; the query rounded to f16.
    const uint32_t* r0 = reinterpret_cast<const uint32_t*>(qs + g0 * C::kQRow);
    const uint32_t* r1 = reinterpret_cast<const uint32_t*>(qs + (g0 + 8) * C::kQRow);
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      const int e0 = (16 * ks + 4 * cq) / 2;
      qa[ks][0] = to_f16x2<T>(r0[e0]);
      qa[ks][1] = to_f16x2<T>(r1[e0]);
      qa[ks][2] = to_f16x2<T>(r0[e0 + 1]);
      qa[ks][3] = to_f16x2<T>(r1[e0 + 1]);
    }
  } else {
    const int rr = (lane & 7) + 8 * ((lane >> 3) & 1), cu = lane >> 4;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks)
      ldsm_x4(qa[ks], smem_u32(qs + rr * C::kQRow + (2 * ks + cu) * 16));
  }
  constexpr int DT = D / 8;  // output column tiles
  float o[DT][4];
#pragma unroll
  for (int dt = 0; dt < DT; ++dt) o[dt][0] = o[dt][1] = o[dt][2] = o[dt][3] = 0.f;
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
  const float sscale = p.score_scale * (F8 ? __ldg(p.k_scale) : 1.f);
  const int min_pos = __shfl_sync(0xffffffffu, pos[0], 0);  // row 0 of the warp: smallest

  bool ok = true;
  for (int c = 0; c < nchunks; ++c) {
    const int stage = c % NS;
    const uint32_t phase = (uint32_t)(c / NS) & 1u;
    ok = __all_sync(0xffffffffu, wait(full + stage, phase, abort));
    if (!ok) break;
    const uint32_t kst = smem_u32(ring + stage * C::kStage);
    const uint32_t vst = kst + C::kKV;
    const int c0 = c * kChunk;
    // ---- S = Q K^T over the chunk's 64 tokens (8 n-tiles of 8 tokens) ----
    float s[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
    {
      // k-steps outermost: the eight n-tiles are eight independent accumulation
      // chains, so consecutive MMAs do not wait on each other.
      const int mi = lane >> 3, rr = lane & 7;
      if constexpr (F8) {
        // One ldmatrix.x4: 16 tokens x two 16-dimension steps of E4M3 codes.
#pragma unroll
        for (int k2 = 0; k2 < KS / 2; ++k2) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int t = 16 * q + rr + 8 * (mi >> 1);
            uint32_t b[4];
            ldsm_x4(b, kst + kv_offset<C::kRowB, C::kPieceB>(t, 2 * k2 + (mi & 1), bs));
#pragma unroll
            for (int x = 0; x < 4; ++x) {
              const uint32_t b0 = e4m3x2_to_f16x2(b[x]), b1 = e4m3x2_to_f16x2(b[x] >> 16);
              Mma<M>::run(s[2 * q + (x >> 1)], qa[2 * k2 + (x & 1)], b0, b1);
            }
          }
        }
      } else {
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int t = 16 * q + rr + 8 * (mi >> 1);
            uint32_t b[4];
            ldsm_x4(b, kst + kv_offset<C::kRowB, C::kPieceB>(t, 2 * ks + (mi & 1), bs));
            Mma<M>::run(s[2 * q], qa[ks], b[0], b[1]);
            Mma<M>::run(s[2 * q + 1], qa[ks], b[2], b[3]);
          }
        }
      }
    }
    // ---- causal mask, online softmax (base 2) ----
    const bool masked = c0 + kChunk - 1 > min_pos;  // some token may lie past a row's position
    float mx[2] = {m[0], m[1]};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int x = e >> 1;
        const int t = c0 + 8 * nt + 2 * cq + (e & 1);
        float v = s[nt][e] * sscale;
        if (masked && t > pos[x]) v = -INFINITY;
        s[nt][e] = v;
        mx[x] = fmaxf(mx[x], v);
      }
    }
    float alpha[2], msub[2];
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      mx[x] = fmaxf(mx[x], __shfl_xor_sync(0xffffffffu, mx[x], 1));
      mx[x] = fmaxf(mx[x], __shfl_xor_sync(0xffffffffu, mx[x], 2));
      msub[x] = mx[x] == -INFINITY ? 0.f : mx[x];
      alpha[x] = fast_exp2(m[x] - msub[x]);
      m[x] = mx[x];
      l[x] *= alpha[x];
    }
#pragma unroll
    for (int dt = 0; dt < DT; ++dt) {
      o[dt][0] *= alpha[0];
      o[dt][1] *= alpha[0];
      o[dt][2] *= alpha[1];
      o[dt][3] *= alpha[1];
    }
    uint32_t pa[4][4];  // P as the A operand of 4 k-steps of 16 tokens
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const float p0 = fast_exp2(s[nt][0] - msub[0]), p1 = fast_exp2(s[nt][1] - msub[0]);
      const float p2 = fast_exp2(s[nt][2] - msub[1]), p3 = fast_exp2(s[nt][3] - msub[1]);
      float r0, r1, r2, r3;  // the rounded values enter the row sums, as the MMA sees them
      const uint32_t lo = Mma<M>::pack(p0, p1, r0, r1);
      const uint32_t hi = Mma<M>::pack(p2, p3, r2, r3);
      l[0] += r0 + r1;
      l[1] += r2 + r3;
      pa[nt >> 1][(nt & 1) * 2 + 0] = lo;
      pa[nt >> 1][(nt & 1) * 2 + 1] = hi;
    }
    // ---- O += P V ----
    const bool vmask = c0 + kChunk > kv_end;  // slots past the range: zero their V
    {
      const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const int t = 16 * kk + rr + 8 * (mi & 1);
        uint32_t keep0 = 0xffffffffu, keep1 = 0xffffffffu;
        if (vmask) {
          const int ta = c0 + 16 * kk + 2 * cq, tb = ta + 8;
          keep0 = (ta < kv_end ? 0x0000ffffu : 0u) | (ta + 1 < kv_end ? 0xffff0000u : 0u);
          keep1 = (tb < kv_end ? 0x0000ffffu : 0u) | (tb + 1 < kv_end ? 0xffff0000u : 0u);
        }
        if constexpr (F8) {
          // Per 8 x 16-byte matrix a lane holds dims (2g0, 2g0+1) of tokens
          // (2cq, 2cq+1); the byte permute gives the pair of tokens at dim 2g0
          // (low half) and at dim 2g0+1 (high half): the even and the odd
          // n-tile of the matrix's 16 dimensions. Masks act on the codes.
#pragma unroll
          for (int dq = 0; dq < D / 32; ++dq) {
            uint32_t b[4];
            ldsm_x4_t(b, vst + kv_offset<C::kRowB, C::kPieceB>(t, 2 * dq + (mi >> 1), bs));
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              const uint32_t lo = __byte_perm(b[2 * half] & keep0, 0, 0x3120);
              const uint32_t hi = __byte_perm(b[2 * half + 1] & keep1, 0, 0x3120);
              const int c16 = 2 * dq + half;  // 16-dimension group
              Mma<M>::run(o[2 * c16], pa[kk], e4m3x2_to_f16x2(lo), e4m3x2_to_f16x2(hi));
              Mma<M>::run(o[2 * c16 + 1], pa[kk], e4m3x2_to_f16x2(lo >> 16),
                          e4m3x2_to_f16x2(hi >> 16));
            }
          }
        } else {
#pragma unroll
          for (int dp = 0; dp < DT / 2; ++dp) {
            uint32_t b[4];
            ldsm_x4_t(b, vst + kv_offset<C::kRowB, C::kPieceB>(t, 2 * dp + (mi >> 1), bs));
            Mma<M>::run(o[2 * dp], pa[kk], b[0] & keep0, b[1] & keep1);
            Mma<M>::run(o[2 * dp + 1], pa[kk], b[2] & keep0, b[3] & keep1);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty + stage);
  }
  if (!ok) return;
  // ---- epilogue: O / l for this thread's two rows ----
#pragma unroll
  for (int x = 0; x < 2; ++x) {
    float lx = l[x];
    lx += __shfl_xor_sync(0xffffffffu, lx, 1);
    lx += __shfl_xor_sync(0xffffffffu, lx, 2);
    const int r = row0 + 16 * w + g0 + 8 * x;
    if (r >= rows) continue;
    const float inv = lx > 0.f ? (F8 ? __ldg(p.v_scale) : 1.f) / lx : 0.f;
    const int tok = r / g, j = r - tok * g;
    T* row = static_cast<T*>(p.out) + ((int64_t)(q0 + tok) * Hq + h * g + j) * D;
    if constexpr (F8) {
      // n-tiles 2c and 2c + 1 hold dims 16c + 4cq + {0, 2} and {1, 3}.
#pragma unroll
      for (int c16 = 0; c16 < D / 16; ++c16) {
        float a, b;
        uint2 w;
        w.x = Mma<T>::pack(o[2 * c16][2 * x] * inv, o[2 * c16 + 1][2 * x] * inv, a, b);
        w.y = Mma<T>::pack(o[2 * c16][2 * x + 1] * inv, o[2 * c16 + 1][2 * x + 1] * inv, a, b);
        *reinterpret_cast<uint2*>(row + 16 * c16 + 4 * cq) = w;
      }
    } else {
      T* dst = row + 2 * cq;
#pragma unroll
      for (int dt = 0; dt < DT; ++dt) {
        float a, b;
        *reinterpret_cast<uint32_t*>(dst + 8 * dt) =
            Mma<T>::pack(o[dt][2 * x] * inv, o[dt][2 * x + 1] * inv, a, b);
      }
    }
  }
}

template <typename T, int D, bool F8>
cudaError_t launch_t(const PrefillParams& p, const CUtensorMap& mk, const CUtensorMap& mv,
                     int max_q_len, int num_seqs, cudaStream_t stream) {
  constexpr int NS = (D == 128 && !F8) ? 2 : 4;  // stages of 32 KB (16-bit, D 128) or less
  using C = Cfg<D, NS, F8 ? 1 : 2>;
  auto kernel = prefill_tc_kernel<T, D, NS, F8>;
  static std::atomic<int> opted_in[64];  // the shared-memory opt-in, once per device
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!opted_in[dev].load(std::memory_order_relaxed)) {
    const cudaError_t e = cudaFuncSetAttribute(
        kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e != cudaSuccess) return e;
    opted_in[dev].store(1, std::memory_order_relaxed);
  }
  const int g = p.num_heads / p.num_kv_heads;
  const int64_t tiles = ((int64_t)max_q_len * g + kRows - 1) / kRows;
  dim3 grid((unsigned)tiles, (unsigned)num_seqs, (unsigned)p.num_kv_heads);
  kernel<<<grid, kThreads, C::kSmem, stream>>>(p, mk, mv);
  return cudaGetLastError();
}

}  // namespace pf

int pf_timeout_flag(bool clear, int* value) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_pf_timeout, sizeof(int)) != cudaSuccess) return -1;
  if (clear && v) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_pf_timeout, &zero, sizeof(int)) != cudaSuccess) return -1;
  }
  *value = v;
  return 0;
}

}  // namespace pkv

extern "C" int paged_attention_prefill(void* out, const void* query, const void* k_cache,
                                       const void* v_cache, const int32_t* block_table,
                                       const int32_t* seq_lens, const int32_t* query_start,
                                       int num_seqs, int num_q_tokens, int max_q_len,
                                       int num_heads, int num_kv_heads, int head_dim,
                                       int block_size, int max_blocks_per_seq, int64_t num_blocks,
                                       float scale, int q_dtype, int cache_dtype,
                                       const float* k_scale, const float* v_scale, unsigned flags,
                                       void* stream) {
  using namespace pkv;
  if (num_seqs < 0 || num_q_tokens < 0 || max_q_len < 0 || num_kv_heads <= 0 ||
      num_heads <= 0 || num_heads % num_kv_heads != 0 || num_blocks <= 0 ||
      num_blocks > INT32_MAX || max_blocks_per_seq <= 0 || num_seqs > 65535 ||
      num_kv_heads > 65535 || !(scale == scale) || (flags & ~PKV_PREFILL_MMA_SYNC))
    return PKV_ERR_SHAPE;
  if (head_dim != 64 && head_dim != 128) return PKV_ERR_UNSUPPORTED;
  if (block_size != 8 && block_size != 16 && block_size != 32) return PKV_ERR_UNSUPPORTED;
  if ((q_dtype != PKV_BF16 && q_dtype != PKV_F16) ||
      (cache_dtype != q_dtype && cache_dtype != PKV_FP8_E4M3))
    return PKV_ERR_DTYPE;
  const bool f8 = cache_dtype == PKV_FP8_E4M3;
  if (num_seqs == 0 || num_q_tokens == 0 || max_q_len == 0) return PKV_OK;
  if (!out || !query || !k_cache || !v_cache || !block_table || !seq_lens || !query_start)
    return PKV_ERR_NULL;
  if (f8 && (!k_scale || !v_scale)) return PKV_ERR_NULL;
  if (((uintptr_t)out | (uintptr_t)query | (uintptr_t)k_cache | (uintptr_t)v_cache) & 15u ||
      ((uintptr_t)block_table | (uintptr_t)seq_lens | (uintptr_t)query_start) & 3u)
    return PKV_ERR_ALIGN;
  const int64_t tiles = ((int64_t)max_q_len * (num_heads / num_kv_heads) + pf::kRows - 1) /
                        pf::kRows;
  if (tiles > INT32_MAX) return PKV_ERR_SHAPE;
  const CUtensorMapDataType dt = f8                   ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                 : q_dtype == PKV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                       : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  // The tcgen05 kernel takes 16-bit and E4M3 caches (the latter widened to f16
  // in shared memory); PKV_PREFILL_MMA_SYNC selects the mma.sync kernel.
  const bool tc5 = !(flags & PKV_PREFILL_MMA_SYNC) && pf::prefill_tc5_supported(head_dim);
  // The tcgen05 kernel numbers its items (tile pairs x sequences x KV heads) in int.
  if (tc5 && (tiles + 1) / 2 * num_seqs * num_kv_heads > INT32_MAX / 2) return PKV_ERR_SHAPE;
  const int e = f8 ? 1 : 2;
  CUtensorMap mk, mv;
  if (!tcx::encode_pool_map(&mk, k_cache, dt, e, head_dim, block_size, num_kv_heads, num_blocks,
                            tc5) ||
      !tcx::encode_pool_map(&mv, v_cache, dt, e, head_dim, block_size, num_kv_heads, num_blocks,
                            tc5))
    return PKV_ERR_CUDA;
  pf::PrefillParams p;
  p.out = out;
  p.query = query;
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.query_start = query_start;
  p.num_heads = num_heads;
  p.num_kv_heads = num_kv_heads;
  p.block_size = block_size;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.num_q_tokens = num_q_tokens;
  p.max_q_len = max_q_len;
  p.num_blocks = (int)num_blocks;
  p.score_scale = scale * 1.4426950408889634f;
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t err;
  const bool bf16 = q_dtype == PKV_BF16, d128 = head_dim == 128;
  if (tc5)
    err = pf::launch_prefill_tc5(p, mk, mv, head_dim, bf16, f8, num_seqs, st);
  else if (f8 && bf16)
    err = d128 ? pf::launch_t<__nv_bfloat16, 128, true>(p, mk, mv, max_q_len, num_seqs, st)
               : pf::launch_t<__nv_bfloat16, 64, true>(p, mk, mv, max_q_len, num_seqs, st);
  else if (f8)
    err = d128 ? pf::launch_t<__half, 128, true>(p, mk, mv, max_q_len, num_seqs, st)
               : pf::launch_t<__half, 64, true>(p, mk, mv, max_q_len, num_seqs, st);
  else if (bf16)
    err = d128 ? pf::launch_t<__nv_bfloat16, 128, false>(p, mk, mv, max_q_len, num_seqs, st)
               : pf::launch_t<__nv_bfloat16, 64, false>(p, mk, mv, max_q_len, num_seqs, st);
  else
    err = d128 ? pf::launch_t<__half, 128, false>(p, mk, mv, max_q_len, num_seqs, st)
               : pf::launch_t<__half, 64, false>(p, mk, mv, max_q_len, num_seqs, st);
  return err == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}
