// Device-side work split for paged decode.
//
// A unit is one (sequence, KV head) pair; its work is the sequence's tokens.
// Units are laid end to end in (sequence, head) order, giving every token of
// every unit a work offset in [0, W), W = num_kv_heads * sum(seq_lens). A unit
// may be cut only at multiples of the partition size P (or never, when P = 0).
// An item (unit, partition p) starts at offset unit_start + p * P and belongs to
// CTA floor(offset * G / W), so every CTA of a grid of G gets about W / G tokens
// of work and a contiguous run of items. Consecutive items of one unit in one
// CTA form a segment and are processed as a single stream; a unit covered by
// one segment is finished by that CTA, and a unit cut into several segments
// leaves one partial (output row, log-sum-exp) per segment; the CTA that
// finishes the last piece of a unit merges its partials (see finish_piece).
//
// The split needs no host knowledge of seq_lens: each CTA reads them (they are
// small and L2-resident) to find its own range.
#pragma once

#include "common.cuh"

namespace pkv {

struct DecodeParams {
  void* out;
  const void* query;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_table;
  const int32_t* seq_lens;
  int num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq;
  int64_t num_blocks;
  int len_cap;        // seq_lens are clamped to [0, len_cap]
  int part;           // partition size in tokens, 0 = never split
  int max_parts;      // partitions per (sequence, head) in the workspace (0 if no split)
  float score_scale;  // scale * log2(e): scores are kept in the base-2 domain
  const float* k_scale;
  const float* v_scale;
  float* ws_o;        // [num_seqs, num_heads, max_parts, head_dim]
  float* ws_lse;      // [num_seqs, num_heads, max_parts], base-2 log-sum-exp
  int* ws_link;       // [num_seqs, num_kv_heads, max_parts]: partition after a segment
  int* ws_done;       // [num_seqs, num_kv_heads]: tokens of split units finished (zeroed per call)
};

constexpr int64_t kNoSplit = int64_t(1) << 30;

__host__ __device__ __forceinline__ int clamp_len(int L, int cap) {
  return L < 0 ? 0 : (L > cap ? cap : L);
}

__host__ __device__ __forceinline__ int load_len(const int32_t* p) {
#ifdef __CUDA_ARCH__
  return __ldg(p);
#else
  return *p;
#endif
}

struct Segment {
  int seq, head;
  int t0, t1;   // token range [t0, t1) of the unit
  int len;      // unit length
};

// Walks the segments of one CTA's range, in order. All threads of a CTA hold
// identical copies and advance them in lockstep.
struct SegmentWalker {
  const int32_t* seq_lens;
  int S, Hkv, cap;
  int64_t P;     // partition size, kNoSplit when the unit is never cut
  int64_t hi;    // first work offset of the next CTA
  int64_t base;  // work offset of sequence i
  int i, h, L;
  int Lnext;     // raw seq_lens[i + 1], loaded one sequence ahead
  int64_t p;     // first partition of unit (i, h) still to take
  bool done;

  __host__ __device__ bool next(Segment& s) {
    while (!done) {
      if (i >= S) { done = true; break; }
      if (h >= Hkv || L == 0) {
        base += (int64_t)Hkv * L;
        ++i;
        h = 0;
        p = 0;
        if (i < S) {
          L = clamp_len(Lnext, cap);
          Lnext = i + 1 < S ? load_len(seq_lens + i + 1) : 0;
        }
        continue;
      }
      if (p * P >= L) { ++h; p = 0; continue; }  // unit started in an earlier CTA
      const int64_t ustart = base + (int64_t)h * L;
      if (ustart + p * P >= hi) { done = true; break; }
      const int64_t nparts = (L + P - 1) / P;
      int64_t q = (hi - 1 - ustart) / P;
      if (q > nparts - 1) q = nparts - 1;
      s.seq = i;
      s.head = h;
      s.len = L;
      s.t0 = (int)(p * P);
      s.t1 = (int)((q + 1) * P < L ? (q + 1) * P : L);
      if (s.t1 < L) {
        done = true;  // the rest of this unit belongs to the next CTA
      } else {
        ++h;
        p = 0;
      }
      return true;
    }
    return false;
  }
};

// Block-wide inclusive scan of one int64 per thread (blockDim.x <= 1024).
__device__ __forceinline__ int64_t block_inclusive_scan(int64_t v, int64_t* sm32, int64_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int64_t n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) sm32[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int64_t w = lane < nw ? sm32[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int64_t n = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += n;
    }
    if (lane < nw) sm32[lane] = w;
  }
  __syncthreads();
  if (warp > 0) v += sm32[warp - 1];
  total = sm32[nw - 1];
  __syncthreads();
  return v;
}

struct SchedShared {
  int64_t scan[32];
  int64_t found_base;
  int64_t total;
  int found_i;
};

// Sets up this CTA's walker (all threads must call it). Also zero-fills the
// output rows of zero-length sequences i with i % gridDim.x == blockIdx.x.
template <typename OT>
__device__ void init_walker(const DecodeParams& prm, SchedShared& sh, SegmentWalker& w) {
  const int S = prm.num_seqs, Hkv = prm.num_kv_heads, cap = prm.len_cap;
  const int G = gridDim.x, c = blockIdx.x;
  // Pass 1: total work; zero rows of empty sequences.
  int64_t sum = 0;
  for (int i = threadIdx.x; i < S; i += blockDim.x) {
    const int L = clamp_len(__ldg(prm.seq_lens + i), cap);
    sum += L;
    if (L == 0 && i % G == c) {
      OT* o = static_cast<OT*>(prm.out) + (int64_t)i * prm.num_heads * prm.head_dim;
      for (int e = 0; e < prm.num_heads * prm.head_dim; ++e) o[e] = from_f32<OT>(0.f);
    }
  }
  int64_t tot;
  block_inclusive_scan(sum, sh.scan, tot);
  const int64_t W = tot * Hkv;
  const int64_t lo = (W * c + G - 1) / G;
  const int64_t hi = (W * (c + 1) + G - 1) / G;
  // Pass 2: the sequence whose work range contains offset lo.
  if (threadIdx.x == 0) sh.found_i = -1;
  __syncthreads();
  int64_t carry = 0;
  for (int i0 = 0; i0 < S && lo < W; i0 += blockDim.x) {
    const int i = i0 + threadIdx.x;
    const int L = i < S ? clamp_len(__ldg(prm.seq_lens + i), cap) : 0;
    int64_t chunk_tot;
    const int64_t incl = block_inclusive_scan((int64_t)L * Hkv, sh.scan, chunk_tot);
    const int64_t b = carry + incl - (int64_t)L * Hkv;
    if (L > 0 && b <= lo && lo < b + (int64_t)L * Hkv) {
      sh.found_i = i;
      sh.found_base = b;
    }
    __syncthreads();
    if (sh.found_i >= 0) break;
    carry += chunk_tot;
  }
  __syncthreads();
  w.seq_lens = prm.seq_lens;
  w.S = S;
  w.Hkv = Hkv;
  w.cap = cap;
  w.P = prm.part > 0 ? prm.part : kNoSplit;
  w.hi = hi;
  const int fi = sh.found_i;
  if (lo >= hi || fi < 0) {
    w.done = true;
    w.i = S;
    w.h = 0;
    w.L = 0;
    w.Lnext = 0;
    w.base = W;
    w.p = 0;
    return;
  }
  w.done = false;
  w.i = fi;
  w.base = sh.found_base;
  w.L = clamp_len(__ldg(prm.seq_lens + fi), cap);
  w.Lnext = fi + 1 < S ? __ldg(prm.seq_lens + fi + 1) : 0;
  const int64_t rel = lo - w.base;
  w.h = (int)(rel / w.L);
  const int64_t r = rel - (int64_t)w.h * w.L;
  w.p = (r + w.P - 1) / w.P;
}

// ---- pieces of split units -------------------------------------------------
//
// A segment that is not a whole unit writes its partial (per query head: the
// normalised output row and the base-2 log-sum-exp of its scores) at partition
// t0 / P, and links that partition to the partition after its last token. It
// then adds its token count to the unit's counter; the CTA whose addition
// completes the unit's length merges all pieces of the unit:
//   M = max_p lse_p,  w_p = 2^(lse_p - M),  out = sum_p w_p o_p / sum_p w_p,
// the blockwise form of the softmax. No CTA ever waits for another.

// Called by `nthreads` threads (index tid) after they wrote the partial rows of
// a piece [t0, t1) of unit (i, h) and the link of its first partition. `flag`
// is a shared int private to these threads; `sync` synchronises them.
template <typename OT, typename Sync>
__device__ void finish_piece(const DecodeParams& prm, int i, int h, int L, int t0, int t1,
                             int tid, int nthreads, volatile int* flag, Sync sync) {
  __threadfence();
  sync();
  const int64_t u = (int64_t)i * prm.num_kv_heads + h;
  if (tid == 0) {
    const int before = atomicAdd(prm.ws_done + u, t1 - t0);
    *flag = before + (t1 - t0) == L;
  }
  sync();
  if (!*flag) return;
  __threadfence();
  const int Hq = prm.num_heads, g = Hq / prm.num_kv_heads, D = prm.head_dim;
  const int MP = prm.max_parts, P = prm.part, nparts = (L + P - 1) / P;
  const int* link = prm.ws_link + u * MP;
  for (int e = tid; e < g * D; e += nthreads) {
    const int j = e / D, d = e - j * D;
    const int64_t row = ((int64_t)i * Hq + h * g + j) * MP;
    float M = -INFINITY;
    int p = 0;
    for (int guard = 0; guard < nparts && p < nparts; ++guard) {
      M = fmaxf(M, __ldcg(prm.ws_lse + row + p));
      const int nx = __ldcg(link + p);
      if (nx <= p) break;
      p = nx;
    }
    float num = 0.f, den = 0.f;
    p = 0;
    for (int guard = 0; guard < nparts && p < nparts; ++guard) {
      const float w = fast_exp2(__ldcg(prm.ws_lse + row + p) - M);
      num = fmaf(w, __ldcg(prm.ws_o + (row + p) * D + d), num);
      den += w;
      const int nx = __ldcg(link + p);
      if (nx <= p) break;
      p = nx;
    }
    static_cast<OT*>(prm.out)[((int64_t)i * Hq + h * g + j) * D + d] = from_f32<OT>(num / den);
  }
}

}  // namespace pkv
