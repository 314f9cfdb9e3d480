// Device-side work split for paged decode.
//
// A unit is one (sequence, KV head) pair; its work is the sequence's tokens
// plus a fixed per-unit cost (the set-up and epilogue a unit costs, counted in
// tokens). Units are laid end to end in (sequence, head) order, giving every
// unit a work range in [0, W), W = sum over units of (cost + L). Partition p of
// a unit (tokens [p P, (p + 1) P)) is an item at work offset
//   first + p P,   first = unit start + cost,
// and belongs to CTA floor(offset G / W) of a grid of G CTAs. So every CTA gets
// about W / G of work and a contiguous run of items; a unit may be cut only at
// multiples of the partition size P (never, when P = 0). Consecutive items of
// one unit in one CTA form a segment, processed as one stream. A unit covered
// by one segment is finished by that CTA. A unit cut into several segments
// ("pieces") leaves one partial per piece, and the CTA that finishes the last
// piece merges them. The split needs no host knowledge of seq_lens: each CTA
// reads them (small, L2-resident) to find its own range.
//
// Partials live in the workspace in two slots per CTA: slot 2c holds CTA c's
// piece that starts inside a unit (only its first segment can), slot 2c + 1
// its piece that starts a unit and ends inside it (only its last segment can).
#pragma once

#include "common.cuh"

namespace pkv {

constexpr int kMaxCtas = 1024;  // grid size bound (two partial slots per CTA)

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
  int unit_cost;      // work charged per non-empty unit, in tokens
  float score_scale;  // scale * log2(e): scores are kept in the base-2 domain
  const float* k_scale;
  const float* v_scale;
  float* ws_o;        // [2 * kMaxCtas, g, head_dim]: normalised partial output rows
  float* ws_lse;      // [2 * kMaxCtas, g]: base-2 log-sum-exp of each partial
  int* ws_done;       // [num_seqs, num_kv_heads]: finished tokens of split units (zeroed per call)
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
  int t0, t1;       // token range [t0, t1) of the unit
  int len;          // unit length
  int64_t first;    // work offset of the unit's partition 0
};

// First work offset owned by CTA c.
__host__ __device__ __forceinline__ int64_t cta_lo(int64_t c, int64_t W, int64_t G) {
  return (W * c + G - 1) / G;
}

// Index of the first partition of a unit (partition 0 at offset `first`) that
// CTA c owns or would own: every partition before it belongs to earlier CTAs.
__host__ __device__ __forceinline__ int64_t cta_first_part(int64_t c, int64_t first, int64_t P,
                                                           int64_t W, int64_t G) {
  const int64_t lo = cta_lo(c, W, G);
  return lo <= first ? 0 : (lo - first + P - 1) / P;
}

// Workspace slot of the piece of a unit held by CTA c; c0 owns partition 0.
__host__ __device__ __forceinline__ int piece_slot(int64_t c, int64_t c0) {
  return (int)(2 * c + (c == c0 ? 1 : 0));
}

// Slot of the piece `s` produced by CTA c (the producing side of piece_slot).
__host__ __device__ __forceinline__ int own_piece_slot(int64_t c, const Segment& s) {
  return (int)(2 * c + (s.t0 == 0 ? 1 : 0));
}

// Walks the segments of one CTA's range. Each role of a CTA holds its own copy
// and advances it independently; all copies see the same sequence. If the range
// ends inside a unit that starts in it, that piece (the "tail") comes first and
// the walk from the range's start stops short of it: its partial is then ready
// early, and the CTA ends on work that needs no merge.
struct SegmentWalker {
  const int32_t* seq_lens;
  int S, Hkv, cap, cost;
  int64_t P;     // partition size, kNoSplit when the unit is never cut
  int64_t W, G;  // total work, grid size
  int64_t hi;    // where the walk from the range's start stops
  int64_t base;  // work offset of sequence i
  int i, h, L;
  int Lnext;     // raw seq_lens[i + 1], loaded one sequence ahead
  int64_t p;     // first partition of unit (i, h) still to take
  bool done;
  bool tail_pending;
  Segment tail;

  __host__ __device__ bool next(Segment& s) {
    if (tail_pending) {
      tail_pending = false;
      s = tail;
      return true;
    }
    while (!done) {
      if (i >= S) { done = true; break; }
      if (h >= Hkv || L == 0) {
        base += L > 0 ? (int64_t)Hkv * (L + cost) : 0;
        ++i;
        h = 0;
        p = 0;
        if (i < S) {
          L = clamp_len(Lnext, cap);
          Lnext = i + 1 < S ? load_len(seq_lens + i + 1) : 0;
        }
        continue;
      }
      if (p * P >= L) { ++h; p = 0; continue; }  // unit's rest belongs to earlier CTAs
      const int64_t first = base + (int64_t)h * (L + cost) + cost;
      if (first + p * P >= hi) { done = true; break; }
      const int64_t nparts = (L + P - 1) / P;
      int64_t q = (hi - 1 - first) / P;
      if (q > nparts - 1) q = nparts - 1;
      s.seq = i;
      s.head = h;
      s.len = L;
      s.first = first;
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

  // Pieces of a split unit: calls f(slot) for each, in token order.
  template <typename F>
  __host__ __device__ void for_each_piece(int64_t first, int L, F f) const {
    const int64_t nparts = (L + P - 1) / P;
    const int64_t c0 = first * G / W;
    const int64_t c1 = (first + (nparts - 1) * P) * G / W;
    for (int64_t c = c0; c <= c1; ++c) {
      const int64_t s0 = c == c0 ? 0 : cta_first_part(c, first, P, W, G);
      const int64_t s1 = c == c1 ? nparts : cta_first_part(c + 1, first, P, W, G);
      if (s0 < s1) f(piece_slot(c, c0));
    }
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
  int64_t found_base, last_base;
  int64_t total;
  int found_i, last_i;
};

// Sets the tail of a walker whose range [lo, hi) has its last offset in
// sequence li (work offset lbase): if the last item lies in a unit that starts
// at or after lo and continues past hi, that piece becomes the tail.
__host__ __device__ __forceinline__ void set_tail(SegmentWalker& w, int li, int64_t lbase, int Lli,
                                                  int64_t lo) {
  w.tail_pending = false;
  if (li < 0 || Lli <= 0) return;
  const int64_t rel = (w.hi - 1) - lbase;
  const int hh = (int)(rel / (Lli + w.cost));
  const int64_t first = lbase + (int64_t)hh * (Lli + w.cost) + w.cost;
  if (w.hi - 1 < first || first < lo) return;  // last item in an earlier unit, or unit began earlier
  const int64_t nparts = (Lli + w.P - 1) / w.P;
  const int64_t q = (w.hi - 1 - first) / w.P;
  if (q >= nparts - 1) return;                  // the unit ends inside the range
  w.tail.seq = li;
  w.tail.head = hh;
  w.tail.len = Lli;
  w.tail.first = first;
  w.tail.t0 = 0;
  w.tail.t1 = (int)((q + 1) * w.P);
  w.tail_pending = true;
  w.hi = first;  // the walk from lo stops before the tail unit
}

// Sets up this CTA's walker (all threads must call it). Also zero-fills the
// output rows of zero-length sequences i with i % gridDim.x == blockIdx.x.
template <typename OT>
__device__ void init_walker(const DecodeParams& prm, SchedShared& sh, SegmentWalker& w) {
  const int S = prm.num_seqs, Hkv = prm.num_kv_heads, cap = prm.len_cap, cost = prm.unit_cost;
  const int G = gridDim.x, c = blockIdx.x;
  // Pass 1: total work; zero rows of empty sequences.
  int64_t sum = 0;
  for (int i = threadIdx.x; i < S; i += blockDim.x) {
    const int L = clamp_len(__ldg(prm.seq_lens + i), cap);
    sum += L > 0 ? (int64_t)Hkv * (L + cost) : 0;
    if (L == 0 && i % G == c) {
      OT* o = static_cast<OT*>(prm.out) + (int64_t)i * prm.num_heads * prm.head_dim;
      for (int e = 0; e < prm.num_heads * prm.head_dim; ++e) o[e] = from_f32<OT>(0.f);
    }
  }
  int64_t W;
  block_inclusive_scan(sum, sh.scan, W);
  const int64_t lo = cta_lo(c, W, G);
  const int64_t hi = cta_lo(c + 1, W, G);
  // Pass 2: the sequences whose work ranges contain offsets lo and hi - 1.
  if (threadIdx.x == 0) {
    sh.found_i = -1;
    sh.last_i = -1;
  }
  __syncthreads();
  int64_t carry = 0;
  for (int i0 = 0; i0 < S && lo < hi; i0 += blockDim.x) {
    const int i = i0 + threadIdx.x;
    const int L = i < S ? clamp_len(__ldg(prm.seq_lens + i), cap) : 0;
    const int64_t wi = L > 0 ? (int64_t)Hkv * (L + cost) : 0;
    int64_t chunk_tot;
    const int64_t incl = block_inclusive_scan(wi, sh.scan, chunk_tot);
    const int64_t b = carry + incl - wi;
    if (wi > 0 && b <= lo && lo < b + wi) {
      sh.found_i = i;
      sh.found_base = b;
    }
    if (wi > 0 && b <= hi - 1 && hi - 1 < b + wi) {
      sh.last_i = i;
      sh.last_base = b;
    }
    __syncthreads();
    if (sh.last_i >= 0) break;
    carry += chunk_tot;
  }
  __syncthreads();
  w.seq_lens = prm.seq_lens;
  w.S = S;
  w.Hkv = Hkv;
  w.cap = cap;
  w.cost = cost;
  w.P = prm.part > 0 ? prm.part : kNoSplit;
  w.W = W;
  w.G = G;
  w.hi = hi;
  w.tail_pending = false;
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
  w.h = (int)(rel / (w.L + cost));
  const int64_t r = rel - (int64_t)w.h * (w.L + cost);  // offset inside unit (fi, h)
  w.p = r <= cost ? 0 : (r - cost + w.P - 1) / w.P;
  const int li = sh.last_i;
  set_tail(w, li, sh.last_base, li >= 0 ? clamp_len(__ldg(prm.seq_lens + li), cap) : 0, lo);
}

// ---- pieces of split units -------------------------------------------------
//
// Each piece writes its partial (per query head: the normalised output row and
// the base-2 log-sum-exp of its scores) to its slot, then adds its token count
// to the unit's counter. The CTA whose addition completes the unit's length
// merges all pieces:
//   M = max_p lse_p,  w_p = 2^(lse_p - M),  out = sum_p w_p o_p / sum_p w_p,
// the blockwise form of the softmax. No CTA ever waits for another.

// Adds piece `s` to its unit's counter; true for the piece that completes it.
// Call from one thread, after the piece's partial is written and fenced.
__device__ __forceinline__ bool complete_piece(const DecodeParams& prm, const Segment& s) {
  const int64_t u = (int64_t)s.seq * prm.num_kv_heads + s.head;
  const int before = atomicAdd(prm.ws_done + u, s.t1 - s.t0);
  return before + (s.t1 - s.t0) == s.len;
}

// Called by `nthreads` threads (index tid) of one CTA after they wrote the
// partial of their piece `s`. `flag` is a shared int private to these
// threads; `sync` synchronises them.
template <typename OT, typename Sync>
__device__ void finish_piece(const DecodeParams& prm, const SegmentWalker& w, const Segment& s,
                             int tid, int nthreads, volatile int* flag, Sync sync) {
  __threadfence();
  sync();
  if (tid == 0) *flag = complete_piece(prm, s);
  sync();
  if (!*flag) return;
  __threadfence();
  const int Hq = prm.num_heads, g = Hq / prm.num_kv_heads, D = prm.head_dim;
  for (int e = tid; e < g * D; e += nthreads) {
    const int j = e / D, d = e - j * D;
    float M = -INFINITY;
    w.for_each_piece(s.first, s.len, [&](int slot) {
      M = fmaxf(M, __ldcg(prm.ws_lse + (int64_t)slot * g + j));
    });
    float num = 0.f, den = 0.f;
    w.for_each_piece(s.first, s.len, [&](int slot) {
      const float wt = fast_exp2(__ldcg(prm.ws_lse + (int64_t)slot * g + j) - M);
      num = fmaf(wt, __ldcg(prm.ws_o + ((int64_t)slot * g + j) * D + d), num);
      den += wt;
    });
    static_cast<OT*>(prm.out)[((int64_t)s.seq * Hq + s.head * g + j) * D + d] =
        from_f32<OT>(num / den);
  }
}

}  // namespace pkv
