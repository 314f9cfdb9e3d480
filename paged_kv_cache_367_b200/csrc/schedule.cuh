// Device-side work split for paged decode.
//
// A unit is one (sequence, KV head) pair; its work is the sequence's tokens
// rounded up to the kernel's chunk (a kernel streams whole chunks, so a partly
// filled chunk costs like a full one) plus a fixed per-unit cost (set-up and
// epilogue, counted in tokens). Units are laid end to end in (sequence, head)
// order, giving every unit a work range in [0, W), W = sum over units of
// (cost + Lw), Lw = L rounded up to the chunk. Partition p of a unit (tokens
// [p P, (p + 1) P)) is an item at work offset
//   first + p P,   first = unit start + cost.
// [0, W) is cut into ranges (Cuts): G "static" ranges of equal size cover
// [0, Ws) and are taken by CTA r = blockIdx.x; Rd "dynamic" ranges of equal size
// cover [Ws, W) and are handed out, in order, to whichever CTA asks next (a
// global counter), so CTAs that run faster take more of the tail. An item
// belongs to the range its offset falls in; a unit may be cut only at multiples
// of the partition size P (never, when P = 0). Consecutive items of one unit in
// one range form a segment, processed as one stream. A unit covered by one
// segment is finished there. A unit cut into several segments ("pieces")
// leaves one partial per piece, and the CTA that finishes the last piece merges
// them. No host knowledge of seq_lens is needed: CTAs read them (small,
// L2-resident) to find their ranges.
//
// Partials live in the workspace in two slots per range: slot 2r holds range
// r's piece that starts inside a unit (only its first segment can), slot
// 2r + 1 its piece that starts a unit and ends inside it (only its last can).
#pragma once

#include "common.cuh"

namespace pkv {

constexpr int kMaxRanges = 1024;  // ranges per launch (two partial slots each)

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
  int unit_round;     // unit lengths are rounded up to a multiple of this (the chunk)
  int dyn_ranges;     // number of dynamic ranges (0: every range is static)
  int static_share;   // share of the work in static ranges, in 1/1024 (when dyn_ranges > 0)
  float score_scale;  // scale * log2(e): scores are kept in the base-2 domain
  const float* k_scale;
  const float* v_scale;
  float* ws_o;        // [2 * kMaxRanges, g, head_dim]: normalised partial output rows
  float* ws_lse;      // [2 * kMaxRanges, g]: base-2 log-sum-exp of each partial
  int* ws_done;       // [num_seqs * num_kv_heads + 1]: finished tokens of split units, then
                      // the dynamic-range counter (zeroed per call)
};

constexpr int64_t kNoSplit = int64_t(1) << 30;

// a / b for a >= 0, b > 0: a 32-bit division when both fit (a 64-bit one is
// several times longer on the GPU, and the set-up runs a chain of them).
__host__ __device__ __forceinline__ int64_t div_nn(int64_t a, int64_t b) {
  if ((((uint64_t)a | (uint64_t)b) >> 32) == 0) return (int64_t)((uint32_t)a / (uint32_t)b);
  return a / b;
}

__host__ __device__ __forceinline__ int clamp_len(int L, int cap) {
  return L < 0 ? 0 : (L > cap ? cap : L);
}

// Work of a unit of L tokens (0 for an empty unit).
__host__ __device__ __forceinline__ int64_t unit_work(int L, int cost, int round) {
  return L > 0 ? (int64_t)(((uint32_t)L + (uint32_t)round - 1u) / (uint32_t)round * (uint32_t)round) + cost
               : 0;
}

__host__ __device__ __forceinline__ int load_len(const int32_t* p) {
#ifdef __CUDA_ARCH__
  return __ldg(p);
#else
  return *p;
#endif
}

// The cut of [0, W) into G static ranges over [0, Ws) and Rd dynamic ranges
// over [Ws, W) (Rd = 0 means Ws = W).
struct Cuts {
  int64_t W, Ws, G, Rd;

  __host__ __device__ int64_t R() const { return G + Rd; }
  // First work offset of range r (r in [0, R]).
  __host__ __device__ int64_t lo(int64_t r) const {
    if (r <= G) return div_nn(Ws * r + G - 1, G);
    return Ws + div_nn((W - Ws) * (r - G) + Rd - 1, Rd);
  }
  // Range holding offset off (0 <= off < W).
  __host__ __device__ int64_t owner(int64_t off) const {
    if (off < Ws) return div_nn(off * G, Ws);
    return G + div_nn((off - Ws) * Rd, W - Ws);
  }
};

__host__ __device__ __forceinline__ Cuts make_cuts(int64_t W, int64_t G, int64_t Rd,
                                                   int static_share) {
  Cuts c;
  c.W = W;
  c.G = G;
  c.Rd = Rd;
  c.Ws = Rd > 0 ? W * static_share / 1024 : W;
  return c;
}

struct Segment {
  int seq, head;
  int t0, t1;       // token range [t0, t1) of the unit
  int len;          // unit length
  int64_t first;    // work offset of the unit's partition 0
};

// Index of the first partition of a unit (partition 0 at offset `first`) that
// range r owns or would own: every partition before it belongs to earlier ranges.
__host__ __device__ __forceinline__ int64_t range_first_part(const Cuts& cu, int64_t r,
                                                             int64_t first, int64_t P) {
  const int64_t lo = cu.lo(r);
  return lo <= first ? 0 : div_nn(lo - first + P - 1, P);
}

// Workspace slot of the piece of a unit held by range r; r0 owns partition 0.
__host__ __device__ __forceinline__ int piece_slot(int64_t r, int64_t r0) {
  return (int)(2 * r + (r == r0 ? 1 : 0));
}

// Slot of the piece `s` produced by range r (the producing side of piece_slot).
__host__ __device__ __forceinline__ int own_piece_slot(int64_t r, const Segment& s) {
  return (int)(2 * r + (s.t0 == 0 ? 1 : 0));
}

// Pieces of a split unit (L tokens, partition 0 at `first`): f(slot) for each,
// in token order.
template <typename F>
__host__ __device__ void for_each_piece(const Cuts& cu, int64_t P, int64_t first, int L, F f) {
  const int64_t nparts = div_nn(L + P - 1, P);
  const int64_t r0 = cu.owner(first);
  const int64_t r1 = cu.owner(first + (nparts - 1) * P);
  for (int64_t r = r0; r <= r1; ++r) {
    const int64_t s0 = r == r0 ? 0 : range_first_part(cu, r, first, P);
    const int64_t s1 = r == r1 ? nparts : range_first_part(cu, r + 1, first, P);
    if (s0 < s1) f(piece_slot(r, r0));
  }
}

// Walks the segments of one range. If the range ends inside a unit that starts
// in it, that piece (the "tail") is taken early: right after the range's first
// segment when that segment is itself a piece of a unit begun in an earlier
// range (a "head"), else first; the walk from the range's start stops short of
// it. Pieces, whose partials need merging, thus come before whole units, and a
// range ends on work that needs no merge.
struct SegmentWalker {
  const int32_t* seq_lens;
  int S, Hkv, cap, cost, round;
  int64_t P;     // partition size, kNoSplit when the unit is never cut
  Cuts cuts;
  int64_t hi;    // where the walk from the range's start stops
  int64_t base;  // work offset of sequence i
  int i, h, L;
  int Lnext;     // raw seq_lens[i + 1], loaded one sequence ahead
  int64_t p;     // first partition of unit (i, h) still to take
  bool done;
  bool tail_pending;
  bool started;   // a segment has been returned
  bool has_head;  // the walk from the range's start begins inside a unit
  Segment tail;

  __host__ __device__ bool next(Segment& s) {
    // The tail goes first, unless the range begins with a head piece (a unit
    // begun in an earlier range, p > 0): then right after it.
    if (tail_pending && (started || !has_head)) {
      tail_pending = false;
      started = true;
      s = tail;
      return true;
    }
    while (!done) {
      if (i >= S) { done = true; break; }
      if (h >= Hkv || L == 0) {
        base += (int64_t)Hkv * unit_work(L, cost, round);
        ++i;
        h = 0;
        p = 0;
        if (i < S) {
          L = clamp_len(Lnext, cap);
          Lnext = i + 1 < S ? load_len(seq_lens + i + 1) : 0;
        }
        continue;
      }
      if (p * P >= L) { ++h; p = 0; continue; }  // unit's rest belongs to earlier ranges
      const int64_t first = base + (int64_t)h * unit_work(L, cost, round) + cost;
      if (first + p * P >= hi) { done = true; break; }
      const int64_t nparts = div_nn(L + P - 1, P);
      int64_t q = div_nn(hi - 1 - first, P);
      if (q > nparts - 1) q = nparts - 1;
      s.seq = i;
      s.head = h;
      s.len = L;
      s.first = first;
      s.t0 = (int)(p * P);
      s.t1 = (int)((q + 1) * P < L ? (q + 1) * P : L);
      if (s.t1 < L) {
        done = true;  // the rest of this unit belongs to the next range
      } else {
        ++h;
        p = 0;
      }
      started = true;
      return true;
    }
    if (tail_pending) {
      tail_pending = false;
      started = true;
      s = tail;
      return true;
    }
    return false;
  }
};

// Sets up `w` for the range [lo, hi): `fi`/`fbase`/`fL` locate the sequence
// holding offset lo (fi < 0: empty range), `li`/`lbase`/`lL` the one holding
// hi - 1, and `fLnext` is the raw length of sequence fi + 1.
__host__ __device__ __forceinline__ void start_range(SegmentWalker& w, int64_t lo, int64_t hi,
                                                     int fi, int64_t fbase, int fL, int fLnext,
                                                     int li, int64_t lbase, int lL) {
  w.hi = hi;
  w.tail_pending = false;
  w.started = false;
  w.has_head = false;
  if (lo >= hi || fi < 0 || fL <= 0) {
    w.done = true;
    w.i = w.S;
    w.h = 0;
    w.L = 0;
    w.Lnext = 0;
    w.base = w.cuts.W;
    w.p = 0;
    return;
  }
  w.done = false;
  w.i = fi;
  w.base = fbase;
  w.L = fL;
  w.Lnext = fLnext;
  const int64_t fw = unit_work(fL, w.cost, w.round);
  const int64_t rel = lo - fbase;
  w.h = (int)div_nn(rel, fw);
  const int64_t r = rel - (int64_t)w.h * fw;  // offset inside unit (fi, h)
  w.p = r <= w.cost ? 0 : div_nn(r - w.cost + w.P - 1, w.P);
  w.has_head = w.p > 0 && w.p * w.P < fL && fbase + (int64_t)w.h * fw + w.cost + w.p * w.P < hi;
  // The tail: the last item lies in a unit that starts at or after lo and
  // continues past hi.
  if (li < 0 || lL <= 0) return;
  const int64_t lw = unit_work(lL, w.cost, w.round);
  const int64_t lrel = (hi - 1) - lbase;
  const int hh = (int)div_nn(lrel, lw);
  const int64_t first = lbase + (int64_t)hh * lw + w.cost;
  if (hi - 1 < first || first < lo) return;
  const int64_t nparts = div_nn(lL + w.P - 1, w.P);
  const int64_t q = div_nn(hi - 1 - first, w.P);
  if (q >= nparts - 1) return;  // the unit ends inside the range
  w.tail.seq = li;
  w.tail.head = hh;
  w.tail.len = lL;
  w.tail.first = first;
  w.tail.t0 = 0;
  w.tail.t1 = (int)((q + 1) * w.P);
  w.tail_pending = true;
  w.hi = first;  // the walk from lo stops before the tail unit
}

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

constexpr int kInitLens = 256;  // batches of at most this many sequences are set up in one pass

struct SchedShared {
  int64_t scan[32];
  int64_t f_base, l_base, d_base;
  Cuts cuts;
  int f_i, l_i, d_i;
  int lens[kInitLens];  // raw seq_lens, in the one-pass set-up
};

// Zero rows of sequence i if it is empty and this CTA owns it (i % G == c).
template <typename OT>
__device__ __forceinline__ void zero_empty_rows(const DecodeParams& prm, int i, int L, int G,
                                                int c) {
  if (i < prm.num_seqs && L == 0 && i % G == c) {
    OT* o = static_cast<OT*>(prm.out) + (int64_t)i * prm.num_heads * prm.head_dim;
    for (int e = 0; e < prm.num_heads * prm.head_dim; ++e) o[e] = from_f32<OT>(0.f);
  }
}

// Records sequence i (work [b, b + wi)) if it holds offset lo, hi - 1 or Ws.
__device__ __forceinline__ void mark_range_seqs(SchedShared& sh, int i, int64_t b, int64_t wi,
                                                int64_t lo, int64_t hi, int64_t ws) {
  if (wi <= 0) return;
  if (lo < hi && b <= lo && lo < b + wi) {
    sh.f_i = i;
    sh.f_base = b;
  }
  if (lo < hi && b <= hi - 1 && hi - 1 < b + wi) {
    sh.l_i = i;
    sh.l_base = b;
  }
  if (b <= ws && ws < b + wi) sh.d_i = i;
}

// Sets up this CTA's walker for its static range r = blockIdx.x (all threads
// must call it; ends with __syncthreads), leaves the cuts in sh.cuts and the
// sequence holding the start of the dynamic ranges in sh.d_i / sh.d_base. Also
// zero-fills the output rows of zero-length sequences i with
// i % gridDim.x == blockIdx.x.
template <typename OT>
__device__ void init_walker(const DecodeParams& prm, SchedShared& sh, SegmentWalker& w) {
  const int S = prm.num_seqs, Hkv = prm.num_kv_heads, cap = prm.len_cap, cost = prm.unit_cost;
  const int round = prm.unit_round;
  const int G = gridDim.x, c = blockIdx.x;
  int64_t W, lo, hi, ws;
  Cuts cu;
  if (threadIdx.x == 0) {
    sh.f_i = -1;
    sh.l_i = -1;
    sh.d_i = S;
  }
  if (S <= (int)blockDim.x && S <= kInitLens) {
    // One pass: each thread holds one sequence; a single scan gives both the
    // total work and every sequence's work offset.
    const int i = threadIdx.x;
    const int raw = i < S ? __ldg(prm.seq_lens + i) : 0;
    const int L = clamp_len(raw, cap);
    if (i < S) sh.lens[i] = raw;
    zero_empty_rows<OT>(prm, i, L, G, c);
    const int64_t wi = i < S ? (int64_t)Hkv * unit_work(L, cost, round) : 0;
    const int64_t incl = block_inclusive_scan(wi, sh.scan, W);  // syncs: defaults above are set
    cu = make_cuts(W, G, prm.dyn_ranges, prm.static_share);
    lo = cu.lo(c);
    hi = cu.lo(c + 1);
    ws = cu.Ws;
    mark_range_seqs(sh, i, incl - wi, wi, lo, hi, ws);
    if (threadIdx.x == 0) {
      sh.d_base = W;
      sh.cuts = cu;
    }
    __syncthreads();
    if (sh.d_i == i) sh.d_base = incl - wi;  // d_base defaults to W, written above
    __syncthreads();
  } else {
    // Pass 1: total work; zero rows of empty sequences.
    int64_t sum = 0;
    for (int i = threadIdx.x; i < S; i += blockDim.x) {
      const int L = clamp_len(__ldg(prm.seq_lens + i), cap);
      sum += (int64_t)Hkv * unit_work(L, cost, round);
      zero_empty_rows<OT>(prm, i, L, G, c);
    }
    block_inclusive_scan(sum, sh.scan, W);
    cu = make_cuts(W, G, prm.dyn_ranges, prm.static_share);
    lo = cu.lo(c);
    hi = cu.lo(c + 1);
    ws = cu.Ws;
    // Pass 2: the sequences holding offsets lo, hi - 1 and Ws.
    if (threadIdx.x == 0) {
      sh.d_base = W;
      sh.cuts = cu;
    }
    __syncthreads();
    int64_t carry = 0;
    for (int i0 = 0; i0 < S; i0 += blockDim.x) {
      const int i = i0 + threadIdx.x;
      const int L = i < S ? clamp_len(__ldg(prm.seq_lens + i), cap) : 0;
      const int64_t wi = (int64_t)Hkv * unit_work(L, cost, round);
      int64_t chunk_tot;
      const int64_t incl = block_inclusive_scan(wi, sh.scan, chunk_tot);
      const int64_t b = carry + incl - wi;
      mark_range_seqs(sh, i, b, wi, lo, hi, ws);
      if (wi > 0 && b <= ws && ws < b + wi) sh.d_base = b;
      __syncthreads();
      const bool have_range = lo >= hi || sh.l_i >= 0;
      const bool have_dyn = ws >= W || sh.d_i < S;
      if (have_range && have_dyn) break;
      carry += chunk_tot;
    }
    __syncthreads();
  }
  w.seq_lens = prm.seq_lens;
  w.S = S;
  w.Hkv = Hkv;
  w.cap = cap;
  w.cost = cost;
  w.round = round;
  w.P = prm.part > 0 ? prm.part : kNoSplit;
  w.cuts = cu;
  const int fi = sh.f_i, li = sh.l_i;
  const bool one_pass = S <= (int)blockDim.x && S <= kInitLens;
  auto raw_len = [&](int i) { return one_pass ? sh.lens[i] : __ldg(prm.seq_lens + i); };
  const int fL = fi >= 0 ? clamp_len(raw_len(fi), cap) : 0;
  const int fLn = fi >= 0 && fi + 1 < S ? raw_len(fi + 1) : 0;
  const int lL = li >= 0 ? clamp_len(raw_len(li), cap) : 0;
  start_range(w, lo, hi, fi, sh.f_base, fL, fLn, li, sh.l_base, lL);
}

// Warp-wide forward search: the sequence whose work range holds offset x,
// starting from sequence *i at work offset *base (all lanes hold the same
// cursor, which only moves forward). On success the cursor points at it and
// *L is its clamped length; returns false if x lies past the last sequence.
__device__ __forceinline__ bool warp_find_seq(const DecodeParams& prm, int64_t x, int& i,
                                              int64_t& base, int& L) {
  const int lane = threadIdx.x & 31;
  const int S = prm.num_seqs, Hkv = prm.num_kv_heads, cap = prm.len_cap, cost = prm.unit_cost;
  while (i < S) {
    const int idx = i + lane;
    const int Li = idx < S ? clamp_len(__ldg(prm.seq_lens + idx), cap) : 0;
    const int64_t wi = (int64_t)Hkv * unit_work(Li, cost, prm.unit_round);
    int64_t incl = wi;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    const int64_t excl = incl - wi;
    const unsigned hit = __ballot_sync(0xffffffffu, wi > 0 && base + excl <= x && x < base + incl);
    if (hit) {
      const int k = __ffs(hit) - 1;
      base += __shfl_sync(0xffffffffu, excl, k);
      L = __shfl_sync(0xffffffffu, Li, k);
      i += k;
      return true;
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
    i += 32;
  }
  return false;
}

// Warp-wide: sets up `w` (whose constant fields are already set) for range r,
// moving the cursor (ci, cbase) forward. Returns false for an empty range.
__device__ __forceinline__ bool warp_start_range(const DecodeParams& prm, SegmentWalker& w,
                                                 int64_t r, int& ci, int64_t& cbase) {
  const int64_t lo = w.cuts.lo(r), hi = w.cuts.lo(r + 1);
  if (lo >= hi) return false;
  int L = 0;
  if (!warp_find_seq(prm, lo, ci, cbase, L)) return false;
  int li = ci, lL = L;
  int64_t lbase = cbase;
  warp_find_seq(prm, hi - 1, li, lbase, lL);
  const int fLn = ci + 1 < w.S ? __ldg(prm.seq_lens + ci + 1) : 0;
  start_range(w, lo, hi, ci, cbase, L, fLn, li, lbase, lL);
  return !w.done || w.tail_pending;
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
// Call from one thread once the piece's partial is written by the threads it is
// synchronised with: the addition releases those writes and acquires the other
// pieces' (acq_rel at GPU scope).
__device__ __forceinline__ bool complete_piece(const DecodeParams& prm, const Segment& s) {
  const int64_t u = (int64_t)s.seq * prm.num_kv_heads + s.head;
  int before;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;"
               : "=r"(before)
               : "l"(prm.ws_done + u), "r"(s.t1 - s.t0)
               : "memory");
  const bool last = before + (s.t1 - s.t0) == s.len;
  // Every piece is in and no other CTA touches this counter again in this
  // call: leave it at zero for the next call on the same workspace.
  if (last) prm.ws_done[u] = 0;
  return last;
}

// Called by `nthreads` threads (index tid) of one CTA after they wrote the
// partial of their piece `s`. `flag` is a shared int private to these
// threads; `sync` synchronises them.
template <typename OT, typename Sync>
__device__ void finish_piece(const DecodeParams& prm, const Cuts& cu, int64_t P, const Segment& s,
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
    for_each_piece(cu, P, s.first, s.len, [&](int slot) {
      M = fmaxf(M, __ldcg(prm.ws_lse + (int64_t)slot * g + j));
    });
    float num = 0.f, den = 0.f;
    for_each_piece(cu, P, s.first, s.len, [&](int slot) {
      const float wt = fast_exp2(__ldcg(prm.ws_lse + (int64_t)slot * g + j) - M);
      num = fmaf(wt, __ldcg(prm.ws_o + ((int64_t)slot * g + j) * D + d), num);
      den += wt;
    });
    static_cast<OT*>(prm.out)[((int64_t)s.seq * Hq + s.head * g + j) * D + d] =
        from_f32<OT>(num / den);
  }
}

}  // namespace pkv
