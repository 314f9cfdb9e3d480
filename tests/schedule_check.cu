// Host check of the decode work split (schedule.cuh). For random length mixes,
// unit costs, grid sizes and partition sizes it walks every CTA's segments with
// the library's SegmentWalker and checks that:
//   - each token of each (sequence, KV head) unit is covered exactly once,
//     with cuts only at partition multiples;
//   - every piece of a split unit has its own workspace slot;
//   - for_each_piece enumerates exactly the slots of a split unit's pieces, in
//     token order (this is what the merging CTA reads).
// The start of each CTA's range is found here by a plain sequential scan.
#include <cstdio>
#include <cstdlib>
#include <map>
#include <set>
#include <vector>

#include "schedule.cuh"

using namespace pkv;

static int check(const std::vector<int32_t>& lens, int Hkv, int cap, int part, int cost, int G) {
  const int S = (int)lens.size();
  int64_t W = 0;
  for (int L : lens) {
    const int c = clamp_len(L, cap);
    W += c > 0 ? (int64_t)Hkv * (c + cost) : 0;
  }
  const int64_t P = part > 0 ? part : kNoSplit;
  std::vector<std::vector<char>> seen(S * Hkv);
  for (int i = 0; i < S; ++i)
    for (int h = 0; h < Hkv; ++h) seen[i * Hkv + h].assign(clamp_len(lens[i], cap), 0);
  std::map<int64_t, std::vector<std::pair<int, int>>> pieces;  // unit -> (t0, slot)
  std::map<int64_t, int64_t> firsts;
  std::set<int> slots;
  for (int c = 0; c < G; ++c) {
    const int64_t lo = cta_lo(c, W, G), hi = cta_lo(c + 1, W, G);
    SegmentWalker w;
    w.seq_lens = lens.data(); w.S = S; w.Hkv = Hkv; w.cap = cap; w.cost = cost; w.P = P;
    w.W = W; w.G = G; w.hi = hi;
    w.done = true; w.i = S; w.h = 0; w.L = 0; w.Lnext = 0; w.base = W; w.p = 0;
    w.tail_pending = false;
    int64_t base = 0;
    int li = -1, Lli = 0;
    int64_t lbase = 0;
    bool found = false;
    for (int i = 0; i < S && lo < hi; ++i) {
      const int L = clamp_len(lens[i], cap);
      const int64_t wi = L > 0 ? (int64_t)Hkv * (L + cost) : 0;
      if (!found && wi > 0 && base <= lo && lo < base + wi) {
        w.done = false; w.i = i; w.base = base; w.L = L;
        w.Lnext = i + 1 < S ? lens[i + 1] : 0;
        const int64_t rel = lo - base;
        w.h = (int)(rel / (L + cost));
        const int64_t r = rel - (int64_t)w.h * (L + cost);
        w.p = r <= cost ? 0 : (r - cost + P - 1) / P;
        found = true;
      }
      if (wi > 0 && base <= hi - 1 && hi - 1 < base + wi) {
        li = i; lbase = base; Lli = L;
        break;
      }
      base += wi;
    }
    if (found) set_tail(w, li, lbase, Lli, lo);
    bool first_seg = true;
    Segment s;
    while (w.next(s)) {
      if (s.t0 >= s.t1 || s.t1 > s.len) return 1;
      if (s.t0 % P != 0) return 2;
      if (s.t1 % P != 0 && s.t1 != s.len) return 3;
      // ownership: the segment's first partition lies in this CTA's range
      const int64_t off = s.first + s.t0;
      if (off < lo || off >= hi) return 6;
      // a piece that ends inside its unit and does not start it is the range's
      // only segment; a piece that starts its unit and ends inside it comes first
      if (s.t0 == 0 && s.t1 < s.len && !first_seg) return 10;
      first_seg = false;
      std::vector<char>& v = seen[s.seq * Hkv + s.head];
      for (int t = s.t0; t < s.t1; ++t) {
        if (v[t]) return 4;
        v[t] = 1;
      }
      if (!(s.t0 == 0 && s.t1 == s.len)) {
        const int slot = own_piece_slot(c, s);
        if (slot < 0 || slot >= 2 * G || !slots.insert(slot).second) return 7;
        const int64_t u = (int64_t)s.seq * Hkv + s.head;
        pieces[u].push_back({s.t0, slot});
        firsts[u] = s.first;
      }
    }
  }
  for (auto& v : seen)
    for (char x : v)
      if (!x) return 5;
  // The merging side enumerates the same slots in the same order.
  for (auto& kv : pieces) {
    const int64_t u = kv.first;
    const int L = clamp_len(lens[u / Hkv], cap);
    SegmentWalker w;
    w.P = P; w.W = W; w.G = G;
    std::vector<int> got;
    w.for_each_piece(firsts[u], L, [&](int slot) { got.push_back(slot); });
    if (got.size() != kv.second.size() || got.size() < 2) return 8;
    for (size_t k = 0; k < got.size(); ++k)
      if (got[k] != kv.second[k].second) return 9;
  }
  return 0;
}

int main() {
  srand(12345);
  int cases = 0;
  for (int trial = 0; trial < 4000; ++trial) {
    const int S = 1 + rand() % 40;
    const int Hkv = 1 + rand() % 9;
    const int bs = 8 << (rand() % 3);
    const int cap = bs * (1 + rand() % 64);
    std::vector<int32_t> lens(S);
    for (int i = 0; i < S; ++i) {
      const int k = rand() % 10;
      lens[i] = k == 0 ? 0 : (k == 1 ? -3 : (k == 2 ? cap + 50 : rand() % (cap + 1)));
    }
    const int part = (rand() % 3 == 0) ? 0 : bs * (1 + rand() % 8);
    const int cost = (rand() % 2) ? 0 : rand() % 130;
    const int G = 1 + rand() % 600;
    const int r = check(lens, Hkv, cap, part, cost, G);
    if (r) {
      printf("FAIL code %d: S=%d Hkv=%d cap=%d part=%d cost=%d G=%d\n", r, S, Hkv, cap, part,
             cost, G);
      return 1;
    }
    ++cases;
  }
  printf("OK %d cases\n", cases);
  return 0;
}
