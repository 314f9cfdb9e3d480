// Host check of the decode work split (schedule.cuh). For random length mixes,
// unit costs, grid sizes, dynamic-range counts, static shares and partition
// sizes it walks every range's segments with the library's SegmentWalker and
// checks that:
//   - each token of each (sequence, KV head) unit is covered exactly once,
//     with cuts only at partition multiples;
//   - every piece of a split unit has its own workspace slot;
//   - for_each_piece enumerates exactly the slots of a split unit's pieces, in
//     token order (this is what the merging CTA reads).
// The sequences holding each range's first and last offsets are found here by a
// plain sequential scan.
#include <cstdio>
#include <cstdlib>
#include <algorithm>
#include <map>
#include <set>
#include <vector>

#include "schedule.cuh"

using namespace pkv;

// Sequential search: the sequence holding offset x (-1 if none).
static int find_seq(const std::vector<int32_t>& lens, int Hkv, int cap, int cost, int round,
                    int64_t x, int64_t* base_out, int* L_out) {
  int64_t base = 0;
  for (int i = 0; i < (int)lens.size(); ++i) {
    const int L = clamp_len(lens[i], cap);
    const int64_t wi = (int64_t)Hkv * unit_work(L, cost, round);
    if (wi > 0 && base <= x && x < base + wi) {
      *base_out = base;
      *L_out = L;
      return i;
    }
    base += wi;
  }
  return -1;
}

static int check(const std::vector<int32_t>& lens, int Hkv, int cap, int part, int cost, int round,
                 int G, int Rd, int share) {
  const int S = (int)lens.size();
  int64_t W = 0;
  for (int L : lens) W += (int64_t)Hkv * unit_work(clamp_len(L, cap), cost, round);
  if (W == 0) return 0;
  const int64_t P = part > 0 ? part : kNoSplit;
  const Cuts cu = make_cuts(W, G, Rd, share);
  if (cu.lo(0) != 0 || cu.lo(cu.R()) != W) return 11;
  std::vector<std::vector<char>> seen(S * Hkv);
  for (int i = 0; i < S; ++i)
    for (int h = 0; h < Hkv; ++h) seen[i * Hkv + h].assign(clamp_len(lens[i], cap), 0);
  std::map<int64_t, std::vector<std::pair<int, int>>> pieces;  // unit -> (t0, slot)
  std::map<int64_t, int64_t> firsts;
  std::set<int> slots;
  for (int64_t r = 0; r < cu.R(); ++r) {
    const int64_t lo = cu.lo(r), hi = cu.lo(r + 1);
    if (hi < lo) return 12;
    for (int64_t off : {lo, hi - 1})
      if (lo < hi && cu.owner(off) != r) return 13;
    SegmentWalker w;
    w.seq_lens = lens.data(); w.S = S; w.Hkv = Hkv; w.cap = cap; w.cost = cost; w.P = P;
    w.round = round;
    w.cuts = cu;
    int64_t fbase = 0, lbase = 0;
    int fL = 0, lL = 0;
    const int fi = lo < hi ? find_seq(lens, Hkv, cap, cost, round, lo, &fbase, &fL) : -1;
    const int li = lo < hi ? find_seq(lens, Hkv, cap, cost, round, hi - 1, &lbase, &lL) : -1;
    const int fLn = fi >= 0 && fi + 1 < S ? lens[fi + 1] : 0;
    start_range(w, lo, hi, fi, fbase, fL, fLn, li, lbase, lL);
    bool first_seg = true, prev_head = false, seen_whole = false;
    Segment s;
    while (w.next(s)) {
      if (s.t0 >= s.t1 || s.t1 > s.len) return 1;
      if (s.t0 % P != 0) return 2;
      if (s.t1 % P != 0 && s.t1 != s.len) return 3;
      // ownership: the segment's first partition lies in this range
      const int64_t off = s.first + s.t0;
      if (off < lo || off >= hi) return 6;
      // pieces come before whole units: a piece that starts its unit and ends
      // inside it is first or follows a piece that starts inside its unit
      if (s.t0 == 0 && s.t1 < s.len && !(first_seg || prev_head)) return 10;
      if (!(s.t0 == 0 && s.t1 == s.len) && seen_whole) return 14;
      seen_whole = seen_whole || (s.t0 == 0 && s.t1 == s.len);
      prev_head = first_seg && s.t0 > 0;
      first_seg = false;
      std::vector<char>& v = seen[s.seq * Hkv + s.head];
      for (int t = s.t0; t < s.t1; ++t) {
        if (v[t]) return 4;
        v[t] = 1;
      }
      if (!(s.t0 == 0 && s.t1 == s.len)) {
        const int slot = own_piece_slot(r, s);
        if (slot < 0 || slot >= 2 * cu.R() || !slots.insert(slot).second) return 7;
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
    std::vector<int> got;
    for_each_piece(cu, P, firsts[u], L, [&](int slot) { got.push_back(slot); });
    std::sort(kv.second.begin(), kv.second.end());
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
    const int Rd = (rand() % 2) ? 0 : rand() % (2 * G + 1);
    const int share = rand() % 1025;
    const int round = (rand() % 2) ? 1 : (8 << (rand() % 4));
    const int r = check(lens, Hkv, cap, part, cost, round, G, Rd, share);
    if (r) {
      printf("FAIL code %d: S=%d Hkv=%d cap=%d part=%d cost=%d round=%d G=%d Rd=%d share=%d\n",
             r, S, Hkv, cap, part, cost, round, G, Rd, share);
      return 1;
    }
    ++cases;
  }
  printf("OK %d cases\n", cases);
  return 0;
}
