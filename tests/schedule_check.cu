// Host check of the decode work split: for random length mixes, grid sizes and
// partition sizes, walk every CTA's segments with the library's SegmentWalker
// and verify that each token of each (sequence, KV head) unit is covered exactly
// once, in order, with cuts only at partition multiples. The start of each
// CTA's range is found here by a plain sequential scan.
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "schedule.cuh"

using namespace pkv;

static int check(const std::vector<int32_t>& lens, int Hkv, int cap, int part, int G) {
  const int S = (int)lens.size();
  int64_t tot = 0;
  for (int L : lens) tot += clamp_len(L, cap);
  const int64_t W = tot * Hkv;
  const int64_t P = part > 0 ? part : kNoSplit;
  std::vector<std::vector<char>> seen(S * Hkv);
  for (int i = 0; i < S; ++i)
    for (int h = 0; h < Hkv; ++h) seen[i * Hkv + h].assign(clamp_len(lens[i], cap), 0);
  for (int c = 0; c < G; ++c) {
    const int64_t lo = (W * c + G - 1) / G, hi = (W * (c + 1) + G - 1) / G;
    SegmentWalker w;
    w.seq_lens = lens.data(); w.S = S; w.Hkv = Hkv; w.cap = cap; w.P = P; w.hi = hi;
    w.done = true; w.i = S; w.h = 0; w.L = 0; w.Lnext = 0; w.base = W; w.p = 0;
    int64_t base = 0;
    for (int i = 0; i < S && lo < hi; ++i) {
      const int L = clamp_len(lens[i], cap);
      if (L > 0 && base <= lo && lo < base + (int64_t)L * Hkv) {
        w.done = false; w.i = i; w.base = base; w.L = L;
        w.Lnext = i + 1 < S ? lens[i + 1] : 0;
        const int64_t rel = lo - base;
        w.h = (int)(rel / L);
        const int64_t r = rel - (int64_t)w.h * L;
        w.p = (r + P - 1) / P;
        break;
      }
      base += (int64_t)L * Hkv;
    }
    Segment s;
    while (w.next(s)) {
      if (s.t0 >= s.t1 || s.t1 > s.len) return 1;
      if (s.t0 % P != 0 && s.t0 != 0) return 2;
      if (s.t1 % P != 0 && s.t1 != s.len) return 3;
      const int64_t ustart = 0;  // ownership: the segment's first item must be in [lo, hi)
      (void)ustart;
      std::vector<char>& v = seen[s.seq * Hkv + s.head];
      for (int t = s.t0; t < s.t1; ++t) {
        if (v[t]) return 4;
        v[t] = 1;
      }
    }
  }
  for (auto& v : seen)
    for (char x : v)
      if (!x) return 5;
  return 0;
}

int main() {
  srand(12345);
  int cases = 0;
  for (int trial = 0; trial < 3000; ++trial) {
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
    const int G = 1 + rand() % 600;
    const int r = check(lens, Hkv, cap, part, G);
    if (r) {
      printf("FAIL code %d: S=%d Hkv=%d cap=%d part=%d G=%d\n", r, S, Hkv, cap, part, G);
      return 1;
    }
    ++cases;
  }
  printf("OK %d cases\n", cases);
  return 0;
}
