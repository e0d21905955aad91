// Host-side check of the scheduling arithmetic in common.cuh, the same
// functions the kernels call: FastDiv against plain division, and the tile
// schedule (contiguous ranges per CTA, the CTA owning a tile, the number of
// CTAs per segment, partial-slot indices) against a brute-force count, on
// many shapes. Compiled by nvcc as host code and run on the CPU; prints
// "ok <checks>" or the first failure.
#include <stdio.h>
#include <stdlib.h>

#include <vector>

#include "common.cuh"

using namespace la;

static unsigned long long rng_state = 0x9E3779B97F4A7C15ull;
static unsigned long long next_rand() {   // splitmix64
  unsigned long long z = (rng_state += 0x9E3779B97F4A7C15ull);
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

static long long checks = 0;
#define REQUIRE(c, ...)                        \
  do {                                         \
    ++checks;                                  \
    if (!(c)) {                                \
      printf("FAIL line %d: ", __LINE__);      \
      printf(__VA_ARGS__);                     \
      printf("\n");                            \
      exit(1);                                 \
    }                                          \
  } while (0)

static void check_fastdiv() {
  const int ds[] = {1, 2, 3, 7, 32, 52, 1560, 4680, 65535, 65536, 1000003, 2147483647};
  const int ns[] = {0, 1, 2, 31, 1559, 1560, 1561, 65535, 2147483646, 2147483647};
  for (int d : ds) {
    const FastDiv f = make_fastdiv(d);
    for (int n : ns) REQUIRE(fdiv(f, n) == n / d, "fdiv %d / %d", n, d);
    for (int i = 0; i < 2000; ++i) {
      const int n = (int)(next_rand() & 0x7fffffff);
      REQUIRE(fdiv(f, n) == n / d, "fdiv %d / %d", n, d);
    }
  }
  for (int i = 0; i < 20000; ++i) {
    const int d = 1 + (int)(next_rand() % 0x7ffffffe);
    const int n = (int)(next_rand() & 0x7fffffff);
    REQUIRE(fdiv(make_fastdiv(d), n) == n / d, "fdiv %d / %d", n, d);
  }
}

// The schedule as the host plan builds it for nseg segments of tps tiles over
// at most G CTAs.
static Sched make_sched(int nseg, int tps, int G) {
  Sched s = {};
  s.nseg = nseg;
  s.tps = tps;
  s.nblk = 1;
  s.U = (long long)nseg * tps;
  s.G = (int)(G < s.U ? G : s.U);
  if (s.G < 1) s.G = 1;
  s.fastU = s.U > 0 && s.U * s.G < (1LL << 31);
  s.divU = make_fastdiv(s.fastU ? (int)s.U : 1);
  s.maxc = 1;
  for (int seg = 0; seg < nseg; ++seg) {
    const long long ub = (long long)seg * tps;
    const int c = cta_of_unit(s, ub + tps - 1) - cta_of_unit(s, ub) + 1;
    if (c > s.maxc) s.maxc = c;
  }
  return s;
}

static void check_sched(int nseg, int tps, int G) {
  const Sched s = make_sched(nseg, tps, G);
  // ranges partition [0, U) in order, every CTA's range owned by that CTA
  REQUIRE(unit_begin(s, 0) == 0 && unit_begin(s, s.G) == s.U, "ends %d %d %d", nseg, tps, G);
  std::vector<std::vector<int>> touching(nseg);
  for (int i = 0; i < s.G; ++i) {
    const long long u0 = unit_begin(s, i), u1 = unit_begin(s, i + 1);
    REQUIRE(u0 <= u1, "order cta %d", i);
    for (long long u = u0; u < u1; ++u) {
      REQUIRE(cta_of_unit(s, u) == i, "owner of %lld (nseg %d tps %d G %d)", u, nseg, tps, G);
      REQUIRE(cta_of_unit_fast(s, u) == i, "fast owner of %lld", u);
      const int seg = (int)(u / tps);
      if (touching[seg].empty() || touching[seg].back() != i) touching[seg].push_back(i);
    }
  }
  for (int seg = 0; seg < nseg; ++seg) {
    const int np = parts_of(s, seg);
    REQUIRE(np == (int)touching[seg].size(), "parts_of(%d) = %d, %zu CTAs", seg, np,
            touching[seg].size());
    REQUIRE(np <= s.maxc, "parts_of(%d) = %d > maxc %d", seg, np, s.maxc);
    for (int k = 0; k < np; ++k) {
      // the k-th contributor in CTA order writes slot k of the segment
      REQUIRE(slot_index(s, seg, touching[seg][k]) == (long long)seg * s.maxc + k,
              "slot of segment %d, CTA %d", seg, touching[seg][k]);
    }
  }
}

int main() {
  check_fastdiv();
  // the workloads' shapes (148 SMs) and their edges
  const int shapes[][3] = {
      {32, 256, 148},      // 480p bidirectional, 128-token tiles
      {224, 37, 148},      // 480p, 7 blocks of 4680 tokens
      {1920, 29, 148},     // 720p, 60 blocks of 3680 tokens
      {128, 64, 148},      // gated D = 128, 64-token tiles
      {8192, 1, 148},      // many one-tile heads
      {17408, 1, 148},     // more heads than arrival counters
      {1, 1, 148},         // one tile
      {3, 5, 148},         // fewer tiles than CTAs
      {148, 1, 148},       // one tile per CTA
      {149, 1, 148},       // one more
  };
  for (const auto& sh : shapes) check_sched(sh[0], sh[1], sh[2]);
  for (int i = 0; i < 300; ++i) {
    const int nseg = 1 + (int)(next_rand() % 3000);
    const int tps = 1 + (int)(next_rand() % 300);
    const int G = 1 + (int)(next_rand() % 600);
    check_sched(nseg, tps, G);
  }
  printf("ok %lld\n", checks);
  return 0;
}
