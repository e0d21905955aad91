// Host-side check of the tensor-core kernels' shared-memory plans (tc.cuh,
// causal.cuh), the functions the launcher calls: for every head dim, gate,
// RoPE table size up to the library's limit and plan budget, the chosen plan
// fits its budget with at least two stages, so every bf16 call the library
// accepts (tables of up to kMaxRopeEntries) has a tensor-core plan; two apply
// CTAs of a half-budget plan fit in one SM's 228 KB with their reserved
// shared memory; the 480p and 720p grids take the intended plans; and the
// apply kernel's weighted tile split covers every tile.
// Compiled by nvcc as host code and run on the CPU; prints "ok <checks>" or
// the first failure.
#include <stdio.h>

#include "causal.cuh"

using namespace la;

static long long checks = 0;
#define REQUIRE(c, ...)                        \
  do {                                         \
    ++checks;                                  \
    if (!(c)) {                                \
      printf("FAIL line %d: ", __LINE__);      \
      printf(__VA_ARGS__);                     \
      printf("\n");                            \
      return 1;                                \
    }                                          \
  } while (0)

int main() {
  const int kSmPerSm = 228 * 1024, kReserved = 1024, kStatic = 1024;
  for (int D : {64, 128}) {
    for (int entries = 0; entries <= kMaxRopeEntries; ++entries) {
      const int s1 = pick_state_stages(D, entries);
      REQUIRE(s1 >= 2, "state D=%d entries=%d: %d stages", D, entries, s1);
      REQUIRE(state_plan(D, entries, s1).total <= (uint32_t)kSmemBudget, "state plan over budget");
      for (int gate = 0; gate < 2; ++gate) {
        int st, sb, gs;
        pick_apply_plan(D, entries, gate, &st, &sb, &gs);
        REQUIRE(st >= 2, "apply D=%d entries=%d gate=%d: %d stages", D, entries, gate, st);
        REQUIRE(apply_plan(D, entries, gate, st, sb, gs).total <= (uint32_t)kSmemBudget,
                "apply plan over budget");
        int sh, sbh, gsh;
        pick_apply_plan(D, entries, gate, &sh, &sbh, &gsh, kSmemBudgetHalf);
        if (sh > 0) {
          const uint32_t t = apply_plan(D, entries, gate, sh, sbh, gsh).total;
          REQUIRE(t <= (uint32_t)kSmemBudgetHalf, "half plan over budget");
          REQUIRE(2 * (t + kReserved + kStatic) <= (uint32_t)kSmPerSm,
                  "two half-budget CTAs do not fit an SM: %u", t);
        }
      }
    }
  }
  for (int entries = 0; entries <= kMaxRopeEntries; ++entries) {
    const int s = pick_causal_stages(entries);
    REQUIRE(s >= 2, "causal entries=%d: %d stages", entries, s);
    REQUIRE(causal_plan(entries, s).total <= (uint32_t)kSmemBudget, "causal plan over budget");
  }
  // the 480p grid (21 x 30 x 52, 16/24/24 at D = 64): 8 q stages and two image
  // slots on one CTA; without RoPE, 4 stages and two slots at half budget
  const int e480 = 21 * 10 + 30 * 14 + 52 * 14;
  int st, sb, gs;
  pick_apply_plan(64, e480, 0, &st, &sb, &gs);
  REQUIRE(st == 8 && sb == 2, "480p apply plan: %d stages, %d slots", st, sb);
  pick_apply_plan(64, 0, 0, &st, &sb, &gs, kSmemBudgetHalf);
  REQUIRE(st >= 3 && sb == 2, "no-RoPE half plan: %d stages, %d slots", st, sb);
  // D = 128 with a gate: a two-tile gate ring on the 480p grid (32/48/48:
  // 2510 table entries), one tile on the 720p grid (21 x 45 x 80: 3628)
  pick_apply_plan(128, 21 * 18 + 30 * 26 + 52 * 26, 1, &st, &sb, &gs);
  REQUIRE(st >= 2 && gs == 2, "gated D=128 480p plan: %d stages, gate ring %d", st, gs);
  pick_apply_plan(128, 21 * 18 + 45 * 26 + 80 * 26, 1, &st, &sb, &gs);
  REQUIRE(st >= 2 && gs == 1, "gated D=128 720p plan: %d stages, gate ring %d", st, gs);
  for (int e : {0, 1358, 2510, 3628, kMaxRopeEntries})
    REQUIRE(tc_supported(true, 128, 1, 32, 48, 48, e) && tc_supported(true, 64, 1, 16, 24, 24, e),
            "no tensor-core plan at %d entries", e);
  // the apply kernel's weighted tile split, as the launcher enables it
  // (u >= 2 g, nlate <= g / 4): every tile once, in order, at least one per
  // CTA; nlate = 0 is the even split c * u / g
  for (int g : {1, 2, 7, 100, 148, 296})
    for (long long u = 2LL * g; u <= 8LL * 148; u += 13)
      for (int nl = 0; 4 * nl <= g; ++nl) {
        REQUIRE(apply_tile_start(0, g, nl, u) == 0 && apply_tile_start(g, g, nl, u) == u,
                "split g=%d u=%lld nlate=%d does not cover the tiles", g, u, nl);
        for (int c = 0; c < g; ++c) {
          const long long a = apply_tile_start(c, g, nl, u), b = apply_tile_start(c + 1, g, nl, u);
          REQUIRE(b - a >= 1, "split g=%d u=%lld nlate=%d: CTA %d gets %lld tiles", g, u, nl, c,
                  b - a);
          if (nl == 0) REQUIRE(a == c * u / g, "even split differs at CTA %d", c);
        }
      }
  // a 720p block step (32 heads x 29 tiles on 148 CTAs, the last 32 light)
  REQUIRE(apply_tile_start(116, 148, 32, 928) - apply_tile_start(115, 148, 32, 928) >= 7 &&
              apply_tile_start(148, 148, 32, 928) - apply_tile_start(147, 148, 32, 928) <= 4,
          "block-step split");
  printf("ok %lld\n", checks);
  return 0;
}
