// Host check of the index arithmetic in geometry.h against plain integer division:
// FastDiv over divisors and numerators, then problem_base, tile_origin and
// tile_row_offset over random nested geometries. Prints "ok <count>" or the first
// mismatch and exits non-zero.
#include "geometry.h"
#include <cstdio>
#include <cstdlib>
#include <random>

using namespace sq;

static int fail(const char* what, long long a, long long b, long long c) {
  std::printf("mismatch %s: %lld %lld %lld\n", what, a, b, c);
  return 1;
}

int main() {
  long long checked = 0;
  std::mt19937_64 rng(12345);
  // FastDiv: every divisor up to 4096 against many numerators, then random large divisors
  for (uint32_t d = 1; d <= 4096; ++d) {
    const FastDiv f = make_fastdiv(d);
    for (int x = 0; x < 20000; ++x) {
      if (fdiv(x, f) != int(uint32_t(x) / d)) return fail("fdiv small", x, d, fdiv(x, f));
      ++checked;
    }
    for (int k = 0; k < 2000; ++k) {
      const int x = int(rng() & 0x7fffffffu);
      if (fdiv(x, f) != int(uint32_t(x) / d)) return fail("fdiv random", x, d, fdiv(x, f));
      ++checked;
    }
    for (int x : {0x7fffffff, 0x7ffffffe, int(0x7fffffffu / d * d), int(0x7fffffffu / d * d) - 1}) {
      if (x < 0) continue;
      if (fdiv(x, f) != int(uint32_t(x) / d)) return fail("fdiv edge", x, d, fdiv(x, f));
      ++checked;
    }
  }
  for (int k = 0; k < 200000; ++k) {
    const uint32_t d = 1u + uint32_t(rng() % 0x7fffffffu);
    const FastDiv f = make_fastdiv(d);
    const int x = int(rng() & 0x7fffffffu);
    if (fdiv(x, f) != int(uint32_t(x) / d)) return fail("fdiv large", x, d, fdiv(x, f));
    ++checked;
  }
  // geometry over random nested tiles
  const int divs[] = {1, 2, 3, 4, 5, 6, 8, 11, 20};
  auto pick = [&](int n) {
    int c[64], k = 0;
    for (int v = 1; v <= n; ++v)
      if (n % v == 0) c[k++] = v;
    return c[rng() % k];
  };
  for (int it = 0; it < 4000; ++it) {
    const int T = divs[rng() % 9] * divs[rng() % 9], H = divs[rng() % 9] * divs[rng() % 9];
    const int W = divs[rng() % 9] * divs[rng() % 9];
    const int cT = pick(T), cH = pick(H), cW = pick(W);
    const int iT = pick(cT), iH = pick(cH), iW = pick(cW);
    Geom g = make_geom_pass(2, 3, T, H, W, iT, iH, iW, cT, cH, cW);
    const bool tiled = plan_tiles(g);
    for (int p = 0; p < g.bh * g.probs; ++p) {
      const int bh = p / g.probs, idx = p % g.probs, q0 = g.p0 * g.p1 * g.p2;
      const int in = idx % q0, out = idx / q0;
      const int ref = bh * g.n + (in % g.p0) * g.o0 + ((in / g.p0) % g.p1) * g.o1 + (in / (g.p0 * g.p1)) * g.o2 +
                      (out % g.p3) * g.o3 + ((out / g.p3) % g.p4) * g.o4 + (out / (g.p3 * g.p4)) * g.o5;
      if (problem_base(g, p) != ref) return fail("problem_base", p, ref, problem_base(g, p));
      ++checked;
    }
    for (int i = 0; i < g.L; ++i) {
      const int ref = (i % g.a_n) * g.sA + ((i / g.a_n) % g.b_n) * g.sB + (i / (g.a_n * g.b_n)) * g.sC;
      if (row_offset(g, i) != ref) return fail("row_offset", i, ref, row_offset(g, i));
      ++checked;
    }
    if (!tiled) continue;
    for (int t = 0; t < g.nt; ++t) {
      int b0, c0;
      tile_origin(g, t, b0, c0);
      if (b0 != (t % g.nb) * g.b_sub || c0 != (t / g.nb) * g.c_sub) return fail("tile_origin", t, b0, c0);
      for (int i = 0; i < g.box_rows; ++i) {
        const int ref = (i % g.a_n) * g.sA + (b0 + (i / g.a_n) % g.b_sub) * g.sB + (c0 + i / (g.a_n * g.b_sub)) * g.sC;
        if (tile_row_offset(g, t, i) != ref) return fail("tile_row_offset", t, i, ref);
        ++checked;
      }
    }
  }
  std::printf("ok %lld\n", checked);
  return 0;
}
