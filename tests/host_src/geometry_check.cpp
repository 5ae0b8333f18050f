// Host check of the index arithmetic in geometry.h against plain integer division:
// FastDiv over divisors and numerators, then problem_base, tile_origin and
// tile_row_offset over random nested geometries. Prints "ok <count>" or the first
// mismatch and exits non-zero.
#include "geometry.h"
#include <cstdio>
#include <cstdlib>
#include <random>
#include <vector>

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
    for (int x = 0; x < 10000; ++x) {
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
  for (int it = 0; it < 1500; ++it) {
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
  // packing: every packed box row maps, through the tensor map's view, to the token of
  // exactly one row of one original problem, rows of a problem share their pack_id, and
  // rows past the packed digit's extent are exactly the out-of-bounds ones
  int packed_geoms = 0;
  for (int it = 0; it < 1000; ++it) {
    const int T = divs[rng() % 9] * divs[rng() % 9], H = divs[rng() % 9] * divs[rng() % 9];
    const int W = divs[rng() % 9] * divs[rng() % 9];
    const int cT = pick(T), cH = pick(H), cW = pick(W);
    const int iT = pick(cT), iH = pick(cH), iW = pick(cW);
    const Geom u = make_geom_pass(2, 3, T, H, W, iT, iH, iW, cT, cH, cW);
    Geom g = u;
    if (!plan_pack(g)) continue;
    if (!plan_tiles(g)) return fail("plan_tiles after pack", it, g.L, 0);
    if (g.nt != 1 || g.box_rows != g.L || g.L > 128) return fail("packed tiling", g.nt, g.box_rows, g.L);
    ++packed_geoms;
    // owner[token] = (original problem) from the unpacked geometry
    const int rows = u.bh * u.n;
    std::vector<int> owner(rows, -1), seen(rows, 0);
    for (int p = 0; p < u.bh * u.probs; ++p)
      for (int i = 0; i < u.L; ++i) owner[problem_base(u, p) + row_offset(u, i)] = p;
    const int mext[3] = {g.pk_dim == 0 ? g.pk_ext : g.a_n, g.pk_dim == 1 ? g.pk_ext : g.b_n,
                         g.pk_dim == 2 ? g.pk_ext : g.c_n};
    for (int p = 0; p < g.bh * g.probs; ++p) {
      int j0 = -1;
      const int base = problem_base(g, p, &j0);
      const int tbase = base - j0 * g.pk_stride;
      if (j0 < 0 || j0 >= g.pk_ext || tbase < 0) return fail("pack origin", p, j0, tbase);
      const int co[3] = {g.pk_dim == 0 ? j0 : 0, g.pk_dim == 1 ? j0 : 0, g.pk_dim == 2 ? j0 : 0};
      int id_owner[128];
      for (int k = 0; k < 128; ++k) id_owner[k] = -1;
      for (int i = 0; i < g.box_rows; ++i) {
        const int a = i % g.a_n, b = (i / g.a_n) % g.b_n, c = i / (g.a_n * g.b_n);
        const bool inb = co[0] + a < mext[0] && co[1] + b < mext[1] && co[2] + c < mext[2];
        const int id = pack_id(g, i);
        const int refid = g.pk_dim == 0 ? a : g.pk_dim == 1 ? b : c;
        if (id != refid) return fail("pack_id", i, id, refid);
        const bool valid = j0 + id < g.pk_ext;
        if (valid != inb) return fail("pack validity", p, i, valid);
        if (!valid) continue;
        const int tok = base + tile_row_offset(g, 0, i);
        const int tma = tbase + (co[0] + a) * g.sA + (co[1] + b) * g.sB + (co[2] + c) * g.sC;
        if (tok != tma || tok < 0 || tok >= rows) return fail("pack token", p, i, tok);
        if (id_owner[id] < 0) id_owner[id] = owner[tok];
        if (owner[tok] != id_owner[id]) return fail("pack grouping", p, i, tok);
        ++seen[tok];
        ++checked;
      }
    }
    for (int t = 0; t < rows; ++t)
      if (seen[t] != 1) return fail("pack coverage", it, t, seen[t]);
  }
  if (packed_geoms < 50) return fail("too few packed geometries", packed_geoms, 0, 0);
  // the three passes over the 27,280-token grid used by the benchmark: 20-token windows six
  // to a box along c (four groups per window column), 11-token groups ten to a box along
  // c, 124-token groups unpacked
  {
    Geom g1 = make_geom_pass(1, 24, 31, 22, 40, 1, 1, 1, 1, 1, 20);
    if (!plan_pack(g1) || g1.pk != 6 || g1.pk_dim != 2 || g1.pk_ext != 22 || g1.probs != 2 * 4 * 31)
      return fail("video pass 1 packing", g1.pk, g1.pk_dim, g1.probs);
    Geom g2 = make_geom_pass(1, 24, 31, 22, 40, 1, 1, 20, 1, 11, 20);
    if (!plan_pack(g2) || g2.pk != 10 || g2.pk_dim != 2 || g2.pk_ext != 20 || g2.probs != 2 * 2 * 2 * 31)
      return fail("video pass 2 packing", g2.pk, g2.pk_dim, g2.probs);
    Geom g3 = make_geom_pass(1, 24, 31, 22, 40, 1, 11, 20, 31, 22, 40);
    if (plan_pack(g3) || g3.pk != 1) return fail("video pass 3 packing", g3.pk, g3.L, 0);
    checked += 3;
  }
  std::printf("ok %lld\n", checked);
  return 0;
}
