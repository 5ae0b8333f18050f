// geometry.h - how the two passes of SQuad-Attention carve the token grid into
// attention problems, shared by the host planner and the kernels.
//
// Operator ("SQuad: Sub-Quadratic Attention Distillation for Efficient Video
// Generation", gist.science technical summary, Methodology section 1): the
// local pass attends inside each tT x tH x tW window; the global pass attends
// across windows among the tokens with the same in-window position.
//
// Both passes are described by one structure. A problem is a 3-D box of tokens
// (a fastest, then b, then c) whose rows sit at token strides sA, sB, sC from
// the problem's first token:
//   local pass : box = (x in window, y in window, t in window),
//                strides (1, W, H*W); problems indexed by the window.
//   global pass: box = (window column, window row, window frame),
//                strides (tW, tH*W, tT*H*W); problems indexed by the position.
// Composing more than two passes (an outlook of the pages: gist.science technical
// summary, Significance and Claims) uses nested tiles t_0 = 1 x 1 x 1 | t_1 | ... | t_k = grid:
// pass j attends among the tokens that share a t_j-window and the position
// inside their t_{j-1}-window, i.e. a box of (t_j / t_{j-1}) sub-windows at
// strides t_{j-1}; problems are indexed by (position in t_{j-1}, t_j-window),
// six digits. The two passes above are j = 1 and j = 2 of k = 2.
// The tensor-core kernels move a problem through TMA boxes ("tiles") of at most
// 128 rows; a tile is a sub-box that is cut along b or along c.
// Packing (forward only): problems of at most 64 rows leave most of a 128-row
// tensor-core tile empty. When one box dimension has extent 1, P problems that are
// consecutive along one problem digit share a box instead: that box dimension runs
// along the digit (stride and tensor-map extent of the digit), the digit's extent
// shrinks to the number of groups, and a key column belongs to the same problem as
// a query row when the two sit at the same position along that dimension.
#pragma once

#include <cstdint>

#ifdef __CUDACC__
#define SQ_HD __host__ __device__ __forceinline__
#else
#define SQ_HD inline
#endif

namespace sq {

// Division by a divisor that is fixed for a launch, as a multiply-high, an add and a
// shift, after the unsigned method of Granlund and Montgomery ("Division by Invariant
// Integers using Multiplication", PLDI 1994): with l = ceil(log2 d) and
// m = floor(2^32 (2^l - d) / d) + 1, the 33-bit multiplier 2^32 + m gives
// floor(x / d) = floor((x (2^32 + m)) / 2^(32 + l)) = (umulhi(x, m) + x) >> l for every
// 0 <= x < 2^32; for x < 2^31 the sum fits in 32 bits. The kernels' scheduling threads
// decode work indices with it, since a hardware-less integer division is a long
// dependent chain on their critical path.
struct FastDiv {
  uint32_t d;  // divisor, 1 <= d < 2^31
  uint32_t m;  // multiplier (low 32 bits of 2^32 + m)
  uint32_t l;  // shift, ceil(log2 d)
};

inline FastDiv make_fastdiv(uint32_t d) {
  FastDiv f{d, 0u, 0u};
  while ((uint64_t(1) << f.l) < d) ++f.l;
  f.m = uint32_t(((uint64_t(1) << 32) * ((uint64_t(1) << f.l) - d)) / d + 1);
  return f;
}

// floor(x / f.d) for 0 <= x < 2^31.
SQ_HD int fdiv(int x, const FastDiv& f) {
#ifdef __CUDA_ARCH__
  const uint32_t hi = __umulhi(uint32_t(x), f.m);
#else
  const uint32_t hi = uint32_t((uint64_t(uint32_t(x)) * f.m) >> 32);
#endif
  return int((hi + uint32_t(x)) >> f.l);
}

struct Geom {
  int a_n, b_n, c_n;  // problem box extents
  int sA, sB, sC;     // token strides of the box dimensions
  int p0, p1, p2;     // problem index extents (p0 fastest): position in the inner window
  int o0, o1, o2;     // token offsets of those index dimensions
  int p3, p4, p5;     // then the outer window (1 when the pass has a single one)
  int o3, o4, o5;
  int probs;          // problems per (batch, head)
  int L;              // rows per problem
  int n;              // tokens per (batch, head)
  int bh;             // batch * heads
  // tiling into <= 128-row TMA boxes (tensor-core path only)
  int b_sub, c_sub;   // tile extent along b and c (a is never cut)
  int nb;             // tiles along b
  int nt;             // tiles per problem
  int box_rows;       // a_n * b_sub * c_sub
  // the divisors above as FastDiv (q0 = p0 p1 p2, problems per outer window)
  FastDiv f_probs, f_q0, f_p0, f_p1, f_p3, f_p4, f_an, f_bn;
  FastDiv f_bsub, f_nb, f_nt;  // set with the tiling
  // packing (plan_pack): pk problems per box along box dimension pk_dim (0 a, 1 b, 2 c;
  // -1: none) and problem digit pk_digit (0..5), whose extent was pk_ext and token
  // offset pk_stride; pk_rowdiv rows separate neighbouring packed problems in a box
  int pk, pk_dim, pk_digit, pk_ext, pk_stride, pk_rowdiv;
  FastDiv f_pk, f_pkrow;
};

// Global token index (b,h offset included) of row 0 of problem `prob`; for a packed
// geometry also the position j0 of its first problem along the packed digit (the
// returned base includes j0 * pk_stride). A group of three digits whose extents are
// all 1 is skipped (the two SQuad passes use one group each), which keeps the
// divisions off the kernels' scheduling path.
SQ_HD int problem_base(const Geom& g, int prob, int* j0 = nullptr) {
  const int bh = fdiv(prob, g.f_probs), idx = prob - bh * g.probs;
  const int q0 = g.p0 * g.p1 * g.p2;  // problems per outer window
  int in = idx, out = 0;
  if (q0 != g.probs) {
    out = fdiv(idx, g.f_q0);
    in = idx - out * q0;
  }
  int base = bh * g.n;
  int dig[6] = {0, 0, 0, 0, 0, 0};
  if (q0 > 1) {
    const int t = fdiv(in, g.f_p0);
    dig[0] = in - t * g.p0;
    dig[2] = fdiv(t, g.f_p1);
    dig[1] = t - dig[2] * g.p1;
    base += dig[0] * g.o0 + dig[1] * g.o1 + dig[2] * g.o2;
  }
  if (out > 0) {
    const int t = fdiv(out, g.f_p3);
    dig[3] = out - t * g.p3;
    dig[5] = fdiv(t, g.f_p4);
    dig[4] = t - dig[5] * g.p4;
    base += dig[3] * g.o3 + dig[4] * g.o4 + dig[5] * g.o5;
  }
  if (j0 != nullptr) {
    const int q = g.pk_digit;
    *j0 = g.pk_dim < 0 ? 0
                       : (q == 0 ? dig[0] : q == 1 ? dig[1] : q == 2 ? dig[2] : q == 3 ? dig[3] : q == 4 ? dig[4] : dig[5]) *
                             g.pk;
  }
  return base;
}

// Packed geometry: the position (0 <= id < pk) of box row i along the packed dimension.
SQ_HD int pack_id(const Geom& g, int i) {
  const int t = fdiv(i, g.f_pkrow);
  return t - fdiv(t, g.f_pk) * g.pk;
}

// Token offset of row i (0 <= i < L) of a problem, rows ordered (c, b, a).
SQ_HD int row_offset(const Geom& g, int i) {
  const int t = fdiv(i, g.f_an), a = i - t * g.a_n;
  const int c = fdiv(t, g.f_bn), b = t - c * g.b_n;
  return a * g.sA + b * g.sB + c * g.sC;
}

// First b and c coordinate of tile t.
SQ_HD void tile_origin(const Geom& g, int t, int& b0, int& c0) {
  const int q = fdiv(t, g.f_nb);
  b0 = (t - q * g.nb) * g.b_sub;
  c0 = q * g.c_sub;
}

// Rows of tile t that lie inside the problem; they are a prefix of the tile.
SQ_HD int tile_valid_rows(const Geom& g, int t) {
  int b0, c0;
  tile_origin(g, t, b0, c0);
  const int nbv = (g.b_n - b0) < g.b_sub ? (g.b_n - b0) : g.b_sub;
  const int ncv = (g.c_n - c0) < g.c_sub ? (g.c_n - c0) : g.c_sub;
  return g.a_n * nbv * ncv;
}

// Token offset (from the problem's first token) of row i of tile t.
SQ_HD int tile_row_offset(const Geom& g, int t, int i) {
  int b0, c0;
  tile_origin(g, t, b0, c0);
  const int r = fdiv(i, g.f_an), a = i - r * g.a_n;
  const int cc = fdiv(r, g.f_bsub), bb = r - cc * g.b_sub;
  return a * g.sA + (b0 + bb) * g.sB + (c0 + cc) * g.sC;
}

SQ_HD int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Fill the tiling fields; returns false when a single box row (a_n) exceeds 128.
inline bool plan_tiles(Geom& g, int max_rows = 128) {
  if (g.a_n > max_rows) return false;
  if (g.a_n * g.b_n <= max_rows) {
    const int cmax = max_rows / (g.a_n * g.b_n);
    const int ntc = ceil_div(g.c_n, cmax);
    g.b_sub = g.b_n;
    g.c_sub = ceil_div(g.c_n, ntc);  // balanced
    g.nb = 1;
    g.nt = ceil_div(g.c_n, g.c_sub);
  } else {
    const int bmax = max_rows / g.a_n;
    const int ntb = ceil_div(g.b_n, bmax);
    g.b_sub = ceil_div(g.b_n, ntb);  // balanced
    g.c_sub = 1;
    g.nb = ceil_div(g.b_n, g.b_sub);
    g.nt = g.nb * g.c_n;
  }
  g.box_rows = g.a_n * g.b_sub * g.c_sub;
  g.f_bsub = make_fastdiv(uint32_t(g.b_sub));
  g.f_nb = make_fastdiv(uint32_t(g.nb));
  g.f_nt = make_fastdiv(uint32_t(g.nt));
  return true;
}

// One pass over nested tiles: attention among the tokens that share a
// (cT, cH, cW)-window and the position inside their (iT, iH, iW)-window. The
// inner tile divides the outer one and the outer one divides the grid.
inline Geom make_geom_pass(int B, int heads, int T, int H, int W, int iT, int iH, int iW, int cT, int cH, int cW) {
  Geom g{};
  g.n = T * H * W;
  g.bh = B * heads;
  g.a_n = cW / iW; g.b_n = cH / iH; g.c_n = cT / iT;
  g.sA = iW; g.sB = iH * W; g.sC = iT * H * W;
  g.p0 = iW; g.p1 = iH; g.p2 = iT;
  g.o0 = 1; g.o1 = W; g.o2 = H * W;
  g.p3 = W / cW; g.p4 = H / cH; g.p5 = T / cT;
  g.o3 = cW; g.o4 = cH * W; g.o5 = cT * H * W;
  g.probs = g.p0 * g.p1 * g.p2 * g.p3 * g.p4 * g.p5;
  g.L = g.a_n * g.b_n * g.c_n;
  g.f_probs = make_fastdiv(uint32_t(g.probs));
  g.f_q0 = make_fastdiv(uint32_t(g.p0 * g.p1 * g.p2));
  g.f_p0 = make_fastdiv(uint32_t(g.p0));
  g.f_p1 = make_fastdiv(uint32_t(g.p1));
  g.f_p3 = make_fastdiv(uint32_t(g.p3));
  g.f_p4 = make_fastdiv(uint32_t(g.p4));
  g.f_an = make_fastdiv(uint32_t(g.a_n));
  g.f_bn = make_fastdiv(uint32_t(g.b_n));
  g.pk = 1;
  g.pk_dim = -1;
  g.pk_digit = 0;
  g.pk_ext = 1;
  g.pk_stride = 0;
  g.pk_rowdiv = 1;
  g.f_pk = make_fastdiv(1u);
  g.f_pkrow = make_fastdiv(1u);
  return g;
}

// Pack several problems into one box when a problem has at most max_rows / 2 rows and
// a box dimension has extent 1 (see the packing note at the top). The slowest such
// dimension is used (c, then b, then a), along the problem digit that fills the box
// best; groups are balanced (the digit's extent p is cut into ceil(p / P) groups of at
// most P problems). Call before plan_tiles. Returns whether the geometry was packed.
inline bool plan_pack(Geom& g, int max_rows = 128) {
  if (2 * g.L > max_rows) return false;
  const int dim = g.c_n == 1 ? 2 : g.b_n == 1 ? 1 : g.a_n == 1 ? 0 : -1;
  if (dim < 0) return false;
  int* ext[6] = {&g.p0, &g.p1, &g.p2, &g.p3, &g.p4, &g.p5};
  int* off[6] = {&g.o0, &g.o1, &g.o2, &g.o3, &g.o4, &g.o5};
  const int cap = max_rows / g.L;
  int q = -1, best = 1;
  for (int i = 0; i < 6; ++i) {
    const int fill = *ext[i] < cap ? *ext[i] : cap;
    if (fill > best) {
      best = fill;
      q = i;
    }
  }
  if (q < 0) return false;
  const int p = *ext[q], groups = ceil_div(p, best), P = ceil_div(p, groups);
  g.pk = P;
  g.pk_dim = dim;
  g.pk_digit = q;
  g.pk_ext = p;
  g.pk_stride = *off[q];
  if (dim == 0) {
    g.a_n = P;
    g.sA = g.pk_stride;
  } else if (dim == 1) {
    g.b_n = P;
    g.sB = g.pk_stride;
  } else {
    g.c_n = P;
    g.sC = g.pk_stride;
  }
  g.pk_rowdiv = dim == 0 ? 1 : dim == 1 ? g.a_n : g.a_n * g.b_n;
  g.probs = g.probs / p * groups;
  *ext[q] = groups;
  *off[q] = g.pk_stride * P;
  g.L = g.a_n * g.b_n * g.c_n;
  g.f_probs = make_fastdiv(uint32_t(g.probs));
  g.f_q0 = make_fastdiv(uint32_t(g.p0 * g.p1 * g.p2));
  g.f_p0 = make_fastdiv(uint32_t(g.p0));
  g.f_p1 = make_fastdiv(uint32_t(g.p1));
  g.f_p3 = make_fastdiv(uint32_t(g.p3));
  g.f_p4 = make_fastdiv(uint32_t(g.p4));
  g.f_an = make_fastdiv(uint32_t(g.a_n));
  g.f_bn = make_fastdiv(uint32_t(g.b_n));
  g.f_pk = make_fastdiv(uint32_t(P));
  g.f_pkrow = make_fastdiv(uint32_t(g.pk_rowdiv));
  return true;
}

// stage 1 = local (window) pass, stage 2 = global (cross-window) pass.
inline Geom make_geom(int stage, int B, int heads, int T, int H, int W, int tT, int tH, int tW) {
  return stage == 1 ? make_geom_pass(B, heads, T, H, W, 1, 1, 1, tT, tH, tW)
                    : make_geom_pass(B, heads, T, H, W, tT, tH, tW, T, H, W);
}

}  // namespace sq
