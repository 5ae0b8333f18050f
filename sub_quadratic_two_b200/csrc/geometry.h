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
#pragma once

#ifdef __CUDACC__
#define SQ_HD __host__ __device__ __forceinline__
#else
#define SQ_HD inline
#endif

namespace sq {

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
};

// Global token index (b,h offset included) of row 0 of problem `prob`.
// A group of three digits whose extents are all 1 is skipped (the two SQuad passes use
// one group each), which keeps the divisions off the kernels' scheduling path.
SQ_HD int problem_base(const Geom& g, int prob) {
  const int bh = prob / g.probs, idx = prob - bh * g.probs;
  const int q0 = g.p0 * g.p1 * g.p2;  // problems per outer window
  int in = idx, out = 0;
  if (q0 != g.probs) {
    out = idx / q0;
    in = idx - out * q0;
  }
  int base = bh * g.n;
  if (q0 > 1) {
    const int t = in / g.p0, i0 = in - t * g.p0;
    const int i2 = t / g.p1, i1 = t - i2 * g.p1;
    base += i0 * g.o0 + i1 * g.o1 + i2 * g.o2;
  }
  if (out > 0) {
    const int t = out / g.p3, i3 = out - t * g.p3;
    const int i5 = t / g.p4, i4 = t - i5 * g.p4;
    base += i3 * g.o3 + i4 * g.o4 + i5 * g.o5;
  }
  return base;
}

// Token offset of row i (0 <= i < L) of a problem, rows ordered (c, b, a).
SQ_HD int row_offset(const Geom& g, int i) {
  const int a = i % g.a_n, b = (i / g.a_n) % g.b_n, c = i / (g.a_n * g.b_n);
  return a * g.sA + b * g.sB + c * g.sC;
}

// First b and c coordinate of tile t.
SQ_HD void tile_origin(const Geom& g, int t, int& b0, int& c0) {
  b0 = (t % g.nb) * g.b_sub;
  c0 = (t / g.nb) * g.c_sub;
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
  const int a = i % g.a_n, bb = (i / g.a_n) % g.b_sub, cc = i / (g.a_n * g.b_sub);
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
  return g;
}

// stage 1 = local (window) pass, stage 2 = global (cross-window) pass.
inline Geom make_geom(int stage, int B, int heads, int T, int H, int W, int tT, int tH, int tW) {
  return stage == 1 ? make_geom_pass(B, heads, T, H, W, 1, 1, 1, tT, tH, tW)
                    : make_geom_pass(B, heads, T, H, W, tT, tH, tW, T, H, W);
}

}  // namespace sq
