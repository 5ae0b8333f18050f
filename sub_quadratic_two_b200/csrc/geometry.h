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
  int p0, p1, p2;     // problem index extents (p0 fastest)
  int o0, o1, o2;     // token offsets of the problem index dimensions
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
SQ_HD int problem_base(const Geom& g, int prob) {
  const int bh = prob / g.probs, idx = prob - bh * g.probs;
  const int i0 = idx % g.p0, i1 = (idx / g.p0) % g.p1, i2 = idx / (g.p0 * g.p1);
  return bh * g.n + i0 * g.o0 + i1 * g.o1 + i2 * g.o2;
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

// stage 1 = local (window) pass, stage 2 = global (cross-window) pass.
inline Geom make_geom(int stage, int B, int heads, int T, int H, int W, int tT, int tH, int tW) {
  Geom g{};
  g.n = T * H * W;
  g.bh = B * heads;
  if (stage == 1) {
    g.a_n = tW; g.b_n = tH; g.c_n = tT;
    g.sA = 1; g.sB = W; g.sC = H * W;
    g.p0 = W / tW; g.p1 = H / tH; g.p2 = T / tT;
    g.o0 = tW; g.o1 = tH * W; g.o2 = tT * H * W;
  } else {
    g.a_n = W / tW; g.b_n = H / tH; g.c_n = T / tT;
    g.sA = tW; g.sB = tH * W; g.sC = tT * H * W;
    g.p0 = tW; g.p1 = tH; g.p2 = tT;
    g.o0 = 1; g.o1 = W; g.o2 = H * W;
  }
  g.probs = g.p0 * g.p1 * g.p2;
  g.L = g.a_n * g.b_n * g.c_n;
  return g;
}

}  // namespace sq
