// sp_plan.h - sequence-parallel layout of SQuad-Attention over G ranks (host only).
//
// The operator's local pass attends inside windows and its global pass across windows
// among tokens that share an in-window position ("SQuad: Sub-Quadratic Attention
// Distillation for Efficient Video Generation", gist.science technical summary,
// Methodology section 1). Sharded by windows, the local pass needs nothing from other
// ranks; the global pass needs, for each in-window position, one row from every window.
// So the forward is: local pass on each rank's windows; one all-to-all that moves Q, K
// and the local-pass output from window-major to position-major; the global pass, on
// each rank, for its share of the positions; a second all-to-all that returns the
// output rows to their owners.
//
// Layouts (per (batch, head) slice; all of them rows of d elements):
//   rank r's shard   : the tokens of frames [t0_r, t0_r + T_r), in token order (a
//                      contiguous range of the full sequence); T_r is a whole number of
//                      tT-frame windows, split as evenly as the frame windows allow.
//   positions        : the w = tT*tH*tW in-window positions are split as evenly as
//                      possible: rank r owns positions [p0_r, p0_r + P_r).
//   position-major   : on rank r, rows [pos in its range][window g], g over all m windows
//                      in window order ((t/tT)*(H/tH) + y/tH)*(W/tW) + x/tW. Viewed as a
//                      grid (P_r * T/tT) x (H/tH) x (W/tW) with tile (T/tT) x (H/tH) x (W/tW),
//                      each window of that grid is one global-pass group, in the row
//                      order of the global pass itself, so the local-pass kernel runs it.
//   exchange buffers : chunk per peer, contiguous: [peer][tensor][slice][rows of that peer].
// Index maps (written by plan_sp, all in rows of one slice):
//   send1[i] : local token of the i-th row sent in the first exchange, rows grouped by
//              destination q, then position (of q), then window (of this rank).
//   recv1[j] : for row j of the position-major layout (j = pos_local * m + g), its
//              source rank s and its row within the chunk s sent.
//   send2[i] : position-major row of the i-th row sent back, grouped by destination s
//              (the owner of the window), then position, then window of s.
//   recv2[p] : for local token p, the rank q that computed it and its row within the
//              chunk q sent back.
#pragma once

#include <cstdint>
#include <vector>

namespace sq {

struct SpShape {
  int T, H, W, tT, tH, tW;  // full grid and window tile
  int G, rank;
};

struct SpPlan {
  int G = 0, rank = 0;
  int w = 0, m = 0;              // positions per window, windows in the full grid
  int nHW = 0;                   // windows per frame window: (H/tH) * (W/tW)
  std::vector<int> fw0, nfw;     // per rank: first frame window and frame windows owned
  std::vector<int> p0, np;       // per rank: first position and positions owned
  int t0 = 0, T = 0;             // this rank's frames
  int n_local = 0;               // this rank's tokens: T * H * W
  int n_pos = 0;                 // this rank's position-major rows: np[rank] * m
  std::vector<int> send1_count, recv1_count, send2_count, recv2_count;  // rows per peer
  std::vector<int> send1, recv1_src, recv1_row, send2, recv2_src, recv2_row;
};

inline void even_split(int total, int parts, std::vector<int>& first, std::vector<int>& count) {
  first.assign(parts, 0);
  count.assign(parts, 0);
  int at = 0;
  for (int r = 0; r < parts; ++r) {
    count[r] = total / parts + (r < total % parts ? 1 : 0);
    first[r] = at;
    at += count[r];
  }
}

// Returns false when the shape is invalid or a rank would own no frame window or no
// position (G larger than either count).
inline bool plan_sp(const SpShape& s, SpPlan& p) {
  if (s.G < 1 || s.rank < 0 || s.rank >= s.G) return false;
  if (s.T <= 0 || s.H <= 0 || s.W <= 0 || s.tT <= 0 || s.tH <= 0 || s.tW <= 0) return false;
  if (s.T % s.tT || s.H % s.tH || s.W % s.tW) return false;
  const int nTw = s.T / s.tT, nHw = s.H / s.tH, nWw = s.W / s.tW;
  p = SpPlan{};
  p.G = s.G;
  p.rank = s.rank;
  p.w = s.tT * s.tH * s.tW;
  p.nHW = nHw * nWw;
  p.m = nTw * p.nHW;
  if (s.G > nTw || s.G > p.w) return false;
  even_split(nTw, s.G, p.fw0, p.nfw);
  even_split(p.w, s.G, p.p0, p.np);
  const int r = s.rank, HW = s.H * s.W;
  p.t0 = p.fw0[r] * s.tT;
  p.T = p.nfw[r] * s.tT;
  p.n_local = p.T * HW;
  p.n_pos = p.np[r] * p.m;
  // token of (window g, position pos) in the full grid
  auto token = [&](int g, int pos) {
    const int fw = g / p.nHW, wh = (g / nWw) % nHw, ww = g % nWw;
    const int pt = pos / (s.tH * s.tW), ph = (pos / s.tW) % s.tH, pw = pos % s.tW;
    return ((fw * s.tT + pt) * s.H + wh * s.tH + ph) * s.W + ww * s.tW + pw;
  };
  const int g0 = p.fw0[r] * p.nHW, nw = p.nfw[r] * p.nHW;  // this rank's windows
  const int tok0 = p.t0 * HW;
  // first exchange: to each q, its positions x this rank's windows
  for (int q = 0; q < s.G; ++q) {
    p.send1_count.push_back(p.np[q] * nw);
    for (int pi = 0; pi < p.np[q]; ++pi)
      for (int j = 0; j < nw; ++j) p.send1.push_back(token(g0 + j, p.p0[q] + pi) - tok0);
  }
  for (int src = 0; src < s.G; ++src) p.recv1_count.push_back(p.np[r] * p.nfw[src] * p.nHW);
  p.recv1_src.resize(p.n_pos);
  p.recv1_row.resize(p.n_pos);
  for (int pi = 0; pi < p.np[r]; ++pi)
    for (int g = 0; g < p.m; ++g) {
      const int fw = g / p.nHW;
      int src = 0;
      while (!(fw >= p.fw0[src] && fw < p.fw0[src] + p.nfw[src])) ++src;
      const int nws = p.nfw[src] * p.nHW;
      p.recv1_src[pi * p.m + g] = src;
      p.recv1_row[pi * p.m + g] = pi * nws + (g - p.fw0[src] * p.nHW);
    }
  // second exchange: to each window owner s, this rank's positions x the windows of s
  for (int dst = 0; dst < s.G; ++dst) {
    const int gs = p.fw0[dst] * p.nHW, nws = p.nfw[dst] * p.nHW;
    p.send2_count.push_back(p.np[r] * nws);
    for (int pi = 0; pi < p.np[r]; ++pi)
      for (int j = 0; j < nws; ++j) p.send2.push_back(pi * p.m + gs + j);
  }
  for (int src = 0; src < s.G; ++src) p.recv2_count.push_back(p.np[src] * nw);
  p.recv2_src.resize(p.n_local);
  p.recv2_row.resize(p.n_local);
  for (int j = 0; j < nw; ++j)
    for (int pos = 0; pos < p.w; ++pos) {
      int src = 0;
      while (!(pos >= p.p0[src] && pos < p.p0[src] + p.np[src])) ++src;
      const int lt = token(g0 + j, pos) - tok0;
      p.recv2_src[lt] = src;
      p.recv2_row[lt] = (pos - p.p0[src]) * nw + j;
    }
  return true;
}

}  // namespace sq
