// fwd_schedule.h - the forward's work-item order (host and device).
//
// The forward kernel (squad_fwd_tc.cuh) takes items (pairs of jobs) in a fixed order
// that every role decodes the same way; the host fills the order's fields. Kept apart
// from the kernel so that a host test can check the order on the CPU: every (pass,
// head, pair) exactly once, and, when passes are chained in one launch, every item of
// pass j-1 of a head before every item of its pass j.
#pragma once
#include <cstdint>
#include "geometry.h"

namespace sq {

enum { FWD_LOCAL = 1, FWD_GLOBAL = 2, FWD_FUSED = 3, FWD_MULTI = 4 };
constexpr int kMaxFwdPasses = 5;

struct PassArgs {
  Geom g;
  void* out;          // [rows, D] bf16 output of this pass
  float* lse;         // natural-log LSE of this pass, or nullptr
  const uint8_t* discard;  // this pass's values when they are scratch read only here (dropped from L2
                           // once read; rows 128-byte aligned), or nullptr
  int jobs_per_bh;    // problems per (batch, head) x boxes per problem
  int pairs_per_bh;   // ceil(jobs_per_bh / 2)
};

struct FwdArgs {
  PassArgs ps[kMaxFwdPasses];    // two-pass modes: [0] local pass, [1] global pass; FWD_MULTI: pass j at [j]
  int mode;                      // FWD_LOCAL, FWD_GLOBAL, FWD_FUSED or FWD_MULTI
  int npass;                     // passes (2 except in FWD_MULTI)
  int bh;                        // batch * heads
  int lag;                       // FWD_FUSED / FWD_MULTI: heads between pass j-1 of a head and its pass j
  int total_items;               // pairs over all (batch, head) and passes run
  FastDiv f_n1, f_n2, f_n12;     // ps[0].pairs_per_bh, ps[1].pairs_per_bh and their sum
  // FWD_MULTI item order (see decode_item): pref[j] = pairs per head of passes before j,
  // the items of the leading blocks, the number of full blocks and the full block size
  int pref[kMaxFwdPasses + 1];
  int lead_items, nmid;
  FastDiv f_full;
  float scale_log2;              // softmax scale * log2(e)
  uint32_t* counters;            // FWD_FUSED / FWD_MULTI: finished jobs per (pass, batch, head), passes < last
  int* err;
  uint64_t timeout_ns;
};

struct Item {
  int pass, bh, pair;
};

// Tensor maps of up to kMaxFwdPasses passes, four per pass: Q, K, values, output.
// FWD_MULTI: pairs of block b, which holds pass j of head b - j*lag for every pass whose
// head exists.
SQ_HD int multi_block_items(const FwdArgs& a, int b) {
  int s = 0;
  for (int j = 0; j < a.npass; ++j) {
    const int h = b - j * a.lag;
    if (h >= 0 && h < a.bh) s += a.ps[j].pairs_per_bh;
  }
  return s;
}


// Work items in launch order. Fused: the local pass of heads 0..lag-1, then for each
// later head h its local pass followed by the global pass of head h-lag, then the
// global passes of the last lag heads. The lag gives the local pass of a head time
// to finish everywhere before its global pass needs it, while its Q, K and O1 are
// still in L2.
SQ_HD Item decode_item(const FwdArgs& a, int i) {
  if (a.mode == FWD_MULTI) {
    // blocks in order; block b: pass 0 of head b, pass 1 of head b - lag, ... (each while
    // that head exists), all pairs of one (pass, head) together. Full blocks, where every
    // pass is present, are decoded directly; the leading and trailing ones by a scan.
    const int N = a.pref[a.npass], first_full = (a.npass - 1) * a.lag;
    int b, r;
    if (i >= a.lead_items && i < a.lead_items + a.nmid * N) {
      const int t = i - a.lead_items, q = fdiv(t, a.f_full);
      b = first_full + q;
      r = t - q * N;
    } else {
      int acc = i < a.lead_items ? 0 : a.lead_items + a.nmid * N;
      b = i < a.lead_items ? 0 : first_full + a.nmid;
      for (;; ++b) {
        const int sz = multi_block_items(a, b);
        if (i < acc + sz) break;
        acc += sz;
      }
      r = i - acc;
    }
    for (int j = 0; j < a.npass; ++j) {
      const int h = b - j * a.lag, n = a.ps[j].pairs_per_bh;
      if (h < 0 || h >= a.bh) continue;
      if (r < n) return {j, h, r};
      r -= n;
    }
    return {a.npass - 1, 0, 0};  // not reached for i < total_items
  }
  const int n1 = a.ps[0].pairs_per_bh, n2 = a.ps[1].pairs_per_bh;
  if (a.mode == FWD_LOCAL) {
    const int q = fdiv(i, a.f_n1);
    return {0, q, i - q * n1};
  }
  if (a.mode == FWD_GLOBAL) {
    const int q = fdiv(i, a.f_n2);
    return {1, q, i - q * n2};
  }
  const int lag = a.lag;
  if (i < lag * n1) {
    const int q = fdiv(i, a.f_n1);
    return {0, q, i - q * n1};
  }
  const int j = i - lag * n1, blk = fdiv(j, a.f_n12), r = j - blk * (n1 + n2);
  if (blk < a.bh - lag) return r < n1 ? Item{0, blk + lag, r} : Item{1, blk, r - n1};
  const int t = j - (a.bh - lag) * (n1 + n2), q = fdiv(t, a.f_n2);
  return {1, a.bh - lag + q, t - q * n2};
}

SQ_HD bool job_valid(const FwdArgs& a, const Item& it, int which) {
  return 2 * it.pair + which < a.ps[it.pass].jobs_per_bh;
}

// FWD_MULTI: the order's fields of a launch whose ps[0..npass), npass, bh and lag are
// set (the closed form covers the blocks where every pass is present).
inline void plan_multi_order(FwdArgs& a) {
  const int np = a.npass;
  a.pref[0] = 0;
  for (int j = 0; j < np; ++j) a.pref[j + 1] = a.pref[j] + a.ps[j].pairs_per_bh;
  a.total_items = a.bh * a.pref[np];
  // blocks 0 .. bh-1 + (np-1)*lag; block b holds pass j of head b - j*lag while that head
  // exists, so blocks (np-1)*lag .. bh-1 hold every pass
  const int first_full = (np - 1) * a.lag;
  a.nmid = a.bh > first_full ? a.bh - first_full : 0;
  a.lead_items = 0;
  for (int b = 0; b < first_full; ++b)
    for (int j = 0; j < np; ++j) {
      const int h = b - j * a.lag;
      if (h >= 0 && h < a.bh) a.lead_items += a.ps[j].pairs_per_bh;
    }
  a.f_full = make_fastdiv(uint32_t(a.pref[np]));
  a.f_n1 = a.f_n2 = a.f_n12 = a.f_full;  // unused in this mode
}

}  // namespace sq
