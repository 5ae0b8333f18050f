// Host check of the forward's work-item order (fwd_schedule.h): for the two-pass fused
// order and the k-pass order, every (pass, head, pair) is decoded exactly once, and every
// item of pass j-1 of a head comes before every item of its pass j. Prints "ok" or the
// first failure.
#include <cstdio>
#include <vector>
#include "fwd_schedule.h"

using namespace sq;

static bool check(const FwdArgs& a, const char* what) {
  const int np = a.mode == FWD_MULTI ? a.npass : 2;
  std::vector<int> first_pos[kMaxFwdPasses], last_pos[kMaxFwdPasses], seen[kMaxFwdPasses];
  for (int j = 0; j < np; ++j) {
    first_pos[j].assign(a.bh, -1);
    last_pos[j].assign(a.bh, -1);
    seen[j].assign(size_t(a.bh) * a.ps[j].pairs_per_bh, 0);
  }
  for (int i = 0; i < a.total_items; ++i) {
    const Item it = decode_item(a, i);
    if (it.pass < 0 || it.pass >= np || it.bh < 0 || it.bh >= a.bh || it.pair < 0 ||
        it.pair >= a.ps[it.pass].pairs_per_bh) {
      std::printf("%s: item %d decodes out of range (%d, %d, %d)\n", what, i, it.pass, it.bh, it.pair);
      return false;
    }
    int& s = seen[it.pass][size_t(it.bh) * a.ps[it.pass].pairs_per_bh + it.pair];
    if (s++) {
      std::printf("%s: (%d, %d, %d) decoded twice\n", what, it.pass, it.bh, it.pair);
      return false;
    }
    if (first_pos[it.pass][it.bh] < 0) first_pos[it.pass][it.bh] = i;
    last_pos[it.pass][it.bh] = i;
  }
  for (int j = 0; j < np; ++j)
    for (int v : seen[j])
      if (v != 1) {
        std::printf("%s: an item of pass %d is missing\n", what, j);
        return false;
      }
  for (int j = 1; j < np; ++j)
    for (int h = 0; h < a.bh; ++h)
      if (!(last_pos[j - 1][h] < first_pos[j][h])) {
        std::printf("%s: head %d, pass %d starts before pass %d ends\n", what, h, j, j - 1);
        return false;
      }
  return true;
}

int main() {
  unsigned rng = 12345u;
  auto next = [&]() { rng = rng * 1664525u + 1013904223u; return rng >> 8; };
  int cases = 0;
  // two passes in one launch (the fused two-pass operator)
  for (int bh = 1; bh <= 40; ++bh)
    for (int lag = 1; lag <= 3; ++lag)
      for (int n1 = 1; n1 <= 6; ++n1)
        for (int n2 = 1; n2 <= 6; ++n2) {
          FwdArgs a{};
          a.mode = FWD_FUSED;
          a.npass = 2;
          a.bh = bh;
          a.lag = lag < bh ? lag : bh;
          a.ps[0].pairs_per_bh = n1;
          a.ps[1].pairs_per_bh = n2;
          a.f_n1 = make_fastdiv(uint32_t(n1));
          a.f_n2 = make_fastdiv(uint32_t(n2));
          a.f_n12 = make_fastdiv(uint32_t(n1 + n2));
          a.total_items = bh * (n1 + n2);
          if (!check(a, "fused")) return 1;
          ++cases;
        }
  // k passes in one launch
  for (int np = 2; np <= kMaxFwdPasses; ++np)
    for (int bh = 1; bh <= 48; bh += (bh < 8 ? 1 : 5))
      for (int lag = 1; lag <= 3; ++lag)
        for (int rep = 0; rep < 12; ++rep) {
          FwdArgs a{};
          a.mode = FWD_MULTI;
          a.npass = np;
          a.bh = bh;
          a.lag = lag < bh ? lag : bh;
          for (int j = 0; j < np; ++j) a.ps[j].pairs_per_bh = 1 + int(next() % 9);
          plan_multi_order(a);
          if (!check(a, "multi")) return 1;
          ++cases;
        }
  std::printf("ok %d orders\n", cases);
  return 0;
}
