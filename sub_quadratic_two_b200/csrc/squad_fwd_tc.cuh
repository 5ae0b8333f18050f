// squad_fwd_tc.cuh - forward of SQuad-Attention on the sm_100a tensor cores.
//
// The operator ("SQuad: Sub-Quadratic Attention Distillation for Efficient Video
// Generation", gist.science technical summary, Methodology section 1) is a local
// pass (softmax attention inside each window, values V, output O1) followed by a
// global pass (softmax attention among the tokens that share an in-window
// position, same Q and K, values O1, output O). One kernel runs either pass, or
// both in one launch with the global pass of a head scheduled right behind the
// local pass of that head, so that its Q, K and O1 are still in L2.
//
// Work decomposition. A problem (a window or a group) is cut into TMA boxes of at
// most 128 rows (geometry.h). A job is one query box of one problem; it runs
// over all key boxes of its problem with an online softmax. Jobs are taken in
// pairs (A, B): A runs on softmax warpgroup 0, B on warpgroup 1, so that the
// tensor core works on one while the other computes its softmax. When A and B
// belong to the same problem (the 220-token windows: two query boxes) they share
// the key and value boxes.
//
// Roles (384 threads):
//   warps 0-3  softmax warpgroup 0, warps 4-7 softmax warpgroup 1
//              (thread = TMEM lane = query row of the box)
//   warp 8     TMA producer: Q boxes (two slots, a box is released after its job's
//              last S) and key/value boxes (one ring of four slots, K and V of a key
//              box in consecutive slots) in the order the tensor core consumes them
//   warps 9,11 one thread each issues tcgen05.mma for one softmax warpgroup:
//              S = Q K^T (both operands K-major) and O += P V (P read from TMEM,
//              V MN-major)
//   warp 10    chained passes: publishes per-(pass, head) completion of the passes
//              other than the last
// The softmax warpgroups write their output rows (through a per-warp transpose patch,
// so that stores are whole 128-byte lines) and, for inference, drop the consumed
// local-pass rows from L2.
// TMEM (512 columns): warpgroup a owns S/P at columns [256a, 256a+128) and O at
// [256a+128, 256a+256). P overwrites S in place as packed bf16.
// Every wait is bounded by the global timer; on expiry the CTA raises an abort
// flag, lets its copies and MMAs in flight land, frees TMEM and returns.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>
#include "fwd_schedule.h"
#include "geometry.h"
#include "sm100.cuh"

namespace sq {

constexpr int kFwdThreads = 384;
constexpr uint32_t kBlk = 128 * 128;  // one 64-column block of a 128-row bf16 box

template <int D>
struct FwdLayout {
  static constexpr int TILE = 128 * D * 2;
  static constexpr int NQ = 2;   // Q boxes (released after the job's last S)
  static constexpr int NKV = 4;  // one ring for key and value boxes, in consumption order
  static constexpr int Q_OFF = 0;
  static constexpr int KV_OFF = Q_OFF + NQ * TILE;
  static constexpr int XP_OFF = KV_OFF + NKV * TILE;   // per softmax warp: 32 rows x 128 B transpose patch
  static constexpr int BAR_OFF = XP_OFF + 8 * 4096;
  static constexpr int NBAR = 24;
  static constexpr int BYTES = BAR_OFF + NBAR * 8 + 16;  // + tmem holder, abort flag, two counters
  static constexpr int ALLOC = BYTES + 1024;
  static constexpr int TMEM_COLS = 512;
};

// barrier indices
// (two Q slots, four key/value slots, two of the rest: one per warpgroup). P is handed to
// the tensor core in two halves of 64 keys: F_PF when the first half (and any rescale of
// O) is in TMEM, F_PF2 when the second is.
enum { F_QF = 0, F_QE = 2, F_KVF = 4, F_KVE = 8, F_SF = 12, F_PF = 14, F_OF = 16, F_PF2 = 18, F_DRAIN = 20 };

struct alignas(64) FwdMaps {
  CUtensorMap m[4 * kMaxFwdPasses];
};

struct Job {
  bool valid;
  int qt;    // query box within the problem
  int prob;  // problem index over all (batch, head)
  int base;  // first token of the problem
  int j0;    // packed geometry: position of its first problem along the packed digit
};

// TMA coordinates (a, b, c, token) of the box of job J whose tile origin is (b0, c0). For
// a packed geometry the packed dimension starts at j0, so that the tensor map's bound on
// that dimension (the digit's extent) zero-fills the rows of a short last group.
__device__ __forceinline__ void box_coords(const Geom& g, const Job& J, int b0, int c0, int& ca, int& cb, int& cc,
                                           int& ct) {
  ca = g.pk_dim == 0 ? J.j0 : 0;
  cb = b0 + (g.pk_dim == 1 ? J.j0 : 0);
  cc = c0 + (g.pk_dim == 2 ? J.j0 : 0);
  ct = J.base - J.j0 * g.pk_stride;
}

__device__ __forceinline__ Job job_of(const FwdArgs& a, const Item& it, int which) {
  const PassArgs& p = a.ps[it.pass];
  const int j = 2 * it.pair + which;
  Job jb;
  jb.valid = j < p.jobs_per_bh;
  const int pl = fdiv(j, p.g.f_nt);
  jb.qt = j - pl * p.g.nt;
  jb.prob = it.bh * p.g.probs + pl;
  jb.j0 = 0;
  jb.base = jb.valid ? problem_base(p.g, jb.prob, &jb.j0) : 0;
  return jb;
}

__device__ __forceinline__ bool wait_count_shared(const uint32_t* c, uint32_t target, volatile int* abort,
                                                  uint64_t timeout_ns) {
  if (ld_acquire_cta_shared(c) >= target) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (ld_acquire_cta_shared(c) >= target) return true;
    __nanosleep(32);
    if ((it & 15u) == 0) {
      if (*abort) return false;
      if (global_timer_ns() - t0 > timeout_ns) {
        *abort = 1;
        return false;
      }
    }
  }
}

__device__ __forceinline__ bool wait_counter(const uint32_t* c, uint32_t target, volatile int* abort,
                                             uint64_t timeout_ns) {
  if (ld_acquire_gpu(c) >= target) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (ld_acquire_gpu(c) >= target) return true;
    __nanosleep(64);
    if ((it & 15u) == 0) {
      if (*abort) return false;
      if (global_timer_ns() - t0 > timeout_ns) {
        *abort = 1;
        return false;
      }
    }
  }
}

// PACKED: the geometry may pack several problems to a box (a per-row key mask then
// applies); the two-pass operator never packs, and its kernel is smaller without it.
template <int D, bool PACKED>
__global__ void __launch_bounds__(kFwdThreads, 1)
    squad_fwd_tc_kernel(const __grid_constant__ FwdMaps maps, const __grid_constant__ FwdArgs args) {
  using Lay = FwdLayout<D>;
  constexpr int DH = D / 64;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::BAR_OFF);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + Lay::BAR_OFF + Lay::NBAR * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::BAR_OFF + Lay::NBAR * 8 + 4);
  // per warpgroup: threads that finished writing their rows of local-pass jobs (monotonic)
  uint32_t* rows_done = reinterpret_cast<uint32_t*>(smem + Lay::BAR_OFF + Lay::NBAR * 8 + 8);
  // tensor map of (pass, role), role: 0 Q, 1 K, 2 values
  auto map_of = [&](int pass, int role) -> const CUtensorMap* { return &maps.m[pass * 4 + role]; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t to = args.timeout_ns;

  // Rows past a TMA box are never written and must stay finite (values are multiplied by P = 0).
  {
    uint4* z = reinterpret_cast<uint4*>(smem);
    for (int i = threadIdx.x; i < Lay::BAR_OFF / 16; i += kFwdThreads) z[i] = make_uint4(0, 0, 0, 0);
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < Lay::NKV; ++i) {
      mbar_init(&bars[F_KVF + i], 1);
      mbar_init(&bars[F_KVE + i], 2);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars[F_QF + i], 1);
      mbar_init(&bars[F_QE + i], 1);
      mbar_init(&bars[F_SF + i], 1);
      mbar_init(&bars[F_PF + i], 128);
      mbar_init(&bars[F_OF + i], 1);
      mbar_init(&bars[F_PF2 + i], 128);
    }
    mbar_init(&bars[F_DRAIN], 1);
    mbar_init(&bars[F_DRAIN + 1], 1);
    *abort_flag = 0;
    rows_done[0] = 0;
    rows_done[1] = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_holder, Lay::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0)
    for (int i = 0; i < 4 * args.npass; ++i) prefetch_tmap(map_of(i >> 2, i & 3));
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t sbase = smem_u32(smem);
  const bool fused = args.mode == FWD_FUSED;
  // passes chained in one launch: pass j of a head reads the output of its pass j - 1
  const bool chained = fused || args.mode == FWD_MULTI;
  const int last_pass = args.npass - 1;
  // 384 threads at up to 168 registers each (the launch bound); no register reallocation

  if (warp == 8) {
    // ================================================================ TMA producer
    if (lane == 0) {
      uint32_t qc = 0, uc = 0;  // Q boxes and key/value ring entries issued
      // L2 policies when passes are chained: Q and K are read again by the next pass (keep)
      // until the last pass; values are read once (drop first).
      const uint64_t pol_keep = make_policy_evict_last(), pol_drop = make_policy_evict_first();
      const uint64_t pol_norm = make_policy_evict_normal();
      bool ok = true;
      for (int i = blockIdx.x; ok && i < args.total_items; i += gridDim.x) {
        const Item it = decode_item(args, i);
        const Geom& g = args.ps[it.pass].g;
        const CUtensorMap* mq = map_of(it.pass, 0);
        const CUtensorMap* mk = map_of(it.pass, 1);
        const CUtensorMap* mv = map_of(it.pass, 2);
        const Job J[2] = {job_of(args, it, 0), job_of(args, it, 1)};
        const bool shared = J[1].valid && J[1].prob == J[0].prob;
        const uint32_t tx = uint32_t(g.box_rows) * D * 2;
        bool dep_done = !(chained && it.pass > 0);
        const uint64_t pol_qk = !chained ? pol_norm : it.pass < last_pass ? pol_keep : pol_drop;
        const uint64_t pol_v = !chained ? pol_norm : pol_drop;
        for (int k = 0; ok && k < g.nt; ++k) {
          for (int x = 0; ok && x < 2; ++x) {
            if (!J[x].valid) continue;
            int b0, c0;
            if (k == 0) {
              const uint32_t s = qc % 2;
              if (!(ok = mbar_wait(&bars[F_QE + s], ((qc / 2) & 1) ^ 1, abort_flag, to))) break;
              tile_origin(g, J[x].qt, b0, c0);
              int ca, cb, cc, ct;
              box_coords(g, J[x], b0, c0, ca, cb, cc, ct);
              mbar_arrive_expect_tx(&bars[F_QF + s], tx);
              for (int dh = 0; dh < DH; ++dh)
                tma_load_5d_hint(smem + Lay::Q_OFF + s * Lay::TILE + dh * kBlk, mq, &bars[F_QF + s], dh * 64, ca, cb,
                                 cc, ct, pol_qk);
              ++qc;
            }
            if (x == 1 && shared) continue;
            tile_origin(g, k, b0, c0);
            int ca, cb, cc, ct;
            box_coords(g, J[x], b0, c0, ca, cb, cc, ct);
            {
              const uint32_t s = uc % Lay::NKV;
              if (!(ok = mbar_wait(&bars[F_KVE + s], ((uc / Lay::NKV) & 1) ^ 1, abort_flag, to))) break;
              mbar_arrive_expect_tx(&bars[F_KVF + s], tx);
              for (int dh = 0; dh < DH; ++dh)
                tma_load_5d_hint(smem + Lay::KV_OFF + s * Lay::TILE + dh * kBlk, mk, &bars[F_KVF + s], dh * 64, ca, cb,
                                 cc, ct, pol_qk);
              ++uc;
            }
            if (!dep_done) {
              // pass j of a head reads the output of its pass j - 1 only once that is complete
              const uint32_t target = uint32_t(args.ps[it.pass - 1].jobs_per_bh);
              if (!(ok = wait_counter(args.counters + (it.pass - 1) * args.bh + it.bh, target, abort_flag, to)))
                break;
              fence_async_global();
              dep_done = true;
            }
            {
              const uint32_t s = uc % Lay::NKV;
              if (!(ok = mbar_wait(&bars[F_KVE + s], ((uc / Lay::NKV) & 1) ^ 1, abort_flag, to))) break;
              mbar_arrive_expect_tx(&bars[F_KVF + s], tx);
              for (int dh = 0; dh < DH; ++dh)
                tma_load_5d_hint(smem + Lay::KV_OFF + s * Lay::TILE + dh * kBlk, mv, &bars[F_KVF + s], dh * 64, ca, cb,
                                 cc, ct, pol_v);
              ++uc;
            }
          }
        }
      }
      // let every issued load land before the CTA may exit
      for (uint32_t s = 0; s < 2; ++s) {
        const uint32_t uses = qc > s ? (qc - s + 1) / 2 : 0;
        if (uses) mbar_wait_drain(&bars[F_QF + s], (uses - 1) & 1, to);
      }
      for (uint32_t s = 0; s < uint32_t(Lay::NKV); ++s) {
        const uint32_t uses = uc > s ? (uc - s + Lay::NKV - 1) / Lay::NKV : 0;
        if (uses) mbar_wait_drain(&bars[F_KVF + s], (uses - 1) & 1, to);
      }
    }
  } else if (warp == 9 || warp == 11) {
    if (lane == 0) {
    // ================================================================ MMA issuers
    // One thread per softmax warpgroup (warp 9 serves jobs A, warp 11 jobs B), so each
    // warpgroup's products are issued as soon as its own operands are ready and the two
    // warpgroups settle into alternation: one computes its softmax while the tensor core
    // runs the other's products. Key/value boxes are released after both users (the
    // "empty" barriers count two arrivals; a box used by one job arrives twice).
    const int x = warp == 9 ? 0 : 1;
    const uint32_t id_s = idesc_bf16_f32(128, 128, 0, 0);
    const uint32_t id_o = idesc_bf16_f32(128, D, 0, 1);
    uint32_t ebase = 0, qbase = 0, pc = 0;
    bool ok = true;
    for (int i = blockIdx.x; ok && i < args.total_items; i += gridDim.x) {
      const Item it = decode_item(args, i);
      const int nk = args.ps[it.pass].g.nt;
      const Job J0 = job_of(args, it, 0), J1 = job_of(args, it, 1);
      const bool shared = J1.valid && J1.prob == J0.prob;
      const uint32_t nvalid = uint32_t(J0.valid) + uint32_t(J1.valid);
      const uint32_t nentries = shared ? uint32_t(nk) : uint32_t(nk) * nvalid;
      if (x == 1 && !J1.valid) {
        ebase += nentries;
        qbase += nvalid;
        continue;
      }
      const uint32_t q = qbase + uint32_t(x);
      for (int k = 0; ok && k < nk; ++k) {
        // key/value entry of this job's key box k; K and V of an entry are consecutive ring slots
        const uint32_t e = ebase + (shared ? uint32_t(k) : uint32_t(k) * nvalid + uint32_t(x));
        const uint32_t uk = 2 * e, uv = 2 * e + 1;
        const uint32_t ks = uk % Lay::NKV, vs = uv % Lay::NKV;
        if (!(ok = mbar_wait(&bars[F_KVF + ks], (uk / Lay::NKV) & 1, abort_flag, to))) break;
        if (k == 0 && !(ok = mbar_wait(&bars[F_QF + q % 2], (q / 2) & 1, abort_flag, to))) break;
        // S overwrites the columns that the previous P.V of this warpgroup reads P from. No
        // wait: the tensor core runs the MMAs that one thread issues in issue order, so the
        // P.V has read its A operand before this S writes there.
        tc_fence_after();
        const uint32_t qa = sbase + Lay::Q_OFF + (q % 2) * Lay::TILE;
        const uint32_t ka = sbase + Lay::KV_OFF + ks * Lay::TILE;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * kBlk + (kk & 3) * 32;
          mma_ss(tmem + x * 256, sdesc_sw128(qa + koff, 16, 1024), sdesc_sw128(ka + koff, 16, 1024), id_s,
                 kk > 0 ? 1u : 0u);
        }
        tc_commit(&bars[F_SF + x]);
        if (k == nk - 1) tc_commit(&bars[F_QE + q % 2]);  // the job's Q box is no longer needed
        tc_commit(&bars[F_KVE + ks]);
        if (!shared) tc_commit(&bars[F_KVE + ks]);
        if (!(ok = mbar_wait(&bars[F_PF + x], pc & 1, abort_flag, to))) break;
        if (!(ok = mbar_wait(&bars[F_KVF + vs], (uv / Lay::NKV) & 1, abort_flag, to))) break;
        tc_fence_after();
        const uint32_t va = sbase + Lay::KV_OFF + vs * Lay::TILE;
        // keys 0-63 as soon as their P is in TMEM, keys 64-127 once the rest is
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ts(tmem + x * 256 + 128, tmem + x * 256 + kk * 8, sdesc_sw128(va + kk * 16 * 128, kBlk, 1024), id_o,
                 (k > 0 || kk > 0) ? 1u : 0u);
        if (!(ok = mbar_wait(&bars[F_PF2 + x], pc & 1, abort_flag, to))) break;
        ++pc;
        tc_fence_after();
#pragma unroll
        for (int kk = 4; kk < 8; ++kk)
          mma_ts(tmem + x * 256 + 128, tmem + x * 256 + kk * 8, sdesc_sw128(va + kk * 16 * 128, kBlk, 1024), id_o, 1u);
        tc_commit(&bars[F_OF + x]);
        tc_commit(&bars[F_KVE + vs]);
        if (!shared) tc_commit(&bars[F_KVE + vs]);
      }
      ebase += nentries;
      qbase += nvalid;
    }
    tc_commit(&bars[F_DRAIN + x]);
    mbar_wait_drain(&bars[F_DRAIN + x], 0, to);
    }
  } else if (warp == 10) {
    // ================================================================ publisher (chained passes)
    // Once all rows of a job of a pass that is not the last are written (the warpgroup's
    // 128 threads each add one to rows_done after their stores), make them visible at GPU
    // scope and count the job for its (pass, head); the next pass of that head starts when
    // its count is complete. Done here so the softmax warpgroups never wait for the fence.
    if (chained && lane == 0) {
      uint32_t pub[2] = {0, 0};
      bool ok = true;
      for (int i = blockIdx.x; ok && i < args.total_items; i += gridDim.x) {
        const Item it = decode_item(args, i);
        if (it.pass == last_pass) continue;
        for (int x = 0; ok && x < 2; ++x) {
          if (!job_valid(args, it, x)) continue;
          ++pub[x];
          if (!(ok = wait_count_shared(&rows_done[x], 128u * pub[x], abort_flag, to))) break;
          fence_acq_rel_gpu();
          red_release_gpu_add(args.counters + it.pass * args.bh + it.bh, 1u);
        }
      }
    }
  } else {
    // ================================================================ softmax warpgroups
    const int a = warp >> 2;  // warpgroup: job A (0) or job B (1) of each pair
    const int row = threadIdx.x & 127;
    const uint32_t tS = tmem + (uint32_t((warp & 3) * 32) << 16) + a * 256;
    const uint32_t tO = tS + 128;
    const float c2 = args.scale_log2;
    uint32_t sc = 0, pvseen = 0;
    bool ok = true;
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, to)) != 0;
    };
    // The next job of this warpgroup and this thread's output row in it, found while the
    // tensor core runs the current job's last P.V (the index arithmetic has divisions).
    struct SJob {
      int i;     // item index (>= total_items: none left)
      int pass;  // 0 local, 1 global
      int qt;    // query box within the problem
      int base;  // first token of the problem
      int tok;   // this thread's output row, or -1 past the box's valid rows
    };
    auto find_job = [&](int i) -> SJob {
      for (; i < args.total_items; i += gridDim.x) {
        const Item it = decode_item(args, i);
        const Job J = job_of(args, it, a);
        if (!J.valid) continue;
        const Geom& g = args.ps[it.pass].g;
        int tok = row < tile_valid_rows(g, J.qt) ? J.base + tile_row_offset(g, J.qt, row) : -1;
        // packed geometry: a row past the packed digit's extent is a zero-filled row
        if (PACKED && g.pk > 1 && J.j0 + pack_id(g, row) >= g.pk_ext) tok = -1;
        return SJob{i, it.pass, J.qt, J.base, tok};
      }
      return SJob{args.total_items, 0, 0, 0, -1};
    };
    SJob cur = find_job(blockIdx.x);
    while (ok && cur.i < args.total_items) {
      const PassArgs& P = args.ps[cur.pass];
      const Geom& g = P.g;
      float m_run = -INFINITY, l_run = 0.f, lr_run = 0.f;
      for (int k = 0; k < g.nt; ++k) {
        if (!(ok = wwait(&bars[F_SF + a], sc & 1))) break;
        ++sc;
        tc_fence_after();
        uint32_t r[128];
        tmem_ld128(tS, r);
        // key columns past the problem (a suffix of the box) -> -inf; only the ragged 32-column chunk is tested
        const int lim = tile_valid_rows(g, k);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (lim < 32 * (j + 1)) {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (32 * j + e >= lim) r[32 * j + e] = 0xff800000u;
          }
        }
        // packed boxes: the 32-key chunks that hold a key of any row of this warp; the
        // exponentials of the other chunks are skipped (their P is zero)
        uint32_t wlive = 0xfu;
        if (PACKED && g.pk > 1) {
          // packed problems: keys of other problems in the box -> -inf. This row's problem
          // holds runs of pk_rowdiv columns, one run every pk * pk_rowdiv columns.
          const int R = g.pk_rowdiv;
          uint64_t mlo = 0ull, mhi = 0ull;
          for (int s0 = pack_id(g, row) * R; s0 < 128; s0 += g.pk * R) {
            const int e = s0 + R < 128 ? s0 + R : 128;
            if (s0 < 64) {
              const int e0 = e < 64 ? e : 64;
              mlo |= (e0 - s0 >= 64 ? ~0ull : ((1ull << (e0 - s0)) - 1ull)) << s0;
            }
            if (e > 64) {
              const int s1 = s0 > 64 ? s0 - 64 : 0, e1 = e - 64;
              mhi |= (e1 - s1 >= 64 ? ~0ull : ((1ull << (e1 - s1)) - 1ull)) << s1;
            }
          }
#pragma unroll
          for (int e = 0; e < 128; ++e)
            if (!(((e < 64 ? mlo : mhi) >> (e & 63)) & 1ull)) r[e] = 0xff800000u;
          const uint32_t mine = (uint32_t(mlo) != 0u ? 1u : 0u) | (uint32_t(mlo >> 32) != 0u ? 2u : 0u) |
                                (uint32_t(mhi) != 0u ? 4u : 0u) | (uint32_t(mhi >> 32) != 0u ? 8u : 0u);
          wlive = __reduce_or_sync(0xffffffffu, mine);
        }
        // row maximum: 8 independent partial maxima of three-input max
        float mp[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) mp[j] = fmaxf(__uint_as_float(r[j]), __uint_as_float(r[j + 8]));
#pragma unroll
        for (int e = 16; e < 128; e += 16)
#pragma unroll
          for (int j = 0; j < 8; ++j) mp[j] = fmax3(mp[j], __uint_as_float(r[e + j]), __uint_as_float(r[e + j + 8]));
        const float mx = fmax3(fmax3(mp[0], mp[1], mp[2]), fmax3(mp[3], mp[4], mp[5]), fmaxf(mp[6], mp[7]));
        // exact running maximum: the largest P of a row is exactly 1 before its bf16
        // rounding, which keeps the dominant term of peaked rows exact
        // the first key box sets the maximum; a later one moves it only when it grows by more
        // than 2^8 (then O and the sums are rescaled), else its probabilities may exceed 1
        float m_use = mx, alpha = 1.f;
        bool grow = false;
        if (k > 0) {
          grow = (mx - m_run) * c2 > 8.f;
          m_use = grow ? mx : m_run;
          alpha = grow ? ex2_approx((m_run - mx) * c2) : 1.f;
        }
        const float neg = -m_use * c2;
        const uint64_t c2x2 = f2(c2, c2), negx2 = f2(neg, neg);
        uint64_t sl[2] = {0ull, 0ull};  // paired partial sums of p
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {  // two 64-column halves: P of a half is packed and stored at once
          if (!PACKED) {
            uint32_t pk[32];
#pragma unroll
            for (int e = 0; e < 64; e += 2) {
              const uint64_t x2 = ffma2(f2(__uint_as_float(r[64 * hh + e]), __uint_as_float(r[64 * hh + e + 1])),
                                        c2x2, negx2);
              const float p0 = ex2_approx(f2_lo(x2));
              const float p1 = ex2_approx(f2_hi(x2));
              sl[(e >> 1) & 1] = fadd2(sl[(e >> 1) & 1], f2(p0, p1));
              pk[e >> 1] = pack_bf16x2(p0, p1);
            }
            tmem_st32(tS + hh * 32, pk);
          } else {
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
              if ((wlive >> (2 * hh + ch)) & 1u) {
                uint32_t pk[16];
#pragma unroll
                for (int e = 32 * ch; e < 32 * ch + 32; e += 2) {
                  const uint64_t x2 = ffma2(f2(__uint_as_float(r[64 * hh + e]), __uint_as_float(r[64 * hh + e + 1])),
                                            c2x2, negx2);
                  const float p0 = ex2_approx(f2_lo(x2));
                  const float p1 = ex2_approx(f2_hi(x2));
                  sl[(e >> 1) & 1] = fadd2(sl[(e >> 1) & 1], f2(p0, p1));
                  pk[(e >> 1) - 16 * ch] = pack_bf16x2(p0, p1);
                }
                tmem_st16(tS + hh * 32 + ch * 16, pk);
              } else {
                tmem_st16_zero(tS + hh * 32 + ch * 16);
              }
            }
          }
          if (hh == 0) {
            // O is rescaled before the first P.V half accumulates into it; the previous P.V
            // has completed (S of this step was issued after it)
            if (__any_sync(0xffffffffu, grow)) {
#pragma unroll
              for (int h = 0; h < 2; ++h) {  // two 64-column halves keep register pressure down
                uint32_t o[64];
                tmem_ld64(tO + h * 64, o);
#pragma unroll
                for (int e = 0; e < 64; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                tmem_st64(tO + h * 64, o);
              }
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&bars[F_PF + a]);
          }
        }
        const uint64_t s2 = fadd2(sl[0], sl[1]);
        const float sum = f2_lo(s2) + f2_hi(s2);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bars[F_PF2 + a]);
        // the box's largest probability enters the normalising sum rounded to bf16, as the
        // tensor core sees it, so that a row dominated by one key returns its value exactly
        const float pmax = ex2_approx(fmaf(mx, c2, neg));
        const float pmax_bf = __uint_as_float(pack_bf16x2(0.f, pmax) & 0xffff0000u);
        l_run = l_run * alpha + sum;
        lr_run = lr_run * alpha + (pmax_bf - pmax);
        m_run = m_use;
      }
      if (!ok) break;
      const SJob nxt = find_job(cur.i + gridDim.x);
      // ---- epilogue: O / l -> bf16, each thread writes its own output row (16-byte stores)
      pvseen += g.nt;
      if (!(ok = wwait(&bars[F_OF + a], (pvseen - 1) & 1))) break;
      tc_fence_after();
      const bool live = cur.tok >= 0;
      const size_t tok = live ? size_t(cur.tok) : 0;
      {
        // Each thread holds its own row. A warp passes its 32 rows through a private
        // 128B-swizzled patch so that every global store writes four whole 128-byte lines.
        const float inv = 1.f / (l_run + lr_run);
        const uint64_t inv2 = f2(inv, inv);
        auto scale_pack = [&](uint32_t a0, uint32_t a1) -> uint32_t {
          uint64_t m;
          asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(m) : "l"(f2(__uint_as_float(a0), __uint_as_float(a1))), "l"(inv2));
          return pack_bf16x2(f2_lo(m), f2_hi(m));
        };
        const uint32_t xp = sbase + Lay::XP_OFF + (warp & 7) * 4096;
        const int lr = lane >> 3, lc = lane & 7;  // read-back: row 4*i + lr, 16-byte chunk lc
        int rtok[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) rtok[i] = __shfl_sync(0xffffffffu, cur.tok, 4 * i + lr);
        // chained passes: an output read by the next pass is kept in L2, the last pass's dropped first
        const uint64_t pol_out = !chained ? make_policy_evict_normal()
                                 : cur.pass < last_pass ? make_policy_evict_last() : make_policy_evict_first();
        uint8_t* outb = static_cast<uint8_t*>(P.out);
#pragma unroll 1
        for (int h = 0; h < D / 64; ++h) {
          uint32_t o[64];
          tmem_ld64(tO + h * 64, o);
#pragma unroll
          for (int c = 0; c < 8; ++c)
            st_shared_v4(xp + lane * 128 + ((c ^ (lane & 7)) << 4), scale_pack(o[8 * c + 0], o[8 * c + 1]),
                         scale_pack(o[8 * c + 2], o[8 * c + 3]), scale_pack(o[8 * c + 4], o[8 * c + 5]),
                         scale_pack(o[8 * c + 6], o[8 * c + 7]));
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int r = 4 * i + lr;  // row of this warp (lane r owns it)
            const uint4 val = ld_shared_v4(xp + r * 128 + ((lc ^ (r & 7)) << 4));
            if (rtok[i] >= 0) st_global_v4_hint(outb + size_t(rtok[i]) * D * 2 + h * 128 + lc * 16, val, pol_out);
          }
          __syncwarp();
        }
      }
      tc_fence_before();
      if (chained && cur.pass < last_pass) red_release_cta_shared_add(&rows_done[a], 1u);  // warp 10 publishes
      if (live && P.discard != nullptr && g.nt == 1) {
        // this row of the previous pass's output was read once, as a value of this group: drop it
        const uint8_t* l1row = P.discard + tok * D * 2;
#pragma unroll
        for (int l = 0; l < D * 2 / 128; ++l) discard_l2_line(l1row + l * 128);
      }
      if (P.lse != nullptr && live)
        P.lse[tok] = (m_run * c2 + log2f(l_run)) * 0.69314718055994530942f;
      cur = nxt;
    }
  }

  __syncthreads();
  if (*abort_flag && threadIdx.x == 0 && args.err != nullptr) atomicCAS(args.err, 0, 1);
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, Lay::TMEM_COLS);
  }
}

}  // namespace sq
