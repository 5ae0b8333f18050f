// squad_fwd_tc.cuh - forward of one SQuad-Attention pass on the sm_100a tensor cores.
//
// One kernel serves both passes of the operator ("SQuad: Sub-Quadratic Attention
// Distillation for Efficient Video Generation", gist.science technical summary,
// Methodology section 1): the local pass (problems = windows, values = V, output
// O1) and the global pass (problems = same-position groups across windows,
// values = O1, output O). Only the tensor maps and the Geom differ.
//
// Design (B200):
//   * Persistent CTAs, one per SM, loop over problems.
//   * Warp-specialised: warp 4 issues TMA loads, warp 5 issues tcgen05.mma from
//     one thread, warps 0-3 (128 threads, thread = TMEM lane = query row) run
//     the softmax and the epilogue.
//   * Every operand tile is a 5-D TMA box (d-block, a, b, c, token) cut from the
//     problem box, so the strided gather of the global pass needs no permute:
//     the box's strides walk across windows. Rows outside the problem are
//     zero-filled by TMA on load and clipped on store.
//   * S = Q K^T accumulates in TMEM (fp32, up to 256 key columns = two key
//     tiles per group). The softmax reads S with tcgen05.ld, writes P as bf16
//     back into the same TMEM columns, and O += P V runs with A = P read from
//     TMEM (no shared-memory round trip for P). Problems with more than two
//     key tiles run an online softmax across groups, rescaling O in TMEM.
//   * The epilogue normalises O, packs bf16 into a 128B-swizzled staging tile
//     and stores it with one TMA store per 64-column block; LSE is written
//     per row.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>
#include "geometry.h"
#include "sm100.cuh"

namespace sq {

struct FwdArgs {
  Geom g;
  int total_probs;      // g.bh * g.probs
  float scale_log2;     // softmax scale * log2(e)
  float* lse;           // [bh*n] natural-log LSE, or nullptr
  int* err;             // device error word
  uint64_t timeout_ns;  // bound for every wait
};

constexpr int kFwdThreads = 192;
constexpr int kTileRowsBytes = 128 * 128;  // one 64-column block of a 128-row tile (bf16)

template <int D, int KT>
struct FwdLayout {
  static constexpr int DH = D / 64;                  // 64-column blocks per row
  static constexpr int TILE = 128 * D * 2;           // bytes of one 128-row tile
  static constexpr int Q_OFF = 0;                    // two Q tiles (double buffer)
  static constexpr int K_OFF = Q_OFF + 2 * TILE;     // KT key tiles: [dh][KT*128 rows][128 B]
  static constexpr int V_OFF = K_OFF + KT * TILE;    // KT value tiles, same layout
  static constexpr int O_OFF = V_OFF + KT * TILE;    // output staging tile
  static constexpr int BAR_OFF = O_OFF + TILE;
  static constexpr int NBAR = 14;  // 13 used
  static constexpr int BYTES = BAR_OFF + NBAR * 8 + 16;
  static constexpr int ALLOC = BYTES + 1024;          // alignment slack
  static constexpr int TMEM_S = 0;                    // S / P columns
  static constexpr int TMEM_O = 128 * KT;             // O accumulator columns
  static constexpr int TMEM_COLS = (128 * KT + D) <= 256 ? 256 : 512;
};

enum { B_QFULL0 = 0, B_QFULL1, B_QEMPTY0, B_QEMPTY1, B_KFULL, B_KEMPTY, B_VFULL, B_VEMPTY, B_SFULL, B_PFULL, B_OFULL,
       B_DRAIN, B_EPI };

__device__ __forceinline__ void flag_error(int* err, int code) {
  if (err != nullptr) atomicCAS(err, 0, code);
}

template <int D, int KT>
__global__ void __launch_bounds__(kFwdThreads, 1)
    squad_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                        const FwdArgs args) {
  using Lay = FwdLayout<D, KT>;
  constexpr int DH = Lay::DH;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::BAR_OFF);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + Lay::BAR_OFF + Lay::NBAR * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::BAR_OFF + Lay::NBAR * 8 + 4);

  const Geom& g = args.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nt = g.nt;
  const int ng = ceil_div(nt, KT);
  const bool kv_resident = (ng == 1);  // key/value tiles loaded once per problem
  const uint64_t to = args.timeout_ns;

  // Zero every operand buffer once: rows past the TMA box are never written and
  // must stay finite (value rows are multiplied by P = 0).
  {
    uint4* z = reinterpret_cast<uint4*>(smem);
    for (int i = threadIdx.x; i < Lay::BAR_OFF / 16; i += kFwdThreads) z[i] = make_uint4(0, 0, 0, 0);
  }
  if (threadIdx.x == 0) {
    mbar_init(&bars[B_QFULL0], 1);
    mbar_init(&bars[B_QFULL1], 1);
    mbar_init(&bars[B_QEMPTY0], 1);
    mbar_init(&bars[B_QEMPTY1], 1);
    mbar_init(&bars[B_KFULL], 1);
    mbar_init(&bars[B_KEMPTY], 1);
    mbar_init(&bars[B_VFULL], 1);
    mbar_init(&bars[B_VEMPTY], 1);
    mbar_init(&bars[B_SFULL], 1);
    mbar_init(&bars[B_PFULL], 128);
    mbar_init(&bars[B_OFULL], 1);
    mbar_init(&bars[B_DRAIN], 1);
    mbar_init(&bars[B_EPI], 128);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_holder, Lay::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_o);
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t sbase = smem_u32(smem);

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t q_iter = 0, kv_iter = 0;
      const uint32_t tile_tx = uint32_t(g.box_rows) * D * 2;
      bool ok = true;
      for (int prob = blockIdx.x; ok && prob < args.total_probs; prob += gridDim.x) {
        const int base = problem_base(g, prob);
        for (int qt = 0; ok && qt < nt; ++qt) {
          const int b = q_iter & 1;
          ok = mbar_wait(&bars[B_QEMPTY0 + b], ((q_iter >> 1) & 1) ^ 1, abort_flag, to);
          if (!ok) break;
          int b0, c0;
          tile_origin(g, qt, b0, c0);
          mbar_arrive_expect_tx(&bars[B_QFULL0 + b], tile_tx);
#pragma unroll
          for (int dh = 0; dh < DH; ++dh)
            tma_load_5d(smem + Lay::Q_OFF + b * Lay::TILE + dh * kTileRowsBytes, &tm_q, &bars[B_QFULL0 + b],
                        dh * 64, 0, b0, c0, base);
          ++q_iter;
          if (kv_resident && qt > 0) continue;
          for (int grp = 0; ok && grp < ng; ++grp) {
            const int kt0 = grp * KT, nkt = min(KT, nt - kt0);
            ok = mbar_wait(&bars[B_KEMPTY], (kv_iter & 1) ^ 1, abort_flag, to);
            if (!ok) break;
            mbar_arrive_expect_tx(&bars[B_KFULL], tile_tx * nkt);
            for (int j = 0; j < nkt; ++j) {
              tile_origin(g, kt0 + j, b0, c0);
#pragma unroll
              for (int dh = 0; dh < DH; ++dh)
                tma_load_5d(smem + Lay::K_OFF + dh * KT * kTileRowsBytes + j * kTileRowsBytes, &tm_k,
                            &bars[B_KFULL], dh * 64, 0, b0, c0, base);
            }
            ok = mbar_wait(&bars[B_VEMPTY], (kv_iter & 1) ^ 1, abort_flag, to);
            if (!ok) break;
            mbar_arrive_expect_tx(&bars[B_VFULL], tile_tx * nkt);
            for (int j = 0; j < nkt; ++j) {
              tile_origin(g, kt0 + j, b0, c0);
#pragma unroll
              for (int dh = 0; dh < DH; ++dh)
                tma_load_5d(smem + Lay::V_OFF + dh * KT * kTileRowsBytes + j * kTileRowsBytes, &tm_v,
                            &bars[B_VFULL], dh * 64, 0, b0, c0, base);
            }
            ++kv_iter;
          }
        }
      }
      // Let every load issued land before the CTA can exit.
      for (int b = 0; b < 2; ++b) {
        const uint32_t uses = q_iter > uint32_t(b) ? (q_iter - b + 1) / 2 : 0;
        if (uses) mbar_wait_drain(&bars[B_QFULL0 + b], (uses - 1) & 1, to);
      }
      if (kv_iter) {
        mbar_wait_drain(&bars[B_KFULL], (kv_iter - 1) & 1, to);
        mbar_wait_drain(&bars[B_VFULL], (kv_iter - 1) & 1, to);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t q_iter = 0, kv_iter = 0, pv_count = 0, p_iter = 0;
      const uint32_t id_o = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t tS = tmem + Lay::TMEM_S, tO = tmem + Lay::TMEM_O;
      bool ok = true;
      for (int prob = blockIdx.x; ok && prob < args.total_probs; prob += gridDim.x) {
        for (int qt = 0; ok && qt < nt; ++qt) {
          const int b = q_iter & 1;
          ok = mbar_wait(&bars[B_QFULL0 + b], (q_iter >> 1) & 1, abort_flag, to);
          if (!ok) break;
          const uint32_t qaddr = sbase + Lay::Q_OFF + b * Lay::TILE;
          for (int grp = 0; grp < ng; ++grp) {
            const int kt0 = grp * KT, nkt = min(KT, nt - kt0);
            const bool fresh = !(kv_resident && qt > 0);
            const bool last_use = !kv_resident || qt == nt - 1;
            if (fresh) {
              ok = mbar_wait(&bars[B_KFULL], kv_iter & 1, abort_flag, to);
              if (!ok) break;
            }
            // the previous P.V must have finished reading P before S is overwritten
            if (pv_count > 0) {
              ok = mbar_wait(&bars[B_OFULL], (pv_count - 1) & 1, abort_flag, to);
              if (!ok) break;
            }
            tc_fence_after();
            const uint32_t id_s = idesc_bf16_f32(128, 128 * nkt, 0, 0);
            const uint32_t kaddr = sbase + Lay::K_OFF;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t koff = (kk >> 2) * kTileRowsBytes + (kk & 3) * 32;
              const uint64_t ad = sdesc_sw128(qaddr + koff, 16, 1024);
              const uint64_t bd = sdesc_sw128(kaddr + (kk >> 2) * KT * kTileRowsBytes + (kk & 3) * 32, 16, 1024);
              mma_ss(tS, ad, bd, id_s, kk > 0 ? 1u : 0u);
            }
            tc_commit(&bars[B_SFULL]);
            if (grp == ng - 1) tc_commit(&bars[B_QEMPTY0 + b]);
            if (last_use) tc_commit(&bars[B_KEMPTY]);
            ok = mbar_wait(&bars[B_PFULL], p_iter & 1, abort_flag, to);
            if (!ok) break;
            ++p_iter;
            if (fresh) {
              ok = mbar_wait(&bars[B_VFULL], kv_iter & 1, abort_flag, to);
              if (!ok) break;
            }
            tc_fence_after();
            const uint32_t vaddr = sbase + Lay::V_OFF;
            for (int j = 0; j < nkt; ++j) {
#pragma unroll
              for (int kk = 0; kk < 8; ++kk) {
                const uint64_t bd = sdesc_sw128(vaddr + (j * 128 + kk * 16) * 128, KT * kTileRowsBytes, 1024);
                mma_ts(tO, tS + j * 64 + kk * 8, bd, id_o, (grp > 0 || j > 0 || kk > 0) ? 1u : 0u);
              }
            }
            tc_commit(&bars[B_OFULL]);
            ++pv_count;
            if (last_use) tc_commit(&bars[B_VEMPTY]);
            if (fresh) ++kv_iter;
          }
          ++q_iter;
        }
      }
      // all issued tensor-core work must finish before TMEM is released
      tc_commit(&bars[B_DRAIN]);
      mbar_wait_drain(&bars[B_DRAIN], 0, to);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue (warps 0-3)
    const int row = threadIdx.x;  // TMEM lane == query row of the tile
    const uint32_t lane_sel = uint32_t(warp * 32) << 16;
    const uint32_t tS = tmem + lane_sel + Lay::TMEM_S, tO = tmem + lane_sel + Lay::TMEM_O;
    const float c2 = args.scale_log2;
    uint32_t s_iter = 0, o_iter = 0, epi_iter = 0;
    bool ok = true;
    // warp-uniform bounded wait: tcgen05.ld/st are warp-collective, so all lanes
    // must take the same branch after a wait
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, to)) != 0;
    };
    // bounded rendezvous of the 128 softmax threads (an mbarrier, so it can time out)
    auto epi_sync = [&]() -> bool {
      mbar_arrive(&bars[B_EPI]);
      const bool r = wwait(&bars[B_EPI], epi_iter & 1);
      ++epi_iter;
      return r;
    };
    for (int prob = blockIdx.x; ok && prob < args.total_probs; prob += gridDim.x) {
      const int base = problem_base(g, prob);
      for (int qt = 0; ok && qt < nt; ++qt) {
        float m_run = -INFINITY, l_run = 0.f;
        for (int grp = 0; grp < ng; ++grp) {
          const int kt0 = grp * KT, nkt = min(KT, nt - kt0);
          int vk[KT];
#pragma unroll
          for (int j = 0; j < KT; ++j) vk[j] = (j < nkt) ? tile_valid_rows(g, kt0 + j) : 0;
          ok = wwait(&bars[B_SFULL], s_iter & 1);
          if (!ok) break;
          ++s_iter;
          tc_fence_after();
          // pass 1: row maximum over valid key columns
          float mx = -INFINITY;
          for (int c = 0; c < nkt * 4; ++c) {
            uint32_t r[32];
            tmem_ld32(tS + c * 32, r);
            const int lim = vk[c >> 2] - (c & 3) * 32;
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (e < lim) mx = fmaxf(mx, __uint_as_float(r[e]));
          }
          const float m_new = fmaxf(m_run, mx);
          const float alpha = ex2_approx((m_run - m_new) * c2);
          const float neg = -m_new * c2;
          // pass 2: P = 2^(S*c2 - m*c2) as bf16 into the S columns already read
          float sum = 0.f;
          for (int c = 0; c < nkt * 4; ++c) {
            uint32_t r[32];
            tmem_ld32(tS + c * 32, r);
            const int lim = vk[c >> 2] - (c & 3) * 32;
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const float p0 = (e < lim) ? ex2_approx(fmaf(__uint_as_float(r[e]), c2, neg)) : 0.f;
              const float p1 = (e + 1 < lim) ? ex2_approx(fmaf(__uint_as_float(r[e + 1]), c2, neg)) : 0.f;
              sum += p0 + p1;
              pk[e >> 1] = pack_bf16x2(p0, p1);
            }
            tmem_st16(tS + c * 16, pk);
          }
          tmem_st_wait();
          if (grp > 0) {
            // rescale the running O (after the previous P.V has landed)
            ok = wwait(&bars[B_OFULL], o_iter & 1);
            if (!ok) break;
            ++o_iter;
            tc_fence_after();
            if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
              for (int c = 0; c < D / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(tO + c * 32, r);
#pragma unroll
                for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
                tmem_st32(tO + c * 32, r);
              }
              tmem_st_wait();
            }
          }
          tc_fence_before();
          mbar_arrive(&bars[B_PFULL]);
          l_run = l_run * alpha + sum;
          m_run = m_new;
        }
        if (!ok) break;
        // ---------------- epilogue: O / l -> bf16 -> staging -> TMA store
        ok = wwait(&bars[B_OFULL], o_iter & 1);
        if (!ok) break;
        ++o_iter;
        tc_fence_after();
        if (row == 0) bulk_wait_read0();  // previous store has finished reading the staging tile
        ok = epi_sync();
        if (!ok) break;
        const float inv = 1.f / l_run;
        const uint32_t obase = sbase + Lay::O_OFF;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tO + c * 32, r);
          const uint32_t blk = obase + (c >> 1) * kTileRowsBytes + row * 128;
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const int chunk = (c & 1) * 4 + q4;  // 16-byte chunk within the 128-byte row
            const uint32_t addr = blk + ((chunk ^ (row & 7)) << 4);
            st_shared_v4(addr,
                         pack_bf16x2(__uint_as_float(r[q4 * 8 + 0]) * inv, __uint_as_float(r[q4 * 8 + 1]) * inv),
                         pack_bf16x2(__uint_as_float(r[q4 * 8 + 2]) * inv, __uint_as_float(r[q4 * 8 + 3]) * inv),
                         pack_bf16x2(__uint_as_float(r[q4 * 8 + 4]) * inv, __uint_as_float(r[q4 * 8 + 5]) * inv),
                         pack_bf16x2(__uint_as_float(r[q4 * 8 + 6]) * inv, __uint_as_float(r[q4 * 8 + 7]) * inv));
          }
        }
        fence_async_smem();
        ok = epi_sync();
        if (!ok) break;
        int b0, c0;
        tile_origin(g, qt, b0, c0);
        if (row == 0) {
#pragma unroll
          for (int dh = 0; dh < DH; ++dh)
            tma_store_5d(&tm_o, smem + Lay::O_OFF + dh * kTileRowsBytes, dh * 64, 0, b0, c0, base);
          bulk_commit();
        }
        if (args.lse != nullptr && row < tile_valid_rows(g, qt)) {
          const float lse2 = m_run * c2 + log2f(l_run);
          args.lse[base + tile_row_offset(g, qt, row)] = lse2 * 0.69314718055994530942f;
        }
      }
    }
    if (row == 0) bulk_wait0();
  }

  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) flag_error(args.err, 1);
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, Lay::TMEM_COLS);
  }
}

}  // namespace sq
