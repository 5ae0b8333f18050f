// squad_bwd_tc.cuh - backward of one SQuad-Attention pass on the sm_100a tensor cores.
//
// The operator ("SQuad: Sub-Quadratic Attention Distillation for Efficient Video
// Generation", gist.science technical summary, Methodology section 1) is two
// softmax-attention passes; training through it (the fine-tuning of Methodology
// section 2) needs the textbook attention gradient of each pass:
//   P = exp(s*Q K^T - lse),  dP = dO Val^T,  D = rowsum(dO o O),  dS = P o (dP - D)
//   dVal = P^T dO,  dK = s * dS^T Q,  dQ = s * dS K.
// One template covers both kernels of a pass, without atomics:
//   MODE_DKDV: a CTA item is (problem, key tile). The key tile (K, Val) stays in
//     shared memory; the query tiles (Q, dO) stream through a double buffer.
//     S^T = K Q^T and dP^T = Val dO^T land in TMEM with lane = key row; the
//     softmax warps turn them into P^T and dS^T (bf16, written back into the
//     same TMEM columns), which are the A operands of dVal += P^T dO and
//     dK += dS^T Q read straight from TMEM.
//   MODE_DQ: a CTA item is (problem, query tile). Q and dO stay; key tiles
//     (K, Val) stream. S = Q K^T, dP = dO Val^T, dS in TMEM, dQ += dS K.
// TMEM columns: [0,128) S, [128,256) dP, [256,256+D) and [384,384+D) accumulators.
// Warp roles as in the forward: warps 0-3 softmax/epilogue (thread = TMEM lane),
// warp 4 TMA producer, warp 5 MMA issuer. Every wait is bounded.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>
#include "geometry.h"
#include "sm100.cuh"

namespace sq {

enum { MODE_DKDV = 0, MODE_DQ = 1 };

struct BwdArgs {
  Geom g;
  int total_items;        // problems * tiles
  float scale;            // softmax scale
  float scale_log2;       // scale * log2(e)
  const float* lse;       // [rows] natural-log LSE of this pass
  const float* Drow;      // [rows] rowsum(dO o O) of this pass
  const float* add;       // fp32 [rows, D] added to dK (DKDV) or dQ (DQ), or nullptr
  void* out_main;         // dK (DKDV) or dQ (DQ): fp32 if OUT_F32 else bf16
  __nv_bfloat16* out_val; // dVal (DKDV only), bf16
  int* err;
  uint64_t timeout_ns;
};

constexpr int kBwdThreads = 192;

template <int D>
struct BwdLayout {
  static constexpr int TILE = 128 * D * 2;
  static constexpr int FIX_OFF = 0;                // fixed pair: 2 tiles
  static constexpr int STR_OFF = 2 * TILE;         // streamed pairs: 2 buffers x 2 tiles
  static constexpr int VEC_OFF = STR_OFF + 4 * TILE;   // 2 buffers x (lse2[128] + D[128]) floats
  static constexpr int BAR_OFF = VEC_OFF + 2 * 2 * 128 * 4;
  static constexpr int NBAR = 12;
  static constexpr int BYTES = BAR_OFF + NBAR * 8 + 16;
  static constexpr int ALLOC = BYTES + 1024;
  static constexpr int TM_S = 0, TM_DP = 128, TM_A1 = 256, TM_A2 = 384;
  static constexpr int TMEM_COLS = 512;
};

enum { C_FIXFULL = 0, C_FIXEMPTY, C_STRFULL0, C_STRFULL1, C_STREMPTY0, C_STREMPTY1, C_SFULL, C_PFULL, C_ACC,
       C_DRAIN, C_VEC };

__device__ __forceinline__ void store_row_out(float* dst, const float* v, int n) {
  float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int i = 0; i < 8; ++i) d4[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
}

template <int D, int MODE, bool OUT_F32>
__global__ void __launch_bounds__(kBwdThreads, 1)
    squad_bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                        const BwdArgs args) {
  using Lay = BwdLayout<D>;
  constexpr int DH = D / 64;
  constexpr uint32_t BLK = 128 * 128;  // one 64-column block of a 128-row tile
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::BAR_OFF);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + Lay::BAR_OFF + Lay::NBAR * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::BAR_OFF + Lay::NBAR * 8 + 4);
  float* vec = reinterpret_cast<float*>(smem + Lay::VEC_OFF);

  const Geom& g = args.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nt = g.nt;
  const uint64_t to = args.timeout_ns;
  // fixed pair: (K, Val) for DKDV, (Q, dO) for DQ; streamed pair: the other two
  const CUtensorMap* fix0 = MODE == MODE_DKDV ? &tm_k : &tm_q;
  const CUtensorMap* fix1 = MODE == MODE_DKDV ? &tm_v : &tm_do;
  const CUtensorMap* str0 = MODE == MODE_DKDV ? &tm_q : &tm_k;
  const CUtensorMap* str1 = MODE == MODE_DKDV ? &tm_do : &tm_v;

  {
    uint4* z = reinterpret_cast<uint4*>(smem);
    for (int i = threadIdx.x; i < Lay::VEC_OFF / 16; i += kBwdThreads) z[i] = make_uint4(0, 0, 0, 0);
  }
  if (threadIdx.x == 0) {
    mbar_init(&bars[C_FIXFULL], 1);
    mbar_init(&bars[C_FIXEMPTY], 1);
    mbar_init(&bars[C_STRFULL0], 1);
    mbar_init(&bars[C_STRFULL1], 1);
    mbar_init(&bars[C_STREMPTY0], 1);
    mbar_init(&bars[C_STREMPTY1], 1);
    mbar_init(&bars[C_SFULL], 1);
    mbar_init(&bars[C_PFULL], 128);
    mbar_init(&bars[C_ACC], 1);
    mbar_init(&bars[C_DRAIN], 1);
    mbar_init(&bars[C_VEC], 128);
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
    prefetch_tmap(&tm_do);
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
      uint32_t it = 0, items = 0;
      const uint32_t tile_tx = uint32_t(g.box_rows) * D * 2;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < args.total_items; item += gridDim.x, ++items) {
        const int prob = item / nt, ft = item - prob * nt;
        const int base = problem_base(g, prob);
        int b0, c0;
        ok = mbar_wait(&bars[C_FIXEMPTY], (items & 1) ^ 1, abort_flag, to);
        if (!ok) break;
        tile_origin(g, ft, b0, c0);
        mbar_arrive_expect_tx(&bars[C_FIXFULL], 2 * tile_tx);
#pragma unroll
        for (int dh = 0; dh < DH; ++dh) {
          tma_load_5d(smem + Lay::FIX_OFF + dh * BLK, fix0, &bars[C_FIXFULL], dh * 64, 0, b0, c0, base);
          tma_load_5d(smem + Lay::FIX_OFF + Lay::TILE + dh * BLK, fix1, &bars[C_FIXFULL], dh * 64, 0, b0, c0, base);
        }
        for (int st = 0; st < nt; ++st, ++it) {
          const int b = it & 1;
          ok = mbar_wait(&bars[C_STREMPTY0 + b], ((it >> 1) & 1) ^ 1, abort_flag, to);
          if (!ok) break;
          tile_origin(g, st, b0, c0);
          uint8_t* dst = smem + Lay::STR_OFF + b * 2 * Lay::TILE;
          mbar_arrive_expect_tx(&bars[C_STRFULL0 + b], 2 * tile_tx);
#pragma unroll
          for (int dh = 0; dh < DH; ++dh) {
            tma_load_5d(dst + dh * BLK, str0, &bars[C_STRFULL0 + b], dh * 64, 0, b0, c0, base);
            tma_load_5d(dst + Lay::TILE + dh * BLK, str1, &bars[C_STRFULL0 + b], dh * 64, 0, b0, c0, base);
          }
        }
      }
      for (int b = 0; b < 2; ++b) {
        const uint32_t uses = it > uint32_t(b) ? (it - b + 1) / 2 : 0;
        if (uses) mbar_wait_drain(&bars[C_STRFULL0 + b], (uses - 1) & 1, to);
      }
      if (items) mbar_wait_drain(&bars[C_FIXFULL], (items - 1) & 1, to);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0, items = 0, acc_count = 0, p_iter = 0;
      const uint32_t id_s = idesc_bf16_f32(128, 128, 0, 0);   // S-like products: both K-major
      const uint32_t id_acc = idesc_bf16_f32(128, D, 0, 1);   // accumulators: B MN-major
      const uint32_t fa = sbase + Lay::FIX_OFF, fb = fa + Lay::TILE;
      bool ok = true;
      for (int item = blockIdx.x; ok && item < args.total_items; item += gridDim.x, ++items) {
        ok = mbar_wait(&bars[C_FIXFULL], items & 1, abort_flag, to);
        if (!ok) break;
        for (int st = 0; st < nt; ++st, ++it) {
          const int b = it & 1;
          ok = mbar_wait(&bars[C_STRFULL0 + b], (it >> 1) & 1, abort_flag, to);
          if (!ok) break;
          if (acc_count > 0) {  // previous accumulation has read P / dS from TMEM
            ok = mbar_wait(&bars[C_ACC], (acc_count - 1) & 1, abort_flag, to);
            if (!ok) break;
          }
          tc_fence_after();
          const uint32_t sa = sbase + Lay::STR_OFF + b * 2 * Lay::TILE, sb = sa + Lay::TILE;
          // S-like product: fixed0 x streamed0^T ; dP-like: fixed1 x streamed1^T
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t koff = (kk >> 2) * BLK + (kk & 3) * 32;
            mma_ss(tmem + Lay::TM_S, sdesc_sw128(fa + koff, 16, 1024), sdesc_sw128(sa + koff, 16, 1024), id_s,
                   kk > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t koff = (kk >> 2) * BLK + (kk & 3) * 32;
            mma_ss(tmem + Lay::TM_DP, sdesc_sw128(fb + koff, 16, 1024), sdesc_sw128(sb + koff, 16, 1024), id_s,
                   kk > 0 ? 1u : 0u);
          }
          tc_commit(&bars[C_SFULL]);
          ok = mbar_wait(&bars[C_PFULL], p_iter & 1, abort_flag, to);
          if (!ok) break;
          ++p_iter;
          tc_fence_after();
          const uint32_t acc_in = st > 0 ? 1u : 0u;
          if (MODE == MODE_DKDV) {
            // dVal += P^T dO_st (A = P^T in TMEM cols [0,64)), dK += dS^T Q_st (A = dS^T in [128,192))
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t bd = sdesc_sw128(sb + kk * 16 * 128, BLK, 1024);
              mma_ts(tmem + Lay::TM_A1, tmem + Lay::TM_S + kk * 8, bd, id_acc, (acc_in | (kk > 0)) ? 1u : 0u);
            }
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t bd = sdesc_sw128(sa + kk * 16 * 128, BLK, 1024);
              mma_ts(tmem + Lay::TM_A2, tmem + Lay::TM_DP + kk * 8, bd, id_acc, (acc_in | (kk > 0)) ? 1u : 0u);
            }
          } else {
            // dQ += dS K_st (A = dS in TMEM cols [128,192))
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t bd = sdesc_sw128(sa + kk * 16 * 128, BLK, 1024);
              mma_ts(tmem + Lay::TM_A1, tmem + Lay::TM_DP + kk * 8, bd, id_acc, (acc_in | (kk > 0)) ? 1u : 0u);
            }
          }
          tc_commit(&bars[C_ACC]);
          ++acc_count;
          tc_commit(&bars[C_STREMPTY0 + b]);
        }
        if (!ok) break;
        tc_commit(&bars[C_FIXEMPTY]);
      }
      tc_commit(&bars[C_DRAIN]);
      mbar_wait_drain(&bars[C_DRAIN], 0, to);
    }
  } else {
    // ------------------------------------------------------------ softmax-gradient + epilogue
    const int row = threadIdx.x;
    const uint32_t lane_sel = uint32_t(warp * 32) << 16;
    const uint32_t tS = tmem + lane_sel + Lay::TM_S, tDP = tmem + lane_sel + Lay::TM_DP;
    const float c2 = args.scale_log2;
    const float log2e = 1.4426950408889634f;
    uint32_t s_iter = 0, acc_seen = 0, vec_iter = 0, items = 0;
    bool ok = true;
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, to)) != 0;
    };
    for (int item = blockIdx.x; ok && item < args.total_items; item += gridDim.x, ++items) {
      const int prob = item / nt, ft = item - prob * nt;
      const int base = problem_base(g, prob);
      const int valid_fixed = tile_valid_rows(g, ft);
      // per-row softmax statistics of the fixed tile (DQ mode: rows are queries)
      float lse_row = 0.f, D_row = 0.f;
      if (MODE == MODE_DQ && row < valid_fixed) {
        const int tok = base + tile_row_offset(g, ft, row);
        lse_row = args.lse[tok] * log2e;
        D_row = args.Drow[tok];
      }
      for (int st = 0; st < nt; ++st) {
        const int valid_str = tile_valid_rows(g, st);
        float* vl = vec + (vec_iter & 1) * 256;  // [0,128) lse*log2e, [128,256) D
        if (MODE == MODE_DKDV) {
          // per-column statistics of the streamed query tile, shared through shared memory
          float l = INFINITY, dd = 0.f;  // rows past the problem: P = 0
          if (row < valid_str) {
            const int tok = base + tile_row_offset(g, st, row);
            l = args.lse[tok] * log2e;
            dd = args.Drow[tok];
          }
          vl[row] = l;
          vl[128 + row] = dd;
          mbar_arrive(&bars[C_VEC]);
          ok = wwait(&bars[C_VEC], vec_iter & 1);
          ++vec_iter;
          if (!ok) break;
        }
        ok = wwait(&bars[C_SFULL], s_iter & 1);
        if (!ok) break;
        ++s_iter;
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t s[32], dp[32];
          tmem_ld32(tS + c * 32, s);
          tmem_ld32(tDP + c * 32, dp);
          uint32_t pk[16], dk[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            float p[2], ds[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int col = c * 32 + e + u;
              float lcol, dcol;
              bool live;
              if (MODE == MODE_DKDV) {
                lcol = vl[col];
                dcol = vl[128 + col];
                live = true;
              } else {
                lcol = lse_row;
                dcol = D_row;
                live = col < valid_str;
              }
              const float pv = live ? ex2_approx(fmaf(__uint_as_float(s[e + u]), c2, -lcol)) : 0.f;
              p[u] = pv;
              ds[u] = pv * (__uint_as_float(dp[e + u]) - dcol);
            }
            pk[e >> 1] = pack_bf16x2(p[0], p[1]);
            dk[e >> 1] = pack_bf16x2(ds[0], ds[1]);
          }
          if (MODE == MODE_DKDV) tmem_st16(tS + c * 16, pk);
          tmem_st16(tDP + c * 16, dk);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bars[C_PFULL]);
      }
      if (!ok) break;
      // ---------------- epilogue: accumulators -> global rows (thread = row of the fixed tile)
      acc_seen += nt;
      ok = wwait(&bars[C_ACC], (acc_seen - 1) & 1);
      if (!ok) break;
      tc_fence_after();
      const bool live = row < valid_fixed;
      const long long tok = live ? (long long)base + tile_row_offset(g, ft, row) : 0;
      // main accumulator: dK (DKDV, columns 384..) or dQ (DQ, columns 256..), times the scale
      const uint32_t tmain = tmem + lane_sel + (MODE == MODE_DKDV ? Lay::TM_A2 : Lay::TM_A1);
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmain + c * 32, r);
        if (live) {
          float v[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(r[e]) * args.scale;
          if (args.add != nullptr) {
            const float4* a4 = reinterpret_cast<const float4*>(args.add + tok * D + c * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float4 x = a4[i];
              v[4 * i] += x.x;
              v[4 * i + 1] += x.y;
              v[4 * i + 2] += x.z;
              v[4 * i + 3] += x.w;
            }
          }
          if (OUT_F32) {
            store_row_out(static_cast<float*>(args.out_main) + tok * D + c * 32, v, 32);
          } else {
            uint4* o4 = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(args.out_main) + tok * D + c * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              o4[i] = make_uint4(pack_bf16x2(v[8 * i], v[8 * i + 1]), pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                                 pack_bf16x2(v[8 * i + 4], v[8 * i + 5]), pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
          }
        }
      }
      if (MODE == MODE_DKDV) {
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tmem + lane_sel + Lay::TM_A1 + c * 32, r);
          if (live) {
            uint4* o4 = reinterpret_cast<uint4*>(args.out_val + tok * D + c * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              o4[i] = make_uint4(pack_bf16x2(__uint_as_float(r[8 * i]), __uint_as_float(r[8 * i + 1])),
                                 pack_bf16x2(__uint_as_float(r[8 * i + 2]), __uint_as_float(r[8 * i + 3])),
                                 pack_bf16x2(__uint_as_float(r[8 * i + 4]), __uint_as_float(r[8 * i + 5])),
                                 pack_bf16x2(__uint_as_float(r[8 * i + 6]), __uint_as_float(r[8 * i + 7])));
          }
        }
      }
      tc_fence_before();  // accumulator reads are done before the next item's first MMA
    }
  }

  __syncthreads();
  if (*abort_flag && threadIdx.x == 0 && args.err != nullptr) atomicCAS(args.err, 0, 1);
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, Lay::TMEM_COLS);
  }
}

}  // namespace sq
