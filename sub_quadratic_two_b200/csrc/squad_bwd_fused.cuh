// squad_bwd_fused.cuh - backward of one SQuad-Attention pass whose problems fit one
// 128-row box, in one kernel on the sm_100a tensor cores.
//
// The pass is softmax attention over independent problems ("SQuad: Sub-Quadratic
// Attention Distillation for Efficient Video Generation", gist.science technical
// summary, Methodology section 1: the groups of the global pass, and the windows of
// the local pass when a window has at most 128 tokens). Its gradient is the textbook
// one:
//   P = exp(s*Q K^T - lse),  dP = dO Val^T,  D = rowsum(dO o O),  dS = P o (dP - D)
//   dVal = P^T dO,  dK = s * dS^T Q,  dQ = s * dS K.
// When a problem is a single box, one CTA item holds the problem's Q, K, Val and dO
// and computes all three gradients from ONE S and ONE dP: five 128-row GEMMs and one
// read of each input, where the split dq / dk-dv kernels take seven and read twice.
//
//   S^T = K Q^T   -> TMEM [0,128)    lane = key row
//   dP^T = Val dO^T -> TMEM [128,256)
//   softmax warps: P^T (bf16, in place in TMEM [0,64)) and dS^T (bf16, to shared memory)
//   dQ  = dS K    (A = dS^T tile read MN-major)      -> TMEM [128,256)
//   dVal = P^T dO (A = P^T from TMEM)                -> TMEM [256,384)
//   dK  = dS^T Q  (A = dS^T tile read K-major)       -> TMEM [384,512)
//
// Warp roles: warps 0-3 softmax gradient (thread = key row = TMEM lane), warps 4-7
// epilogue (thread = token row; stores pass through a per-warp transpose patch so that
// each warp store writes whole lines), warp 8 TMA producer, warp 9 MMA issuer.
// Input tiles live in a pool of five slots: the next item's K and Q go into the spare
// slot and the slot Val leaves when dP is done, so the next S can start while the
// current item's gradients are still accumulating. Every wait is bounded.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>
#include "geometry.h"
#include "sm100.cuh"

namespace sq {

struct BwdFusedArgs {
  Geom g;                  // the pass's geometry; g.nt == 1
  int total_items;         // problems
  float scale;             // softmax scale
  float scale_log2;        // scale * log2(e)
  const float* lse;        // [rows] natural-log LSE of this pass
  const float* Drow;       // [rows] rowsum(dO o O) of this pass
  const float* add_q;      // fp32 [rows, D] added to dQ, or nullptr
  const float* add_k;      // fp32 [rows, D] added to dK, or nullptr
  void* out_q;             // dQ: fp32 if OUT_F32 else bf16
  void* out_k;             // dK: fp32 if OUT_F32 else bf16
  __nv_bfloat16* out_val;  // dVal, bf16
  int* err;
  uint64_t timeout_ns;
};

constexpr int kBwdFusedThreads = 320;

template <int D>
struct BwdFusedLayout {
  static constexpr int TILE = 128 * D * 2;
  static constexpr int NSLOT = 5;
  static constexpr int SLOT_OFF = 0;
  static constexpr int DS_OFF = NSLOT * TILE;           // dS^T: 128 key rows x 128 query columns, bf16
  static constexpr int XP_OFF = DS_OFF + 128 * 128 * 2;  // 4 epilogue warps x (32 rows x 128 B)
  static constexpr int VEC_OFF = XP_OFF + 4 * 4096;      // 2 buffers x (lse*log2e[128], D[128])
  static constexpr int BAR_OFF = VEC_OFF + 2 * 256 * 4;
  static constexpr int NBAR = 20;
  static constexpr int BYTES = BAR_OFF + NBAR * 8 + 16;
  static constexpr int ALLOC = BYTES + 1024;
  static constexpr int TM_S = 0, TM_DP = 128, TM_DV = 256, TM_DK = 384;  // dQ reuses TM_DP
  static constexpr int TMEM_COLS = 512;
};

enum { G_FULL = 0, G_EMPTY = 5, G_SFULL = 10, G_PFULL, G_DQDONE, G_ACC, G_DQFREE, G_ACCFREE, G_VEC, G_DRAIN };

// Slot roles of one item. After each item: the spare takes K, Val's slot (free once
// dP is done) takes Q, K's and Q's slots take Val and dO, dO's slot becomes the spare.
struct SlotRoles {
  int k = 0, q = 1, v = 2, o = 3, sp = 4;
  __device__ __forceinline__ void next() {
    const int nk = sp, nq = v, nv = k, no = q, nsp = o;
    k = nk;
    q = nq;
    v = nv;
    o = no;
    sp = nsp;
  }
};

// Epilogue of one fp32 accumulator (thread = row): out = acc * scale (+ add), written
// as fp32 or bf16 rows through the warp's 128B-swizzled patch, 32 columns per round.
template <int D, bool OUT_F32>
__device__ __forceinline__ void epi_rows_f32(uint32_t taddr, uint32_t xp, int lane, size_t tok, bool live,
                                             float scale, const float* add, void* out) {
  const int lr = lane >> 3, lc = lane & 7;
#pragma unroll 1
  for (int rd = 0; rd < D / 32; ++rd) {
    uint32_t v[32];
    tmem_ld32(taddr + rd * 32, v);
#pragma unroll
    for (int c = 0; c < 8; ++c)
      st_shared_v4(xp + lane * 128 + ((c ^ (lane & 7)) << 4), __float_as_uint(__uint_as_float(v[4 * c]) * scale),
                   __float_as_uint(__uint_as_float(v[4 * c + 1]) * scale),
                   __float_as_uint(__uint_as_float(v[4 * c + 2]) * scale),
                   __float_as_uint(__uint_as_float(v[4 * c + 3]) * scale));
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = 4 * i + lr;
      const size_t rtok = __shfl_sync(0xffffffffu, tok, r);
      const bool rlive = __shfl_sync(0xffffffffu, live, r);
      const uint4 x = ld_shared_v4(xp + r * 128 + ((lc ^ (r & 7)) << 4));
      if (rlive) {
        float4 f = make_float4(__uint_as_float(x.x), __uint_as_float(x.y), __uint_as_float(x.z), __uint_as_float(x.w));
        const size_t e = rtok * D + rd * 32 + lc * 4;
        if (add != nullptr) {
          const float4 a = *reinterpret_cast<const float4*>(add + e);
          f.x += a.x;
          f.y += a.y;
          f.z += a.z;
          f.w += a.w;
        }
        if (OUT_F32)
          *reinterpret_cast<float4*>(static_cast<float*>(out) + e) = f;
        else
          *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(out) + e) =
              make_uint2(pack_bf16x2(f.x, f.y), pack_bf16x2(f.z, f.w));
      }
    }
    __syncwarp();
  }
}

// Epilogue of one fp32 accumulator written as bf16 rows, 64 columns per round.
template <int D>
__device__ __forceinline__ void epi_rows_bf16(uint32_t taddr, uint32_t xp, int lane, size_t tok, bool live,
                                              __nv_bfloat16* out) {
  const int lr = lane >> 3, lc = lane & 7;
#pragma unroll 1
  for (int h = 0; h < D / 64; ++h) {
    uint32_t o[64];
    tmem_ld64(taddr + h * 64, o);
#pragma unroll
    for (int c = 0; c < 8; ++c)
      st_shared_v4(xp + lane * 128 + ((c ^ (lane & 7)) << 4),
                   pack_bf16x2(__uint_as_float(o[8 * c + 0]), __uint_as_float(o[8 * c + 1])),
                   pack_bf16x2(__uint_as_float(o[8 * c + 2]), __uint_as_float(o[8 * c + 3])),
                   pack_bf16x2(__uint_as_float(o[8 * c + 4]), __uint_as_float(o[8 * c + 5])),
                   pack_bf16x2(__uint_as_float(o[8 * c + 6]), __uint_as_float(o[8 * c + 7])));
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = 4 * i + lr;
      const size_t rtok = __shfl_sync(0xffffffffu, tok, r);
      const bool rlive = __shfl_sync(0xffffffffu, live, r);
      const uint4 x = ld_shared_v4(xp + r * 128 + ((lc ^ (r & 7)) << 4));
      if (rlive) *reinterpret_cast<uint4*>(out + rtok * D + h * 64 + lc * 8) = x;
    }
    __syncwarp();
  }
}

template <int D, bool OUT_F32>
__global__ void __launch_bounds__(kBwdFusedThreads, 1)
    squad_bwd_fused_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                           const __grid_constant__ BwdFusedArgs args) {
  using Lay = BwdFusedLayout<D>;
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
  const uint64_t to = args.timeout_ns;

  {
    // TMA writes rows [0, box_rows) of each slot; rows past the box stay zero for good
    uint4* z = reinterpret_cast<uint4*>(smem + Lay::SLOT_OFF);
    for (int i = threadIdx.x; i < Lay::NSLOT * Lay::TILE / 16; i += kBwdFusedThreads) z[i] = make_uint4(0, 0, 0, 0);
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < Lay::NSLOT; ++s) {
      mbar_init(&bars[G_FULL + s], 1);
      mbar_init(&bars[G_EMPTY + s], 1);
    }
    mbar_init(&bars[G_SFULL], 1);
    mbar_init(&bars[G_PFULL], 128);
    mbar_init(&bars[G_DQDONE], 1);
    mbar_init(&bars[G_ACC], 1);
    mbar_init(&bars[G_DQFREE], 128);
    mbar_init(&bars[G_ACCFREE], 128);
    mbar_init(&bars[G_VEC], 128);
    mbar_init(&bars[G_DRAIN], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_holder, Lay::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
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
  auto slot_addr = [&](int s) -> uint32_t { return sbase + Lay::SLOT_OFF + s * Lay::TILE; };

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      SlotRoles R;
      uint32_t pu = 0, used = 0;  // per slot: parity of its use count; ever used
      const uint32_t tx = uint32_t(g.box_rows) * D * 2;
      int b0, c0;
      tile_origin(g, 0, b0, c0);
      auto load = [&](int s, const CUtensorMap* m, int base) -> bool {
        if (!mbar_wait(&bars[G_EMPTY + s], ((pu >> s) & 1u) ^ 1u, abort_flag, to)) return false;
        mbar_arrive_expect_tx(&bars[G_FULL + s], tx);
#pragma unroll
        for (int dh = 0; dh < DH; ++dh)
          tma_load_5d(smem + Lay::SLOT_OFF + s * Lay::TILE + dh * BLK, m, &bars[G_FULL + s], dh * 64, 0, b0, c0,
                      base);
        pu ^= 1u << s;
        used |= 1u << s;
        return true;
      };
      for (int item = blockIdx.x; item < args.total_items; item += gridDim.x) {
        const int base = problem_base(g, item);
        // K and Q first: they go to slots that free early, so the next S can start soon
        if (!(load(R.k, &tm_k, base) && load(R.q, &tm_q, base) && load(R.v, &tm_v, base) &&
              load(R.o, &tm_do, base)))
          break;
        R.next();
      }
      for (int s = 0; s < Lay::NSLOT; ++s)
        if ((used >> s) & 1u) mbar_wait_drain(&bars[G_FULL + s], ((pu >> s) & 1u) ^ 1u, to);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      SlotRoles R;
      uint32_t cu = 0, i = 0;
      const uint32_t id_s = idesc_bf16_f32(128, 128, 0, 0);   // S^T, dP^T: both operands K-major
      const uint32_t id_kv = idesc_bf16_f32(128, D, 0, 1);    // dVal, dK: B MN-major
      const uint32_t id_q = idesc_bf16_f32(128, D, 1, 1);     // dQ: A (dS^T tile) and B MN-major
      const uint32_t ds = sbase + Lay::DS_OFF;
      bool ok = true;
      auto wait_full = [&](int s) -> bool {
        return mbar_wait(&bars[G_FULL + s], (cu >> s) & 1u, abort_flag, to);
      };
      for (int item = blockIdx.x; item < args.total_items; item += gridDim.x, ++i) {
        const uint32_t sk = slot_addr(R.k), sq_ = slot_addr(R.q), sv = slot_addr(R.v), so = slot_addr(R.o);
        // S^T into [0,128): the previous dVal has read P^T from there
        if (i > 0) ok = mbar_wait(&bars[G_ACC], (i - 1) & 1u, abort_flag, to);
        ok = ok && wait_full(R.k) && wait_full(R.q);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * BLK + (kk & 3) * 32;
          mma_ss(tmem + Lay::TM_S, sdesc_sw128(sk + koff, 16, 1024), sdesc_sw128(sq_ + koff, 16, 1024), id_s,
                 kk > 0 ? 1u : 0u);
        }
        // dP^T into [128,256): the epilogue has drained the previous dQ from there
        if (i > 0) ok = mbar_wait(&bars[G_DQFREE], (i - 1) & 1u, abort_flag, to);
        ok = ok && wait_full(R.v) && wait_full(R.o);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * BLK + (kk & 3) * 32;
          mma_ss(tmem + Lay::TM_DP, sdesc_sw128(sv + koff, 16, 1024), sdesc_sw128(so + koff, 16, 1024), id_s,
                 kk > 0 ? 1u : 0u);
        }
        tc_commit(&bars[G_SFULL]);
        tc_commit(&bars[G_EMPTY + R.v]);  // Val is done
        cu ^= (1u << R.k) | (1u << R.q) | (1u << R.v) | (1u << R.o);
        if (!(ok = mbar_wait(&bars[G_PFULL], i & 1u, abort_flag, to))) break;
        tc_fence_after();
        // dQ = dS K (K = key rows): A = dS^T tile (rows = keys, query-contiguous: MN-major)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tmem + Lay::TM_DP, sdesc_sw128(ds + kk * 2048, BLK, 1024), sdesc_sw128(sk + kk * 2048, BLK, 1024),
                 id_q, kk > 0 ? 1u : 0u);
        tc_commit(&bars[G_DQDONE]);
        if (i > 0 && !(ok = mbar_wait(&bars[G_ACCFREE], (i - 1) & 1u, abort_flag, to))) break;
        tc_fence_after();
        // dVal = P^T dO (K = query rows): A = P^T in TMEM columns [0,64)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + Lay::TM_DV, tmem + Lay::TM_S + kk * 8, sdesc_sw128(so + kk * 2048, BLK, 1024), id_kv,
                 kk > 0 ? 1u : 0u);
        // dK = dS^T Q (K = query rows): A = dS^T tile, K-major
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tmem + Lay::TM_DK, sdesc_sw128(ds + (kk >> 2) * BLK + (kk & 3) * 32, 16, 1024),
                 sdesc_sw128(sq_ + kk * 2048, BLK, 1024), id_kv, kk > 0 ? 1u : 0u);
        tc_commit(&bars[G_ACC]);
        tc_commit(&bars[G_EMPTY + R.k]);
        tc_commit(&bars[G_EMPTY + R.q]);
        tc_commit(&bars[G_EMPTY + R.o]);
        R.next();
      }
      tc_commit(&bars[G_DRAIN]);
      mbar_wait_drain(&bars[G_DRAIN], 0, to);
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ softmax gradient (thread = key row)
    const int row = threadIdx.x;
    const uint32_t lane_sel = uint32_t(warp * 32) << 16;
    const uint32_t tS = tmem + lane_sel + Lay::TM_S, tDP = tmem + lane_sel + Lay::TM_DP;
    const uint32_t ds_row = sbase + Lay::DS_OFF + row * 128;
    const float c2 = args.scale_log2;
    const float log2e = 1.4426950408889634f;
    const int valid = tile_valid_rows(g, 0);
    const bool rlive = row < valid;
    const int roff = rlive ? tile_row_offset(g, 0, row) : 0;
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, to)) != 0;
    };
    uint32_t i = 0;
    for (int item = blockIdx.x; item < args.total_items; item += gridDim.x, ++i) {
      // per-query statistics (the query box is the key box): row r publishes column r
      float* vl = vec + (i & 1u) * 256;
      float l = INFINITY, dd = 0.f;  // query columns past the problem: P = 0
      if (rlive) {
        const int tok = problem_base(g, item) + roff;
        l = args.lse[tok] * log2e;
        dd = args.Drow[tok];
      }
      vl[row] = l;
      vl[128 + row] = dd;
      mbar_arrive(&bars[G_VEC]);
      if (!wwait(&bars[G_VEC], i & 1u)) break;
      if (!wwait(&bars[G_SFULL], i & 1u)) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t s[32], dp[32];
        tmem_ld32(tS + c * 32, s);
        tmem_ld32(tDP + c * 32, dp);
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int e4 = 0; e4 < 32; e4 += 4) {
          const float4 lc4 = *reinterpret_cast<const float4*>(vl + c * 32 + e4);
          const float4 dc4 = *reinterpret_cast<const float4*>(vl + 128 + c * 32 + e4);
          const float lcol[4] = {lc4.x, lc4.y, lc4.z, lc4.w};
          const float dcol[4] = {dc4.x, dc4.y, dc4.z, dc4.w};
          float p[4], dsv[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            // key rows past the problem: P = dS = 0 (a select: exp2 of a zero score may overflow)
            p[u] = rlive ? ex2_approx(fmaf(__uint_as_float(s[e4 + u]), c2, -lcol[u])) : 0.f;
            dsv[u] = p[u] * (__uint_as_float(dp[e4 + u]) - dcol[u]);
          }
          pk[e4 >> 1] = pack_bf16x2(p[0], p[1]);
          pk[(e4 >> 1) + 1] = pack_bf16x2(p[2], p[3]);
          dk[e4 >> 1] = pack_bf16x2(dsv[0], dsv[1]);
          dk[(e4 >> 1) + 1] = pack_bf16x2(dsv[2], dsv[3]);
        }
        tmem_st16(tS + c * 16, pk);
        // dS^T row: query columns [32c, 32c+32) are 16-byte chunks 4(c&1)..4(c&1)+3 of block c>>1
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int chunk = (c & 1) * 4 + j;
          st_shared_v4(ds_row + (c >> 1) * BLK + ((chunk ^ (row & 7)) << 4), dk[4 * j], dk[4 * j + 1], dk[4 * j + 2],
                       dk[4 * j + 3]);
        }
      }
      tmem_st_wait();
      fence_async_smem();  // the dS^T tile is read by the tensor core
      tc_fence_before();
      mbar_arrive(&bars[G_PFULL]);
    }
  } else {
    // ------------------------------------------------------------ epilogue (thread = token row)
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const uint32_t lane_sel = uint32_t(q4 * 32) << 16;
    const uint32_t xp = sbase + Lay::XP_OFF + q4 * 4096;
    const int valid = tile_valid_rows(g, 0);
    const bool live = row < valid;
    const int roff = live ? tile_row_offset(g, 0, row) : 0;
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, to)) != 0;
    };
    uint32_t i = 0;
    for (int item = blockIdx.x; item < args.total_items; item += gridDim.x, ++i) {
      const size_t tok = live ? size_t(problem_base(g, item) + roff) : 0;
      if (!wwait(&bars[G_DQDONE], i & 1u)) break;
      tc_fence_after();
      epi_rows_f32<D, OUT_F32>(tmem + lane_sel + Lay::TM_DP, xp, lane, tok, live, args.scale, args.add_q,
                               args.out_q);
      tc_fence_before();
      mbar_arrive(&bars[G_DQFREE]);
      if (!wwait(&bars[G_ACC], i & 1u)) break;
      tc_fence_after();
      epi_rows_bf16<D>(tmem + lane_sel + Lay::TM_DV, xp, lane, tok, live, args.out_val);
      epi_rows_f32<D, OUT_F32>(tmem + lane_sel + Lay::TM_DK, xp, lane, tok, live, args.scale, args.add_k,
                               args.out_k);
      tc_fence_before();
      mbar_arrive(&bars[G_ACCFREE]);
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
