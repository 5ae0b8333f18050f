// squad_bwd_fused.cuh - backward of one SQuad-Attention pass in one kernel on the
// sm_100a tensor cores.
//
// The pass is softmax attention over independent problems ("SQuad: Sub-Quadratic
// Attention Distillation for Efficient Video Generation", gist.science technical
// summary, Methodology section 1: the windows of the local pass, the groups of the
// global pass). Its gradient is the textbook one:
//   P = exp(s*Q K^T - lse),  dP = dO Val^T,  D = rowsum(dO o O),  dS = P o (dP - D)
//   dVal = P^T dO,  dK = s * dS^T Q,  dQ = s * dS K.
// D of a query row is read from a vector (a row-dot pass makes it for the first backward
// launch). The epilogue can also produce the D of the pass that made Val: rowsum(dVal o
// Val) over the rows it writes (the global pass gives the local pass its D this way).
// A problem of L tokens is cut into nt boxes of at most 128 rows. A CTA item is
// (problem, key box kb): K_kb and Val_kb stay, the query boxes (Q_qb, dO_qb) stream,
// and every (qb, kb) block is done once, with five GEMMs and no recomputation:
//
//   S^T = K Q^T      -> TMEM [0,128)    lane = key row
//   dP^T = Val dO^T  -> TMEM [128,256)
//   softmax warps: P^T (bf16, in place in TMEM [0,64)) and dS^T (bf16, to shared memory)
//   dQ_qb part = dS K  (A = dS^T tile read MN-major)   -> TMEM [128,256)
//   dVal_kb += P^T dO  (A = P^T from TMEM)             -> TMEM [256,384)
//   dK_kb  += dS^T Q   (A = dS^T tile read K-major)    -> TMEM [384,512)
//
// dVal and dK of a key box are complete when its item ends. dQ of a query box is
// complete in one block when nt == 1 (stored, plus an optional fp32 addend); for
// nt > 1 each block adds its part into an fp32 buffer with vector reductions
// (red.global.add.v4.f32) and the host converts that buffer afterwards.
//
// Packed geometry (PACKED, problems of at most 64 tokens, several to a box; nt == 1):
// the softmax-gradient warps zero P and dS between a key row and the query columns of
// the other problems in the box, and rows past the packed digit's extent are dead on
// both sides (not read as statistics, not written).
//
// Warp roles: warps 0-3 softmax gradient (thread = key row = TMEM lane), then the drain of
// the block's dQ part (thread = query row); warps 4-7 epilogue, the drain of dVal and dK
// (thread = token row); warp 8 TMA producer, warp 9 MMA issuer. Drains pass through
// per-warp transpose patches so that each warp instruction writes whole lines.
// Input tiles live in a pool of five slots handed out in the order they are freed, so
// the next block's Q (and, at an item boundary, K) load while the current block's
// gradients are still accumulating. Every wait is bounded.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>
#include "geometry.h"
#include "sm100.cuh"

namespace sq {

struct BwdFusedArgs {
  Geom g;                  // the pass's geometry
  int total_items;         // problems * nt
  float scale;             // softmax scale
  float scale_log2;        // scale * log2(e)
  const float* lse;        // [rows] natural-log LSE of this pass
  const float* Drow;          // [rows] D = rowsum(dO o O) of this pass
  const __nv_bfloat16* val;   // [rows, D] values of this pass (read when d_next != nullptr)
  float* d_next;              // [rows] rowsum(dVal o Val), the D of the pass that produced Val, or nullptr
  const float* add_q;      // nt == 1: fp32 [rows, D] added to dQ, or nullptr
  float* acc_q;            // nt > 1: fp32 [rows, D] that the dQ parts are added into
  const float* add_k;      // fp32 [rows, D] added to dK, or nullptr
  void* out_q;             // nt == 1: dQ, fp32 if OUT_F32 else bf16
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
  static constexpr int XPS_OFF = XP_OFF + 4 * 4096;      // 4 softmax warps x (16 rows x 128 B)
  static constexpr int VEC_OFF = XPS_OFF + 4 * 2048;     // 2 buffers x (lse*log2e[128], D[128])
  static constexpr int BAR_OFF = VEC_OFF + 2 * 256 * 4;
  static constexpr int NBAR = 20;
  static constexpr int BYTES = BAR_OFF + NBAR * 8 + 16;
  static constexpr int ALLOC = BYTES + 1024;
  static constexpr int TM_S = 0, TM_DP = 128, TM_DV = 256, TM_DK = 384;  // dQ reuses TM_DP
  static constexpr int TMEM_COLS = 512;
};

enum {
  G_FULL = 0, G_EMPTY = 5,
  G_SFULL = 10,   // per block: S^T and dP^T are in TMEM
  G_PFULL,        // per block: P^T and dS^T written (128 softmax threads)
  G_DQDONE,       // per block: the dQ part is in TMEM
  G_STEPACC,      // per block: dVal and dK MMAs done (P^T and dS^T consumed)
  G_ITEMACC,      // per item: dVal and dK complete
  G_DQFREE,       // per block: the epilogue drained the dQ part (128 threads)
  G_ACCFREE,      // per item: the epilogue drained dVal and dK (128 threads)
  G_VEC,          // per block: column statistics published (128 softmax threads)
  G_DRAIN
};

// Tile slots of the blocks, identical on the producer and the MMA issuer. Slots are
// handed out first-freed first-used: the five free slots, then the releases of the
// blocks in order (Val after the item's last dP; Q, dO after each block's
// accumulation; K after the item's last one). A release is taken into the queue only
// when the queue runs dry, which fixes the order independently of timing.
struct SlotPlan {
  struct Rec {
    int k, v, q, o;
    bool last;
  };
  uint32_t fifo = 0x43210u;  // 4 bits per free slot, front in the low bits
  int n = 5;
  // blocks whose releases are not yet queued: [head, tail); at most two (the current block
  // and the one before it) are ever pending, kept in r0 / r1 by parity
  Rec r0{}, r1{};
  int head = 0, tail = 0;
  int ck = 0, cv = 0;
  __device__ __forceinline__ void push(int s) {
    fifo |= uint32_t(s) << (4 * n);
    ++n;
  }
  __device__ __forceinline__ int pop() {
    while (n == 0 && head < tail) {
      const Rec r = (head & 1) ? r1 : r0;
      if (r.last) push(r.v);
      push(r.q);
      push(r.o);
      if (r.last) push(r.k);
      ++head;
    }
    const int s = int(fifo & 15u);
    fifo >>= 4;
    --n;
    return s;
  }
  // slots of the next block: all four tiles at an item's first block, Q and dO after
  __device__ __forceinline__ Rec next(bool first, bool last) {
    Rec r;
    if (first) {
      r.k = pop();
      r.q = pop();
      r.v = pop();
      r.o = pop();
      ck = r.k;
      cv = r.v;
    } else {
      r.k = ck;
      r.v = cv;
      r.q = pop();
      r.o = pop();
    }
    r.last = last;
    if (tail & 1)
      r1 = r;
    else
      r0 = r;
    ++tail;
    return r;
  }
};

// Dot product of two 8-element bf16 chunks (widened exactly), added to acc.
__device__ __forceinline__ float dot8_bf16(const uint4& x, const uint4& y, float acc) {
  const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    acc = fmaf(__uint_as_float(xs[u] << 16), __uint_as_float(ys[u] << 16), acc);
    acc = fmaf(__uint_as_float(xs[u] & 0xffff0000u), __uint_as_float(ys[u] & 0xffff0000u), acc);
  }
  return acc;
}

// Rows an epilogue lane writes: a warp drains its 32 TMEM lanes (one row each) through
// a 128B-swizzled patch and writes them back four rows per instruction; lane l handles
// rows 4i + l/8 (i < 8), 16-byte column chunk l%8. Token rows are shuffled once per box.
struct EpiRows {
  int tok[8];
  uint32_t live;  // bit r: warp row r is inside the problem
};

__device__ __forceinline__ EpiRows epi_rows_of(int lane, int my_tok, bool my_live) {
  EpiRows e;
#pragma unroll
  for (int i = 0; i < 8; ++i) e.tok[i] = __shfl_sync(0xffffffffu, my_tok, 4 * i + (lane >> 3));
  e.live = __ballot_sync(0xffffffffu, my_live);
  return e;
}

__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}

enum { EPI_F32 = 0, EPI_BF16 = 1, EPI_RED = 2 };

// Paired fp32 multiply (two lanes of one 64-bit register, rounded as two scalar multiplies).
__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// The 16-byte chunk of scaled accumulator values v[0..3] for the transpose patch.
__device__ __forceinline__ void st_scaled4(uint32_t addr, const uint32_t* v, uint64_t scale2) {
  const uint64_t a = fmul2(f2(__uint_as_float(v[0]), __uint_as_float(v[1])), scale2);
  const uint64_t b = fmul2(f2(__uint_as_float(v[2]), __uint_as_float(v[3])), scale2);
  st_shared_v4(addr, uint32_t(a), uint32_t(a >> 32), uint32_t(b), uint32_t(b >> 32));
}

// x + a over a 16-byte chunk, in pairs.
__device__ __forceinline__ float4 add4(const uint4& x, const float4& a) {
  const uint64_t lo = fadd2(f2(__uint_as_float(x.x), __uint_as_float(x.y)), f2(a.x, a.y));
  const uint64_t hi = fadd2(f2(__uint_as_float(x.z), __uint_as_float(x.w)), f2(a.z, a.w));
  return make_float4(f2_lo(lo), f2_hi(lo), f2_lo(hi), f2_hi(hi));
}

// Drain one fp32 accumulator (D columns): value = acc * scale (+ add), then stored as
// fp32 (EPI_F32) or bf16 (EPI_BF16), or added into fp32 memory (EPI_RED). The addend
// loads of 64 columns are issued before their TMEM loads so the latencies overlap.
template <int D, int KIND>
__device__ __forceinline__ void epi_acc(uint32_t taddr, uint32_t xp, int lane, const EpiRows& R, float scale,
                                        const float* add, void* out) {
  const int lr = lane >> 3, lc = lane & 7;
#pragma unroll 1
  for (int h = 0; h < D / 64; ++h) {
    float4 a[2][8];
#pragma unroll
    for (int rr = 0; rr < 2; ++rr)
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        a[rr][i] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (add != nullptr && ((R.live >> (4 * i + lr)) & 1u))
          a[rr][i] = __ldg(reinterpret_cast<const float4*>(add + size_t(R.tok[i]) * D + h * 64 + rr * 32 + lc * 4));
      }
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      uint32_t v[32];
      tmem_ld32(taddr + h * 64 + rr * 32, v);
      const uint64_t scale2 = f2(scale, scale);
#pragma unroll
      for (int c = 0; c < 8; ++c) st_scaled4(xp + lane * 128 + ((c ^ (lane & 7)) << 4), v + 4 * c, scale2);
      __syncwarp();
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = 4 * i + lr;
        const uint4 x = ld_shared_v4(xp + r * 128 + ((lc ^ (r & 7)) << 4));
        if ((R.live >> r) & 1u) {
          const float4 f = add4(x, a[rr][i]);
          const float f0 = f.x, f1 = f.y, f2 = f.z, f3 = f.w;
          const size_t e = size_t(R.tok[i]) * D + h * 64 + rr * 32 + lc * 4;
          if (KIND == EPI_F32)
            *reinterpret_cast<float4*>(static_cast<float*>(out) + e) = make_float4(f0, f1, f2, f3);
          else if (KIND == EPI_BF16)
            *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(out) + e) =
                make_uint2(pack_bf16x2(f0, f1), pack_bf16x2(f2, f3));
          else
            red_add_v4(static_cast<float*>(out) + e, f0, f1, f2, f3);
        }
      }
      __syncwarp();
    }
  }
}

// The same drain through a patch of 16 rows (the softmax warps' patches are half the size
// of the epilogue warps'): per 32-column chunk, lanes 0-15 and then lanes 16-31 write their
// rows, and each round is written back four rows per instruction (lane l: patch row
// 4i + l/8, 16-byte chunk l%8).
template <int D, int KIND>
__device__ __forceinline__ void epi_acc16(uint32_t taddr, uint32_t xp, int lane, int my_tok, bool my_live,
                                          float scale, const float* add, void* out) {
  const int pr = lane >> 3, lc = lane & 7;
  const uint32_t live = __ballot_sync(0xffffffffu, my_live);
  int tok[2][4];
#pragma unroll
  for (int r = 0; r < 2; ++r)
#pragma unroll
    for (int i = 0; i < 4; ++i) tok[r][i] = __shfl_sync(0xffffffffu, my_tok, 16 * r + 4 * i + pr);
  const int prow = lane & 15;
#pragma unroll 1
  for (int ch = 0; ch < D / 32; ++ch) {
    float4 a[2][4];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[r][i] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (add != nullptr && ((live >> (16 * r + 4 * i + pr)) & 1u))
          a[r][i] = __ldg(reinterpret_cast<const float4*>(add + size_t(tok[r][i]) * D + ch * 32 + lc * 4));
      }
    uint32_t v[32];
    tmem_ld32(taddr + ch * 32, v);
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      if ((lane >> 4) == r) {
        const uint64_t scale2 = f2(scale, scale);
#pragma unroll
        for (int c = 0; c < 8; ++c) st_scaled4(xp + prow * 128 + ((c ^ (prow & 7)) << 4), v + 4 * c, scale2);
      }
      __syncwarp();
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int q = 4 * i + pr;
        const uint4 x = ld_shared_v4(xp + q * 128 + ((lc ^ (q & 7)) << 4));
        if ((live >> (16 * r + q)) & 1u) {
          const float4 f = add4(x, a[r][i]);
          const float f0 = f.x, f1 = f.y, f2 = f.z, f3 = f.w;
          const size_t e = size_t(tok[r][i]) * D + ch * 32 + lc * 4;
          if (KIND == EPI_F32)
            *reinterpret_cast<float4*>(static_cast<float*>(out) + e) = make_float4(f0, f1, f2, f3);
          else if (KIND == EPI_BF16)
            *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(out) + e) =
                make_uint2(pack_bf16x2(f0, f1), pack_bf16x2(f2, f3));
          else
            red_add_v4(static_cast<float*>(out) + e, f0, f1, f2, f3);
        }
      }
      __syncwarp();
    }
  }
}

// Drain one fp32 accumulator as bf16 rows (no scale), 64 columns per round; with
// d_next, also rowsum(value o val) of the written (bf16) values, one float per row.
template <int D>
__device__ __forceinline__ void epi_acc_bf16(uint32_t taddr, uint32_t xp, int lane, const EpiRows& R,
                                             __nv_bfloat16* out, const __nv_bfloat16* val, float* d_next) {
  const int lr = lane >> 3, lc = lane & 7;
  float dn[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) dn[i] = 0.f;
#pragma unroll 1
  for (int h = 0; h < D / 64; ++h) {
    uint4 y[8];
    if (d_next != nullptr) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        y[i] = ((R.live >> (4 * i + lr)) & 1u)
                   ? __ldg(reinterpret_cast<const uint4*>(val + size_t(R.tok[i]) * D + h * 64 + lc * 8))
                   : make_uint4(0, 0, 0, 0);
    }
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
      const uint4 x = ld_shared_v4(xp + r * 128 + ((lc ^ (r & 7)) << 4));
      if ((R.live >> r) & 1u) *reinterpret_cast<uint4*>(out + size_t(R.tok[i]) * D + h * 64 + lc * 8) = x;
      if (d_next != nullptr) dn[i] = dot8_bf16(x, y[i], dn[i]);
    }
    __syncwarp();
  }
  if (d_next != nullptr) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float v = dn[i];
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      v += __shfl_xor_sync(0xffffffffu, v, 4);
      if (lc == 0 && ((R.live >> (4 * i + lr)) & 1u)) d_next[R.tok[i]] = v;
    }
  }
}

// D_t = rowsum(a_t o b_t) of bf16 rows (d a multiple of 8, at most 256): d/8 threads per
// row, one 16-byte chunk of each operand per thread, a shuffle sum over the row's lanes.
// Coalesced and HBM-bound; it gives the first backward launch its D as a vector.
__global__ void rowdot_bf16_kernel(const __nv_bfloat16* __restrict__ a, const __nv_bfloat16* __restrict__ b,
                                   float* __restrict__ out, long long rows, int d) {
  const int per = d / 8;  // lanes per row: a power of two dividing 32 (d = 64 or 128)
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long row = gid / per;
  const int c = int(gid - row * per);
  float acc = 0.f;
  if (row < rows) {
    const uint4 x = __ldg(reinterpret_cast<const uint4*>(a + row * d) + c);
    const uint4 y = __ldg(reinterpret_cast<const uint4*>(b + row * d) + c);
    acc = dot8_bf16(x, y, 0.f);
  }
  for (int off = per >> 1; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (row < rows && c == 0) out[row] = acc;
}

// dq = bf16(acc), 8 elements per thread (rows * d is a multiple of 8)
__global__ void f32_to_bf16_kernel(const float* __restrict__ in, __nv_bfloat16* __restrict__ out, size_t n8) {
  const size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const float4 a = reinterpret_cast<const float4*>(in)[2 * i];
  const float4 b = reinterpret_cast<const float4*>(in)[2 * i + 1];
  reinterpret_cast<uint4*>(out)[i] =
      make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
}

// Packed geometry: whether box row `row` of the box whose first problem is j0 along the
// packed digit holds a problem (rows past the digit's extent are padding).
__device__ __forceinline__ bool packed_row_live(const Geom& g, int j0, int row) {
  return j0 + pack_id(g, row) < g.pk_ext;
}

template <int D, bool OUT_F32, bool PACKED>
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
    mbar_init(&bars[G_STEPACC], 1);
    mbar_init(&bars[G_ITEMACC], 1);
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

  const int nt = g.nt;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      SlotPlan plan;
      uint32_t pu = 0, used = 0;  // per slot: parity of its use count; ever used
      const uint32_t tx = uint32_t(g.box_rows) * D * 2;
      auto load = [&](int s, const CUtensorMap* m, int base, int t) -> bool {
        if (!mbar_wait(&bars[G_EMPTY + s], ((pu >> s) & 1u) ^ 1u, abort_flag, to)) return false;
        int b0, c0;
        tile_origin(g, t, b0, c0);
        mbar_arrive_expect_tx(&bars[G_FULL + s], tx);
#pragma unroll
        for (int dh = 0; dh < DH; ++dh)
          tma_load_5d(smem + Lay::SLOT_OFF + s * Lay::TILE + dh * BLK, m, &bars[G_FULL + s], dh * 64, 0, b0, c0,
                      base);
        pu ^= 1u << s;
        used |= 1u << s;
        return true;
      };
      bool ok = true;
      for (int item = blockIdx.x; ok && item < args.total_items; item += gridDim.x) {
        const int prob = fdiv(item, g.f_nt), kb = item - prob * nt;
        const int base = problem_base(g, prob);
        for (int qb = 0; qb < nt; ++qb) {
          const SlotPlan::Rec r = plan.next(qb == 0, qb == nt - 1);
          // K and Q first: S needs only them
          if (qb == 0)
            ok = load(r.k, &tm_k, base, kb) && load(r.q, &tm_q, base, qb) && load(r.v, &tm_v, base, kb) &&
                 load(r.o, &tm_do, base, qb);
          else
            ok = load(r.q, &tm_q, base, qb) && load(r.o, &tm_do, base, qb);
          if (!ok) break;
        }
      }
      for (int s = 0; s < Lay::NSLOT; ++s)
        if ((used >> s) & 1u) mbar_wait_drain(&bars[G_FULL + s], ((pu >> s) & 1u) ^ 1u, to);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      SlotPlan plan;
      uint32_t cu = 0, i = 0, t = 0;  // consumer parities; item and block counters
      const uint32_t id_s = idesc_bf16_f32(128, 128, 0, 0);   // S^T, dP^T: both operands K-major
      const uint32_t id_kv = idesc_bf16_f32(128, D, 0, 1);    // dVal, dK: B MN-major
      const uint32_t id_q = idesc_bf16_f32(128, D, 1, 1);     // dQ: A (dS^T tile) and B MN-major
      const uint32_t ds = sbase + Lay::DS_OFF;
      bool ok = true;
      auto wait_full = [&](int s) -> bool {
        const bool r = mbar_wait(&bars[G_FULL + s], (cu >> s) & 1u, abort_flag, to);
        cu ^= 1u << s;
        return r;
      };
      for (int item = blockIdx.x; ok && item < args.total_items; item += gridDim.x, ++i) {
        for (int qb = 0; qb < nt; ++qb, ++t) {
          const bool first = qb == 0, last = qb == nt - 1;
          const SlotPlan::Rec r = plan.next(first, last);
          const uint32_t sk = slot_addr(r.k), sq_ = slot_addr(r.q), sv = slot_addr(r.v), so = slot_addr(r.o);
          // S^T into [0,128): the previous block's dVal has read P^T from there
          if (t > 0) ok = mbar_wait(&bars[G_STEPACC], (t - 1) & 1u, abort_flag, to);
          if (ok && first) ok = wait_full(r.k);
          ok = ok && wait_full(r.q);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t koff = (kk >> 2) * BLK + (kk & 3) * 32;
            mma_ss(tmem + Lay::TM_S, sdesc_sw128(sk + koff, 16, 1024), sdesc_sw128(sq_ + koff, 16, 1024), id_s,
                   kk > 0 ? 1u : 0u);
          }
          // dP^T into [128,256): the epilogue has drained the previous dQ part from there
          if (t > 0) ok = mbar_wait(&bars[G_DQFREE], (t - 1) & 1u, abort_flag, to);
          if (ok && first) ok = wait_full(r.v);
          ok = ok && wait_full(r.o);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t koff = (kk >> 2) * BLK + (kk & 3) * 32;
            mma_ss(tmem + Lay::TM_DP, sdesc_sw128(sv + koff, 16, 1024), sdesc_sw128(so + koff, 16, 1024), id_s,
                   kk > 0 ? 1u : 0u);
          }
          tc_commit(&bars[G_SFULL]);
          if (last) tc_commit(&bars[G_EMPTY + r.v]);  // Val is done
          if (!(ok = mbar_wait(&bars[G_PFULL], t & 1u, abort_flag, to))) break;
          tc_fence_after();
          // dQ part = dS K (K = key rows): A = dS^T tile (rows = keys, query-contiguous: MN-major)
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(tmem + Lay::TM_DP, sdesc_sw128(ds + kk * 2048, BLK, 1024), sdesc_sw128(sk + kk * 2048, BLK, 1024),
                   id_q, kk > 0 ? 1u : 0u);
          tc_commit(&bars[G_DQDONE]);
          // the first block of an item overwrites dVal and dK: the epilogue has drained the last item's
          if (first && i > 0 && !(ok = mbar_wait(&bars[G_ACCFREE], (i - 1) & 1u, abort_flag, to))) break;
          tc_fence_after();
          // dVal += P^T dO (K = query rows): A = P^T in TMEM columns [0,64)
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tmem + Lay::TM_DV, tmem + Lay::TM_S + kk * 8, sdesc_sw128(so + kk * 2048, BLK, 1024), id_kv,
                   (!first || kk > 0) ? 1u : 0u);
          // dK += dS^T Q (K = query rows): A = dS^T tile, K-major
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(tmem + Lay::TM_DK, sdesc_sw128(ds + (kk >> 2) * BLK + (kk & 3) * 32, 16, 1024),
                   sdesc_sw128(sq_ + kk * 2048, BLK, 1024), id_kv, (!first || kk > 0) ? 1u : 0u);
          tc_commit(&bars[G_STEPACC]);
          tc_commit(&bars[G_EMPTY + r.q]);
          tc_commit(&bars[G_EMPTY + r.o]);
          if (last) {
            tc_commit(&bars[G_EMPTY + r.k]);
            tc_commit(&bars[G_ITEMACC]);
          }
        }
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
    const uint32_t xps = sbase + Lay::XPS_OFF + warp * 2048;
    const float c2 = args.scale_log2;
    const uint64_t c2x2 = f2(c2, c2);
    const float log2e = 1.4426950408889634f;
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, to)) != 0;
    };
    // packed boxes: the query columns in this key row's problem (the same for every box)
    uint32_t pmask[4] = {~0u, ~0u, ~0u, ~0u};
    if (PACKED && g.pk > 1) {
      const int me = pack_id(g, row);
#pragma unroll 1
      for (int j = 0; j < 128; ++j)
        if (pack_id(g, j) != me) pmask[j >> 5] &= ~(1u << (j & 31));
    }
    // the statistics (lse, D) of this thread's query row in a block, read one block ahead so
    // that their latency overlaps the previous block's dQ drain
    auto stats_of = [&](int item, int qb, float& lse_l2, float& dv) {
      lse_l2 = INFINITY;  // query columns past the problem: P = 0
      dv = 0.f;
      if (item >= args.total_items) return;
      const int prob = fdiv(item, g.f_nt);
      int j0 = 0;
      const int base = problem_base(g, prob, &j0);
      if (row < tile_valid_rows(g, qb) && (!PACKED || g.pk <= 1 || packed_row_live(g, j0, row))) {
        const int tk = base + tile_row_offset(g, qb, row);
        lse_l2 = __ldg(args.lse + tk) * log2e;
        dv = __ldg(args.Drow + tk);
      }
    };
    float nx_lse, nx_d;
    stats_of(blockIdx.x, 0, nx_lse, nx_d);
    uint32_t t = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < args.total_items; item += gridDim.x) {
      const int prob = fdiv(item, g.f_nt), kb = item - prob * nt;
      int j0 = 0;
      const int base = problem_base(g, prob, &j0);
      const bool rlive = row < tile_valid_rows(g, kb) && (!PACKED || g.pk <= 1 || packed_row_live(g, j0, row));
      for (int qb = 0; qb < nt; ++qb, ++t) {
        // per-query statistics of the block's query box: row r publishes column r
        float* vl = vec + (t & 1u) * 256;
        const bool qlive = row < tile_valid_rows(g, qb) && (!PACKED || g.pk <= 1 || packed_row_live(g, j0, row));
        const int tok = qlive ? base + tile_row_offset(g, qb, row) : 0;
        vl[row] = -nx_lse;  // negated: the gradient step adds them with paired instructions
        vl[128 + row] = -nx_d;
        mbar_arrive(&bars[G_VEC]);
        if (!(ok = wwait(&bars[G_VEC], t & 1u))) break;
        if (!(ok = wwait(&bars[G_SFULL], t & 1u))) break;
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          // this chunk's 32 query columns of the packed-box mask (selected, not indexed)
          const uint32_t pm = c == 0 ? pmask[0] : c == 1 ? pmask[1] : c == 2 ? pmask[2] : pmask[3];
          if (PACKED && __all_sync(0xffffffffu, pm == 0u)) {
            // no key row of this warp shares a problem with these query columns: P = dS = 0
            tmem_st16_zero(tS + c * 16);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int chunk = (c & 1) * 4 + j;
              st_shared_v4(ds_row + (c >> 1) * BLK + ((chunk ^ (row & 7)) << 4), 0u, 0u, 0u, 0u);
            }
            continue;
          }
          uint32_t s[32], dp[32];
          tmem_ld32(tS + c * 32, s);
          tmem_ld32(tDP + c * 32, dp);
          uint32_t pk[16], dk[16];
#pragma unroll
          for (int e4 = 0; e4 < 32; e4 += 4) {
            // column statistics, negated: -lse * log2(e) and -D of the block's query columns
            const float4 lc4 = *reinterpret_cast<const float4*>(vl + c * 32 + e4);
            const float4 dc4 = *reinterpret_cast<const float4*>(vl + 128 + c * 32 + e4);
            const uint64_t nl[2] = {f2(lc4.x, lc4.y), f2(lc4.z, lc4.w)};
            const uint64_t nd[2] = {f2(dc4.x, dc4.y), f2(dc4.z, dc4.w)};
#pragma unroll
            for (int u2 = 0; u2 < 2; ++u2) {
              const int e = e4 + 2 * u2;
              const uint64_t x2 = ffma2(f2(__uint_as_float(s[e]), __uint_as_float(s[e + 1])), c2x2, nl[u2]);
              // key rows past the problem, and in a packed box the query columns of other
              // problems: P = dS = 0 (a select: exp2 of a zero score may overflow)
              const bool same0 = !PACKED || ((pm >> e) & 1u), same1 = !PACKED || ((pm >> (e + 1)) & 1u);
              const float p0 = rlive && same0 ? ex2_approx(f2_lo(x2)) : 0.f;
              const float p1 = rlive && same1 ? ex2_approx(f2_hi(x2)) : 0.f;
              const uint64_t d2 = fadd2(f2(__uint_as_float(dp[e]), __uint_as_float(dp[e + 1])), nd[u2]);
              uint64_t ds2;
              asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(ds2) : "l"(f2(p0, p1)), "l"(d2));
              pk[e >> 1] = pack_bf16x2(p0, p1);
              dk[e >> 1] = pack_bf16x2(f2_lo(ds2), f2_hi(ds2));
            }
          }
          tmem_st16(tS + c * 16, pk);
          // dS^T row: query columns [32c, 32c+32) are 16-byte chunks 4(c&1)..4(c&1)+3 of block c>>1
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int chunk = (c & 1) * 4 + j;
            st_shared_v4(ds_row + (c >> 1) * BLK + ((chunk ^ (row & 7)) << 4), dk[4 * j], dk[4 * j + 1],
                         dk[4 * j + 2], dk[4 * j + 3]);
          }
        }
        tmem_st_wait();
        fence_async_smem();  // the dS^T tile is read by the tensor core
        tc_fence_before();
        mbar_arrive(&bars[G_PFULL]);
        if (qb + 1 < nt)
          stats_of(item, qb + 1, nx_lse, nx_d);
        else
          stats_of(item + int(gridDim.x), 0, nx_lse, nx_d);
        // the block's dQ part (TMEM lane = query row): drained here while the epilogue warps
        // drain dVal and dK, so the next block's dP^T, which reuses its columns, is not
        // queued behind the item's other accumulators
        if (!(ok = wwait(&bars[G_DQDONE], t & 1u))) break;
        tc_fence_after();
        if (nt > 1)
          epi_acc16<D, EPI_RED>(tDP, xps, lane, tok, qlive, args.scale, nullptr, args.acc_q);
        else
          epi_acc16<D, OUT_F32 ? EPI_F32 : EPI_BF16>(tDP, xps, lane, tok, qlive, args.scale, args.add_q, args.out_q);
        tc_fence_before();
        mbar_arrive(&bars[G_DQFREE]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (thread = token row)
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const uint32_t lane_sel = uint32_t(q4 * 32) << 16;
    const uint32_t xp = sbase + Lay::XP_OFF + q4 * 4096;
    auto wwait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, to)) != 0;
    };
    uint32_t i = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < args.total_items; item += gridDim.x, ++i) {
      const int prob = fdiv(item, g.f_nt), kb = item - prob * nt;
      int j0 = 0;
      const int base = problem_base(g, prob, &j0);
      const bool prow = !PACKED || g.pk <= 1 || packed_row_live(g, j0, row);
      const bool livek = row < tile_valid_rows(g, kb) && prow;
      const EpiRows RK = epi_rows_of(lane, livek ? base + tile_row_offset(g, kb, row) : 0, livek);
      if (!(ok = wwait(&bars[G_ITEMACC], i & 1u))) break;
      tc_fence_after();
      epi_acc_bf16<D>(tmem + lane_sel + Lay::TM_DV, xp, lane, RK, args.out_val, args.val, args.d_next);
      epi_acc<D, OUT_F32 ? EPI_F32 : EPI_BF16>(tmem + lane_sel + Lay::TM_DK, xp, lane, RK, args.scale, args.add_k,
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
