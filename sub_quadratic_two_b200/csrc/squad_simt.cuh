// squad_simt.cuh - CUDA-core (FMA) kernels for one pass of SQuad-Attention.
//
// These serve the fp32 path (float inputs, float arithmetic, expf/logf) and the
// backward of the bf16 path. One warp owns one query row (forward, dq) or one
// key row (dk, dv); the 32 lanes split the head dimension and reduce dot
// products with warp shuffles. Every pass is described by a Geom (geometry.h),
// so the same kernels run the local (window) pass and the global
// (cross-window) pass.
//
// Pass backward, for P_ij = exp(s*<q_i,k_j> - lse_i), dP_ij = <dO_i, val_j>,
// D_i = <dO_i, O_i> (= sum_j P_ij dP_ij) and dS_ij = P_ij (dP_ij - D_i):
//   dq_i = s * sum_j dS_ij k_j,  dk_j = s * sum_i dS_ij q_i,  dval_j = sum_i P_ij dO_i.
#pragma once
#include <cuda_bf16.h>
#include "geometry.h"

namespace sq {

constexpr int kSimtWarps = 4;

__device__ __forceinline__ float ld_f(const float* p) { return *p; }
__device__ __forceinline__ float ld_f(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st_f(float* p, float x) { *p = x; }
__device__ __forceinline__ void st_f(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Forward of one pass: out_i = sum_j softmax_j(s <q_i,k_j>) val_j, online over j.
template <typename T, int DPL>
__global__ void __launch_bounds__(kSimtWarps * 32) simt_fwd_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                                  const T* __restrict__ val, T* __restrict__ out,
                                                                  float* __restrict__ lse, Geom g, int d,
                                                                  float scale) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.y * kSimtWarps + warp;
  if (i >= g.L) return;
  const int base = problem_base(g, blockIdx.x);
  const long long ti = base + row_offset(g, i);
  float qv[DPL], acc[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) {
    qv[e] = ld_f(q + ti * d + lane + 32 * e);
    acc[e] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  for (int j = 0; j < g.L; ++j) {
    const long long tj = base + row_offset(g, j);
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < DPL; ++e) s = fmaf(qv[e], ld_f(k + tj * d + lane + 32 * e), s);
    s = warp_sum(s) * scale;
    const float m_new = fmaxf(m, s);
    const float corr = expf(m - m_new);
    const float p = expf(s - m_new);
    l = l * corr + p;
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[e] = fmaf(acc[e], corr, p * ld_f(val + tj * d + lane + 32 * e));
    m = m_new;
  }
  const float inv = 1.f / l;
#pragma unroll
  for (int e = 0; e < DPL; ++e) st_f(out + ti * d + lane + 32 * e, acc[e] * inv);
  if (lse != nullptr && lane == 0) lse[ti] = m + logf(l);
}

// D_t = <a_t, b_t> for every token t (one warp per token).
template <typename T, int DPL>
__global__ void __launch_bounds__(kSimtWarps * 32) simt_rowdot_kernel(const T* __restrict__ a, const T* __restrict__ b,
                                                                     float* __restrict__ out, long long rows, int d) {
  const long long t = (long long)blockIdx.x * kSimtWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= rows) return;
  float s = 0.f;
#pragma unroll
  for (int e = 0; e < DPL; ++e) s = fmaf(ld_f(a + t * d + lane + 32 * e), ld_f(b + t * d + lane + 32 * e), s);
  s = warp_sum(s);
  if (lane == 0) out[t] = s;
}

// dq_i = s * sum_j dS_ij k_j (+ dq_add_i), one warp per query row.
template <typename T, typename TO, int DPL>
__global__ void __launch_bounds__(kSimtWarps * 32) simt_bwd_dq_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ val, const T* __restrict__ dout,
    const float* __restrict__ lse, const float* __restrict__ Drow, const float* __restrict__ dq_add,
    TO* __restrict__ dq, Geom g, int d, float scale) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.y * kSimtWarps + warp;
  if (i >= g.L) return;
  const int base = problem_base(g, blockIdx.x);
  const long long ti = base + row_offset(g, i);
  float qv[DPL], gv[DPL], acc[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) {
    qv[e] = ld_f(q + ti * d + lane + 32 * e);
    gv[e] = ld_f(dout + ti * d + lane + 32 * e);
    acc[e] = 0.f;
  }
  const float li = lse[ti], Di = Drow[ti];
  for (int j = 0; j < g.L; ++j) {
    const long long tj = base + row_offset(g, j);
    float s = 0.f, dp = 0.f;
#pragma unroll
    for (int e = 0; e < DPL; ++e) {
      s = fmaf(qv[e], ld_f(k + tj * d + lane + 32 * e), s);
      dp = fmaf(gv[e], ld_f(val + tj * d + lane + 32 * e), dp);
    }
    s = warp_sum(s);
    dp = warp_sum(dp);
    const float p = expf(s * scale - li);
    const float ds = p * (dp - Di);
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[e] = fmaf(ds, ld_f(k + tj * d + lane + 32 * e), acc[e]);
  }
#pragma unroll
  for (int e = 0; e < DPL; ++e) {
    float r = acc[e] * scale;
    if (dq_add != nullptr) r += dq_add[ti * d + lane + 32 * e];
    st_f(dq + ti * d + lane + 32 * e, r);
  }
}

// dk_j = s * sum_i dS_ij q_i (+ dk_add_j), dval_j = sum_i P_ij dO_i, one warp per key row.
template <typename T, typename TOK, typename TOV, int DPL>
__global__ void __launch_bounds__(kSimtWarps * 32) simt_bwd_dkdv_kernel(
    const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ val, const T* __restrict__ dout,
    const float* __restrict__ lse, const float* __restrict__ Drow, const float* __restrict__ dk_add,
    TOK* __restrict__ dk, TOV* __restrict__ dval, Geom g, int d, float scale) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.y * kSimtWarps + warp;
  if (j >= g.L) return;
  const int base = problem_base(g, blockIdx.x);
  const long long tj = base + row_offset(g, j);
  float kv[DPL], vv[DPL], ak[DPL], av[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) {
    kv[e] = ld_f(k + tj * d + lane + 32 * e);
    vv[e] = ld_f(val + tj * d + lane + 32 * e);
    ak[e] = 0.f;
    av[e] = 0.f;
  }
  for (int i = 0; i < g.L; ++i) {
    const long long ti = base + row_offset(g, i);
    float s = 0.f, dp = 0.f;
#pragma unroll
    for (int e = 0; e < DPL; ++e) {
      s = fmaf(ld_f(q + ti * d + lane + 32 * e), kv[e], s);
      dp = fmaf(ld_f(dout + ti * d + lane + 32 * e), vv[e], dp);
    }
    s = warp_sum(s);
    dp = warp_sum(dp);
    const float p = expf(s * scale - lse[ti]);
    const float ds = p * (dp - Drow[ti]);
#pragma unroll
    for (int e = 0; e < DPL; ++e) {
      ak[e] = fmaf(ds, ld_f(q + ti * d + lane + 32 * e), ak[e]);
      av[e] = fmaf(p, ld_f(dout + ti * d + lane + 32 * e), av[e]);
    }
  }
#pragma unroll
  for (int e = 0; e < DPL; ++e) {
    float r = ak[e] * scale;
    if (dk_add != nullptr) r += dk_add[tj * d + lane + 32 * e];
    st_f(dk + tj * d + lane + 32 * e, r);
    st_f(dval + tj * d + lane + 32 * e, av[e]);
  }
}

}  // namespace sq
