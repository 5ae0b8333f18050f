// squad_api.cu - the C ABI of libsquad (declared in include/squad.h).
//
// Host side only: argument checks, the per-pass geometry, TMA tensor maps and
// kernel launches on the caller's stream. No allocation, no synchronisation
// (except squad_poll_device_error, which says so).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "squad.h"
#include "geometry.h"
#include "squad_bwd_fused.cuh"
#include "squad_fwd_tc.cuh"
#include "squad_simt.cuh"
#include "tmap_cache.h"
#include "sp_plan.h"
#include "squad_sp.cuh"

namespace {

using sq::Geom;

constexpr int kVersion = 1 * 10000 + 0 * 100 + 0;
constexpr int kMaxDevices = 64;
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;  // 2 s per wait: far above any legitimate wait
constexpr int kFusedLag = 2;  // heads between a local pass and its global pass (see decode_item)
constexpr int kMultiLag = 2;  // heads between pass j-1 and pass j of a head in the k-pass launch

thread_local int t_last_cuda = 0;

__device__ int g_squad_dev_err;  // set by kernels that gave up on a bounded wait

squad_status cuda_fail(int code) {
  t_last_cuda = code;
  return SQUAD_ERR_CUDA;
}

#define SQ_CUDA(call)                                   \
  do {                                                  \
    cudaError_t e_ = (call);                            \
    if (e_ != cudaSuccess) return cuda_fail(int(e_));   \
  } while (0)

// ---------------------------------------------------------------- per-device state

struct DeviceState {
  bool ready = false;
  int sms = 0;
  int l2_bytes = 0;
  int* err = nullptr;          // device address of g_squad_dev_err
  bool fwd_attr_set[2][2] = {};  // [D=64/128][packed]
  bool fused_attr_set[2][2][2] = {};   // [D=64/128][out_f32][packed]
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

squad_status device_state(DeviceState** out) {
  int dev = 0;
  SQ_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return SQUAD_ERR_UNSUPPORTED;
  // binds the device's primary context to this thread (a thread that has made no runtime
  // call yet, such as an autograd worker, has none, and the tensor-map encoder needs it)
  SQ_CUDA(cudaSetDevice(dev));
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState& s = g_dev[dev];
  if (!s.ready) {
    SQ_CUDA(cudaDeviceGetAttribute(&s.sms, cudaDevAttrMultiProcessorCount, dev));
    SQ_CUDA(cudaDeviceGetAttribute(&s.l2_bytes, cudaDevAttrL2CacheSize, dev));
    void* p = nullptr;
    SQ_CUDA(cudaGetSymbolAddress(&p, g_squad_dev_err));
    s.err = static_cast<int*>(p);
    if (g_encode == nullptr) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
      SQ_CUDA(cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q));
      if (q != cudaDriverEntryPointSuccess || fn == nullptr) return cuda_fail(int(cudaErrorSymbolNotFound));
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    s.ready = true;
  }
  *out = &s;
  return SQUAD_OK;
}

// ---------------------------------------------------------------- argument checks

struct Plan {
  Geom g1, g2;        // local pass, global pass
  long long rows;     // B*heads*n
  size_t elem;        // bytes per element of q/k/v/o
  float scale;
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// with_passes = false checks the tensors only (the k-pass entry points plan their own passes)
squad_status make_plan(const squad_desc* d, Plan* p, bool with_passes = true) {
  if (d == nullptr) return SQUAD_ERR_INVALID_ARG;
  if (d->dtype != SQUAD_F32 && d->dtype != SQUAD_BF16) return SQUAD_ERR_INVALID_ARG;
  if (d->B <= 0 || d->heads <= 0 || d->d <= 0 || d->T <= 0 || d->H <= 0 || d->W <= 0 || d->tT <= 0 ||
      d->tH <= 0 || d->tW <= 0)
    return SQUAD_ERR_SHAPE;
  if (d->T % d->tT || d->H % d->tH || d->W % d->tW) return SQUAD_ERR_SHAPE;
  const long long n = (long long)d->T * d->H * d->W;
  const long long rows = n * d->B * d->heads;
  if (rows >= (1ll << 31) || rows * d->d >= (1ll << 40)) return SQUAD_ERR_SHAPE;
  if (!(d->scale > 0.f) && !(d->scale <= 0.f)) return SQUAD_ERR_INVALID_ARG;  // NaN
  if (d->dtype == SQUAD_BF16) {
    if (d->d != 64 && d->d != 128) return SQUAD_ERR_UNSUPPORTED;
  } else {
    if (d->d % 32 != 0 || d->d > 256) return SQUAD_ERR_UNSUPPORTED;
  }
  if (with_passes) {
    p->g1 = sq::make_geom(1, d->B, d->heads, d->T, d->H, d->W, d->tT, d->tH, d->tW);
    p->g2 = sq::make_geom(2, d->B, d->heads, d->T, d->H, d->W, d->tT, d->tH, d->tW);
    if (d->dtype == SQUAD_BF16) {
      if (!sq::plan_tiles(p->g1) || !sq::plan_tiles(p->g2)) return SQUAD_ERR_UNSUPPORTED;
    }
  }
  p->rows = rows;
  p->elem = d->dtype == SQUAD_BF16 ? 2 : 4;
  p->scale = d->scale > 0.f ? d->scale : 1.0f / std::sqrt(float(d->d));
  return SQUAD_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Forward workspace: [local-pass output, only when the caller passes no o1][per-head counters].
size_t fwd_o1_bytes(const Plan& p, const squad_desc* d) { return align256(p.rows * d->d * p.elem); }
size_t fwd_counter_bytes(const squad_desc* d) { return align256(size_t(d->B) * d->heads * sizeof(uint32_t)); }
size_t fwd_workspace(const Plan& p, const squad_desc* d) { return fwd_o1_bytes(p, d) + fwd_counter_bytes(d); }

struct BwdWs {
  size_t do1, dq2, dk2, D2, D1, total;
};

BwdWs bwd_workspace(const Plan& p, const squad_desc* d) {
  BwdWs w{};
  const size_t big = p.rows * d->d;
  w.do1 = 0;
  w.dq2 = w.do1 + align256(big * p.elem);
  w.dk2 = w.dq2 + align256(big * 4);
  w.D2 = w.dk2 + align256(big * 4);
  w.D1 = w.D2 + align256(p.rows * 4);
  w.total = w.D1 + align256(p.rows * 4);
  return w;
}

// ---------------------------------------------------------------- tensor maps

// 5-D map over a [rows, d] bf16 tensor: (d, a, b, c, token) with the problem box's
// token strides; boxes of (64, a_n, b_sub, c_sub, 1), 128-byte swizzle.
// Encoded maps are reused by later calls with the same pointers and shapes (tmap_cache.h).
sq::TmapCache<128> g_tmaps;

squad_status encode_map(CUtensorMap* m, const void* base, const Geom& g, int d, long long rows) {
  const cuuint64_t esz = 2;
  // a packed dimension spans the packed digit's full extent (its rows past that extent read as zeros)
  cuuint64_t dims[5] = {cuuint64_t(d), cuuint64_t(g.pk_dim == 0 ? g.pk_ext : g.a_n),
                        cuuint64_t(g.pk_dim == 1 ? g.pk_ext : g.b_n), cuuint64_t(g.pk_dim == 2 ? g.pk_ext : g.c_n),
                        cuuint64_t(rows)};
  cuuint64_t strides[4] = {cuuint64_t(g.sA) * d * esz, cuuint64_t(g.sB) * d * esz, cuuint64_t(g.sC) * d * esz,
                           cuuint64_t(d) * esz};
  cuuint32_t box[5] = {64u, cuuint32_t(g.a_n), cuuint32_t(g.b_sub), cuuint32_t(g.c_sub), 1u};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  int dev = 0;
  SQ_CUDA(cudaGetDevice(&dev));
  const sq::TmapKey key = sq::make_tmap_key(dev, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, CU_TENSOR_MAP_SWIZZLE_128B, 5, base,
                                            dims, strides, box);
  CUresult r = g_tmaps.get(key, m, [&](CUtensorMap* out) {
    return g_encode(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  });
  if (r != CUDA_SUCCESS) return cuda_fail(int(r));
  return SQUAD_OK;
}

// ---------------------------------------------------------------- launches

sq::PassArgs pass_args(const Geom& g, void* out, float* lse) {
  sq::PassArgs pa{};
  pa.g = g;
  pa.out = out;
  pa.lse = lse;
  pa.jobs_per_bh = g.probs * g.nt;
  pa.pairs_per_bh = (pa.jobs_per_bh + 1) / 2;
  return pa;
}

template <int D, bool PACKED>
squad_status launch_fwd_tc_t(DeviceState* ds, const sq::FwdMaps& m, const sq::FwdArgs& a, cudaStream_t st) {
  using Lay = sq::FwdLayout<D>;
  auto kern = sq::squad_fwd_tc_kernel<D, PACKED>;
  bool& attr = ds->fwd_attr_set[D == 128 ? 1 : 0][PACKED ? 1 : 0];
  if (!attr) {
    SQ_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::ALLOC));
    attr = true;
  }
  const int grid = a.total_items < ds->sms ? a.total_items : ds->sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(grid));
  cfg.blockDim = dim3(sq::kFwdThreads);
  cfg.dynamicSmemBytes = Lay::ALLOC;
  cfg.stream = st;
  cudaLaunchAttribute attrs[1];
  // Chained passes have CTAs wait on other CTAs' progress: require co-residency.
  attrs[0].id = cudaLaunchAttributeCooperative;
  attrs[0].val.cooperative = (a.mode == sq::FWD_FUSED || a.mode == sq::FWD_MULTI) ? 1 : 0;
  cfg.attrs = attrs;
  cfg.numAttrs = 1;
  SQ_CUDA(cudaLaunchKernelEx(&cfg, kern, m, a));
  return SQUAD_OK;
}

// Forward launch. mode FWD_LOCAL: out1 = local pass of (q, k, val1). FWD_GLOBAL: out2 =
// global pass of (q, k, val2). FWD_FUSED: both, the global pass reading out1 (= val2).
squad_status launch_fwd_tc(DeviceState* ds, int d, int mode, const Plan& p, const void* q, const void* k,
                           const void* val1, void* out1, float* lse1, const void* val2, void* out2, float* lse2,
                           uint32_t* counters, const void* discard, cudaStream_t st) {
  sq::FwdMaps maps;
  CUtensorMap* m = maps.m;
  squad_status s;
  const bool do1 = mode != sq::FWD_GLOBAL, do2 = mode != sq::FWD_LOCAL;
  if (do1) {
    if ((s = encode_map(&m[0], q, p.g1, d, p.rows)) != SQUAD_OK) return s;
    if ((s = encode_map(&m[1], k, p.g1, d, p.rows)) != SQUAD_OK) return s;
    if ((s = encode_map(&m[2], val1, p.g1, d, p.rows)) != SQUAD_OK) return s;
    if ((s = encode_map(&m[3], out1, p.g1, d, p.rows)) != SQUAD_OK) return s;
  }
  if (do2) {
    if ((s = encode_map(&m[4], q, p.g2, d, p.rows)) != SQUAD_OK) return s;
    if ((s = encode_map(&m[5], k, p.g2, d, p.rows)) != SQUAD_OK) return s;
    if ((s = encode_map(&m[6], val2, p.g2, d, p.rows)) != SQUAD_OK) return s;
    if ((s = encode_map(&m[7], out2, p.g2, d, p.rows)) != SQUAD_OK) return s;
  }
  for (int i = 0; i < 4; ++i) {  // the pass that does not run gets copies of valid maps
    if (!do1) m[i] = m[4 + i];
    if (!do2) m[4 + i] = m[i];
  }
  for (int i = 8; i < 4 * sq::kMaxFwdPasses; ++i) m[i] = m[i & 7];  // unused
  sq::FwdArgs a{};
  a.npass = 2;
  a.ps[0] = pass_args(p.g1, out1, lse1);
  a.ps[1] = pass_args(p.g2, out2, lse2);
  a.mode = mode;
  a.bh = p.g1.bh;
  a.lag = kFusedLag < a.bh ? kFusedLag : a.bh;
  a.total_items = (do1 ? a.bh * a.ps[0].pairs_per_bh : 0) + (do2 ? a.bh * a.ps[1].pairs_per_bh : 0);
  a.f_n1 = sq::make_fastdiv(uint32_t(a.ps[0].pairs_per_bh));
  a.f_n2 = sq::make_fastdiv(uint32_t(a.ps[1].pairs_per_bh));
  a.f_n12 = sq::make_fastdiv(uint32_t(a.ps[0].pairs_per_bh + a.ps[1].pairs_per_bh));
  a.scale_log2 = p.scale * 1.4426950408889634f;
  a.counters = counters;
  a.ps[1].discard = static_cast<const uint8_t*>(discard);
  a.err = ds->err;
  a.timeout_ns = kWaitTimeoutNs;
  if (mode == sq::FWD_FUSED) SQ_CUDA(cudaMemsetAsync(counters, 0, size_t(a.bh) * sizeof(uint32_t), st));
  const bool packed = p.g1.pk > 1 || p.g2.pk > 1;
  if (d == 128) return packed ? launch_fwd_tc_t<128, true>(ds, maps, a, st) : launch_fwd_tc_t<128, false>(ds, maps, a, st);
  return packed ? launch_fwd_tc_t<64, true>(ds, maps, a, st) : launch_fwd_tc_t<64, false>(ds, maps, a, st);
}

dim3 simt_grid(const Geom& g) { return dim3(unsigned(g.bh * g.probs), unsigned(sq::ceil_div(g.L, sq::kSimtWarps))); }

template <typename T, int DPL>
squad_status simt_fwd_t(const Geom& g, const void* q, const void* k, const void* val, void* out, float* lse, int d,
                        float scale, cudaStream_t st) {
  sq::simt_fwd_kernel<T, DPL><<<simt_grid(g), sq::kSimtWarps * 32, 0, st>>>(
      static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(val), static_cast<T*>(out), lse, g,
      d, scale);
  SQ_CUDA(cudaGetLastError());
  return SQUAD_OK;
}

template <typename T>
squad_status simt_fwd(const Geom& g, const void* q, const void* k, const void* val, void* out, float* lse, int d,
                      float scale, cudaStream_t st) {
  switch (d / 32) {
    case 1: return simt_fwd_t<T, 1>(g, q, k, val, out, lse, d, scale, st);
    case 2: return simt_fwd_t<T, 2>(g, q, k, val, out, lse, d, scale, st);
    case 3: return simt_fwd_t<T, 3>(g, q, k, val, out, lse, d, scale, st);
    case 4: return simt_fwd_t<T, 4>(g, q, k, val, out, lse, d, scale, st);
    case 5: return simt_fwd_t<T, 5>(g, q, k, val, out, lse, d, scale, st);
    case 6: return simt_fwd_t<T, 6>(g, q, k, val, out, lse, d, scale, st);
    case 7: return simt_fwd_t<T, 7>(g, q, k, val, out, lse, d, scale, st);
    case 8: return simt_fwd_t<T, 8>(g, q, k, val, out, lse, d, scale, st);
  }
  return SQUAD_ERR_UNSUPPORTED;
}

// Backward of one pass on the CUDA cores: D = rowdot(dout, out); dq; dk and dval.
template <typename T, typename TOQ, typename TOK, typename TOV, int DPL>
squad_status simt_pass_bwd_t(const Geom& g, long long rows, const T* q, const T* k, const T* val, const T* out,
                             const T* dout, const float* lse, float* Drow, const float* dq_add, TOQ* dq,
                             const float* dk_add, TOK* dk, TOV* dval, int d, float scale, cudaStream_t st) {
  const unsigned rblocks = unsigned((rows + sq::kSimtWarps - 1) / sq::kSimtWarps);
  sq::simt_rowdot_kernel<T, DPL><<<rblocks, sq::kSimtWarps * 32, 0, st>>>(dout, out, Drow, rows, d);
  SQ_CUDA(cudaGetLastError());
  sq::simt_bwd_dq_kernel<T, TOQ, DPL>
      <<<simt_grid(g), sq::kSimtWarps * 32, 0, st>>>(q, k, val, dout, lse, Drow, dq_add, dq, g, d, scale);
  SQ_CUDA(cudaGetLastError());
  sq::simt_bwd_dkdv_kernel<T, TOK, TOV, DPL>
      <<<simt_grid(g), sq::kSimtWarps * 32, 0, st>>>(q, k, val, dout, lse, Drow, dk_add, dk, dval, g, d, scale);
  SQ_CUDA(cudaGetLastError());
  return SQUAD_OK;
}

template <typename T, int DPL>
squad_status simt_bwd_t(const Plan& p, const BwdWs& w, uint8_t* ws, const void* q, const void* k, const void* v,
                        const void* o, const void* o1, const float* lse1, const float* lse2, const void* dout,
                        void* dq, void* dk, void* dv, int d, cudaStream_t st) {
  const T* Q = static_cast<const T*>(q);
  const T* K = static_cast<const T*>(k);
  T* dO1 = reinterpret_cast<T*>(ws + w.do1);
  float* dQ2 = reinterpret_cast<float*>(ws + w.dq2);
  float* dK2 = reinterpret_cast<float*>(ws + w.dk2);
  float* D2 = reinterpret_cast<float*>(ws + w.D2);
  float* D1 = reinterpret_cast<float*>(ws + w.D1);
  squad_status s;
  // global pass: values O1, upstream dout -> dQ2, dK2 (fp32) and dO1
  s = simt_pass_bwd_t<T, float, float, T, DPL>(p.g2, p.rows, Q, K, static_cast<const T*>(o1),
                                               static_cast<const T*>(o), static_cast<const T*>(dout), lse2, D2,
                                               nullptr, dQ2, nullptr, dK2, dO1, d, p.scale, st);
  if (s != SQUAD_OK) return s;
  // local pass: values V, upstream dO1 -> dq = dq1 + dQ2, dk = dk1 + dK2, dv
  return simt_pass_bwd_t<T, T, T, T, DPL>(p.g1, p.rows, Q, K, static_cast<const T*>(v), static_cast<const T*>(o1),
                                          dO1, lse1, D1, dQ2, static_cast<T*>(dq), dK2, static_cast<T*>(dk),
                                          static_cast<T*>(dv), d, p.scale, st);
}

// ---------------- tensor-core backward (bf16)

template <int D, bool F32, bool PACKED>
squad_status launch_bwd_fused_t(DeviceState* ds, const CUtensorMap* maps, const sq::BwdFusedArgs& a,
                                cudaStream_t st) {
  using Lay = sq::BwdFusedLayout<D>;
  auto kern = sq::squad_bwd_fused_kernel<D, F32, PACKED>;
  bool& attr = ds->fused_attr_set[D == 128 ? 1 : 0][F32 ? 1 : 0][PACKED ? 1 : 0];
  if (!attr) {
    SQ_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Lay::ALLOC));
    attr = true;
  }
  const int grid = a.total_items < ds->sms ? a.total_items : ds->sms;
  kern<<<grid, sq::kBwdFusedThreads, Lay::ALLOC, st>>>(maps[0], maps[1], maps[2], maps[3], a);
  SQ_CUDA(cudaGetLastError());
  return SQUAD_OK;
}

// Backward of one pass on the tensor cores. q, k: inputs; val: the pass's values;
// out: the pass's output; dout: its upstream gradient. f32_out selects fp32 dq/dk
// (the global pass, whose parts are summed into the local pass's results).
squad_status tc_pass_bwd(DeviceState* ds, const Plan& p, int d, const Geom& g, const void* q, const void* k,
                         const void* val, const void* out, const void* dout, const float* lse, const float* Drow,
                         float* d_next, const float* dq_add, float* dq_acc, void* dq, const float* dk_add, void* dk,
                         __nv_bfloat16* dval, bool f32_out, cudaStream_t st) {
  CUtensorMap maps[4];
  squad_status s;
  if ((s = encode_map(&maps[0], q, g, d, p.rows)) != SQUAD_OK) return s;
  if ((s = encode_map(&maps[1], k, g, d, p.rows)) != SQUAD_OK) return s;
  if ((s = encode_map(&maps[2], val, g, d, p.rows)) != SQUAD_OK) return s;
  if ((s = encode_map(&maps[3], dout, g, d, p.rows)) != SQUAD_OK) return s;
  // one kernel: every (query box, key box) block once; dk and dval complete per key box
  sq::BwdFusedArgs f{};
  f.g = g;
  f.total_items = g.bh * g.probs * g.nt;
  f.scale = p.scale;
  f.scale_log2 = p.scale * 1.4426950408889634f;
  f.lse = lse;
  if (Drow == nullptr) return SQUAD_ERR_INVALID_ARG;
  f.Drow = Drow;
  f.val = static_cast<const __nv_bfloat16*>(val);
  f.d_next = d_next;
  f.add_k = dk_add;
  f.out_k = dk;
  f.out_val = dval;
  f.err = ds->err;
  f.timeout_ns = kWaitTimeoutNs;
  const size_t n_el = size_t(p.rows) * d;
  if (g.nt == 1) {
    f.add_q = dq_add;  // dq = part (+ add), stored directly
    f.out_q = dq;
  } else if (f32_out) {
    // dq (fp32) = add + sum of the parts of every key box
    f.acc_q = static_cast<float*>(dq);
    if (dq_add != nullptr)
      SQ_CUDA(cudaMemcpyAsync(dq, dq_add, n_el * sizeof(float), cudaMemcpyDeviceToDevice, st));
    else
      SQ_CUDA(cudaMemsetAsync(dq, 0, n_el * sizeof(float), st));
  } else {
    // dq (bf16) = bf16(add + sum of the parts): the parts are added into the fp32 addend
    if (dq_acc == nullptr) return SQUAD_ERR_INVALID_ARG;
    f.acc_q = dq_acc;
  }
  // packed boxes (problems of at most 64 tokens several to a box) take the masked instance
  const bool packed = g.pk > 1;
  squad_status s2;
  if (d == 128)
    s2 = f32_out ? (packed ? launch_bwd_fused_t<128, true, true>(ds, maps, f, st)
                           : launch_bwd_fused_t<128, true, false>(ds, maps, f, st))
                 : (packed ? launch_bwd_fused_t<128, false, true>(ds, maps, f, st)
                           : launch_bwd_fused_t<128, false, false>(ds, maps, f, st));
  else
    s2 = f32_out ? (packed ? launch_bwd_fused_t<64, true, true>(ds, maps, f, st)
                           : launch_bwd_fused_t<64, true, false>(ds, maps, f, st))
                 : (packed ? launch_bwd_fused_t<64, false, true>(ds, maps, f, st)
                           : launch_bwd_fused_t<64, false, false>(ds, maps, f, st));
  if (s2 != SQUAD_OK || g.nt == 1 || f32_out) return s2;
  const unsigned cblocks = unsigned((n_el / 8 + 255) / 256);
  sq::f32_to_bf16_kernel<<<cblocks, 256, 0, st>>>(dq_acc, static_cast<__nv_bfloat16*>(dq), n_el / 8);
  SQ_CUDA(cudaGetLastError());
  return SQUAD_OK;
}

// D = rowsum(a o b) over bf16 [rows, d] tensors into an fp32 vector.
squad_status rowdot_bf16(const void* a, const void* b, float* out, long long rows, int d, cudaStream_t st) {
  const long long threads = rows * (d / 8);
  sq::rowdot_bf16_kernel<<<unsigned((threads + 255) / 256), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(a), static_cast<const __nv_bfloat16*>(b), out, rows, d);
  SQ_CUDA(cudaGetLastError());
  return SQUAD_OK;
}

squad_status tc_bwd(DeviceState* ds, const Plan& p, const BwdWs& w, uint8_t* ws, const void* q, const void* k,
                    const void* v, const void* o, const void* o1, const float* lse1, const float* lse2,
                    const void* dout, void* dq, void* dk, void* dv, int d, cudaStream_t st) {
  auto* dO1 = reinterpret_cast<__nv_bfloat16*>(ws + w.do1);
  float* dQ2 = reinterpret_cast<float*>(ws + w.dq2);
  float* dK2 = reinterpret_cast<float*>(ws + w.dk2);
  float* D1 = reinterpret_cast<float*>(ws + w.D1);
  float* D2 = reinterpret_cast<float*>(ws + w.D2);
  squad_status s;
  // D2 = rowsum(dout o O) by a bandwidth-bound row-dot pass (in the backward kernel these
  // loads would sit on each block's critical path)
  if ((s = rowdot_bf16(dout, o, D2, p.rows, d, st)) != SQUAD_OK) return s;
  // global pass: values O1, output O, upstream dout -> dQ2, dK2 (fp32), dO1 and the
  // local pass's D1 = rowsum(dO1 o O1)
  s = tc_pass_bwd(ds, p, d, p.g2, q, k, o1, o, dout, lse2, D2, D1, nullptr, nullptr, dQ2, nullptr, dK2, dO1,
                  true, st);
  if (s != SQUAD_OK) return s;
  // local pass: values V, output O1, upstream dO1 -> dq = dq1 + dQ2, dk = dk1 + dK2, dv
  return tc_pass_bwd(ds, p, d, p.g1, q, k, v, o1, dO1, lse1, D1, nullptr, dQ2, dQ2, dq, dK2, dk,
                     static_cast<__nv_bfloat16*>(dv), false, st);
}

template <typename T>
squad_status simt_bwd(const Plan& p, const BwdWs& w, uint8_t* ws, const void* q, const void* k, const void* v,
                      const void* o, const void* o1, const float* lse1, const float* lse2, const void* dout, void* dq,
                      void* dk, void* dv, int d, cudaStream_t st) {
  switch (d / 32) {
    case 1: return simt_bwd_t<T, 1>(p, w, ws, q, k, v, o, o1, lse1, lse2, dout, dq, dk, dv, d, st);
    case 2: return simt_bwd_t<T, 2>(p, w, ws, q, k, v, o, o1, lse1, lse2, dout, dq, dk, dv, d, st);
    case 3: return simt_bwd_t<T, 3>(p, w, ws, q, k, v, o, o1, lse1, lse2, dout, dq, dk, dv, d, st);
    case 4: return simt_bwd_t<T, 4>(p, w, ws, q, k, v, o, o1, lse1, lse2, dout, dq, dk, dv, d, st);
    case 5: return simt_bwd_t<T, 5>(p, w, ws, q, k, v, o, o1, lse1, lse2, dout, dq, dk, dv, d, st);
    case 6: return simt_bwd_t<T, 6>(p, w, ws, q, k, v, o, o1, lse1, lse2, dout, dq, dk, dv, d, st);
    case 7: return simt_bwd_t<T, 7>(p, w, ws, q, k, v, o, o1, lse1, lse2, dout, dq, dk, dv, d, st);
    case 8: return simt_bwd_t<T, 8>(p, w, ws, q, k, v, o, o1, lse1, lse2, dout, dq, dk, dv, d, st);
  }
  return SQUAD_ERR_UNSUPPORTED;
}

}  // namespace

// One thread waits on a barrier that nothing completes: the bounded wait gives up
// after timeout_ns and the error word is set (the test of the device timeout path).
__global__ void selftest_timeout_kernel(int* err, uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    sq::mbar_init(&bar, 1);
    abort_flag = 0;
    sq::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !sq::mbar_wait(&bar, 0, &abort_flag, timeout_ns)) atomicCAS(err, 0, 1);
}

// ==================================================================== C ABI

extern "C" {

squad_status squad_attn_workspace_size(const squad_desc* desc, int which, size_t* bytes) {
  if (bytes == nullptr) return SQUAD_ERR_INVALID_ARG;
  Plan p;
  squad_status s = make_plan(desc, &p);
  if (s != SQUAD_OK) return s;
  if (which == 0) {
    *bytes = fwd_workspace(p, desc);
  } else if (which == 2) {
    *bytes = fwd_counter_bytes(desc);
  } else if (which == 1) {
    *bytes = bwd_workspace(p, desc).total;
  } else {
    return SQUAD_ERR_INVALID_ARG;
  }
  return SQUAD_OK;
}

squad_status squad_attn_fwd(const squad_desc* desc, const void* q, const void* k, const void* v, void* o, void* o1,
                            float* lse1, float* lse2, void* workspace, size_t workspace_bytes, void* stream) {
  Plan p;
  squad_status s = make_plan(desc, &p);
  if (s != SQUAD_OK) return s;
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) return SQUAD_ERR_INVALID_ARG;
  void* o1buf = o1;
  uint32_t* counters = nullptr;
  if (o1buf == nullptr) {
    if (workspace == nullptr || workspace_bytes < fwd_workspace(p, desc)) return SQUAD_ERR_WORKSPACE;
    o1buf = workspace;
    counters = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) + fwd_o1_bytes(p, desc));
  } else if (workspace != nullptr && workspace_bytes >= fwd_counter_bytes(desc)) {
    counters = static_cast<uint32_t*>(workspace);
  }
  for (const void* ptr : {q, k, v, static_cast<const void*>(o), static_cast<const void*>(o1buf),
                          static_cast<const void*>(lse1), static_cast<const void*>(lse2),
                          static_cast<const void*>(counters)})
    if (!aligned16(ptr)) return SQUAD_ERR_ALIGN;
  DeviceState* ds = nullptr;
  if ((s = device_state(&ds)) != SQUAD_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int d = desc->d;
  if (desc->dtype == SQUAD_BF16) {
    // One launch, the global pass of each head right behind its local pass, only pays when
    // the heads in flight (the lag plus one) keep their Q, K and O1 in L2; otherwise (the
    // 53,680-token shape: 3 x 41 MB) the global pass reads them from DRAM anyway and its
    // waits on the local pass cost time, so the passes run as two launches.
    const double head_bytes = 3.0 * double(p.g1.n) * d * p.elem;
    const bool fits = (kFusedLag + 1) * head_bytes <= 0.6 * double(ds->l2_bytes);
    if (counters != nullptr && fits) {
      // one launch: the global pass of each head runs right behind its local pass; without
      // a caller o1 the local-pass rows are dropped from L2 once the global pass has read them
      const bool drop = o1 == nullptr && (reinterpret_cast<uintptr_t>(o1buf) & 127u) == 0;
      return launch_fwd_tc(ds, d, sq::FWD_FUSED, p, q, k, v, o1buf, lse1, o1buf, o, lse2, counters,
                           drop ? o1buf : nullptr, st);
    }
    if ((s = launch_fwd_tc(ds, d, sq::FWD_LOCAL, p, q, k, v, o1buf, lse1, nullptr, nullptr, nullptr, nullptr,
                           nullptr, st)) != SQUAD_OK)
      return s;
    return launch_fwd_tc(ds, d, sq::FWD_GLOBAL, p, q, k, nullptr, nullptr, nullptr, o1buf, o, lse2, nullptr,
                         nullptr, st);
  }
  if ((s = simt_fwd<float>(p.g1, q, k, v, o1buf, lse1, d, p.scale, st)) != SQUAD_OK) return s;
  return simt_fwd<float>(p.g2, q, k, o1buf, o, lse2, d, p.scale, st);
}

// ---- forward from host memory, copies overlapped with compute
// The (batch, head) slices are independent problems, so the forward runs on chunks of
// slices: the copy of chunk i+1 in, the forward of chunk i and the copy of chunk i-1 out
// proceed on three streams at once. Device buffers: two sets (q, k, v, o of one chunk)
// used in turn, then the fused forward's workspace for one chunk.
namespace {

struct HostFwdWs {
  size_t set_bytes, chunk_bytes, fwd_ws, total;
};

HostFwdWs host_fwd_workspace(const squad_desc* d, const Plan& p, int chunk) {
  squad_desc dc = *d;
  dc.B = 1;
  dc.heads = chunk;
  Plan pc;
  HostFwdWs w{};
  w.chunk_bytes = size_t(chunk) * (p.rows / (long long)(d->B * d->heads)) * d->d * p.elem;
  w.set_bytes = 4 * align256(w.chunk_bytes);
  w.fwd_ws = make_plan(&dc, &pc) == SQUAD_OK ? fwd_workspace(pc, &dc) : 0;
  w.total = 2 * w.set_bytes + w.fwd_ws;
  return w;
}

struct EventSet {  // events of one call, released when the call has enqueued everything
  cudaEvent_t e[7] = {};
  int n = 0;
  ~EventSet() {
    for (int i = 0; i < n; ++i) cudaEventDestroy(e[i]);
  }
};

}  // namespace

squad_status squad_attn_fwd_host_workspace_size(const squad_desc* desc, int slices_per_chunk, size_t* bytes) {
  if (bytes == nullptr) return SQUAD_ERR_INVALID_ARG;
  Plan p;
  squad_status s = make_plan(desc, &p);
  if (s != SQUAD_OK) return s;
  if (slices_per_chunk < 1) return SQUAD_ERR_INVALID_ARG;
  const int S = desc->B * desc->heads;
  const int chunk = slices_per_chunk < S ? slices_per_chunk : S;
  *bytes = host_fwd_workspace(desc, p, chunk).total;
  return SQUAD_OK;
}

squad_status squad_attn_fwd_host(const squad_desc* desc, const void* q, const void* k, const void* v, void* o,
                                 int slices_per_chunk, void* workspace, size_t workspace_bytes,
                                 void* stream, void* stream_in, void* stream_out) {
  Plan p;
  squad_status s = make_plan(desc, &p);
  if (s != SQUAD_OK) return s;
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr || slices_per_chunk < 1)
    return SQUAD_ERR_INVALID_ARG;
  if (stream_in == nullptr || stream_out == nullptr || stream_in == stream_out || stream_in == stream ||
      stream_out == stream)
    return SQUAD_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return SQUAD_ERR_ALIGN;
  const int S = desc->B * desc->heads;
  const int chunk = slices_per_chunk < S ? slices_per_chunk : S;
  const HostFwdWs w = host_fwd_workspace(desc, p, chunk);
  if (workspace == nullptr || workspace_bytes < w.total) return SQUAD_ERR_WORKSPACE;
  cudaStream_t sc = static_cast<cudaStream_t>(stream), si = static_cast<cudaStream_t>(stream_in),
               so = static_cast<cudaStream_t>(stream_out);
  const size_t slice_bytes = w.chunk_bytes / size_t(chunk);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  auto buf = [&](int set, int which) { return ws + size_t(set) * w.set_bytes + size_t(which) * align256(w.chunk_bytes); };
  uint8_t* fws = ws + 2 * w.set_bytes;
  EventSet ev;  // [0] entry, [1..2] copied in, [3..4] computed, [5..6] copied out (per buffer set)
  for (; ev.n < 7; ++ev.n) SQ_CUDA(cudaEventCreateWithFlags(&ev.e[ev.n], cudaEventDisableTiming));
  // ordered after the work already on `stream`
  SQ_CUDA(cudaEventRecord(ev.e[0], sc));
  SQ_CUDA(cudaStreamWaitEvent(si, ev.e[0], 0));
  SQ_CUDA(cudaStreamWaitEvent(so, ev.e[0], 0));
  const uint8_t* hq = static_cast<const uint8_t*>(q);
  const uint8_t* hk = static_cast<const uint8_t*>(k);
  const uint8_t* hv = static_cast<const uint8_t*>(v);
  uint8_t* ho = static_cast<uint8_t*>(o);
  for (int c0 = 0, i = 0; c0 < S; c0 += chunk, ++i) {
    const int cs = S - c0 < chunk ? S - c0 : chunk;
    const int b = i & 1;
    const size_t off = size_t(c0) * slice_bytes, nb = size_t(cs) * slice_bytes;
    // set b was last read by the forward of chunk i-2 (inputs) and the copy out of chunk i-2 (output)
    if (i >= 2) SQ_CUDA(cudaStreamWaitEvent(si, ev.e[3 + b], 0));
    SQ_CUDA(cudaMemcpyAsync(buf(b, 0), hq + off, nb, cudaMemcpyHostToDevice, si));
    SQ_CUDA(cudaMemcpyAsync(buf(b, 1), hk + off, nb, cudaMemcpyHostToDevice, si));
    SQ_CUDA(cudaMemcpyAsync(buf(b, 2), hv + off, nb, cudaMemcpyHostToDevice, si));
    SQ_CUDA(cudaEventRecord(ev.e[1 + b], si));
    SQ_CUDA(cudaStreamWaitEvent(sc, ev.e[1 + b], 0));
    if (i >= 2) SQ_CUDA(cudaStreamWaitEvent(sc, ev.e[5 + b], 0));
    squad_desc dc = *desc;
    dc.B = 1;
    dc.heads = cs;
    if ((s = squad_attn_fwd(&dc, buf(b, 0), buf(b, 1), buf(b, 2), buf(b, 3), nullptr, nullptr, nullptr, fws, w.fwd_ws,
                            sc)) != SQUAD_OK)
      return s;
    SQ_CUDA(cudaEventRecord(ev.e[3 + b], sc));
    SQ_CUDA(cudaStreamWaitEvent(so, ev.e[3 + b], 0));
    SQ_CUDA(cudaMemcpyAsync(ho + off, buf(b, 3), nb, cudaMemcpyDeviceToHost, so));
    SQ_CUDA(cudaEventRecord(ev.e[5 + b], so));
  }
  // later work on `stream` (and a synchronisation of it) sees o complete: the copies out
  // run in order on stream_out, so the last one's event covers them all
  const int last = ((S + chunk - 1) / chunk - 1) & 1;
  SQ_CUDA(cudaStreamWaitEvent(sc, ev.e[5 + last], 0));
  return SQUAD_OK;
}

squad_status squad_attn_fwd_pass(const squad_desc* desc, int stage, const void* q, const void* k,
                                 const void* val, void* out, float* lse, void* stream) {
  Plan p;
  squad_status s = make_plan(desc, &p);
  if (s != SQUAD_OK) return s;
  if (stage != 1 && stage != 2) return SQUAD_ERR_INVALID_ARG;
  if (q == nullptr || k == nullptr || val == nullptr || out == nullptr) return SQUAD_ERR_INVALID_ARG;
  for (const void* ptr : {q, k, val, static_cast<const void*>(out), static_cast<const void*>(lse)})
    if (!aligned16(ptr)) return SQUAD_ERR_ALIGN;
  DeviceState* ds = nullptr;
  if ((s = device_state(&ds)) != SQUAD_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Geom& g = stage == 1 ? p.g1 : p.g2;
  if (desc->dtype == SQUAD_BF16) {
    if (stage == 1)
      return launch_fwd_tc(ds, desc->d, sq::FWD_LOCAL, p, q, k, val, out, lse, nullptr, nullptr, nullptr, nullptr,
                           nullptr, st);
    return launch_fwd_tc(ds, desc->d, sq::FWD_GLOBAL, p, q, k, nullptr, nullptr, nullptr, val, out, lse, nullptr,
                         nullptr, st);
  }
  return simt_fwd<float>(g, q, k, val, out, lse, desc->d, p.scale, st);
}

}  // extern "C"

// ---------------------------------------------------------------- forward without allocation
// Scratch for squad_attn_fwd_noalloc: the local-pass output of problems that fit.
// Device code could name it directly, but the kernels take plain pointers, so the
// host looks up its device address once per device (see noalloc_scratch below).
static __device__ __align__(256) unsigned char g_squad_noalloc_scratch[SQUAD_NOALLOC_SCRATCH_BYTES];

namespace {
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device. In host code the
// array's name is only a host-side stand-in, so the address must come from
// cudaGetSymbolAddress, called with the device current; it is cached per device.
squad_status noalloc_scratch(void** out) {
  int dev = 0;
  SQ_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return SQUAD_ERR_UNSUPPORTED;
  // binds the device's primary context to this thread (a thread that has made no runtime
  // call yet, such as an autograd worker, has none, and the tensor-map encoder needs it)
  SQ_CUDA(cudaSetDevice(dev));
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    SQ_CUDA(cudaGetSymbolAddress(&p, g_squad_noalloc_scratch));
    if (p == nullptr) return cuda_fail(int(cudaErrorInvalidSymbol));
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return SQUAD_OK;
}
}  // namespace

extern "C" squad_status squad_attn_fwd_noalloc(const squad_desc* desc, const void* q, const void* k, const void* v,
                                               void* o, float* lse1, float* lse2, void* stream) {
  Plan p;
  squad_status s = make_plan(desc, &p);
  if (s != SQUAD_OK) return s;
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) return SQUAD_ERR_INVALID_ARG;
  const size_t need = size_t(p.rows) * size_t(desc->d) * p.elem;
  if (need > size_t(SQUAD_NOALLOC_SCRATCH_BYTES)) return SQUAD_ERR_WORKSPACE;
  for (const void* ptr : {q, k, v, static_cast<const void*>(o), static_cast<const void*>(lse1),
                          static_cast<const void*>(lse2)})
    if (!aligned16(ptr)) return SQUAD_ERR_ALIGN;
  void* scratch = nullptr;
  if ((s = noalloc_scratch(&scratch)) != SQUAD_OK) return s;
  DeviceState* ds = nullptr;
  if ((s = device_state(&ds)) != SQUAD_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int d = desc->d;
  // The local pass writes every element of the scratch that the global pass reads.
  if (desc->dtype == SQUAD_BF16) {
    if ((s = launch_fwd_tc(ds, d, sq::FWD_LOCAL, p, q, k, v, scratch, lse1, nullptr, nullptr, nullptr, nullptr,
                           nullptr, st)) != SQUAD_OK)
      return s;
    return launch_fwd_tc(ds, d, sq::FWD_GLOBAL, p, q, k, nullptr, nullptr, nullptr, scratch, o, lse2, nullptr,
                         nullptr, st);
  }
  if ((s = simt_fwd<float>(p.g1, q, k, v, scratch, lse1, d, p.scale, st)) != SQUAD_OK) return s;
  return simt_fwd<float>(p.g2, q, k, scratch, o, lse2, d, p.scale, st);
}

extern "C" {

squad_status squad_attn_bwd(const squad_desc* desc, const void* q, const void* k, const void* v, const void* o,
                            const void* o1, const float* lse1, const float* lse2, const void* dout, void* dq,
                            void* dk, void* dv, void* workspace, size_t workspace_bytes, void* stream) {
  Plan p;
  squad_status s = make_plan(desc, &p);
  if (s != SQUAD_OK) return s;
  for (const void* ptr : {q, k, v, o, o1, static_cast<const void*>(lse1), static_cast<const void*>(lse2), dout,
                          static_cast<const void*>(dq), static_cast<const void*>(dk), static_cast<const void*>(dv)})
    if (ptr == nullptr) return SQUAD_ERR_INVALID_ARG;
  for (const void* ptr : {q, k, v, o, o1, static_cast<const void*>(lse1), static_cast<const void*>(lse2), dout,
                          static_cast<const void*>(dq), static_cast<const void*>(dk), static_cast<const void*>(dv),
                          static_cast<const void*>(workspace)})
    if (!aligned16(ptr)) return SQUAD_ERR_ALIGN;
  const BwdWs w = bwd_workspace(p, desc);
  if (workspace == nullptr || workspace_bytes < w.total) return SQUAD_ERR_WORKSPACE;
  DeviceState* ds = nullptr;
  if ((s = device_state(&ds)) != SQUAD_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (desc->dtype == SQUAD_BF16)
    return tc_bwd(ds, p, w, ws, q, k, v, o, o1, lse1, lse2, dout, dq, dk, dv, desc->d, st);
  return simt_bwd<float>(p, w, ws, q, k, v, o, o1, lse1, lse2, dout, dq, dk, dv, desc->d, st);
}

squad_status squad_plan_info(const squad_desc* desc, int stage, int* info) {
  if (info == nullptr || (stage != 1 && stage != 2)) return SQUAD_ERR_INVALID_ARG;
  Plan p;
  squad_status s = make_plan(desc, &p);
  if (s != SQUAD_OK) return s;
  Geom g = stage == 1 ? p.g1 : p.g2;
  if (desc->dtype != SQUAD_BF16 && !sq::plan_tiles(g)) return SQUAD_ERR_UNSUPPORTED;
  info[0] = g.L;
  info[1] = g.probs;
  info[2] = g.nt;
  info[3] = g.box_rows;
  info[4] = g.a_n;
  info[5] = g.b_sub;
  info[6] = g.c_sub;
  info[7] = g.nt >= 2 ? 2 : 1;
  return SQUAD_OK;
}

squad_status squad_selftest_wait_timeout(unsigned long long timeout_ns, void* stream) {
  if (timeout_ns < 1000ull || timeout_ns > 10000000000ull) return SQUAD_ERR_INVALID_ARG;
  DeviceState* ds = nullptr;
  squad_status s;
  if ((s = device_state(&ds)) != SQUAD_OK) return s;
  selftest_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(ds->err, timeout_ns);
  SQ_CUDA(cudaGetLastError());
  return SQUAD_OK;
}

squad_status squad_poll_device_error(void* stream) {
  SQ_CUDA(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  int v = 0;
  SQ_CUDA(cudaMemcpyFromSymbol(&v, g_squad_dev_err, sizeof(int)));
  if (v != 0) {
    const int zero = 0;
    SQ_CUDA(cudaMemcpyToSymbol(g_squad_dev_err, &zero, sizeof(int)));
    return v == 2 ? SQUAD_ERR_INDEX : SQUAD_ERR_TIMEOUT;
  }
  return SQUAD_OK;
}

const char* squad_strerror(int status) {
  switch (status) {
    case SQUAD_OK: return "ok";
    case SQUAD_ERR_INVALID_ARG: return "invalid argument";
    case SQUAD_ERR_SHAPE: return "invalid shape";
    case SQUAD_ERR_ALIGN: return "pointer not 16-byte aligned";
    case SQUAD_ERR_UNSUPPORTED: return "unsupported configuration";
    case SQUAD_ERR_CUDA: return "CUDA error";
    case SQUAD_ERR_TIMEOUT: return "device wait timed out";
    case SQUAD_ERR_WORKSPACE: return "workspace missing or too small";
    case SQUAD_ERR_INDEX: return "a row index given to a shuffle was out of range";
  }
  return "unknown status";
}

int squad_last_cuda_error(void) { return t_last_cuda; }

squad_status squad_tmap_cache_stats(unsigned long long* hits, unsigned long long* misses) {
  if (hits == nullptr && misses == nullptr) return SQUAD_ERR_INVALID_ARG;
  g_tmaps.stats(hits, misses);
  return SQUAD_OK;
}

int squad_version(void) { return kVersion; }

}  // extern "C"

// ---------------------------------------------------------------- more than two passes
// k = ntiles + 1 passes over nested tiles t_1 | ... | t_{k-1} | grid (innermost first):
// pass j attends among the tokens of one t_j-window at the same position inside their
// t_{j-1}-window; its values are the previous pass's output. The pages name composing
// more than two passes as an outlook (gist.science technical summary, Significance and
// Claims); k = 2 is the operator above. Each pass runs on the same kernels as the two
// SQuad passes: on bf16 with a workspace, all k passes in one launch (pass j of a head
// starts once pass j-1 of that head is done everywhere), else one launch per pass.

namespace {

constexpr int kMaxTiles = 4;

struct MultiPlan {
  Plan base;                 // scale, rows, element size (its g1/g2 are unused)
  int k;                     // passes
  Geom g[kMaxTiles + 1];     // pass j at g[j - 1]
  Geom gf[kMaxTiles + 1];    // the same for the bf16 forward, small problems packed several to a box
};

squad_status make_multi_plan(const squad_desc* d, int ntiles, const int* tiles, MultiPlan* mp) {
  if (d == nullptr || tiles == nullptr) return SQUAD_ERR_INVALID_ARG;
  if (ntiles < 1 || ntiles > kMaxTiles) return SQUAD_ERR_UNSUPPORTED;
  // the base plan validates the tensors; the tiles are checked here (nested)
  squad_desc d1 = *d;
  d1.tT = d1.tH = d1.tW = 1;
  squad_status s = make_plan(&d1, &mp->base, false);
  if (s != SQUAD_OK) return s;
  mp->k = ntiles + 1;
  const int grid[3] = {d->T, d->H, d->W};
  for (int j = 1; j <= mp->k; ++j) {
    int in[3], out[3];
    for (int a = 0; a < 3; ++a) {
      in[a] = j == 1 ? 1 : tiles[3 * (j - 2) + a];
      out[a] = j == mp->k ? grid[a] : tiles[3 * (j - 1) + a];
      if (in[a] <= 0 || out[a] <= 0 || out[a] % in[a] != 0 || grid[a] % out[a] != 0) return SQUAD_ERR_SHAPE;
    }
    Geom g = sq::make_geom_pass(d->B, d->heads, d->T, d->H, d->W, in[0], in[1], in[2], out[0], out[1], out[2]);
    Geom gf = g;
    if (d->dtype == SQUAD_BF16) {
      if (!sq::plan_tiles(g)) return SQUAD_ERR_UNSUPPORTED;
      sq::plan_pack(gf);
      if (!sq::plan_tiles(gf)) return SQUAD_ERR_UNSUPPORTED;
    }
    mp->g[j - 1] = g;
    mp->gf[j - 1] = gf;
  }
  return SQUAD_OK;
}

// Forward workspace: [outputs of passes 1..k-1, only when the caller passes no inter]
// [finished jobs per (pass, batch, head) for passes 2..k].
size_t multi_fwd_inter_bytes(const MultiPlan& mp, const squad_desc* d) {
  return align256(size_t(mp.k - 1) * mp.base.rows * d->d * mp.base.elem);
}
size_t multi_fwd_counter_bytes(const MultiPlan& mp) {
  return align256(size_t(mp.k - 1) * mp.g[0].bh * sizeof(uint32_t));
}

// All k passes of the bf16 forward in one cooperative launch (FWD_MULTI item order, see
// decode_item): val[j] / out[j] / lse[j] are pass j's values, output and LSE.
squad_status launch_fwd_multi(DeviceState* ds, int d, const MultiPlan& mp, const void* q, const void* k,
                              const void* const* val, void* const* out, float* const* lse, uint32_t* counters,
                              bool drop_inter, cudaStream_t st) {
  sq::FwdMaps maps;
  sq::FwdArgs a{};
  squad_status s;
  const int np = mp.k;
  if (np > sq::kMaxFwdPasses) return SQUAD_ERR_UNSUPPORTED;
  bool packed = false;
  for (int j = 0; j < np; ++j) {
    const Geom& g = mp.gf[j];
    CUtensorMap* m = &maps.m[4 * j];
    if ((s = encode_map(&m[0], q, g, d, mp.base.rows)) != SQUAD_OK) return s;
    if ((s = encode_map(&m[1], k, g, d, mp.base.rows)) != SQUAD_OK) return s;
    if ((s = encode_map(&m[2], val[j], g, d, mp.base.rows)) != SQUAD_OK) return s;
    if ((s = encode_map(&m[3], out[j], g, d, mp.base.rows)) != SQUAD_OK) return s;
    a.ps[j] = pass_args(g, out[j], lse[j]);
    // scratch values (a previous pass's output nobody else reads) leave L2 once read
    if (drop_inter && j > 0 && (reinterpret_cast<uintptr_t>(val[j]) & 127u) == 0)
      a.ps[j].discard = static_cast<const uint8_t*>(val[j]);
    packed = packed || g.pk > 1;
  }
  for (int i = 4 * np; i < 4 * sq::kMaxFwdPasses; ++i) maps.m[i] = maps.m[i % (4 * np)];  // unused
  a.mode = sq::FWD_MULTI;
  a.npass = np;
  a.bh = mp.gf[0].bh;
  a.lag = kMultiLag < a.bh ? kMultiLag : a.bh;
  sq::plan_multi_order(a);
  a.scale_log2 = mp.base.scale * 1.4426950408889634f;
  a.counters = counters;
  a.err = ds->err;
  a.timeout_ns = kWaitTimeoutNs;
  SQ_CUDA(cudaMemsetAsync(counters, 0, size_t(np - 1) * a.bh * sizeof(uint32_t), st));
  if (d == 128) return packed ? launch_fwd_tc_t<128, true>(ds, maps, a, st) : launch_fwd_tc_t<128, false>(ds, maps, a, st);
  return packed ? launch_fwd_tc_t<64, true>(ds, maps, a, st) : launch_fwd_tc_t<64, false>(ds, maps, a, st);
}

// Backward workspace: two upstream gradients (dtype) used in turn, two fp32 dQ and two
// fp32 dK accumulators used in turn (the pass reads one and writes the other), one fp32
// row vector.
struct MultiWs {
  size_t up[2], dq[2], dk[2], drow, dvec[2], total;
};

MultiWs multi_workspace(const MultiPlan& mp, const squad_desc* d) {
  MultiWs w{};
  const size_t big = size_t(mp.base.rows) * d->d;
  size_t off = 0;
  for (int i = 0; i < 2; ++i) { w.up[i] = off; off += align256(big * mp.base.elem); }
  for (int i = 0; i < 2; ++i) { w.dq[i] = off; off += align256(big * 4); }
  for (int i = 0; i < 2; ++i) { w.dk[i] = off; off += align256(big * 4); }
  w.drow = off;
  off += align256(size_t(mp.base.rows) * 4);
  for (int i = 0; i < 2; ++i) { w.dvec[i] = off; off += align256(size_t(mp.base.rows) * 4); }
  w.total = off;
  return w;
}

template <int DPL>
squad_status simt_pass_bwd_f32(const Geom& g, long long rows, const float* q, const float* k, const float* val,
                               const float* out, const float* dout, const float* lse, float* Drow,
                               const float* dq_add, float* dq, const float* dk_add, float* dk, float* dval, int d,
                               float scale, cudaStream_t st) {
  return simt_pass_bwd_t<float, float, float, float, DPL>(g, rows, q, k, val, out, dout, lse, Drow, dq_add, dq,
                                                          dk_add, dk, dval, d, scale, st);
}

squad_status simt_pass_bwd_f32_any(int d, const Geom& g, long long rows, const float* q, const float* k,
                                   const float* val, const float* out, const float* dout, const float* lse,
                                   float* Drow, const float* dq_add, float* dq, const float* dk_add, float* dk,
                                   float* dval, float scale, cudaStream_t st) {
  switch (d / 32) {
#define SQ_CASE(n) \
  case n: return simt_pass_bwd_f32<n>(g, rows, q, k, val, out, dout, lse, Drow, dq_add, dq, dk_add, dk, dval, d, scale, st);
    SQ_CASE(1) SQ_CASE(2) SQ_CASE(3) SQ_CASE(4) SQ_CASE(5) SQ_CASE(6) SQ_CASE(7) SQ_CASE(8)
#undef SQ_CASE
  }
  return SQUAD_ERR_UNSUPPORTED;
}

}  // namespace

extern "C" {

squad_status squad_attn_multi_bwd_workspace_size(const squad_desc* desc, int ntiles, const int* tiles,
                                                 size_t* bytes) {
  MultiPlan mp;
  squad_status s = make_multi_plan(desc, ntiles, tiles, &mp);
  if (s != SQUAD_OK) return s;
  if (bytes == nullptr) return SQUAD_ERR_INVALID_ARG;
  *bytes = multi_workspace(mp, desc).total;
  return SQUAD_OK;
}

squad_status squad_attn_multi_fwd_workspace_size(const squad_desc* desc, int ntiles, const int* tiles,
                                                 int save_inter, size_t* bytes) {
  if (bytes == nullptr) return SQUAD_ERR_INVALID_ARG;
  MultiPlan mp;
  squad_status s = make_multi_plan(desc, ntiles, tiles, &mp);
  if (s != SQUAD_OK) return s;
  *bytes = (save_inter ? 0 : multi_fwd_inter_bytes(mp, desc)) + multi_fwd_counter_bytes(mp);
  return SQUAD_OK;
}

squad_status squad_attn_multi_fwd(const squad_desc* desc, int ntiles, const int* tiles, const void* q,
                                  const void* k, const void* v, void* o, void* inter, float* lse, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  MultiPlan mp;
  squad_status s = make_multi_plan(desc, ntiles, tiles, &mp);
  if (s != SQUAD_OK) return s;
  for (const void* ptr : {q, k, v, static_cast<const void*>(o)})
    if (ptr == nullptr) return SQUAD_ERR_INVALID_ARG;
  for (const void* ptr : {q, k, v, static_cast<const void*>(o), static_cast<const void*>(inter),
                          static_cast<const void*>(lse), static_cast<const void*>(workspace)})
    if (!aligned16(ptr)) return SQUAD_ERR_ALIGN;
  const bool save = inter != nullptr;
  if (!save && workspace == nullptr) return SQUAD_ERR_WORKSPACE;
  const size_t inter_ws = save ? 0 : multi_fwd_inter_bytes(mp, desc);
  if (workspace != nullptr && workspace_bytes < inter_ws + multi_fwd_counter_bytes(mp)) return SQUAD_ERR_WORKSPACE;
  if (!save) inter = workspace;
  DeviceState* ds = nullptr;
  if ((s = device_state(&ds)) != SQUAD_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t big = size_t(mp.base.rows) * desc->d * mp.base.elem;
  if (desc->dtype == SQUAD_BF16 && workspace != nullptr) {
    const void* vals[sq::kMaxFwdPasses];
    void* outs[sq::kMaxFwdPasses];
    float* lses[sq::kMaxFwdPasses];
    for (int j = 0; j < mp.k; ++j) {
      outs[j] = j == mp.k - 1 ? o : static_cast<uint8_t*>(inter) + big * j;
      vals[j] = j == 0 ? v : outs[j - 1];
      lses[j] = lse == nullptr ? nullptr : lse + size_t(mp.base.rows) * j;
    }
    uint32_t* counters = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) + inter_ws);
    return launch_fwd_multi(ds, desc->d, mp, q, k, vals, outs, lses, counters, !save, st);
  }
  const void* val = v;
  for (int j = 1; j <= mp.k; ++j) {
    void* out = j == mp.k ? o : static_cast<uint8_t*>(inter) + big * (j - 1);
    float* l = lse == nullptr ? nullptr : lse + size_t(mp.base.rows) * (j - 1);
    if (desc->dtype == SQUAD_BF16) {
      Plan p = mp.base;
      p.g1 = p.g2 = mp.gf[j - 1];
      s = launch_fwd_tc(ds, desc->d, sq::FWD_LOCAL, p, q, k, val, out, l, val, out, l, nullptr, nullptr, st);
    } else {
      s = simt_fwd<float>(mp.g[j - 1], q, k, val, out, l, desc->d, mp.base.scale, st);
    }
    if (s != SQUAD_OK) return s;
    val = out;
  }
  return SQUAD_OK;
}

squad_status squad_attn_multi_bwd(const squad_desc* desc, int ntiles, const int* tiles, const void* q,
                                  const void* k, const void* v, const void* o, const void* inter, const float* lse,
                                  const void* dout, void* dq, void* dk, void* dv, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  MultiPlan mp;
  squad_status s = make_multi_plan(desc, ntiles, tiles, &mp);
  if (s != SQUAD_OK) return s;
  for (const void* ptr : {q, k, v, o, inter, static_cast<const void*>(lse), dout, static_cast<const void*>(dq),
                          static_cast<const void*>(dk), static_cast<const void*>(dv)})
    if (ptr == nullptr) return SQUAD_ERR_INVALID_ARG;
  for (const void* ptr : {q, k, v, o, inter, static_cast<const void*>(lse), dout, static_cast<const void*>(dq),
                          static_cast<const void*>(dk), static_cast<const void*>(dv),
                          static_cast<const void*>(workspace)})
    if (!aligned16(ptr)) return SQUAD_ERR_ALIGN;
  const MultiWs w = multi_workspace(mp, desc);
  if (workspace == nullptr || workspace_bytes < w.total) return SQUAD_ERR_WORKSPACE;
  DeviceState* ds = nullptr;
  if ((s = device_state(&ds)) != SQUAD_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t big = size_t(mp.base.rows) * desc->d * mp.base.elem;
  const bool bf16 = desc->dtype == SQUAD_BF16;
  auto inter_at = [&](int j) -> const void* { return static_cast<const uint8_t*>(inter) + big * (j - 1); };
  // Last pass first. Pass j reads the upstream gradient of its output and writes that of
  // its values (the output of pass j-1); dQ and dK accumulate in fp32 across passes (each
  // pass reads the sum so far from one buffer and writes the new sum to the other), and
  // the first pass writes the final dq, dk, dv.
  const void* up = dout;
  int acc = 0;  // accumulator holding the sum so far (valid for j < k)
  // bf16: D of pass k = rowsum(dout o o) by a row-dot pass; pass j writes the D of pass j-1
  // (rowsum(dVal o Val) of its own results) into the other vector
  if (bf16 && (s = rowdot_bf16(dout, o, reinterpret_cast<float*>(ws + w.dvec[mp.k & 1]), mp.base.rows, desc->d,
                               st)) != SQUAD_OK)
    return s;
  for (int j = mp.k; j >= 1; --j) {
    // bf16: small problems packed several to a box, as in the forward
    const Geom& g = bf16 ? mp.gf[j - 1] : mp.g[j - 1];
    const void* val = j == 1 ? v : inter_at(j - 1);
    const void* out = j == mp.k ? o : inter_at(j);
    const float* l = lse + size_t(mp.base.rows) * (j - 1);
    void* dval = j == 1 ? dv : ws + w.up[j & 1];
    const float* q_add = j == mp.k ? nullptr : reinterpret_cast<const float*>(ws + w.dq[acc]);
    const float* k_add = j == mp.k ? nullptr : reinterpret_cast<const float*>(ws + w.dk[acc]);
    void* q_out = j == 1 ? dq : ws + w.dq[acc ^ 1];
    void* k_out = j == 1 ? dk : ws + w.dk[acc ^ 1];
    if (bf16) {
      // the last step (j = 1) writes bf16 and, for multi-box problems, adds its dQ parts
      // into the fp32 sum before the conversion
      float* q_acc = j == 1 ? const_cast<float*>(q_add) : nullptr;
      const float* drow = reinterpret_cast<const float*>(ws + w.dvec[j & 1]);
      float* d_next = j > 1 ? reinterpret_cast<float*>(ws + w.dvec[(j - 1) & 1]) : nullptr;
      s = tc_pass_bwd(ds, mp.base, desc->d, g, q, k, val, out, up, l, drow, d_next, q_add, q_acc, q_out,
                      k_add, k_out, static_cast<__nv_bfloat16*>(dval), j > 1, st);
    } else {
      s = simt_pass_bwd_f32_any(desc->d, g, mp.base.rows, static_cast<const float*>(q),
                                static_cast<const float*>(k), static_cast<const float*>(val),
                                static_cast<const float*>(out), static_cast<const float*>(up), l,
                                reinterpret_cast<float*>(ws + w.drow), q_add, static_cast<float*>(q_out), k_add,
                                static_cast<float*>(k_out), static_cast<float*>(dval), mp.base.scale, st);
    }
    if (s != SQUAD_OK) return s;
    up = dval;
    acc ^= 1;
  }
  return SQUAD_OK;
}

}  // extern "C"

// ---------------------------------------------------------------- sequence-parallel forward
// Plan (host only) and row shuffles around the two all-to-alls; see sp_plan.h.

namespace {

squad_status sp_plan_of(const squad_desc* d, int G, int rank, sq::SpPlan& p) {
  if (d == nullptr) return SQUAD_ERR_INVALID_ARG;
  if (G < 1 || G > sq::kSpMaxPeers || rank < 0 || rank >= G) return SQUAD_ERR_INVALID_ARG;
  Plan base;
  squad_status s = make_plan(d, &base, false);
  if (s != SQUAD_OK) return s;
  if (d->T % d->tT || d->H % d->tH || d->W % d->tW) return SQUAD_ERR_SHAPE;
  const sq::SpShape sh{d->T, d->H, d->W, d->tT, d->tH, d->tW, G, rank};
  if (!sq::plan_sp(sh, p)) return SQUAD_ERR_UNSUPPORTED;
  return SQUAD_OK;
}

squad_status sp_shuffle_args(int ntensors, int slices, int rows_in, int rows_out, int row_bytes, int G,
                             const int* counts, sq::SpShuffleArgs* a) {
  if (ntensors < 1 || ntensors > sq::kSpMaxTensors || slices < 1 || rows_in < 0 || rows_out < 0 || row_bytes <= 0 ||
      row_bytes % 16 != 0 || G < 1 || G > sq::kSpMaxPeers || counts == nullptr)
    return SQUAD_ERR_INVALID_ARG;
  *a = sq::SpShuffleArgs{};
  a->ntensors = ntensors;
  a->slices = slices;
  a->rows_in = rows_in;
  a->rows_out = rows_out;
  a->row_bytes = row_bytes;
  a->G = G;
  long long at = 0;
  for (int q = 0; q < G; ++q) {
    if (counts[q] < 0) return SQUAD_ERR_INVALID_ARG;
    a->prefix[q] = int(at);
    at += counts[q];
  }
  a->prefix[G] = int(at);
  if ((long long)ntensors * slices * (at > rows_out ? at : rows_out) * row_bytes >= (1ll << 40) || at >= (1ll << 31))
    return SQUAD_ERR_SHAPE;
  return SQUAD_OK;
}

unsigned sp_blocks(long long chunks, int sms) {
  const long long b = (chunks + 255) / 256;
  const long long cap = 8ll * sms;
  return unsigned(b < 1 ? 1 : b > cap ? cap : b);
}

}  // namespace

extern "C" {

squad_status squad_sp_plan_info(const squad_desc* desc, int G, int rank, int* info) {
  if (info == nullptr) return SQUAD_ERR_INVALID_ARG;
  sq::SpPlan p;
  squad_status s = sp_plan_of(desc, G, rank, p);
  if (s != SQUAD_OK) return s;
  info[0] = p.t0;
  info[1] = p.T;
  info[2] = p.n_local;
  info[3] = p.n_pos;
  info[4] = p.p0[rank];
  info[5] = p.np[rank];
  info[6] = p.w;
  info[7] = p.m;
  return SQUAD_OK;
}

squad_status squad_sp_plan_maps(const squad_desc* desc, int G, int rank, int* counts, int* send1, int* recv1_src,
                                int* recv1_row, int* send2, int* recv2_src, int* recv2_row) {
  for (const void* ptr : {static_cast<const void*>(counts), static_cast<const void*>(send1),
                          static_cast<const void*>(recv1_src), static_cast<const void*>(recv1_row),
                          static_cast<const void*>(send2), static_cast<const void*>(recv2_src),
                          static_cast<const void*>(recv2_row)})
    if (ptr == nullptr) return SQUAD_ERR_INVALID_ARG;
  sq::SpPlan p;
  squad_status s = sp_plan_of(desc, G, rank, p);
  if (s != SQUAD_OK) return s;
  for (int q = 0; q < G; ++q) {
    counts[q] = p.send1_count[q];
    counts[G + q] = p.recv1_count[q];
    counts[2 * G + q] = p.send2_count[q];
    counts[3 * G + q] = p.recv2_count[q];
  }
  std::memcpy(send1, p.send1.data(), sizeof(int) * p.send1.size());
  std::memcpy(recv1_src, p.recv1_src.data(), sizeof(int) * p.recv1_src.size());
  std::memcpy(recv1_row, p.recv1_row.data(), sizeof(int) * p.recv1_row.size());
  std::memcpy(send2, p.send2.data(), sizeof(int) * p.send2.size());
  std::memcpy(recv2_src, p.recv2_src.data(), sizeof(int) * p.recv2_src.size());
  std::memcpy(recv2_row, p.recv2_row.data(), sizeof(int) * p.recv2_row.size());
  return SQUAD_OK;
}

squad_status squad_sp_pack(const void* const* srcs, int ntensors, int slices, int rows_in, int row_bytes, int G,
                           const int* counts, const int* idx, void* dst, void* stream) {
  sq::SpShuffleArgs a;
  squad_status s = sp_shuffle_args(ntensors, slices, rows_in, 0, row_bytes, G, counts, &a);
  if (s != SQUAD_OK) return s;
  if (srcs == nullptr || idx == nullptr || dst == nullptr) return SQUAD_ERR_INVALID_ARG;
  for (int t = 0; t < ntensors; ++t) {
    if (srcs[t] == nullptr) return SQUAD_ERR_INVALID_ARG;
    if (!aligned16(srcs[t])) return SQUAD_ERR_ALIGN;
    a.src[t] = static_cast<const uint8_t*>(srcs[t]);
  }
  if (!aligned16(dst) || (reinterpret_cast<uintptr_t>(idx) & 3u)) return SQUAD_ERR_ALIGN;
  a.dst[0] = static_cast<uint8_t*>(dst);
  DeviceState* ds = nullptr;
  if ((s = device_state(&ds)) != SQUAD_OK) return s;
  a.err = ds->err;
  const long long chunks = (long long)ntensors * slices * a.prefix[G] * (row_bytes / 16);
  if (chunks == 0) return SQUAD_OK;
  sq::sp_pack_kernel<<<sp_blocks(chunks, ds->sms), 256, 0, static_cast<cudaStream_t>(stream)>>>(a, idx);
  SQ_CUDA(cudaGetLastError());
  return SQUAD_OK;
}

squad_status squad_sp_unpack(const void* src, int ntensors, int slices, int rows_out, int row_bytes, int G,
                             const int* counts, const int* src_rank, const int* src_row, void* const* dsts,
                             void* stream) {
  sq::SpShuffleArgs a;
  squad_status s = sp_shuffle_args(ntensors, slices, 0, rows_out, row_bytes, G, counts, &a);
  if (s != SQUAD_OK) return s;
  if (src == nullptr || src_rank == nullptr || src_row == nullptr || dsts == nullptr) return SQUAD_ERR_INVALID_ARG;
  if (!aligned16(src) || (reinterpret_cast<uintptr_t>(src_rank) & 3u) || (reinterpret_cast<uintptr_t>(src_row) & 3u))
    return SQUAD_ERR_ALIGN;
  a.src[0] = static_cast<const uint8_t*>(src);
  for (int t = 0; t < ntensors; ++t) {
    if (dsts[t] == nullptr) return SQUAD_ERR_INVALID_ARG;
    if (!aligned16(dsts[t])) return SQUAD_ERR_ALIGN;
    a.dst[t] = static_cast<uint8_t*>(dsts[t]);
  }
  DeviceState* ds = nullptr;
  if ((s = device_state(&ds)) != SQUAD_OK) return s;
  a.err = ds->err;
  const long long chunks = (long long)ntensors * slices * rows_out * (row_bytes / 16);
  if (chunks == 0) return SQUAD_OK;
  sq::sp_unpack_kernel<<<sp_blocks(chunks, ds->sms), 256, 0, static_cast<cudaStream_t>(stream)>>>(a, src_rank,
                                                                                                  src_row);
  SQ_CUDA(cudaGetLastError());
  return SQUAD_OK;
}

}  // extern "C"
