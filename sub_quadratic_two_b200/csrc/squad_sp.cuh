// squad_sp.cuh - row shuffles of the sequence-parallel forward (see sp_plan.h).
//
// Both kernels copy whole rows (row_bytes, a multiple of 16) with 16-byte loads and
// stores, one thread per 16-byte chunk, grid-stride. They are HBM-bound copies around
// the two all-to-alls; the attention itself runs in the tensor-core kernels. Every index
// is checked against the extent it addresses: a row whose index is out of range is
// skipped and the device error word is set (the host reads it as SQUAD_ERR_INDEX).
#pragma once
#include <cstdint>

namespace sq {

constexpr int kSpMaxPeers = 64;
constexpr int kSpMaxTensors = 3;

struct SpShuffleArgs {
  const uint8_t* src[kSpMaxTensors];  // pack: the tensors [slices, rows_in, row]; unpack: [0] = exchange buffer
  uint8_t* dst[kSpMaxTensors];        // pack: [0] = exchange buffer; unpack: the tensors [slices, rows_out, row]
  int ntensors, slices, rows_in, rows_out, row_bytes, G;
  int prefix[kSpMaxPeers + 1];        // rows per slice before each peer's chunk (prefix[G] = all rows)
  int* err;
};

// pack: exchange buffer row (peer q, tensor t, slice s, i) = tensor t, slice s, row idx[prefix[q] + i]
__global__ void sp_pack_kernel(SpShuffleArgs a, const int* __restrict__ idx) {
  const int per_row = a.row_bytes / 16;
  const long long nt_s = (long long)a.ntensors * a.slices;
  const long long total = nt_s * a.prefix[a.G] * per_row;
  for (long long c = blockIdx.x * (long long)blockDim.x + threadIdx.x; c < total; c += (long long)gridDim.x * blockDim.x) {
    const long long o = c / per_row;
    const int part = int(c - o * per_row);
    int q = 0;
    while (q + 1 < a.G && o >= nt_s * a.prefix[q + 1]) ++q;
    const int cnt = a.prefix[q + 1] - a.prefix[q];
    const long long rem = o - nt_s * a.prefix[q];
    const int ts = int(rem / cnt), i = int(rem - (long long)ts * cnt);
    const int t = ts / a.slices, s = ts - t * a.slices;
    const int row = idx[a.prefix[q] + i];
    if (row < 0 || row >= a.rows_in) {
      if (part == 0) atomicCAS(a.err, 0, 2);
      continue;
    }
    const uint4* src = reinterpret_cast<const uint4*>(a.src[t] + ((long long)s * a.rows_in + row) * a.row_bytes);
    reinterpret_cast<uint4*>(a.dst[0] + o * a.row_bytes)[part] = src[part];
  }
}

// unpack: tensor t, slice s, row j = exchange buffer row (peer src_rank[j], tensor t, slice s, src_row[j])
__global__ void sp_unpack_kernel(SpShuffleArgs a, const int* __restrict__ src_rank, const int* __restrict__ src_row) {
  const int per_row = a.row_bytes / 16;
  const long long total = (long long)a.ntensors * a.slices * a.rows_out * per_row;
  const long long nt_s = (long long)a.ntensors * a.slices;
  for (long long c = blockIdx.x * (long long)blockDim.x + threadIdx.x; c < total; c += (long long)gridDim.x * blockDim.x) {
    const long long o = c / per_row;
    const int part = int(c - o * per_row);
    const int ts = int(o / a.rows_out), j = int(o - (long long)ts * a.rows_out);
    const int t = ts / a.slices, s = ts - t * a.slices;
    const int q = src_rank[j], k = src_row[j];
    if (q < 0 || q >= a.G || k < 0 || k >= a.prefix[q + 1] - a.prefix[q]) {
      if (part == 0) atomicCAS(a.err, 0, 2);
      continue;
    }
    const long long srow = nt_s * a.prefix[q] + (long long)(t * a.slices + s) * (a.prefix[q + 1] - a.prefix[q]) + k;
    const uint4* src = reinterpret_cast<const uint4*>(a.src[0] + srow * a.row_bytes);
    reinterpret_cast<uint4*>(a.dst[t] + ((long long)s * a.rows_out + j) * a.row_bytes)[part] = src[part];
  }
}

}  // namespace sq
