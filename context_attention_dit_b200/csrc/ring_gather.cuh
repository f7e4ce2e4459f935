// ring_gather.cuh - the Ring Anything pad -> all-gather buffer, simulated as one local copy.
//
// "Context parallelism", "Ring Anything Attention": ranks whose K/V blocks differ in length
// pad their local block to the longest one, all-gather the padded blocks, and slice every
// gathered block back to its true length before attention.  On one GPU the gathered buffer
// is built directly from the unsharded tensor:
//   X   [B][S][H][D]                    block c = rows [bounds[c], bounds[c+1])
//   Y   [n][B][max_len][H][D]           Y[c][b][r] = X[b][bounds[c] + r]  for r < len_c,
//                                       0 for len_c <= r < max_len (the padding)
// Block c's true-length view is Y[c][:, :len_c], a [B][len_c][H][D] tensor with batch stride
// max_len*H*D, which the strided attention reads in place.
//
// A destination row is H*D contiguous elements and so is its source row, so the copy is a
// row gather: grid.x covers the vectors of a row, grid.y walks groups of kGatherRows
// destination rows (strided by gridDim.y), grid.z is the tensor.
#pragma once

#include <cstdint>

#include "ptx_sm100.cuh"

namespace cpattn {

constexpr int kGatherThreads = 128;
constexpr int kGatherRows = 4;  // destination rows per thread and pass (all loads before the stores)
constexpr int kGatherMaxTensors = 8;
constexpr int kGatherMaxChunks = 64;

struct GatherArgs {
  const void* src[kGatherMaxTensors];
  void* dst[kGatherMaxTensors];
  int bounds[kGatherMaxChunks + 1];
  int n_chunks, B, S, max_len;
};

// Source row of destination row R = (c * B + b) * max_len + r, or -1 for a padding row.
__device__ __forceinline__ long long gather_src_row(const GatherArgs& a, long long R) {
  const long long per_c = static_cast<long long>(a.B) * a.max_len;
  const int c = static_cast<int>(R / per_c);
  const long long rem = R - c * per_c;
  const int b = static_cast<int>(rem / a.max_len);
  const int r = static_cast<int>(rem - static_cast<long long>(b) * a.max_len);
  if (r >= a.bounds[c + 1] - a.bounds[c]) return -1;
  return static_cast<long long>(b) * a.S + a.bounds[c] + r;
}

template <typename V>
__global__ void __launch_bounds__(kGatherThreads)
    ring_anything_gather_kernel(const __grid_constant__ GatherArgs a, int row_vecs, long long rows) {
  const int i = blockIdx.x * kGatherThreads + threadIdx.x;  // vector within the row
  if (i >= row_vecs) return;
  const V* __restrict__ src = static_cast<const V*>(a.src[blockIdx.z]);
  V* __restrict__ dst = static_cast<V*>(a.dst[blockIdx.z]);
  const long long src_total = static_cast<long long>(a.B) * a.S * row_vecs;
  const long long dst_total = rows * row_vecs;
  for (long long R0 = static_cast<long long>(blockIdx.y) * kGatherRows; R0 < rows;
       R0 += static_cast<long long>(gridDim.y) * kGatherRows) {
    V v[kGatherRows];
#pragma unroll
    for (int k = 0; k < kGatherRows; ++k) {
      v[k] = V{};
      const long long R = R0 + k;
      if (R < rows) {
        const long long sr = gather_src_row(a, R);
        const long long si = sr * row_vecs + i;
        if (sr >= 0 && in_bounds(si, 1, src_total)) v[k] = src[si];
      }
    }
#pragma unroll
    for (int k = 0; k < kGatherRows; ++k) {
      const long long R = R0 + k;
      const long long di = R * row_vecs + i;
      if (R < rows && in_bounds(di, 1, dst_total)) dst[di] = v[k];
    }
  }
}

}  // namespace cpattn
