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

template <typename V>
__global__ void __launch_bounds__(kGatherThreads)
    ring_anything_gather_kernel(const __grid_constant__ GatherArgs a, int row_vecs, int rows) {
  const int i = blockIdx.x * kGatherThreads + threadIdx.x;  // vector within the row
  if (i >= row_vecs) return;
  const V* __restrict__ src = static_cast<const V*>(a.src[blockIdx.z]);
  V* __restrict__ dst = static_cast<V*>(a.dst[blockIdx.z]);
  const long long src_total = static_cast<long long>(a.B) * a.S * row_vecs;
  const long long dst_total = static_cast<long long>(rows) * row_vecs;
  const int per_c = a.B * a.max_len;  // destination rows per block
  for (int R0 = blockIdx.y * kGatherRows; R0 < rows; R0 += gridDim.y * kGatherRows) {
    // Destination row R = (c * B + b) * max_len + r; the rows of a group are consecutive,
    // so (c, b, r) is found once and stepped.
    int c = R0 / per_c;
    const int rem = R0 - c * per_c;
    int b = rem / a.max_len;
    int r = rem - b * a.max_len;
    V v[kGatherRows];
#pragma unroll
    for (int k = 0; k < kGatherRows; ++k) {
      v[k] = V{};
      if (R0 + k < rows && r < a.bounds[c + 1] - a.bounds[c]) {  // a true row of block c, else padding
        const long long si = (static_cast<long long>(b) * a.S + a.bounds[c] + r) * row_vecs + i;
        if (in_bounds(si, 1, src_total)) v[k] = src[si];
      }
      if (++r == a.max_len) {
        r = 0;
        if (++b == a.B) {
          b = 0;
          ++c;
        }
      }
    }
#pragma unroll
    for (int k = 0; k < kGatherRows; ++k) {
      const long long di = static_cast<long long>(R0 + k) * row_vecs + i;
      if (R0 + k < rows && in_bounds(di, 1, dst_total)) dst[di] = v[k];
    }
  }
}

}  // namespace cpattn
