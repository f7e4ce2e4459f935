// ulysses_permute.cuh - the Ulysses all-to-all simulated as one local copy.
//
// "Context parallelism", "Ulysses Attention": the first all-to-all regroups the data
// so that each GPU holds every token for a subset of heads; the second regroups the
// results by token.  With P ranks stacked rank-major:
//   sequence-sharded  X[p][b][s_local][h][d]   ([P][B][S/P][H][D])
//   head-sharded      Y[q][b][s][j][d]         ([P][B][S][H/P][D])
//   Y[q][b][p*S/P + s_local][j][:] = X[p][b][s_local][q*H/P + j][:]
// Direction 0 copies X -> Y (first exchange), direction 1 copies Y -> X (second).
//
// Both directions walk the sequence-sharded token rows: block (x, y, z) covers the
// vectors [x*blockDim, ...) of kPermuteRows consecutive rows (p, b, s_local) of one tensor.
// A row of H*D elements splits into P contiguous pieces of (H/P)*D elements, one per
// head group q, which are contiguous rows of Y.  So the X side is one contiguous row
// per block and the Y side is P contiguous runs; every access is one vector of type V.
#pragma once

#include <cstdint>

namespace cpattn {

constexpr int kPermuteThreads = 128;
constexpr int kPermuteRows = 4;       // token rows per thread (all loads in flight before the stores)
constexpr int kPermuteMaxTensors = 8;

struct PermuteArgs {
  const void* src[kPermuteMaxTensors];
  void* dst[kPermuteMaxTensors];
};

// grid.x covers the vectors of a token row, grid.y groups of kPermuteRows rows of a
// shard (strided by gridDim.y), grid.z = tensor * P * B + p * B + b.
template <typename V>
__global__ void __launch_bounds__(kPermuteThreads)
    ulysses_permute_kernel(const __grid_constant__ PermuteArgs a, int P, int B, int Sp, int row_vecs, int piece_vecs,
                           int direction) {
  const int i = blockIdx.x * kPermuteThreads + threadIdx.x;  // vector within the token row
  if (i >= row_vecs) return;
  const int q = i / piece_vecs;  // head group of this vector
  const int w = i - q * piece_vecs;
  const int tz = blockIdx.z;
  const int n = tz / (P * B);
  const int pb = tz - n * (P * B);
  const int p = pb / B;
  const int b = pb - p * B;
  const V* __restrict__ src = static_cast<const V*>(a.src[n]);
  V* __restrict__ dst = static_cast<V*>(a.dst[n]);
  const long long S = static_cast<long long>(Sp) * P;
  const long long x0 = static_cast<long long>(pb) * Sp * row_vecs + i;                     // X row stride row_vecs
  const long long y0 = ((static_cast<long long>(q) * B + b) * S + static_cast<long long>(p) * Sp) * piece_vecs + w;
  for (int s0 = blockIdx.y * kPermuteRows; s0 < Sp; s0 += gridDim.y * kPermuteRows) {
    V v[kPermuteRows];
#pragma unroll
    for (int r = 0; r < kPermuteRows; ++r) {
      const int sl = s0 + r;
      if (sl < Sp) v[r] = direction == 0 ? src[x0 + static_cast<long long>(sl) * row_vecs]
                                         : src[y0 + static_cast<long long>(sl) * piece_vecs];
    }
#pragma unroll
    for (int r = 0; r < kPermuteRows; ++r) {
      const int sl = s0 + r;
      if (sl < Sp) {
        if (direction == 0)
          dst[y0 + static_cast<long long>(sl) * piece_vecs] = v[r];
        else
          dst[x0 + static_cast<long long>(sl) * row_vecs] = v[r];
      }
    }
  }
}

}  // namespace cpattn
