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
// vectors [x*blockDim, ...) of row (p = z / B, b = z % B, s_local = y, y + gridDim.y, ...).
// A row of H*D elements splits into P contiguous pieces of (H/P)*D elements, one per
// head group q, which are contiguous rows of Y.  So the X side is one contiguous row
// per block and the Y side is P contiguous runs; every access is one vector of type V.
#pragma once

#include <cstdint>

namespace cpattn {

constexpr int kPermuteThreads = 128;

template <typename V>
__global__ void __launch_bounds__(kPermuteThreads)
    ulysses_permute_kernel(const V* __restrict__ src, V* __restrict__ dst, int P, int B, int Sp, int row_vecs,
                           int piece_vecs, int direction) {
  const int i = blockIdx.x * kPermuteThreads + threadIdx.x;  // vector within the token row
  if (i >= row_vecs) return;
  const int q = i / piece_vecs;  // head group of this vector
  const int w = i - q * piece_vecs;
  const int pb = blockIdx.z;
  const int p = pb / B;
  const int b = pb - p * B;
  const long long S = static_cast<long long>(Sp) * P;
  for (int sl = blockIdx.y; sl < Sp; sl += gridDim.y) {
    const long long x_idx = (static_cast<long long>(pb) * Sp + sl) * row_vecs + i;
    const long long y_idx = ((static_cast<long long>(q) * B + b) * S + static_cast<long long>(p) * Sp + sl) *
                                piece_vecs + w;
    if (direction == 0)
      dst[y_idx] = src[x_idx];
    else
      dst[x_idx] = src[y_idx];
  }
}

}  // namespace cpattn
