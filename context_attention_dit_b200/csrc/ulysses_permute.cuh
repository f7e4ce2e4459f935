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

#include "ptx_sm100.cuh"

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
  const long long total = static_cast<long long>(P) * B * Sp * row_vecs;  // vectors per tensor
  for (int s0 = blockIdx.y * kPermuteRows; s0 < Sp; s0 += gridDim.y * kPermuteRows) {
    V v[kPermuteRows];
#pragma unroll
    for (int r = 0; r < kPermuteRows; ++r) {
      const int sl = s0 + r;
      const long long xi = x0 + static_cast<long long>(sl) * row_vecs, yi = y0 + static_cast<long long>(sl) * piece_vecs;
      if (sl < Sp && in_bounds(direction == 0 ? xi : yi, 1, total)) v[r] = src[direction == 0 ? xi : yi];
    }
#pragma unroll
    for (int r = 0; r < kPermuteRows; ++r) {
      const int sl = s0 + r;
      const long long xi = x0 + static_cast<long long>(sl) * row_vecs, yi = y0 + static_cast<long long>(sl) * piece_vecs;
      if (sl < Sp && in_bounds(direction == 0 ? yi : xi, 1, total)) dst[direction == 0 ? yi : xi] = v[r];
    }
  }
}

// The exchange for shards of unequal size ("Ulysses Anything Attention": the sequence
// length and head count need not be divisible by the degree).  Sequence shard p holds
// tokens [seq[p], seq[p+1]) of every head, packed at element offset B*seq[p]*H*D as
// [B][S_p][H][D]; head shard q holds heads [head[q], head[q+1]) of every token, packed at
// B*S*head[q]*D as [B][S][H_q][D].  With equal shards both are the stacked layouts above.
constexpr int kPermuteMaxDegree = 64;

struct AnyBounds {
  int seq[kPermuteMaxDegree + 1];
  int head[kPermuteMaxDegree + 1];
};

// Walks the sequence-sharded rows: grid.x covers the vectors of a token row (VE elements
// each, D a multiple of VE so no vector crosses a head), grid.y groups of kPermuteRows rows
// of a shard (strided by gridDim.y), grid.z = (tensor * P + p) * B + b.  Each thread finds
// the head group of its vector once and reuses it for every row.
template <typename V>
__global__ void __launch_bounds__(kPermuteThreads)
    ulysses_anything_kernel(const __grid_constant__ PermuteArgs a, const __grid_constant__ AnyBounds bd, int P, int B,
                            int S, int H, int D, int VE, int direction) {
  const int row_vecs = H * D / VE;
  const int i = blockIdx.x * kPermuteThreads + threadIdx.x;
  if (i >= row_vecs) return;
  const int n = blockIdx.z / (P * B);
  const int pb = blockIdx.z - n * (P * B);
  const int p = pb / B;
  const int b = pb - p * B;
  const V* __restrict__ src = static_cast<const V*>(a.src[n]);
  V* __restrict__ dst = static_cast<V*>(a.dst[n]);
  const int s0 = bd.seq[p];
  const int Sp = bd.seq[p + 1] - s0;
  const long long e = static_cast<long long>(i) * VE;  // element within the token row
  const int h = static_cast<int>(e / D);
  int q = 0;
  while (bd.head[q + 1] <= h) ++q;  // the group holding head h (groups may be empty)
  const int hq = bd.head[q];
  const long long Hq = bd.head[q + 1] - hq;
  const long long w = e - static_cast<long long>(hq) * D;  // element within the group's row
  // Vector offsets of row s_local of this (p, b) on each side.
  const long long x0 = (static_cast<long long>(B) * s0 * H * D + static_cast<long long>(b) * Sp * H * D + e) / VE;
  const long long xs = static_cast<long long>(H) * D / VE;
  const long long y0 = (static_cast<long long>(B) * S * hq * D + (static_cast<long long>(b) * S + s0) * Hq * D + w) / VE;
  const long long ys = Hq * D / VE;
  const long long total = static_cast<long long>(B) * S * H * D / VE;  // vectors per buffer
  for (int sl0 = blockIdx.y * kPermuteRows; sl0 < Sp; sl0 += gridDim.y * kPermuteRows) {
    V v[kPermuteRows];
#pragma unroll
    for (int r = 0; r < kPermuteRows; ++r) {
      const int sl = sl0 + r;
      const long long si = direction == 0 ? x0 + sl * xs : y0 + sl * ys;
      if (sl < Sp && in_bounds(si, 1, total)) v[r] = src[si];
    }
#pragma unroll
    for (int r = 0; r < kPermuteRows; ++r) {
      const int sl = sl0 + r;
      const long long di = direction == 0 ? y0 + sl * ys : x0 + sl * xs;
      if (sl < Sp && in_bounds(di, 1, total)) dst[di] = v[r];
    }
  }
}

// LSE of attention computed on the head-sharded layout, [P][B][H/P][S] (head group p =
// heads [p*H/P, (p+1)*H/P)), regrouped to [B][H][S]: the (p, b) block of (H/P)*S floats is
// contiguous on both sides.  grid.y = p*B + b; grid.x strides over the block.
__global__ void __launch_bounds__(256) lse_regroup_kernel(const float* __restrict__ src, float* __restrict__ dst,
                                                          int P, int B, long long block) {
  const int pb = blockIdx.y;
  const int p = pb / B;
  const int b = pb - p * B;
  const float* s = src + static_cast<long long>(pb) * block;
  float* d = dst + (static_cast<long long>(b) * P + p) * block;
  const long long total = static_cast<long long>(P) * B * block;
  for (long long i = blockIdx.x * 256LL + threadIdx.x; i < block; i += gridDim.x * 256LL)
    if (in_bounds(static_cast<long long>(pb) * block + i, 1, total) &&
        in_bounds((static_cast<long long>(b) * P + p) * block + i, 1, total))
      d[i] = s[i];
}

}  // namespace cpattn
