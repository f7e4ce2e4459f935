// peer.cuh - the Ulysses exchange and the step barrier with one process per GPU.
//
// "Context parallelism", "Ulysses Attention": the two all-to-alls, done by pushes into
// peer memory (buffers of the other GPUs mapped into this process with CUDA IPC).  Per
// rank, with no leading degree dimension (P ranks, Sp = S/P tokens and Hp = H/P heads
// per shard):
//   sequence shard of rank r   X_r[b][s][h][:]    [B][Sp][H][D]
//   head shard of rank q       Y_q[b][t][j][:]    [B][S][Hp][D]
//   forward (direction 0): rank r stores, for every q,
//       Y_q[b][r*Sp + s][j] = X_r[b][s][q*Hp + j]
//   inverse (direction 1): rank r stores, for every p,
//       X_p[b][s][r*Hp + j] = Y_r[b][p*Sp + s][j]
// Run on every rank, the forward push fills exactly the layout of the single-GPU
// exchange (ulysses_permute.cuh) split by rank.  Reads are local and writes go to the
// owner, so every byte crosses NVLink once, as a store.
//
// The barrier orders the steps of one exchange across ranks: each rank writes the step's
// epoch into its slot of every rank's signal pad, then waits, bounded, until every slot
// of its own pad has reached the epoch.
#pragma once

#include <cstdint>

#include "ptx_sm100.cuh"
#include "ulysses_permute.cuh"

namespace cpattn {

constexpr int kPeerMax = 16;  // ranks in one exchange group

struct PushArgs {
  const void* src[kPermuteMaxTensors];
  void* dst[kPermuteMaxTensors][kPeerMax];  // dst[t][q]: tensor t's buffer on rank q
};

// Work row (b, s) for s < Sp: P pieces of piece_vecs vectors, piece q going to (dir 0) or
// coming from (dir 1) rank q.  grid.x covers the P*piece_vecs vectors of a work row,
// grid.y groups of kPermuteRows rows (strided by gridDim.y), grid.z = tensor * B + b.
template <typename V>
__global__ void __launch_bounds__(kPermuteThreads)
    ulysses_push_kernel(const __grid_constant__ PushArgs a, int rank, int P, int B, int Sp, int piece_vecs,
                        int direction) {
  const int row_vecs = P * piece_vecs;  // H*D elements of a sequence-shard row
  const int i = blockIdx.x * kPermuteThreads + threadIdx.x;
  if (i >= row_vecs) return;
  const int q = i / piece_vecs;
  const int w = i - q * piece_vecs;
  const int n = blockIdx.z / B;
  const int b = blockIdx.z - n * B;
  const V* __restrict__ src = static_cast<const V*>(a.src[n]);
  V* __restrict__ dst = static_cast<V*>(a.dst[n][q]);
  const long long S = static_cast<long long>(Sp) * P;
  // Vector offsets of work row 0 and the row strides, on the source and destination side.
  const long long x0 = static_cast<long long>(b) * Sp * row_vecs;  // X row (b, 0)
  long long s0, ss, d0, ds;
  if (direction == 0) {
    s0 = x0 + i;
    ss = row_vecs;
    d0 = (static_cast<long long>(b) * S + static_cast<long long>(rank) * Sp) * piece_vecs + w;
    ds = piece_vecs;
  } else {
    s0 = (static_cast<long long>(b) * S + static_cast<long long>(q) * Sp) * piece_vecs + w;
    ss = piece_vecs;
    d0 = x0 + static_cast<long long>(rank) * piece_vecs + w;
    ds = row_vecs;
  }
  const long long total = static_cast<long long>(B) * Sp * row_vecs;  // vectors of X_r and of Y_q alike
  for (int sl0 = blockIdx.y * kPermuteRows; sl0 < Sp; sl0 += gridDim.y * kPermuteRows) {
    V v[kPermuteRows];
#pragma unroll
    for (int r = 0; r < kPermuteRows; ++r) {
      const int sl = sl0 + r;
      if (sl < Sp && in_bounds(s0 + sl * ss, 1, total)) v[r] = src[s0 + sl * ss];
    }
#pragma unroll
    for (int r = 0; r < kPermuteRows; ++r) {
      const int sl = sl0 + r;
      if (sl < Sp && in_bounds(d0 + sl * ds, 1, total)) dst[d0 + sl * ds] = v[r];
    }
  }
  // No fence here: a kernel's stores, to other GPUs included, are performed when it
  // completes, before the barrier kernel that follows it on the stream signals anyone.
}

// "Ulysses Anything Attention" with one process per GPU: shards of unequal size.  Sequence
// shard p holds tokens [seq[p], seq[p+1]) and head shard q heads [head[q], head[q+1])
// (either may be empty); per rank, X_r is [B][S_r][H][D] and Y_q is [B][S][H_q][D]:
//   forward (direction 0): rank r stores, for every q,
//       Y_q[b][seq[r] + s][j] = X_r[b][s][head[q] + j]
//   inverse (direction 1): rank r stores, for every p,
//       X_p[b][s][head[r] + j] = Y_r[b][seq[p] + s][j]
struct AnyPushArgs {
  const void* src[kPermuteMaxTensors];
  void* dst[kPermuteMaxTensors][kPeerMax];
  int seq[kPeerMax + 1];
  int head[kPeerMax + 1];
};

// Forward: grid.x covers the vectors (VE elements, never crossing a head) of an X_r row,
// grid.y groups of kPermuteRows rows of X_r (strided), grid.z = tensor * B + b.
// Inverse: grid.x covers the vectors of a Y_r row, grid.y groups of rows of the
// destination shard p, grid.z = (tensor * B + b) * P + p.
template <typename V>
__global__ void __launch_bounds__(kPermuteThreads)
    ulysses_anything_push_kernel(const __grid_constant__ AnyPushArgs a, int rank, int P, int B, int H, int D, int VE,
                                 int direction) {
  const int S = a.seq[P];
  const long long i = static_cast<long long>(blockIdx.x) * kPermuteThreads + threadIdx.x;
  long long s0, ss, d0, ds, src_total, dst_total;  // vector offsets of row 0, row strides, extents
  int rows;
  V* __restrict__ dst;
  const V* __restrict__ src;
  if (direction == 0) {
    if (i * VE >= static_cast<long long>(H) * D) return;
    const int n = blockIdx.z / B, b = blockIdx.z - (blockIdx.z / B) * B;
    const long long e = i * VE;
    const int h = static_cast<int>(e / D);
    int q = 0;
    while (a.head[q + 1] <= h) ++q;  // the head group holding h (groups may be empty)
    const long long Hq = a.head[q + 1] - a.head[q];
    const int Sr = a.seq[rank + 1] - a.seq[rank];
    rows = Sr;
    src = static_cast<const V*>(a.src[n]);
    dst = static_cast<V*>(a.dst[n][q]);
    s0 = (static_cast<long long>(b) * Sr * H * D + e) / VE;
    ss = static_cast<long long>(H) * D / VE;
    d0 = ((static_cast<long long>(b) * S + a.seq[rank]) * Hq * D + e - static_cast<long long>(a.head[q]) * D) / VE;
    ds = Hq * D / VE;
    src_total = static_cast<long long>(B) * Sr * H * D / VE;
    dst_total = static_cast<long long>(B) * S * Hq * D / VE;
  } else {
    const long long Hr = a.head[rank + 1] - a.head[rank];
    if (i * VE >= Hr * D) return;
    const int z = blockIdx.z / P, p = blockIdx.z - (blockIdx.z / P) * P;
    const int n = z / B, b = z - (z / B) * B;
    const long long e = i * VE;
    const int Sp = a.seq[p + 1] - a.seq[p];
    rows = Sp;
    src = static_cast<const V*>(a.src[n]);
    dst = static_cast<V*>(a.dst[n][p]);
    s0 = ((static_cast<long long>(b) * S + a.seq[p]) * Hr * D + e) / VE;
    ss = Hr * D / VE;
    d0 = (static_cast<long long>(b) * Sp * H * D + static_cast<long long>(a.head[rank]) * D + e) / VE;
    ds = static_cast<long long>(H) * D / VE;
    src_total = static_cast<long long>(B) * S * Hr * D / VE;
    dst_total = static_cast<long long>(B) * Sp * H * D / VE;
  }
  for (int sl0 = blockIdx.y * kPermuteRows; sl0 < rows; sl0 += gridDim.y * kPermuteRows) {
    V v[kPermuteRows];
#pragma unroll
    for (int r = 0; r < kPermuteRows; ++r) {
      const int sl = sl0 + r;
      if (sl < rows && in_bounds(s0 + sl * ss, 1, src_total)) v[r] = src[s0 + sl * ss];
    }
#pragma unroll
    for (int r = 0; r < kPermuteRows; ++r) {
      const int sl = sl0 + r;
      if (sl < rows && in_bounds(d0 + sl * ds, 1, dst_total)) dst[d0 + sl * ds] = v[r];
    }
  }
}

struct SignalTable {
  uint32_t* pad[kPeerMax];  // pad[q]: rank q's signal pad, one word per rank
};

__device__ __forceinline__ void st_release_sys(uint32_t* p, uint32_t v) {
  asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_sys(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// One warp.  Lane q < P signals rank q (after a system-scope fence, so that this rank's
// earlier writes, the stream's previous kernels included, are visible first), then lane q
// waits for rank q's signal in this rank's pad.  Epochs increase by one per barrier and
// are compared modulo 2^32.  A wait that runs past `limit_ns` of wall-clock time (the
// global timer) gives up and records kDevTimeout in `status`; the kernel then returns.
__global__ void __launch_bounds__(32)
    peer_barrier_kernel(const __grid_constant__ SignalTable t, int rank, int P, uint32_t epoch, uint64_t limit_ns,
                        int* status) {
  const int q = threadIdx.x;
  if (q < P) {
    __threadfence_system();
    st_release_sys(t.pad[q] + rank, epoch);
  }
  bool ok = true;
  if (q < P) {
    const uint32_t* w = t.pad[rank] + q;
    const uint64_t t0 = global_ns();
    int polls = 0;
    while (static_cast<int>(ld_acquire_sys(w) - epoch) < 0) {
      if ((++polls & 15) == 0 && global_ns() - t0 > limit_ns) {
        ok = false;
        break;
      }
      __nanosleep(128);
    }
  }
  if (!__all_sync(0xffffffffu, ok) && q == 0) atomicExch(status, kDevTimeout);
}

}  // namespace cpattn
