// lse_merge.cuh - merge per-block attention partials through their log-sum-exps.
//
// "Context parallelism", "Ring Attention": a GPU's queries see the K/V blocks one
// after another; ContextParallelConfig.convert_to_fp32 ("Parallelism" API page)
// keeps every block's output and LSE in float32 for this accumulation.  The merge
// (the standard log-sum-exp combination; the pages do not print it) is
//   M = max_i lse_i,  L = M + ln sum_i exp(lse_i - M),  O = sum_i exp(lse_i - L) O_i
// with empty blocks (lse_i = -inf) weighted 0 and all-empty rows giving O = 0, L = -inf.
//
// Work layout: a block takes ST consecutive query positions s of one batch b (all heads),
// i.e. ST*H rows.  It first stages their LSEs (n blocks x H heads x ST positions) in
// shared memory with loads that are contiguous along s, then its warps walk the rows with
// the head fastest, so consecutive warps read consecutive 512-byte partial rows (one
// contiguous H*D*4-byte run per position) and write consecutive output rows.  Per row,
// lane i holds lse_i and lse_{i+32}; the max and the sum are warp-shuffle reductions;
// each lane then streams D/32 floats of every block with one vector load per block.
#pragma once

#include <cuda_bf16.h>

#include "ptx_sm100.cuh"

namespace cpattn {

constexpr int kMergeThreads = 256;
constexpr int kPeerMergeMax = 16;  // ranks of a Ulysses group

// kUlysses: the partials are those of attention on Ulysses head shards (batch P*Bs, H heads
// per shard, shard p = heads [p*H, (p+1)*H) of P*H), and the merged output goes straight to
// the sequence-sharded layout of the inverse exchange, [P][Bs][Sq/P][P*H][D] (the merge and
// the second all-to-all of "Ulysses Attention" in one pass), with the LSE as [Bs][P*H][Sq].
//
// kPeer (one process per GPU): the partials are this rank's head shard only (batch Bs, H
// heads, shard index `shard` of P), and the merged row of token s goes to rank s/(Sq/P)'s
// sequence shard, peer_out[s/(Sq/P)] as [Bs][Sq/P][P*H][D], over peer memory: the merge and
// this rank's half of the second all-to-all in one kernel.  No LSE is written.
struct MergePeers {
  void* out[kPeerMergeMax];
};

template <int D, bool kOutBf16, bool kUlysses, bool kPeer = false>
__global__ void __launch_bounds__(kMergeThreads)
    lse_merge_kernel(const float* __restrict__ partials, const float* __restrict__ lses, int n, void* __restrict__ out,
                     float* __restrict__ out_lse, int H, int Sq, int ST, long long part_stride, long long lse_stride,
                     int P, int Bs, const __grid_constant__ MergePeers peers = MergePeers{}, int shard = 0) {
  constexpr int kVec = D / 32;  // floats per lane: 4 (D=128) or 2 (D=64)
  constexpr float kLog2e = 1.4426950408889634f;
  constexpr float kLn2 = 0.69314718055994530942f;
  extern __shared__ float lse_s[];  // [n][H][ST]
  const int b = blockIdx.y;
  const int s0 = blockIdx.x * ST;
  const int HS = H * ST;
  for (int idx = threadIdx.x; idx < n * HS; idx += kMergeThreads) {
    const int c = idx / HS;
    const int rem = idx - c * HS;
    const int h = rem / ST;
    const int st = rem - h * ST;
    const int s = s0 + st;
#ifdef CP_DEBUG
    const long long li = c * lse_stride + (static_cast<long long>(b) * H + h) * Sq + s;
    lse_s[idx] = s < Sq && in_bounds(li, 1, n * lse_stride) ? __ldg(lses + li) : -INFINITY;
#else
    lse_s[idx] = s < Sq ? __ldg(lses + c * lse_stride + (static_cast<long long>(b) * H + h) * Sq + s) : -INFINITY;
#endif
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  for (int r = threadIdx.x >> 5; r < HS; r += kMergeThreads / 32) {
    const int st = r / H;
    const int h = r - st * H;
    const int s = s0 + st;
    if (s >= Sq) break;  // rows are ordered by st: every later row is past Sq too
    const float l0 = lane < n ? lse_s[(lane * H + h) * ST + st] : -INFINITY;
    const float l1 = lane + 32 < n ? lse_s[((lane + 32) * H + h) * ST + st] : -INFINITY;
    float M = fmaxf(l0, l1);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const long long row = (static_cast<long long>(b) * Sq + s) * H + h;  // BSHD row
    const long long eoff = row * D + lane * kVec;
    long long ooff = eoff;                                                 // output element
    long long lrow = (static_cast<long long>(b) * H + h) * Sq + s;        // [B][H][Sq]
    void* dst = out;
    if (kUlysses) {
      const int p = b / Bs, bs = b - (b / Bs) * Bs;  // head shard, batch
      const int Sp = Sq / P;
      const int ps = s / Sp, sl = s - (s / Sp) * Sp;  // sequence shard, token within it
      ooff = (((static_cast<long long>(ps) * Bs + bs) * Sp + sl) * (static_cast<long long>(P) * H) + p * H + h) * D +
             lane * kVec;
      lrow = (static_cast<long long>(bs) * P * H + p * H + h) * Sq + s;
    }
    if (kPeer) {
      const int Sp = Sq / P;
      const int ps = s / Sp, sl = s - (s / Sp) * Sp;  // owner rank, token within its shard
      dst = peers.out[ps];
      ooff = ((static_cast<long long>(b) * Sp + sl) * (static_cast<long long>(P) * H) + shard * H + h) * D + lane * kVec;
    }
#ifdef CP_DEBUG
    // The row's partial vectors (every block), its output vector and its LSE.  The whole
    // warp skips the row, so that the shuffles below stay converged.
    const long long rows_total = lse_stride;  // B*H*Sq rows in every block and in the output
    const bool ok = in_bounds(eoff + (n - 1) * part_stride, kVec, n * part_stride) &&
                    in_bounds(ooff, kVec, rows_total * D) && in_bounds(lrow, 1, rows_total);
    if (!__all_sync(0xffffffffu, ok)) continue;
#endif
    if (M == -INFINITY) {  // every block empty
      if (kOutBf16) {
        if (kVec == 4)
          *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(dst) + ooff) = make_uint2(0u, 0u);
        else
          *reinterpret_cast<uint32_t*>(static_cast<__nv_bfloat16*>(dst) + ooff) = 0u;
      } else {
        float* o = static_cast<float*>(dst) + ooff;
#pragma unroll
        for (int i = 0; i < kVec; ++i) o[i] = 0.f;
      }
      if (!kPeer && lane == 0 && out_lse) out_lse[lrow] = -INFINITY;
      continue;
    }
    // exp(x - M) = 2^((x - M) * log2 e); exp(-inf) = 0 for empty blocks.
    float tot = ex2_approx((l0 - M) * kLog2e) + ex2_approx((l1 - M) * kLog2e);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
    const float L2 = M * kLog2e + __log2f(tot);  // merged LSE in base 2
    const float w0 = ex2_approx(l0 * kLog2e - L2);
    const float w1 = ex2_approx(l1 * kLog2e - L2);

    float acc[kVec];
#pragma unroll
    for (int i = 0; i < kVec; ++i) acc[i] = 0.f;
    const float* src = partials + eoff;
#pragma unroll 8
    for (int c = 0; c < n; ++c) {
      const float w = __shfl_sync(0xffffffffu, c < 32 ? w0 : w1, c & 31);
      if (kVec == 4) {
        const float4 v = __ldcs(reinterpret_cast<const float4*>(src + c * part_stride));
        acc[0] = fmaf(w, v.x, acc[0]);
        acc[1] = fmaf(w, v.y, acc[1]);
        acc[2] = fmaf(w, v.z, acc[2]);
        acc[3] = fmaf(w, v.w, acc[3]);
      } else {
        const float2 v = __ldcs(reinterpret_cast<const float2*>(src + c * part_stride));
        acc[0] = fmaf(w, v.x, acc[0]);
        acc[1] = fmaf(w, v.y, acc[1]);
      }
    }
    if (kOutBf16) {
      __nv_bfloat16* o = static_cast<__nv_bfloat16*>(dst) + ooff;
      if (kVec == 4)
        *reinterpret_cast<uint2*>(o) = make_uint2(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]));
      else
        *reinterpret_cast<uint32_t*>(o) = pack_bf16x2(acc[0], acc[1]);
    } else {
      float* o = static_cast<float*>(dst) + ooff;
      if (kVec == 4)
        *reinterpret_cast<float4*>(o) = make_float4(acc[0], acc[1], acc[2], acc[3]);
      else
        *reinterpret_cast<float2*>(o) = make_float2(acc[0], acc[1]);
    }
    if (!kPeer && lane == 0 && out_lse) out_lse[lrow] = L2 * kLn2;
  }
}

}  // namespace cpattn
