// attn_fwd_sm100.cuh - non-causal blockwise attention with LSE for B200 (sm_100a).
//
// Computes, for every (batch b, head h, K/V block c, query row i),
//   S_ij = scale * q_i . k_j  over the keys j of block c,
//   O_i  = sum_j softmax_j(S_ij) v_j,   lse_i = ln sum_j exp(S_ij)
// ("Attention backends", "Available backends": scaled_dot_product_attention; the
// per-block fp32 output + LSE follow ContextParallelConfig.convert_to_fp32 on the
// "Parallelism" API page, so that ring blocks can be merged afterwards).
//
// Design (one CTA per SM, persistent over work items (b, h, c, q-tile)):
//   warp 0      TMA producer: Q tile (128 rows x D) once per item, then K and V tiles
//               (128 keys x D) through a ring of kStages shared-memory stages.
//   warp 1      allocates TMEM; one elected thread issues every tcgen05.mma:
//               S = Q K^T (SS form, K-major operands) into a double-buffered S in TMEM,
//               O += P V (TS form: P read from TMEM, V MN-major from shared memory).
//   warps 2..5  softmax warpgroup: thread t of warp w owns query row 32*(w%4)+t, which
//               is TMEM lane 32*(w%4)+t.  It loads its S row (fp32), masks keys past the
//               block end, updates the running max m / sum l (base-2 domain), writes
//               P = 2^(S*scale*log2e - m) as bf16 pairs over the first 64 columns of
//               the same S buffer, and after the last tile writes O/l and the LSE.
// The running max is updated lazily: O (in TMEM) is rescaled only when a row's max
// grows by more than 8 (a factor 256); otherwise the stale max stays, which is exact
// because O and l share it and 2^8 cannot overflow fp32 or bf16.
// TMEM columns: S buffers at [0,128) and [128,256), O at [256, 256+D).
// Every mbarrier wait is bounded (see ptx_sm100.cuh); on a timeout every role leaves
// its loop, in-flight TMA loads and MMAs are drained, TMEM is freed and the kernel
// returns with CP_ERR_TIMEOUT recorded in the device status word.
#pragma once

#include <cuda.h>

#include "ptx_sm100.cuh"

namespace cpattn {

constexpr int kBM = 128;          // query rows per tile (TMEM lanes)
constexpr int kBN = 128;          // keys per K/V tile
constexpr int kStages = 2;        // K/V shared-memory stages
constexpr int kAttnThreads = 192; // 6 warps
constexpr int kTmemCols = 512;
constexpr int kMaxChunks = 64;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct AttnParams {
  int B, H, Sq;
  int n_chunks;
  int n_qt;                  // ceil(Sq / kBM)
  int total_items;           // B * H * n_chunks * n_qt
  float scale_log2;          // scale * log2(e)
  void* out;                 // chunk c at out + c*out_chunk_stride elements, [B][Sq][H][D]
  int out_f32;               // 1: fp32 output, 0: bf16 output
  long long out_chunk_stride;
  float* lse;                // chunk c at lse + c*lse_chunk_stride, [B][H][Sq]; may be null
  long long lse_chunk_stride;
  int* status;               // device status word
  int bounds[kMaxChunks + 1];  // K/V row bounds of the blocks
};

template <int D>
struct AttnSmem {
  static constexpr int kHalfBytes = kBM * 64 * 2;          // 128 rows x 64 bf16 = one 128B-swizzled box
  static constexpr int kTileBytes = kBM * D * 2;           // 128 rows x D bf16
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTileBytes;
  static constexpr int kV = kK + kStages * kTileBytes;
  static constexpr int kBar = kV + kStages * kTileBytes;
  static constexpr int kNumBars = 17;
  static constexpr int kUsed = kBar + kNumBars * 8 + 16;
  // Ask for more than half an SM's shared memory so that exactly one CTA (which owns
  // all 512 TMEM columns) is resident per SM.
  static constexpr int kRequest = (kUsed + 1024) > 120 * 1024 ? (kUsed + 1024) : 120 * 1024;
};

struct ItemCoord {
  int b, h, c, qt;
};

__device__ __forceinline__ ItemCoord decode_item(int item, const AttnParams& p) {
  ItemCoord r;
  r.qt = item % p.n_qt;
  int t = item / p.n_qt;
  r.c = t % p.n_chunks;
  t /= p.n_chunks;
  r.h = t % p.H;
  r.b = t / p.H;
  return r;
}

// All lanes wait; the warp proceeds only if every lane saw the phase complete.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status) {
  const bool ok = mbar_wait(bar, parity, abort_flag, status);
  return __all_sync(0xffffffffu, ok);
}

// Wait bounded by time only (used to drain in-flight work after an abort).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitLimitCycles) return;
  }
}

template <int D>
__device__ __forceinline__ void attn_producer(const CUtensorMap* tm_q, const CUtensorMap* tm_k,
                                              const CUtensorMap* tm_v, const AttnParams& p, uint8_t* smem,
                                              uint64_t* bars, volatile int* abort_flag) {
  using L = AttnSmem<D>;
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;
  uint64_t* k_empty = bars + 4;
  uint64_t* v_full = bars + 6;
  uint64_t* v_empty = bars + 8;
  uint32_t kc_k = 0, kc_v = 0;  // tiles issued into the K and V rings
  int t_ne = 0;                 // items with at least one K/V tile
  bool ok = true;
  for (int item = blockIdx.x; item < p.total_items && ok; item += gridDim.x) {
    const ItemCoord ic = decode_item(item, p);
    const int kv0 = p.bounds[ic.c];
    const int kvlen = p.bounds[ic.c + 1] - kv0;
    const int n_kv = (kvlen + kBN - 1) / kBN;
    if (n_kv == 0) continue;
    if (t_ne > 0 && !mbar_wait(q_empty, (t_ne - 1) & 1, abort_flag, p.status)) break;
    mbar_arrive_expect_tx(q_full, L::kTileBytes);
#pragma unroll
    for (int hf = 0; hf < D / 64; ++hf)
      tma_load_4d(smem + L::kQ + hf * L::kHalfBytes, tm_q, q_full, hf * 64, ic.h, ic.qt * kBM, ic.b);
    ++t_ne;
    for (int j = 0; j < n_kv; ++j) {
      const int row = kv0 + j * kBN;
      {
        const int st = kc_k % kStages;
        const uint32_t u = kc_k / kStages;
        if (u > 0 && !mbar_wait(k_empty + st, (u - 1) & 1, abort_flag, p.status)) { ok = false; break; }
        mbar_arrive_expect_tx(k_full + st, L::kTileBytes);
#pragma unroll
        for (int hf = 0; hf < D / 64; ++hf)
          tma_load_4d(smem + L::kK + st * L::kTileBytes + hf * L::kHalfBytes, tm_k, k_full + st, hf * 64, ic.h,
                      row, ic.b);
        ++kc_k;
      }
      {
        const int st = kc_v % kStages;
        const uint32_t u = kc_v / kStages;
        if (u > 0 && !mbar_wait(v_empty + st, (u - 1) & 1, abort_flag, p.status)) { ok = false; break; }
        mbar_arrive_expect_tx(v_full + st, L::kTileBytes);
#pragma unroll
        for (int hf = 0; hf < D / 64; ++hf)
          tma_load_4d(smem + L::kV + st * L::kTileBytes + hf * L::kHalfBytes, tm_v, v_full + st, hf * 64, ic.h,
                      row, ic.b);
        ++kc_v;
      }
    }
  }
  // Drain: every issued load lands before the CTA may exit (normal path: already done).
  if (t_ne > 0) drain_wait(q_full, (t_ne - 1) & 1);
  for (int st = 0; st < kStages; ++st) {
    const uint32_t uk = kc_k / kStages + (st < static_cast<int>(kc_k % kStages) ? 1u : 0u);
    const uint32_t uv = kc_v / kStages + (st < static_cast<int>(kc_v % kStages) ? 1u : 0u);
    if (uk > 0) drain_wait(k_full + st, (uk - 1) & 1);
    if (uv > 0) drain_wait(v_full + st, (uv - 1) & 1);
  }
}

template <int D>
__device__ __forceinline__ void attn_mma(const AttnParams& p, uint8_t* smem, uint64_t* bars, uint32_t tmem,
                                         volatile int* abort_flag) {
  using L = AttnSmem<D>;
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;
  uint64_t* k_empty = bars + 4;
  uint64_t* v_full = bars + 6;
  uint64_t* v_empty = bars + 8;
  uint64_t* s_full = bars + 10;
  uint64_t* p_ready = bars + 12;
  uint64_t* o_done = bars + 14;
  uint64_t* o_free = bars + 15;
  uint64_t* drain = bars + 16;
  constexpr uint32_t kIdescQK = idesc_bf16_f32(kBM, kBN, 0);
  constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, D, 1);
  const uint32_t sQ = smem_u32(smem + L::kQ);
  const uint32_t sK = smem_u32(smem + L::kK);
  const uint32_t sV = smem_u32(smem + L::kV);
  const uint32_t tmem_o = tmem + 256;

  uint32_t kc_k = 0, kc_v = 0;  // K/V ring positions consumed
  uint32_t g = 0;               // global tile counter (S buffer = g & 1)
  int t_ne = 0;

  // S[g&1] = Q K_tile^T over D/16 k-steps of 16 (128B-swizzled K-major operands:
  // step k sits in 64-column half k/4 at byte offset 32*(k%4)).
  auto issue_qk = [&](uint32_t gg) -> bool {
    const int st = kc_k % kStages;
    if (!mbar_wait(k_full + st, (kc_k / kStages) & 1, abort_flag, p.status)) return false;
    tc_fence_after();
    const uint32_t d_tmem = tmem + (gg & 1) * kBN;
    const uint32_t kbase = sK + st * L::kTileBytes;
#pragma unroll
    for (int k = 0; k < D / 16; ++k) {
      const uint32_t off = (k >> 2) * L::kHalfBytes + (k & 3) * 32;
      tc_mma_ss(d_tmem, sdesc_sw128(sQ + off, 16, 1024), sdesc_sw128(kbase + off, 16, 1024), kIdescQK, k > 0);
    }
    tc_commit(k_empty + st);
    tc_commit(s_full + (gg & 1));
    ++kc_k;
    return true;
  };
  // O (+)= P V: P (bf16 pairs) in TMEM columns [S buffer, +64); V tile MN-major: 16 keys
  // per k-step = 2048 bytes; the two 64-wide D halves are 16 KB apart (leading offset).
  auto issue_pv = [&](uint32_t gg, bool accumulate) -> bool {
    const int st = kc_v % kStages;
    if (!mbar_wait(v_full + st, (kc_v / kStages) & 1, abort_flag, p.status)) return false;
    tc_fence_after();
    const uint32_t a_tmem = tmem + (gg & 1) * kBN;
    const uint32_t vbase = sV + st * L::kTileBytes;
#pragma unroll
    for (int k = 0; k < kBN / 16; ++k) {
      tc_mma_ts(tmem_o, a_tmem + k * 8, sdesc_sw128(vbase + k * 2048, L::kHalfBytes, 1024), kIdescPV,
                (accumulate || k > 0) ? 1u : 0u);
    }
    tc_commit(v_empty + st);
    tc_commit(o_done);
    ++kc_v;
    return true;
  };

  for (int item = blockIdx.x; item < p.total_items; item += gridDim.x) {
    const ItemCoord ic = decode_item(item, p);
    const int kvlen = p.bounds[ic.c + 1] - p.bounds[ic.c];
    const int n_kv = (kvlen + kBN - 1) / kBN;
    if (n_kv == 0) continue;
    if (!mbar_wait(q_full, t_ne & 1, abort_flag, p.status)) goto done;
    tc_fence_after();
    if (!issue_qk(g)) goto done;
    if (n_kv == 1) tc_commit(q_empty);
    for (int j = 0; j < n_kv; ++j, ++g) {
      if (j + 1 < n_kv) {
        if (!issue_qk(g + 1)) goto done;
        if (j + 2 == n_kv) tc_commit(q_empty);
      }
      if (!mbar_wait(p_ready + (g & 1), (g >> 1) & 1, abort_flag, p.status)) goto done;
      if (j == 0 && t_ne > 0) {
        if (!mbar_wait(o_free, (t_ne - 1) & 1, abort_flag, p.status)) goto done;
      }
      tc_fence_after();
      if (!issue_pv(g, j > 0)) goto done;
    }
    ++t_ne;
  }
done:
  // Drain: wait until every MMA this thread issued has completed.
  tc_commit(drain);
  drain_wait(drain, 0);
}

template <int D>
__device__ __forceinline__ void attn_softmax(const AttnParams& p, uint64_t* bars, uint32_t tmem,
                                             volatile int* abort_flag) {
  uint64_t* s_full = bars + 10;
  uint64_t* p_ready = bars + 12;
  uint64_t* o_done = bars + 14;
  uint64_t* o_free = bars + 15;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int quarter = warp & 3;
  const int row = quarter * 32 + lane;
  const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
  const uint32_t taddr_o = taddr + 256;
  const float sl2 = p.scale_log2;
  uint32_t g = 0;

  for (int item = blockIdx.x; item < p.total_items; item += gridDim.x) {
    const ItemCoord ic = decode_item(item, p);
    const int kvlen = p.bounds[ic.c + 1] - p.bounds[ic.c];
    const int n_kv = (kvlen + kBN - 1) / kBN;
    const int s_row = ic.qt * kBM + row;
    const bool row_ok = s_row < p.Sq;
    const size_t o_off = static_cast<size_t>(ic.c) * p.out_chunk_stride +
                         ((static_cast<size_t>(ic.b) * p.Sq + s_row) * p.H + ic.h) * D;
    const size_t l_off = static_cast<size_t>(ic.c) * p.lse_chunk_stride +
                         (static_cast<size_t>(ic.b) * p.H + ic.h) * p.Sq + s_row;
    if (n_kv == 0) {  // no keys: O = 0, lse = -inf
      if (row_ok) {
        if (p.out_f32) {
          float4* o = reinterpret_cast<float4*>(static_cast<float*>(p.out) + o_off);
          for (int i = 0; i < D / 4; ++i) o[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        } else {
          uint4* o = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + o_off);
          for (int i = 0; i < D / 8; ++i) o[i] = make_uint4(0u, 0u, 0u, 0u);
        }
        if (p.lse) p.lse[l_off] = -INFINITY;
      }
      continue;
    }

    float m = -INFINITY;  // running max of S*scale*log2e (possibly stale by < 8)
    float l = 0.f;        // running sum of 2^(S*scale*log2e - m)
    for (int j = 0; j < n_kv; ++j, ++g) {
      const uint32_t sb = g & 1;
      if (!warp_wait(s_full + sb, (g >> 1) & 1, abort_flag, p.status)) return;
      tc_fence_after();
      float s[kBN];
#pragma unroll
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(taddr + sb * kBN + c * 32, r);
#pragma unroll
        for (int i = 0; i < 32; ++i) s[c * 32 + i] = __uint_as_float(r[i]);
      }
      const int valid = kvlen - j * kBN;
      if (valid < kBN) {
#pragma unroll
        for (int i = 0; i < kBN; ++i)
          if (i >= valid) s[i] = -INFINITY;
      }
      float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
      for (int i = 4; i < kBN; i += 4) {
        mx0 = fmaxf(mx0, s[i]);
        mx1 = fmaxf(mx1, s[i + 1]);
        mx2 = fmaxf(mx2, s[i + 2]);
        mx3 = fmaxf(mx3, s[i + 3]);
      }
      const float m_tile = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * sl2;
      bool prev_consumed = (j == 0);
      if (j == 0) {
        m = m_tile;
      } else {
        const bool need = m_tile > m + kRescaleThreshold;
        if (__any_sync(0xffffffffu, need)) {
          // O must hold PV of the previous tile before it is rescaled.
          if (!warp_wait(o_done, (g - 1) & 1, abort_flag, p.status)) return;
          prev_consumed = true;
          tc_fence_after();
          const float m_new = need ? m_tile : m;
          const float alpha = ex2_approx(m - m_new);
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(taddr_o + c * 32, r);
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
            tmem_st32(taddr_o + c * 32, r);
          }
          tmem_wait_st();
          l *= alpha;
          m = m_new;
        }
      }
      const float neg_m = -m;
      float ls0 = 0.f, ls1 = 0.f;
      uint32_t pk[kBN / 2];
#pragma unroll
      for (int i = 0; i < kBN / 2; ++i) {
        const float p0 = ex2_approx(fmaf(s[2 * i], sl2, neg_m));
        const float p1 = ex2_approx(fmaf(s[2 * i + 1], sl2, neg_m));
        ls0 += p0;
        ls1 += p1;
        pk[i] = pack_bf16x2(p0, p1);
      }
      l += ls0 + ls1;
#pragma unroll
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t r[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) r[i] = pk[c * 16 + i];
        tmem_st16(taddr + sb * kBN + c * 16, r);
      }
      tmem_wait_st();
      // Consume PV(g-1)'s completion in order (it is long done by now).
      if (!prev_consumed) {
        if (!warp_wait(o_done, (g - 1) & 1, abort_flag, p.status)) return;
      }
      tc_fence_before();
      mbar_arrive(p_ready + sb);
    }

    // Epilogue: wait for the last PV, write O / l and the LSE, release O.
    if (!warp_wait(o_done, (g - 1) & 1, abort_flag, p.status)) return;
    tc_fence_after();
    const float inv_l = 1.f / l;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t r[32];
      tmem_ld32(taddr_o + c * 32, r);
      if (row_ok) {
        if (p.out_f32) {
          float4* o = reinterpret_cast<float4*>(static_cast<float*>(p.out) + o_off + c * 32);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            o[i] = make_float4(__uint_as_float(r[4 * i]) * inv_l, __uint_as_float(r[4 * i + 1]) * inv_l,
                               __uint_as_float(r[4 * i + 2]) * inv_l, __uint_as_float(r[4 * i + 3]) * inv_l);
        } else {
          uint4* o = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + o_off + c * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            o[i] = make_uint4(pack_bf16x2(__uint_as_float(r[8 * i + 0]) * inv_l, __uint_as_float(r[8 * i + 1]) * inv_l),
                              pack_bf16x2(__uint_as_float(r[8 * i + 2]) * inv_l, __uint_as_float(r[8 * i + 3]) * inv_l),
                              pack_bf16x2(__uint_as_float(r[8 * i + 4]) * inv_l, __uint_as_float(r[8 * i + 5]) * inv_l),
                              pack_bf16x2(__uint_as_float(r[8 * i + 6]) * inv_l, __uint_as_float(r[8 * i + 7]) * inv_l));
        }
      }
    }
    if (row_ok && p.lse) p.lse[l_off] = (m + log2f(l)) * 0.69314718055994530942f;
    tc_fence_before();
    mbar_arrive(o_free);
  }
}

template <int D>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ AttnParams p) {
  using L = AttnSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + L::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5;

  if (threadIdx.x == 0) {
    mbar_init(bars + 0, 1);   // q_full (TMA tx)
    mbar_init(bars + 1, 1);   // q_empty (MMA commit)
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bars + 2 + s, 1);  // k_full
      mbar_init(bars + 4 + s, 1);  // k_empty
      mbar_init(bars + 6 + s, 1);  // v_full
      mbar_init(bars + 8 + s, 1);  // v_empty
    }
    mbar_init(bars + 10, 1);   // s_full[0]
    mbar_init(bars + 11, 1);   // s_full[1]
    mbar_init(bars + 12, 128); // p_ready[0] (softmax threads)
    mbar_init(bars + 13, 128); // p_ready[1]
    mbar_init(bars + 14, 1);   // o_done (MMA commit after each PV)
    mbar_init(bars + 15, 128); // o_free (softmax epilogue done with O)
    mbar_init(bars + 16, 1);   // drain
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && (threadIdx.x & 31) == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Producer and MMA roles run on lane 0 of their warp; the other lanes wait at the
  // __syncwarp so that each warp is converged again for the teardown below.
  if (warp == 0) {
    if ((threadIdx.x & 31) == 0) attn_producer<D>(&tm_q, &tm_k, &tm_v, p, smem, bars, abort_flag);
    __syncwarp();
  } else if (warp == 1) {
    if ((threadIdx.x & 31) == 0) attn_mma<D>(p, smem, bars, tmem, abort_flag);
    __syncwarp();
  } else {
    attn_softmax<D>(p, bars, tmem, abort_flag);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace cpattn
