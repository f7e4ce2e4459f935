// attn_pair_sm100.cuh - non-causal blockwise attention with LSE for B200 (sm_100a), two
// 128-row Q tiles per CTA sharing every K/V tile.
//
// Computes what attn_fwd_sm100.cuh computes ("Attention backends", "Available backends":
// scaled_dot_product_attention; per-block fp32 output + LSE as ContextParallelConfig.
// convert_to_fp32 on the "Parallelism" page), with a different division of the work:
//
//   A work unit is (batch b, head h, pair of 128-row Q tiles = 256 query rows).  Each K/V
//   tile is staged in shared memory once and used by both Q tiles, which halves the
//   shared-memory operand traffic per FLOP of the QK^T and P.V products (the K and V tiles
//   are written once and read twice) and the K/V reads from L2.
//   warps 0-3   softmax warpgroup 0: rows of Q tile 0, one row per thread (= TMEM lane),
//               all 128 keys of every K/V tile;
//   warps 4-7   softmax warpgroup 1: the same for Q tile 1.
//               Each keeps its own running max m_i, sum l_i and accumulator O_i, so the two
//               groups never wait for each other: while one computes its softmax, the
//               tensor cores run the other's products.
//   warp 8      TMA producer of Q (both tiles) and K (two stages);
//   warp 9      TMEM owner (512 columns) and QK issuer: S_i(t) = Q_i K(t)^T, i = 0, 1;
//   warp 10     TMA producer of V (two stages);
//   warp 11     P.V issuer: O_i += P_i(t) V(t) (TS form, P from TMEM), i = 0, 1;
//   warps 12-15 epilogue: at a segment's end (one K/V block, or every block when fused)
//               it reads O_i, releases it, and writes O_i / l_i and the LSE m_i + ln l_i.
// TMEM columns: S_0 [0,128), S_1 [128,256) (P_i as bf16 pairs over columns 0..63 of S_i),
// O_0 [256,256+D), O_1 [384,384+D).
// Dependencies per Q tile i: softmax_i(t) -> P.V_i(t) -> QK_i(t+1) (S_i holds P_i(t)) ->
// softmax_i(t+1).  The lazy max (rescale of O_i only when a row's max grows by more than
// 8 in log2 units), the software 2^x for one pair in four, the bounded waits and the
// abort/drain path follow attn_fwd_sm100.cuh.
#pragma once

#include <cuda.h>

#include "attn_fwd_sm100.cuh"

namespace cpattn {
namespace pair {

constexpr int kRows = 256;            // query rows per work unit (two Q tiles)
constexpr int kThreads = 512;
constexpr int kProducerWarp = 8;      // Q and K loads
constexpr int kQkWarp = 9;            // TMEM owner, QK issuer
constexpr int kVProducerWarp = 10;    // V loads
constexpr int kPvWarp = 11;           // P.V issuer
constexpr int kEpilogueWarp0 = 12;
// setmaxnreg split of the 128 x 512 launch budget: softmax (a whole 128-key S row per
// thread), control warps, epilogue (32 columns of an O row at a time).
constexpr int kSoftmaxRegs = 200;
constexpr int kControlRegs = 48;
constexpr int kEpilogueRegs = 64;
constexpr int kLaunchRegs = 65536 / kThreads;  // registers per thread at launch (128)
static_assert(2 * kSoftmaxRegs + kControlRegs + kEpilogueRegs == 4 * kLaunchRegs,
              "register split must use the launch budget");
constexpr int kTmemO = 256;           // O_i at kTmemO + 128 i

template <int D>
struct Smem {
  static constexpr int kHalfBytes = kBM * 64 * 2;   // one 128-row x 64-column 128B-swizzled box
  static constexpr int kTileBytes = kBM * D * 2;
  static constexpr int kQ = 0;                                // Q_0, Q_1
  static constexpr int kK = kQ + 2 * kTileBytes;              // two K stages
  static constexpr int kV = kK + kStages * kTileBytes;        // two V stages
  static constexpr int kStat = kV + kStages * kTileBytes;     // float2 [2 tiles][2 parities][128]
  static constexpr int kBar = kStat + 2 * 2 * kBM * 8;
  static constexpr int kNumBars = 28;
  static constexpr int kUsed = kBar + kNumBars * 8 + 16;
  static constexpr int kRequest = (kUsed + 1024) > 120 * 1024 ? (kUsed + 1024) : 120 * 1024;
};

// Barrier indices (i = Q tile, st = stage).
enum : int {
  kQFull = 0,       // [2]  Q_i loaded (TMA transaction count)
  kQEmpty = 2,      // [2]  the unit's last QK_i completed: Q_i may be replaced
  kKFull = 4,       // [2]  K stage loaded
  kKFree = 6,       // [2]  both QKs of the K stage's tile completed
  kVFull = 8,       // [2]  V stage loaded
  kVFree = 10,      // [2]  both P.Vs of the V stage's tile completed
  kSReady = 12,     // [2]  S_i(t) computed (one phase per tile)
  kPReady = 14,     // [2]  softmax_i stored P_i(t) (4 warp arrivals per tile)
  kPvDone = 16,     // [2]  P.V_i(t) completed: S_i free, O_i holds every product up to t
  kODone = 18,      // [2]  a segment's last P.V_i completed
  kOFree = 20,      // [2]  the epilogue has read O_i (4 warp arrivals)
  kStatReady = 22,  // [2]  softmax_i wrote the segment's (m_i, l_i) (4 warp arrivals)
  kDrainQk = 24,
  kDrainPv = 25,
};

struct PairCoord {
  int b, h, qp;  // batch, head, Q tile pair
};

__device__ __forceinline__ PairCoord decode_pair(int u, const AttnParams& p) {
  const int n_qp = (p.n_qt + 1) / 2;
  PairCoord r;
  r.qp = u % n_qp;
  const int bh = u / n_qp;
  r.h = bh % p.H;
  r.b = bh / p.H;
  return r;
}

__device__ __forceinline__ int n_units(const AttnParams& p) { return p.B * p.H * ((p.n_qt + 1) / 2); }

// ------------------------------------------------------------------------------- producers

template <int D>
__device__ __forceinline__ void producer_qk(const CUtensorMap* tm_q, const CUtensorMap* tm_k, const AttnParams& p,
                                            uint8_t* smem, uint64_t* bars, volatile int* abort_flag) {
  using L = Smem<D>;
  if (p.tiles_per_unit == 0) return;
  uint32_t kc = 0;            // K tiles issued
  uint32_t nq[2] = {0u, 0u};  // Q_i loads issued (one per unit)
  bool ok = true;
  const int nun = n_units(p);
  for (int u = blockIdx.x; u < nun && ok; u += gridDim.x) {
    const PairCoord uc = decode_pair(u, p);
    for (int i = 0; i < 2; ++i) {
      if (nq[i] > 0 && !mbar_wait(bars + kQEmpty + i, (nq[i] - 1) & 1, abort_flag, p.status, 32)) {
        ok = false;
        break;
      }
      mbar_arrive_expect_tx(bars + kQFull + i, L::kTileBytes);
#pragma unroll
      for (int hf = 0; hf < D / 64; ++hf)
        tma_load_4d(smem + L::kQ + i * L::kTileBytes + hf * L::kHalfBytes, tm_q, bars + kQFull + i, hf * 64, uc.h,
                    uc.qp * kRows + i * kBM, uc.b);
      ++nq[i];
    }
    if (!ok) break;
    Tile t;
    bool have = first_tile_from(p, 0, t);
    while (have) {
      const int st = kc % kStages;
      const uint32_t use = kc / kStages;
      if (use > 0 && !mbar_wait(bars + kKFree + st, (use - 1) & 1, abort_flag, p.status, 32)) {
        ok = false;
        break;
      }
      // Test hook (p.fault == 1): skip the CTA's first K tile, so that the consumers'
      // bounded waits run out and the kernel returns CP_ERR_TIMEOUT.
      if (!(p.fault == 1 && kc == 0)) {
        mbar_arrive_expect_tx(bars + kKFull + st, L::kTileBytes);
#pragma unroll
        for (int hf = 0; hf < D / 64; ++hf)
          tma_load_4d(smem + L::kK + st * L::kTileBytes + hf * L::kHalfBytes, tm_k, bars + kKFull + st, hf * 64,
                      uc.h, t.row0, uc.b);
      }
      ++kc;
      have = next_tile(p, t, t);
    }
  }
  // Drain: every issued load lands before the CTA may exit.
  for (int i = 0; i < 2; ++i)
    if (nq[i] > 0) drain_wait(bars + kQFull + i, (nq[i] - 1) & 1);
  for (int st = 0; st < kStages; ++st) {
    const uint32_t uk = kc / kStages + (st < static_cast<int>(kc % kStages) ? 1u : 0u);
    if (uk > 0) drain_wait(bars + kKFull + st, (uk - 1) & 1);
  }
}

template <int D>
__device__ __forceinline__ void producer_v(const CUtensorMap* tm_v, const AttnParams& p, uint8_t* smem,
                                           uint64_t* bars, volatile int* abort_flag) {
  using L = Smem<D>;
  if (p.tiles_per_unit == 0) return;
  uint32_t vc = 0;
  bool ok = true;
  const int nun = n_units(p);
  for (int u = blockIdx.x; u < nun && ok; u += gridDim.x) {
    const PairCoord uc = decode_pair(u, p);
    Tile t;
    bool have = first_tile_from(p, 0, t);
    while (have) {
      const int st = vc % kStages;
      const uint32_t use = vc / kStages;
      if (use > 0 && !mbar_wait(bars + kVFree + st, (use - 1) & 1, abort_flag, p.status, 32)) {
        ok = false;
        break;
      }
      mbar_arrive_expect_tx(bars + kVFull + st, L::kTileBytes);
#pragma unroll
      for (int hf = 0; hf < D / 64; ++hf)
        tma_load_4d(smem + L::kV + st * L::kTileBytes + hf * L::kHalfBytes, tm_v, bars + kVFull + st, hf * 64, uc.h,
                    t.row0, uc.b);
      ++vc;
      have = next_tile(p, t, t);
    }
  }
  for (int st = 0; st < kStages; ++st) {
    const uint32_t uv = vc / kStages + (st < static_cast<int>(vc % kStages) ? 1u : 0u);
    if (uv > 0) drain_wait(bars + kVFull + st, (uv - 1) & 1);
  }
}

// ------------------------------------------------------------------------------- MMA issuers

// Warp 9, lane 0: for every K/V tile t, S_0(t) = Q_0 K(t)^T, then S_1(t) = Q_1 K(t)^T.
// S_i held P_i(t-1), so QK_i(t) waits for P.V_i(t-1) (MMAs of different threads are not
// ordered with each other).
template <int D>
__device__ __forceinline__ void mma_qk(const AttnParams& p, uint8_t* smem, uint64_t* bars, uint32_t tmem,
                                       volatile int* abort_flag) {
  using L = Smem<D>;
  if (p.tiles_per_unit == 0) return;
  constexpr uint32_t kIdesc128 = idesc_bf16_f32(kBM, 128, 0);
  constexpr uint32_t kIdesc64 = idesc_bf16_f32(kBM, 64, 0);
  const uint32_t sQ = smem_u32(smem + L::kQ);
  const uint32_t sK = smem_u32(smem + L::kK);
  uint32_t kc = 0;  // K tiles consumed (= tiles issued: one K tile per tile)
  uint32_t nu = 0;
  const int nun = n_units(p);
  for (int u = blockIdx.x; u < nun; u += gridDim.x, ++nu) {
    Tile t;
    bool have = first_tile_from(p, 0, t);
    bool q_ready = false;
    while (have) {
      Tile nxt;
      const bool more = next_tile(p, t, nxt);
      const int kst = kc % kStages;
      if (!mbar_wait(bars + kKFull + kst, (kc / kStages) & 1, abort_flag, p.status)) goto done;
      const uint64_t kd = sdesc_sw128(sK + kst * L::kTileBytes, 16, 1024);
      const uint32_t idesc = t.valid() > kHalfN ? kIdesc128 : kIdesc64;
#pragma unroll 1
      for (int i = 0; i < 2; ++i) {
        if (!q_ready && !mbar_wait(bars + kQFull + i, nu & 1, abort_flag, p.status)) goto done;
        if (kc > 0 && !mbar_wait(bars + kPvDone + i, (kc - 1) & 1, abort_flag, p.status)) goto done;
        tc_fence_after();
        const uint64_t qd = sdesc_sw128(sQ + i * L::kTileBytes, 16, 1024);
        const uint32_t d_tmem = tmem + i * kBN;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = ((k >> 2) * L::kHalfBytes + (k & 3) * 32) >> 4;
          tc_mma_ss(d_tmem, qd + off, kd + off, idesc, k > 0);
        }
        tc_commit(bars + kSReady + i);
        if (!more) tc_commit(bars + kQEmpty + i);  // the unit's last QK_i: Q_i frees
      }
      q_ready = true;
      tc_commit(bars + kKFree + kst);
      ++kc;
      t = nxt;
      have = more;
    }
  }
done:
  tc_commit(bars + kDrainQk);
  drain_wait(bars + kDrainQk, 0);
}

// Warp 11, lane 0: O_i (+)= P_i(t) V(t) for i = 0, 1 once softmax_i stored P_i(t).  P_i is
// the bf16 pairs in columns 0..63 of S_i (16 keys = 8 columns per k-step); V is MN-major,
// 16 keys per k-step = 2048 bytes, the two 64-wide D halves 16 KB apart.
template <int D>
__device__ __forceinline__ void mma_pv(const AttnParams& p, uint8_t* smem, uint64_t* bars, uint32_t tmem,
                                       volatile int* abort_flag) {
  using L = Smem<D>;
  if (p.tiles_per_unit == 0) return;
  constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, D, 1);
  const uint32_t sV = smem_u32(smem + L::kV);
  uint32_t vc = 0;   // tiles consumed
  uint32_t nch = 0;  // segments finished
  const int nun = n_units(p);
  for (int u = blockIdx.x; u < nun; u += gridDim.x) {
    Tile t;
    bool have = first_tile_from(p, 0, t);
    while (have) {
      const int vst = vc % kStages;
      if (!mbar_wait(bars + kVFull + vst, (vc / kStages) & 1, abort_flag, p.status)) goto done;
      const uint64_t vd = sdesc_sw128(sV + vst * L::kTileBytes, L::kHalfBytes, 1024);
      const int ksteps = t.valid() > kHalfN ? kBN / 16 : kHalfN / 16;  // P is 0 past the valid keys
#pragma unroll 1
      for (int i = 0; i < 2; ++i) {
        if (!mbar_wait(bars + kPReady + i, vc & 1, abort_flag, p.status)) goto done;
        if (t.first() && nch > 0 && !mbar_wait(bars + kOFree + i, (nch - 1) & 1, abort_flag, p.status)) goto done;
        tc_fence_after();
        const uint32_t a = tmem + i * kBN;
        const uint32_t o = tmem + kTmemO + i * 128;
        const uint32_t acc0 = t.first() ? 0u : 1u;
        for (int ks = 0; ks < ksteps; ++ks)
          tc_mma_ts(o, a + ks * 8, vd + ks * (2048 >> 4), kIdescPV, ks > 0 ? 1u : acc0);
        tc_commit(bars + kPvDone + i);
        if (t.last()) tc_commit(bars + kODone + i);
      }
      if (t.last()) ++nch;
      tc_commit(bars + kVFree + vst);
      ++vc;
      have = next_tile(p, t, t);
    }
  }
done:
  tc_commit(bars + kDrainPv);
  drain_wait(bars + kDrainPv, 0);
}

// ------------------------------------------------------------------------------- softmax

// Softmax of one tile for this thread's row over its `N` (128 or 64) columns in one pass:
// load the S values, mask keys at or past `valid` (MASK), row max, lazy max update,
// P = 2^(S*scale*log2e - m) (packed FMAs, MUFU ex2, one pair in four on the FMA pipe when
// nothing is masked, packed sums), stored as bf16 pairs over the first N/2 columns.  A
// rescale of O_i waits for P.V_i of the previous tile (`pv_prev`, already complete: QK_i
// of this tile waited for it); if that wait gives up, false is returned.
template <int D, int N, bool MASK>
__device__ __forceinline__ bool softmax_row(uint32_t ts, uint32_t to, int valid, bool fresh, float sl2, float& m,
                                            float& l, uint64_t* pv_prev, uint32_t pv_par, volatile int* abort_flag,
                                            int* status) {
  uint32_t r[N];
  if constexpr (N == 128)
    tmem_ld128(ts, r);
  else
    tmem_ld64(ts, r);
  if (MASK) {
#pragma unroll
    for (int i = 0; i < N; ++i)
      if (i >= valid) r[i] = __float_as_uint(-INFINITY);
  }
  float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
#pragma unroll
  for (int i = 0; i < N; i += 8) {
    a0 = fmax3(a0, __uint_as_float(r[i]), __uint_as_float(r[i + 1]));
    a1 = fmax3(a1, __uint_as_float(r[i + 2]), __uint_as_float(r[i + 3]));
    a2 = fmax3(a2, __uint_as_float(r[i + 4]), __uint_as_float(r[i + 5]));
    a3 = fmax3(a3, __uint_as_float(r[i + 6]), __uint_as_float(r[i + 7]));
  }
  const float m_tile = fmaxf(fmaxf(a0, a1), fmaxf(a2, a3)) * sl2;
  float alpha = 1.f;
  bool rescale = false;
  if (fresh) {
    m = m_tile;
  } else {
    const bool need = m_tile > m + kRescaleThreshold;
    rescale = __any_sync(0xffffffffu, need);
    if (need) {
      alpha = ex2_approx(m - m_tile);
      l *= alpha;
      m = m_tile;
    }
  }
  const uint64_t scale2 = f2_pack(sl2, sl2);
  const uint64_t negm2 = f2_pack(-m, -m);
  uint64_t sum_a = 0, sum_b = 0;  // packed fp32 pairs (+0.0f, +0.0f)
#pragma unroll
  for (int c = 0; c < N / 32; ++c) {
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int k = c * 32 + 2 * i;
      const uint64_t x = fma_f32x2(f2_pack(__uint_as_float(r[k]), __uint_as_float(r[k + 1])), scale2, negm2);
      float p0, p1;
      if (!MASK && kEmuEvery > 0 && (i % kEmuEvery) == kEmuEvery - 1) {
        // x >= -125 keeps 2^n a normal number; smaller terms are below 2^-125 of a sum >= 1.
        const uint64_t xc = f2_pack(fmaxf(f2_lo(x), -125.f), fmaxf(f2_hi(x), -125.f));
        const uint64_t shift = f2_pack(12582912.f, 12582912.f);
        const uint64_t tt = add_f32x2(xc, shift);
        const uint64_t fr = add_f32x2(xc, add_f32x2(shift, f2_pack(-f2_lo(tt), -f2_hi(tt))));
        uint64_t q = fma_f32x2(fr, f2_pack(kExp2C3, kExp2C3), f2_pack(kExp2C2, kExp2C2));
        q = fma_f32x2(fr, q, f2_pack(kExp2C1, kExp2C1));
        q = fma_f32x2(fr, q, f2_pack(kExp2C0, kExp2C0));
        p0 = __uint_as_float(__float_as_uint(f2_lo(q)) + (__float_as_uint(f2_lo(tt)) << 23));
        p1 = __uint_as_float(__float_as_uint(f2_hi(q)) + (__float_as_uint(f2_hi(tt)) << 23));
      } else {
        p0 = ex2_approx(f2_lo(x));
        p1 = ex2_approx(f2_hi(x));
      }
      const uint64_t pp = f2_pack(p0, p1);
      if (i & 1)
        sum_b = add_f32x2(sum_b, pp);
      else
        sum_a = add_f32x2(sum_a, pp);
      pk[i] = pack_bf16x2(p0, p1);
    }
    tmem_st16(ts + c * 16, pk);
  }
  const uint64_t sum = add_f32x2(sum_a, sum_b);
  l += f2_lo(sum) + f2_hi(sum);
  if (rescale) {
    // Rows whose max grew by more than 8 rescale O_i by alpha (1 for the other rows of the
    // warp).  This tile's P.V adds to O_i only after p_ready, i.e. after these stores.
    if (!warp_wait(pv_prev, pv_par, abort_flag, status)) {
      tmem_wait_st();
      return false;
    }
    tc_fence_after();
#pragma unroll 1
    for (int c = 0; c < D / 32; ++c) {
      uint32_t o[32];
      tmem_ld32(to + c * 32, o);
#pragma unroll
      for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
      tmem_st32(to + c * 32, o);
    }
  }
  tmem_wait_st();
  return true;
}

// Softmax warpgroup i: every tile of every block of every unit for the rows of Q tile i; at
// a segment's end it hands the rows' (m_i, l_i) to the epilogue warpgroup.
template <int D>
__device__ __forceinline__ void softmax(const AttnParams& p, uint8_t* smem, uint64_t* bars, uint32_t tmem,
                                        volatile int* abort_flag) {
  using L = Smem<D>;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int qi = warp >> 2;       // Q tile
  const int quarter = warp & 3;   // TMEM lane quarter
  const int row = quarter * 32 + lane;
  const uint32_t lanes = static_cast<uint32_t>(quarter * 32) << 16;
  const uint32_t ts = tmem + lanes + qi * kBN;
  const uint32_t to = tmem + lanes + kTmemO + qi * 128;
  float2* stat = reinterpret_cast<float2*>(smem + L::kStat) + qi * 2 * kBM;
  uint64_t* s_ready = bars + kSReady + qi;
  uint64_t* p_ready = bars + kPReady + qi;
  uint64_t* pv_done = bars + kPvDone + qi;
  const float sl2 = p.scale_log2;
  uint32_t g = 0;     // tiles seen
  uint32_t nch = 0;   // segments finished
  bool alive = true;
  const int nun = n_units(p);
  for (int u = blockIdx.x; u < nun; u += gridDim.x) {
    const PairCoord uc = decode_pair(u, p);
    const int s_row = uc.qp * kRows + qi * kBM + row;
    const ::cpattn::UnitCoord oc{uc.b, uc.h, 0};
    float m = -INFINITY, l = 0.f;
    bool fresh = true;
    if (p.fuse && p.first_c < 0 && s_row < p.Sq) write_empty_row<D>(p, 0, oc, s_row);  // no keys at all
    for (int c = 0; c < p.n_chunks; ++c) {
      const int n_kv = block_tiles(p, c);
      if (n_kv == 0) {  // no keys: O = 0, lse = -inf (fused: the block adds nothing)
        if (!p.fuse && s_row < p.Sq) write_empty_row<D>(p, c, oc, s_row);
        continue;
      }
      if (!p.fuse || c == p.first_c) {
        m = -INFINITY;
        l = 0.f;
        fresh = true;
      }
      for (int j = 0; j < n_kv; ++j, ++g) {
        const Tile t = make_tile(p, c, j);
        if (!warp_wait(s_ready, g & 1, abort_flag, p.status) || !alive) return;
        tc_fence_after();
        const int v = t.valid();
        const uint32_t pv_par = (g - 1) & 1;  // rescales happen only after a segment's first tile (g >= 1)
        bool ok;
        if (v == kBN)
          ok = softmax_row<D, 128, false>(ts, to, v, fresh, sl2, m, l, pv_done, pv_par, abort_flag, p.status);
        else if (v > kHalfN)
          ok = softmax_row<D, 128, true>(ts, to, v, fresh, sl2, m, l, pv_done, pv_par, abort_flag, p.status);
        else
          ok = softmax_row<D, 64, true>(ts, to, v, fresh, sl2, m, l, pv_done, pv_par, abort_flag, p.status);
        alive = alive && ok;
        fresh = false;
        tc_fence_before();
        warp_arrive(p_ready);
      }
      if (p.fuse && c != p.last_c) continue;  // the segment goes on with the next block
      // Hand (m, l) to the epilogue, after it has released O_i of the previous segment (it
      // reads that segment's stats first): without this wait one-tile segments could run
      // two stat_ready phases ahead of the epilogue.
      if (nch > 0 && (!warp_wait(bars + kOFree + qi, (nch - 1) & 1, abort_flag, p.status) || !alive)) return;
      stat[(nch & 1) * kBM + row] = make_float2(m, l);
      warp_arrive(bars + kStatReady + qi);
      ++nch;
    }
  }
}

// ------------------------------------------------------------------------------- epilogue

// Epilogue warpgroup: for every segment and Q tile i, wait for the last P.V_i and the
// rows' (m_i, l_i), then write O_i / l_i 32 columns at a time and the LSE.  O_i is
// released as soon as its last columns are in registers: the next segment's first
// P.V_i comes only after softmax_i of that segment's first tile, so the release is
// rarely waited for.
template <int D>
__device__ __forceinline__ void epilogue(const AttnParams& p, uint8_t* smem, uint64_t* bars, uint32_t tmem,
                                         volatile int* abort_flag) {
  using L = Smem<D>;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int quarter = warp & 3;
  const int row = quarter * 32 + lane;
  const uint32_t lanes = static_cast<uint32_t>(quarter * 32) << 16;
  const float2* stat = reinterpret_cast<const float2*>(smem + L::kStat);
  uint32_t nch = 0;
  if (p.tiles_per_unit == 0) return;
  const int nun = n_units(p);
  for (int u = blockIdx.x; u < nun; u += gridDim.x) {
    const PairCoord uc = decode_pair(u, p);
    for (int c0 = 0; c0 < p.n_chunks; ++c0) {
      if (block_tiles(p, c0) == 0) continue;
      if (p.fuse && c0 != p.last_c) continue;  // one merged output per unit
      const int c = p.fuse ? 0 : c0;             // output block index
#pragma unroll 1
      for (int qi = 0; qi < 2; ++qi) {
        if (!group_wait(bars + kStatReady + qi, nch & 1, kBarEpilogue, true, abort_flag, p.status, 64)) return;
        if (!group_wait(bars + kODone + qi, nch & 1, kBarEpilogue, true, abort_flag, p.status, 64)) return;
        tc_fence_after();
        const float2 s = stat[(qi * 2 + (nch & 1)) * kBM + row];
        const float inv = 1.f / s.y;
        const int s_row = uc.qp * kRows + qi * kBM + row;
        const bool row_ok = s_row < p.Sq;
        const size_t o_off = row_ok ? static_cast<size_t>(out_row_offset<D>(p, c, uc.b, s_row, uc.h)) : 0;
        const bool store = row_ok && in_bounds(static_cast<long long>(o_off), D, p.out_elems);
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t r[32];
          tmem_ld32(tmem + lanes + kTmemO + qi * 128 + cc * 32, r);
          if (cc == D / 32 - 1) {
            tc_fence_before();
            warp_arrive(bars + kOFree + qi);
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * inv);
          if (store) store_row<D>(p, o_off, r, cc);
        }
        if (row_ok) {
          if (p.lse) {
            const long long li = lse_index(p, c, uc.b, s_row, uc.h);
            if (in_bounds(li, 1, p.lse_elems)) p.lse[li] = (s.x + log2f(s.y)) * 0.69314718055994530942f;
          }
        }
      }
      ++nch;
    }
  }
}

// ------------------------------------------------------------------------------- kernel

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_pair_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ AttnParams p) {
  using L = Smem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + L::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bars + kQFull + i, 1);
      mbar_init(bars + kQEmpty + i, 1);
      mbar_init(bars + kKFull + i, 1);
      mbar_init(bars + kKFree + i, 1);
      mbar_init(bars + kVFull + i, 1);
      mbar_init(bars + kVFree + i, 1);
      mbar_init(bars + kSReady + i, 1);
      mbar_init(bars + kPReady + i, 4);     // the 4 warps of softmax warpgroup i
      mbar_init(bars + kPvDone + i, 1);
      mbar_init(bars + kODone + i, 1);
      mbar_init(bars + kOFree + i, 4);      // the 4 epilogue warps
      mbar_init(bars + kStatReady + i, 4);  // the 4 warps of softmax warpgroup i
    }
    mbar_init(bars + kDrainQk, 1);
    mbar_init(bars + kDrainPv, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == kProducerWarp && (threadIdx.x & 31) == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
  }
  if (warp == kVProducerWarp && (threadIdx.x & 31) == 0) tma_prefetch_desc(&tm_v);
  if (warp == kQkWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= kEpilogueWarp0) {
    regs_set<kEpilogueRegs, kLaunchRegs>();
    epilogue<D>(p, smem, bars, tmem, abort_flag);
  } else if (warp >= 8) {
    regs_set<kControlRegs, kLaunchRegs>();
    if (warp == kProducerWarp) {
      if ((threadIdx.x & 31) == 0) producer_qk<D>(&tm_q, &tm_k, p, smem, bars, abort_flag);
    } else if (warp == kVProducerWarp) {
      if ((threadIdx.x & 31) == 0) producer_v<D>(&tm_v, p, smem, bars, abort_flag);
    } else if (warp == kQkWarp) {
      if ((threadIdx.x & 31) == 0) mma_qk<D>(p, smem, bars, tmem, abort_flag);
    } else if (warp == kPvWarp) {
      if ((threadIdx.x & 31) == 0) mma_pv<D>(p, smem, bars, tmem, abort_flag);
    }
    __syncwarp();
  } else {
    regs_set<kSoftmaxRegs, kLaunchRegs>();
    softmax<D>(p, smem, bars, tmem, abort_flag);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kQkWarp) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace pair
}  // namespace cpattn
