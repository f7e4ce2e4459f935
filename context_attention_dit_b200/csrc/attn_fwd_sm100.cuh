// attn_fwd_sm100.cuh - non-causal blockwise attention with LSE for B200 (sm_100a).
//
// Computes, for every (batch b, head h, K/V block c, query row i),
//   S_ij = scale * q_i . k_j  over the keys j of block c,
//   O_i  = sum_j softmax_j(S_ij) v_j,   lse_i = ln sum_j exp(S_ij)
// ("Attention backends", "Available backends": scaled_dot_product_attention; the
// per-block fp32 output + LSE follow ContextParallelConfig.convert_to_fp32 on the
// "Parallelism" API page, so that ring blocks can be merged afterwards).
//
// Design (one CTA per SM, persistent over work units (b, h, pair of 128-row Q tiles);
// each unit walks every K/V block and, inside a block, its 128-key tiles):
//   warps 0-3   softmax warpgroup 0, Q tile 0 of the pair; thread t of warp w owns
//   warps 4-7   softmax warpgroup 1, Q tile 1; its query row 32*(w%4)+t = TMEM lane.
//               Per K/V tile: load the S row from TMEM, mask keys past the block end,
//               update the running max m and sum l (base 2), write P = 2^(S*scale*log2e
//               - m) as bf16 pairs into the first columns of the same S buffer.  After
//               a block's last tile: hand the row's (m, l) to the epilogue warpgroup.
//   warp 8      TMA producer: both Q tiles once per unit; K and V tiles (128 keys x D)
//               through two 2-stage rings.  Warps 8-11 form the control warpgroup, which
//               hands registers to the softmax warpgroups (setmaxnreg 88 / 184 / 56).
//   warps 12-15 epilogue warpgroup: after a block's last P.V, read O_w from TMEM, release
//               it for the next block, write O/l (fp32 partial or final bf16/fp32) and lse.
//   warp 9      TMEM owner (512 columns) and MMA issuer (one thread), in the order
//               QK0(t) QK1(t) | PV0(t) QK0(t+1) PV1(t) QK1(t+1) | ...
//               S_w = Q_w K^T: SS form, both operands K-major and 128B-swizzled;
//               O_w += P_w V: TS form, P_w read from TMEM, V MN-major in shared memory.
//               Because QK_w(t+1) is issued after PV_w(t), the commit that signals "S_w
//               full" also certifies that O_w holds every earlier P.V product.
// TMEM columns: S0 [0,128), S1 [128,256), O0 [256,256+D), O1 [384,384+D).
// A tile whose block has at most 64 keys left runs N = 64 (QK) and K = 64 (PV) MMAs and
// a 64-column softmax.
// The running max is updated lazily: O_w is rescaled in TMEM only when a row's max grows
// by more than 8 (a factor 256); otherwise the stale max stays, which is exact because O
// and l share it and 2^8 cannot overflow fp32 or bf16.
// Every mbarrier wait is bounded (see ptx_sm100.cuh); on a timeout every role leaves its
// loop, in-flight TMA loads and MMAs are drained, TMEM is freed and the kernel returns
// with CP_ERR_TIMEOUT recorded in the device status word.
#pragma once

#include <cuda.h>

#include "ptx_sm100.cuh"

namespace cpattn {

constexpr int kBM = 128;           // query rows per Q tile (TMEM lanes)
constexpr int kQTiles = 2;         // Q tiles per work unit, one softmax warpgroup each
constexpr int kBN = 128;           // keys per K/V tile
constexpr int kStages = 2;         // stages of each of the K and V rings
constexpr int kAttnThreads = 512;  // 16 warps: 2 softmax, 1 control, 1 epilogue warpgroup
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kEpilogueWarp0 = 12;
// Registers per thread after the split (launch: 128 = 65536 / 512).
// 256 * kSoftmaxRegs + 128 * kControlRegs + 128 * kEpilogueRegs = 512 * 128.
constexpr int kSoftmaxRegs = 184;
constexpr int kControlRegs = 88;
constexpr int kEpilogueRegs = 56;
static_assert(2 * kSoftmaxRegs + kControlRegs + kEpilogueRegs == 4 * 128, "register split must use the launch budget");
constexpr int kTmemCols = 512;
constexpr int kMaxChunks = 64;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct AttnParams {
  int B, H, Sq;
  int n_chunks;
  int n_qp;                  // ceil(Sq / (kQTiles * kBM)) Q-tile pairs
  int n_units;               // B * H * n_qp
  int tiles_per_unit;        // sum over blocks of ceil(len / kBN)
  float scale_log2;          // scale * log2(e)
  void* out;                 // block c at out + c*out_chunk_stride elements, [B][Sq][H][D]
  int out_f32;               // 1: fp32 output, 0: bf16 output
  int out_v8;                // 1: out is 32-byte aligned (32-byte stores)
  long long out_chunk_stride;
  float* lse;                // block c at lse + c*lse_chunk_stride, [B][H][Sq]; may be null
  long long lse_chunk_stride;
  int* status;               // device status word
  int fuse;                  // 1: one running softmax over all blocks, one merged output
  int fault;                 // test hook: 1 = the producer never loads the CTA's first K tile
  int first_c, last_c;       // first / last non-empty block (-1 if none)
  int bounds[kMaxChunks + 1];  // K/V row bounds of the blocks
};

template <int D>
struct AttnSmem {
  static constexpr int kHalfBytes = kBM * 64 * 2;  // 128 rows x 64 bf16: one 128B-swizzled box
  static constexpr int kTileBytes = kBM * D * 2;   // 128 rows x D bf16
  static constexpr int kQ = 0;                     // kQTiles Q tiles
  static constexpr int kK = kQ + kQTiles * kTileBytes;
  static constexpr int kV = kK + kStages * kTileBytes;
  static constexpr int kStat = kV + kStages * kTileBytes;  // float2 [kQTiles][2][kBM]: (m, l) per row
  static constexpr int kBar = kStat + kQTiles * 2 * kBM * 8;
  static constexpr int kNumBars = 21;
  static constexpr int kUsed = kBar + kNumBars * 8 + 16;
  // More than half an SM's shared memory: exactly one CTA (owning all 512 TMEM
  // columns) is resident per SM.
  static constexpr int kRequest = (kUsed + 1024) > 120 * 1024 ? (kUsed + 1024) : 120 * 1024;
};

// Barrier indices.
enum : int {
  kQFull = 0, kQEmpty = 1, kKFull = 2, kKEmpty = 4, kVFull = 6, kVEmpty = 8,
  kSFull = 10, kPReady = 12, kODone = 14, kOFree = 16, kStatReady = 18, kDrain = 20
};

struct UnitCoord {
  int b, h, qp;
};

__device__ __forceinline__ UnitCoord decode_unit(int u, const AttnParams& p) {
  UnitCoord r;
  r.qp = u % p.n_qp;
  const int bh = u / p.n_qp;
  r.h = bh % p.H;
  r.b = bh / p.H;
  return r;
}

// One 128-key (or shorter) tile of K/V block c.
struct Tile {
  int c, j;   // block, tile within the block
  int row0;   // first K/V row
  int info;   // bits 0-7: keys of the block in this tile (1..128); bit 8: last tile of its
              // block (drives the tile walk); bits 9/10: first / last tile of a softmax
              // segment (a block, or every block if fused)
  __device__ __forceinline__ int valid() const { return info & 0xFF; }
  __device__ __forceinline__ bool block_last() const { return (info >> 8) & 1; }
  __device__ __forceinline__ bool first() const { return (info >> 9) & 1; }
  __device__ __forceinline__ bool last() const { return (info >> 10) & 1; }
};

__device__ __forceinline__ int block_tiles(const AttnParams& p, int c) {
  return (p.bounds[c + 1] - p.bounds[c] + kBN - 1) / kBN;
}

__device__ __forceinline__ Tile make_tile(const AttnParams& p, int c, int j) {
  Tile t;
  t.c = c;
  t.j = j;
  const int len = p.bounds[c + 1] - p.bounds[c];
  t.row0 = p.bounds[c] + j * kBN;
  // first / last: the tile starts / ends a softmax segment (a block, or with p.fuse the
  // whole run of blocks).
  const int block_last = (j == (len + kBN - 1) / kBN - 1);
  const int first = (j == 0) && (!p.fuse || c == p.first_c);
  const int last = block_last && (!p.fuse || c == p.last_c);
  t.info = min(kBN, len - j * kBN) | (block_last << 8) | (first << 9) | (last << 10);
  return t;
}

// First tile at or after block c (skipping empty blocks); false if none.
__device__ __forceinline__ bool first_tile_from(const AttnParams& p, int c, Tile& t) {
  for (; c < p.n_chunks; ++c)
    if (block_tiles(p, c) > 0) {
      t = make_tile(p, c, 0);
      return true;
    }
  return false;
}

__device__ __forceinline__ bool next_tile(const AttnParams& p, const Tile& cur, Tile& nxt) {
  if (!cur.block_last()) {
    nxt = make_tile(p, cur.c, cur.j + 1);
    return true;
  }
  return first_tile_from(p, cur.c + 1, nxt);
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

// ------------------------------------------------------------------------------- producer

template <int D>
__device__ __forceinline__ void attn_producer(const CUtensorMap* tm_q, const CUtensorMap* tm_k,
                                              const CUtensorMap* tm_v, const AttnParams& p, uint8_t* smem,
                                              uint64_t* bars, volatile int* abort_flag) {
  using L = AttnSmem<D>;
  if (p.tiles_per_unit == 0) return;
  uint32_t kc_k = 0, kc_v = 0;  // tiles issued into the K and V rings
  uint32_t n_q = 0;             // Q pairs issued
  bool ok = true;
  for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
    const UnitCoord uc = decode_unit(u, p);
    if (n_q > 0 && !mbar_wait(bars + kQEmpty, (n_q - 1) & 1, abort_flag, p.status)) break;
    mbar_arrive_expect_tx(bars + kQFull, kQTiles * L::kTileBytes);
#pragma unroll
    for (int w = 0; w < kQTiles; ++w)
#pragma unroll
      for (int hf = 0; hf < D / 64; ++hf)
        tma_load_4d(smem + L::kQ + w * L::kTileBytes + hf * L::kHalfBytes, tm_q, bars + kQFull, hf * 64, uc.h,
                    (uc.qp * kQTiles + w) * kBM, uc.b);
    ++n_q;
    Tile t;
    bool have = first_tile_from(p, 0, t);
    while (have) {
      {
        const int st = kc_k % kStages;
        const uint32_t use = kc_k / kStages;
        if (use > 0 && !mbar_wait(bars + kKEmpty + st, (use - 1) & 1, abort_flag, p.status)) { ok = false; break; }
        // Test hook (p.fault == 1): skip the CTA's first K tile, so that the consumer's
        // bounded wait runs out and the kernel returns CP_ERR_TIMEOUT.
        if (!(p.fault == 1 && kc_k == 0)) {
          mbar_arrive_expect_tx(bars + kKFull + st, L::kTileBytes);
#pragma unroll
          for (int hf = 0; hf < D / 64; ++hf)
            tma_load_4d(smem + L::kK + st * L::kTileBytes + hf * L::kHalfBytes, tm_k, bars + kKFull + st, hf * 64,
                        uc.h, t.row0, uc.b);
        }
        ++kc_k;
      }
      {
        const int st = kc_v % kStages;
        const uint32_t use = kc_v / kStages;
        if (use > 0 && !mbar_wait(bars + kVEmpty + st, (use - 1) & 1, abort_flag, p.status)) { ok = false; break; }
        mbar_arrive_expect_tx(bars + kVFull + st, L::kTileBytes);
#pragma unroll
        for (int hf = 0; hf < D / 64; ++hf)
          tma_load_4d(smem + L::kV + st * L::kTileBytes + hf * L::kHalfBytes, tm_v, bars + kVFull + st, hf * 64,
                      uc.h, t.row0, uc.b);
        ++kc_v;
      }
      have = next_tile(p, t, t);
    }
  }
  // Drain: every issued load lands before the CTA may exit (normal path: already done).
  if (n_q > 0) drain_wait(bars + kQFull, (n_q - 1) & 1);
  for (int st = 0; st < kStages; ++st) {
    const uint32_t uk = kc_k / kStages + (st < static_cast<int>(kc_k % kStages) ? 1u : 0u);
    const uint32_t uv = kc_v / kStages + (st < static_cast<int>(kc_v % kStages) ? 1u : 0u);
    if (uk > 0) drain_wait(bars + kKFull + st, (uk - 1) & 1);
    if (uv > 0) drain_wait(bars + kVFull + st, (uv - 1) & 1);
  }
}

// ------------------------------------------------------------------------------- MMA issuer

template <int D>
__device__ __forceinline__ void attn_mma(const AttnParams& p, uint8_t* smem, uint64_t* bars, uint32_t tmem,
                                         volatile int* abort_flag) {
  using L = AttnSmem<D>;
  if (p.tiles_per_unit == 0) return;
  constexpr uint32_t kIdescQK128 = idesc_bf16_f32(kBM, 128, 0);
  constexpr uint32_t kIdescQK64 = idesc_bf16_f32(kBM, 64, 0);
  constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, D, 1);
  const uint32_t sQ = smem_u32(smem + L::kQ);
  const uint32_t sK = smem_u32(smem + L::kK);
  const uint32_t sV = smem_u32(smem + L::kV);

  uint32_t kc_k = 0, kc_v = 0;  // K/V ring positions consumed
  uint32_t g = 0;               // tiles processed (S_w / P_w phase)
  uint32_t nch = 0;             // non-empty blocks finished (O_w phase)
  uint32_t n_q = 0;             // units started (Q phase)

  // S_w = Q_w K^T: D/16 k-steps of 16; step k sits in 64-column half k/4 at byte 32*(k%4).
  auto issue_qk = [&](int w, const Tile& t, int kst) {
    const uint32_t d_tmem = tmem + w * kBN;
    const uint32_t qbase = sQ + w * L::kTileBytes;
    const uint32_t kbase = sK + kst * L::kTileBytes;
    const uint32_t idesc = t.valid() > 64 ? kIdescQK128 : kIdescQK64;
#pragma unroll
    for (int k = 0; k < D / 16; ++k) {
      const uint32_t off = (k >> 2) * L::kHalfBytes + (k & 3) * 32;
      tc_mma_ss(d_tmem, sdesc_sw128(qbase + off, 16, 1024), sdesc_sw128(kbase + off, 16, 1024), idesc, k > 0);
    }
    tc_commit(bars + kSFull + w);
  };
  // O_w (+)= P_w V: P_w (bf16 pairs) in the S_w columns; V MN-major, 16 keys per k-step
  // = 2048 bytes; the two 64-wide D halves are 16 KB apart (leading byte offset).
  auto issue_pv = [&](int w, const Tile& t, int vst) {
    const uint32_t a_tmem = tmem + w * kBN;
    const uint32_t o_tmem = tmem + 256 + w * 128;
    const uint32_t vbase = sV + vst * L::kTileBytes;
    const int ksteps = t.valid() > 64 ? kBN / 16 : 64 / 16;
    for (int k = 0; k < ksteps; ++k)
      tc_mma_ts(o_tmem, a_tmem + k * 8, sdesc_sw128(vbase + k * 2048, L::kHalfBytes, 1024), kIdescPV,
                (!t.first() || k > 0) ? 1u : 0u);
  };
  auto wait_k = [&]() -> bool {
    if (!mbar_wait(bars + kKFull + (kc_k % kStages), (kc_k / kStages) & 1, abort_flag, p.status)) return false;
    tc_fence_after();
    return true;
  };

  for (int u = blockIdx.x; u < p.n_units; u += gridDim.x) {
    if (!mbar_wait(bars + kQFull, n_q & 1, abort_flag, p.status)) goto done;
    tc_fence_after();
    ++n_q;
    Tile cur, nxt;
    first_tile_from(p, 0, cur);
    // Prologue: S for the unit's first tile, both Q tiles.
    if (!wait_k()) goto done;
    issue_qk(0, cur, kc_k % kStages);
    issue_qk(1, cur, kc_k % kStages);
    tc_commit(bars + kKEmpty + (kc_k % kStages));
    ++kc_k;
    bool more = next_tile(p, cur, nxt);
    if (!more) tc_commit(bars + kQEmpty);
    while (true) {
      const int vst = kc_v % kStages;
      if (!mbar_wait(bars + kVFull + vst, (kc_v / kStages) & 1, abort_flag, p.status)) goto done;
#pragma unroll
      for (int w = 0; w < kQTiles; ++w) {
        if (!mbar_wait(bars + kPReady + w, g & 1, abort_flag, p.status)) goto done;
        if (cur.first() && nch > 0) {
          if (!mbar_wait(bars + kOFree + w, (nch - 1) & 1, abort_flag, p.status)) goto done;
        }
        tc_fence_after();
        issue_pv(w, cur, vst);
        if (cur.last()) tc_commit(bars + kODone + w);
        if (more) {
          if (w == 0 && !wait_k()) goto done;
          issue_qk(w, nxt, kc_k % kStages);
        }
      }
      tc_commit(bars + kVEmpty + vst);
      ++kc_v;
      if (more) {
        tc_commit(bars + kKEmpty + (kc_k % kStages));
        ++kc_k;
      }
      ++g;
      if (cur.last()) ++nch;
      if (!more) break;
      cur = nxt;
      more = next_tile(p, cur, nxt);
      if (!more) tc_commit(bars + kQEmpty);  // the unit's last QK has been issued
    }
  }
done:
  // Drain: wait until every MMA this thread issued has completed.
  tc_commit(bars + kDrain);
  drain_wait(bars + kDrain, 0);
}

// ------------------------------------------------------------------------------- softmax

// Softmax of one tile of NC (128 or 64) columns for this thread's row, in one pass over
// TMEM: the whole S row is loaded into registers (one round trip), keys at or past
// `valid` are masked when MASK (only a block's last tile), then the row max, the lazy
// max update, and P = 2^(S*scale*log2e - m) with packed fp32x2 FMAs, MUFU ex2 and packed
// sums.  On return P is stored as bf16 pairs in columns [0, NC/2) of the S buffer (the
// whole row is already in registers, so the overwrite is safe) and l/m are updated.
template <int D, int NC, bool MASK>
__device__ __forceinline__ void softmax_tile(uint32_t ts, uint32_t to, int valid, bool first, float sl2, float& m,
                                             float& l) {
  uint32_t r[NC];
  if (NC == 128)
    tmem_ld128(ts, *reinterpret_cast<uint32_t(*)[128]>(r));
  else
    tmem_ld64(ts, *reinterpret_cast<uint32_t(*)[64]>(r));
  if (MASK) {
#pragma unroll
    for (int i = 0; i < NC; ++i)
      if (i >= valid) r[i] = __float_as_uint(-INFINITY);
  }
  float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
#pragma unroll
  for (int i = 0; i < NC; i += 8) {
    a0 = fmax3(a0, __uint_as_float(r[i]), __uint_as_float(r[i + 1]));
    a1 = fmax3(a1, __uint_as_float(r[i + 2]), __uint_as_float(r[i + 3]));
    a2 = fmax3(a2, __uint_as_float(r[i + 4]), __uint_as_float(r[i + 5]));
    a3 = fmax3(a3, __uint_as_float(r[i + 6]), __uint_as_float(r[i + 7]));
  }
  const float m_tile = fmaxf(fmaxf(a0, a1), fmaxf(a2, a3)) * sl2;
  float alpha = 1.f;
  bool rescale = false;
  if (first) {
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
  for (int c = 0; c < NC / 32; ++c) {
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int k = c * 32 + 2 * i;
      const uint64_t x = fma_f32x2(f2_pack(__uint_as_float(r[k]), __uint_as_float(r[k + 1])), scale2, negm2);
      const float p0 = ex2_approx(f2_lo(x));
      const float p1 = ex2_approx(f2_hi(x));
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
    // Rows whose max grew by more than 8 rescale O by alpha (1 for the other rows of the
    // warp).  O holds every earlier P.V product (see the MMA issue order), and the P.V of
    // this tile is issued only after P_ready, i.e. after these stores complete.
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t o[32];
      tmem_ld32(to + c * 32, o);
#pragma unroll
      for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
      tmem_st32(to + c * 32, o);
    }
  }
  tmem_wait_st();
}

// Write 32 columns (block cc) of this thread's output row, scaled by 1/l: fp32 or bf16,
// with 32-byte stores when the output base is 32-byte aligned (p.out_v8), else 16-byte.
template <int D>
__device__ __forceinline__ void store_row(const AttnParams& p, size_t o_off, const uint32_t (&r)[32], int cc,
                                          float inv_l) {
  auto sc = [&](int i) { return __uint_as_float(r[i]) * inv_l; };
  if (p.out_f32) {
    float* o = static_cast<float*>(p.out) + o_off + cc * 32;
    if (p.out_v8) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        st_global_v8(o + 8 * i, __float_as_uint(sc(8 * i)), __float_as_uint(sc(8 * i + 1)),
                     __float_as_uint(sc(8 * i + 2)), __float_as_uint(sc(8 * i + 3)), __float_as_uint(sc(8 * i + 4)),
                     __float_as_uint(sc(8 * i + 5)), __float_as_uint(sc(8 * i + 6)), __float_as_uint(sc(8 * i + 7)));
    } else {
      float4* o4 = reinterpret_cast<float4*>(o);
#pragma unroll
      for (int i = 0; i < 8; ++i) o4[i] = make_float4(sc(4 * i), sc(4 * i + 1), sc(4 * i + 2), sc(4 * i + 3));
    }
  } else {
    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out) + o_off + cc * 32;
    if (p.out_v8) {
#pragma unroll
      for (int i = 0; i < 2; ++i)
        st_global_v8(o + 16 * i, pack_bf16x2(sc(16 * i + 0), sc(16 * i + 1)), pack_bf16x2(sc(16 * i + 2), sc(16 * i + 3)),
                     pack_bf16x2(sc(16 * i + 4), sc(16 * i + 5)), pack_bf16x2(sc(16 * i + 6), sc(16 * i + 7)),
                     pack_bf16x2(sc(16 * i + 8), sc(16 * i + 9)), pack_bf16x2(sc(16 * i + 10), sc(16 * i + 11)),
                     pack_bf16x2(sc(16 * i + 12), sc(16 * i + 13)), pack_bf16x2(sc(16 * i + 14), sc(16 * i + 15)));
    } else {
      uint4* o4 = reinterpret_cast<uint4*>(o);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        o4[i] = make_uint4(pack_bf16x2(sc(8 * i + 0), sc(8 * i + 1)), pack_bf16x2(sc(8 * i + 2), sc(8 * i + 3)),
                           pack_bf16x2(sc(8 * i + 4), sc(8 * i + 5)), pack_bf16x2(sc(8 * i + 6), sc(8 * i + 7)));
    }
  }
}

template <int D>
__device__ __forceinline__ void write_empty_row(const AttnParams& p, int c, const UnitCoord& uc, int s_row) {
  const size_t o_off = static_cast<size_t>(c) * p.out_chunk_stride +
                       ((static_cast<size_t>(uc.b) * p.Sq + s_row) * p.H + uc.h) * D;
  if (p.out_f32) {
    float4* o = reinterpret_cast<float4*>(static_cast<float*>(p.out) + o_off);
    for (int i = 0; i < D / 4; ++i) o[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  } else {
    uint4* o = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + o_off);
    for (int i = 0; i < D / 8; ++i) o[i] = make_uint4(0u, 0u, 0u, 0u);
  }
  if (p.lse)
    p.lse[static_cast<size_t>(c) * p.lse_chunk_stride + (static_cast<size_t>(uc.b) * p.H + uc.h) * p.Sq + s_row] =
        -INFINITY;
}

// Softmax warpgroup w: every tile of every block of every unit; at a block's end it hands
// the row's (m, l) to the epilogue warpgroup and carries on with the next block.
template <int D>
__device__ __forceinline__ void attn_softmax(const AttnParams& p, uint8_t* smem, uint64_t* bars, uint32_t tmem,
                                             volatile int* abort_flag) {
  using L = AttnSmem<D>;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int w = warp >> 2;        // warpgroup = Q tile of the pair
  const int quarter = warp & 3;   // TMEM lane quarter
  const int row = quarter * 32 + lane;
  const uint32_t lanes = static_cast<uint32_t>(quarter * 32) << 16;
  const uint32_t ts = tmem + lanes + w * kBN;          // S_w
  const uint32_t to = tmem + lanes + 256 + w * 128;    // O_w
  float2* stat = reinterpret_cast<float2*>(smem + L::kStat) + w * 2 * kBM;
  const float sl2 = p.scale_log2;
  uint32_t g = 0, nch = 0;

  for (int u = blockIdx.x; u < p.n_units; u += gridDim.x) {
    const UnitCoord uc = decode_unit(u, p);
    const int s_row = (uc.qp * kQTiles + w) * kBM + row;
    float m = -INFINITY;  // running max of S*scale*log2e (possibly stale by < 8)
    float l = 0.f;        // running sum of 2^(S*scale*log2e - m)
    if (p.fuse && p.first_c < 0 && s_row < p.Sq) write_empty_row<D>(p, 0, uc, s_row);  // no keys at all
    for (int c = 0; c < p.n_chunks; ++c) {
      const int n_kv = block_tiles(p, c);
      if (n_kv == 0) {  // no keys: O = 0, lse = -inf (fused: the block simply adds nothing)
        if (!p.fuse && s_row < p.Sq) write_empty_row<D>(p, c, uc, s_row);
        continue;
      }
      if (!p.fuse || c == p.first_c) {
        m = -INFINITY;
        l = 0.f;
      }
      for (int j = 0; j < n_kv; ++j, ++g) {
        const Tile t = make_tile(p, c, j);
        if (!warp_wait(bars + kSFull + w, g & 1, abort_flag, p.status)) return;
        tc_fence_after();
        if (t.valid() == 128)
          softmax_tile<D, 128, false>(ts, to, t.valid(), t.first(), sl2, m, l);
        else if (t.valid() > 64)
          softmax_tile<D, 128, true>(ts, to, t.valid(), t.first(), sl2, m, l);
        else if (t.valid() == 64)
          softmax_tile<D, 64, false>(ts, to, t.valid(), t.first(), sl2, m, l);
        else
          softmax_tile<D, 64, true>(ts, to, t.valid(), t.first(), sl2, m, l);
        tc_fence_before();
        mbar_arrive(bars + kPReady + w);
      }
      if (p.fuse && c != p.last_c) continue;  // the segment goes on with the next block
      // Hand (m, l) of this block to the epilogue warpgroup.  First wait until the epilogue
      // has finished the previous block (it releases O_w only after reading that block's
      // stats): without this wait, blocks of a single tile let this warpgroup run two
      // stat_ready phases ahead of the epilogue, which a parity wait cannot tell apart.
      if (nch > 0 && !warp_wait(bars + kOFree + w, (nch - 1) & 1, abort_flag, p.status)) return;
      stat[(nch & 1) * kBM + row] = make_float2(m, l);
      mbar_arrive(bars + kStatReady + w);
      ++nch;
    }
  }
}

// Epilogue warpgroup: for every non-empty block and both Q tiles, wait for the block's
// last P.V and its (m, l), read O_w from TMEM 32 columns at a time, write O/l and the LSE,
// then release O_w for the next block's first P.V.
template <int D>
__device__ __forceinline__ void attn_epilogue(const AttnParams& p, uint8_t* smem, uint64_t* bars, uint32_t tmem,
                                              volatile int* abort_flag) {
  using L = AttnSmem<D>;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int quarter = warp & 3;
  const int row = quarter * 32 + lane;
  const uint32_t lanes = static_cast<uint32_t>(quarter * 32) << 16;
  const float2* stat = reinterpret_cast<const float2*>(smem + L::kStat);
  uint32_t nch = 0;
  if (p.tiles_per_unit == 0) return;
  for (int u = blockIdx.x; u < p.n_units; u += gridDim.x) {
    const UnitCoord uc = decode_unit(u, p);
    for (int c0 = 0; c0 < p.n_chunks; ++c0) {
      if (block_tiles(p, c0) == 0) continue;
      if (p.fuse && c0 != p.last_c) continue;  // one merged output per unit
      const int c = p.fuse ? 0 : c0;             // output block index
#pragma unroll 1
      for (int w = 0; w < kQTiles; ++w) {
        if (!warp_wait(bars + kStatReady + w, nch & 1, abort_flag, p.status)) return;
        if (!warp_wait(bars + kODone + w, nch & 1, abort_flag, p.status)) return;
        tc_fence_after();
        const float2 ml = stat[(w * 2 + (nch & 1)) * kBM + row];
        const float inv_l = 1.f / ml.y;
        const int s_row = (uc.qp * kQTiles + w) * kBM + row;
        const bool row_ok = s_row < p.Sq;
        const size_t o_off = static_cast<size_t>(c) * p.out_chunk_stride +
                             ((static_cast<size_t>(uc.b) * p.Sq + s_row) * p.H + uc.h) * D;
        const uint32_t to = tmem + lanes + 256 + w * 128;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t r[32];
          tmem_ld32(to + cc * 32, r);
          if (row_ok) store_row<D>(p, o_off, r, cc, inv_l);
        }
        tc_fence_before();
        mbar_arrive(bars + kOFree + w);
        if (row_ok && p.lse)
          p.lse[static_cast<size_t>(c) * p.lse_chunk_stride + (static_cast<size_t>(uc.b) * p.H + uc.h) * p.Sq +
                s_row] = (ml.x + log2f(ml.y)) * 0.69314718055994530942f;
      }
      ++nch;
    }
  }
}

// ------------------------------------------------------------------------------- kernel

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
    mbar_init(bars + kQFull, 1);    // TMA transaction count
    mbar_init(bars + kQEmpty, 1);   // MMA commit
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bars + kKFull + s, 1);
      mbar_init(bars + kKEmpty + s, 1);
      mbar_init(bars + kVFull + s, 1);
      mbar_init(bars + kVEmpty + s, 1);
    }
    for (int w = 0; w < kQTiles; ++w) {
      mbar_init(bars + kSFull + w, 1);     // MMA commit after QK_w
      mbar_init(bars + kPReady + w, 128);  // the 128 threads of softmax warpgroup w
      mbar_init(bars + kODone + w, 1);     // MMA commit after a block's last PV_w
      mbar_init(bars + kOFree + w, 128);   // the epilogue warpgroup has read O_w
      mbar_init(bars + kStatReady + w, 128);  // warpgroup w has written a block's (m, l)
    }
    mbar_init(bars + kDrain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == kProducerWarp && (threadIdx.x & 31) == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Producer and MMA roles run on lane 0 of their warp; the other lanes wait at the
  // __syncwarp so that each warp is converged again for the teardown below.
  // Warps 10 and 11 only give their registers back to the softmax warpgroups.
  if (warp >= kEpilogueWarp0) {
    regs_decrease<kEpilogueRegs>();
    attn_epilogue<D>(p, smem, bars, tmem, abort_flag);
  } else if (warp >= kQTiles * 4) {
    regs_decrease<kControlRegs>();
    if (warp == kProducerWarp) {
      if ((threadIdx.x & 31) == 0) attn_producer<D>(&tm_q, &tm_k, &tm_v, p, smem, bars, abort_flag);
    } else if (warp == kMmaWarp) {
      if ((threadIdx.x & 31) == 0) attn_mma<D>(p, smem, bars, tmem, abort_flag);
    }
    __syncwarp();
  } else {
    regs_increase<kSoftmaxRegs>();
    attn_softmax<D>(p, smem, bars, tmem, abort_flag);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace cpattn
