// attn_fwd_sm100.cuh - non-causal blockwise attention with LSE for B200 (sm_100a).
//
// Computes, for every (batch b, head h, K/V block c, query row i),
//   S_ij = scale * q_i . k_j  over the keys j of block c,
//   O_i  = sum_j softmax_j(S_ij) v_j,   lse_i = ln sum_j exp(S_ij)
// ("Attention backends", "Available backends": scaled_dot_product_attention; the
// per-block fp32 output + LSE follow ContextParallelConfig.convert_to_fp32 on the
// "Parallelism" API page, so that ring blocks can be merged afterwards).
//
// Design (one CTA per SM, persistent over work units (b, h, 128-row Q tile); each unit
// walks every K/V block and, inside a block, its 128-key tiles):
//   warps 0-3   softmax warpgroup 0: keys 0-63 of every K/V tile;
//   warps 4-7   softmax warpgroup 1: keys 64-127.  Thread t of warp w owns query row
//               32*(w%4)+t (= TMEM lane) and keeps its own running max m_k, sum l_k and
//               accumulator O_k over its half k of the keys.  Per tile it loads its 64 S
//               columns from TMEM, masks keys past the block end, updates m_k (lazily)
//               and l_k, and stores P = 2^(S*scale*log2e - m_k) as bf16 over the first
//               32 of those columns.  At a segment's end it hands (m_k, l_k) over.
//   warp 8      TMA producer of Q (two slots, so the next unit's tile arrives early) and
//               K (two stages).
//   warp 10     TMA producer of V (two stages).
//   warp 9      TMEM owner (512 columns) and QK issuer (one thread):
//               S(t) = Q K(t)^T        SS form, into S buffer t%2, as soon as K(t) is
//                                      loaded and PV(t-2) has consumed that buffer;
//   warp 11     P.V issuer (one thread):
//               O_k += P_k(t) V_k(t)   TS form (P from TMEM), once both warpgroups have
//                                      stored P(t); V_k = rows 64k..64k+63 of V.
//               The next S is computed while the softmax works on this tile, and each
//               issuer's bookkeeping overlaps the other's MMAs.
//   warps 12-15 epilogue warpgroup: after a segment's last P.V, merge the two halves,
//               m = max(m_0, m_1), w_k = 2^(m_k - m),
//               O = (w_0 O_0 + w_1 O_1) / (w_0 l_0 + w_1 l_1),
//               lse = ln 2 * (m + log2(w_0 l_0 + w_1 l_1)),
//               release O and write O (fp32 partial, or bf16/fp32) and lse.
// A segment is one K/V block, or every block with p.fuse (cp_ring_sim_fused).
// TMEM columns: S buffers [0,128) and [128,256) (P_k over columns 64k .. 64k+31 of its
// buffer), O_0 [256,256+D), O_1 [384,384+D).
// A tile with at most 64 keys runs an N = 64 QK and no P.V for half 1.
// Lazy max: O_k is rescaled in TMEM only when a row's max grows by more than 8 (a factor
// 256); otherwise the stale max stays, which is exact because O_k and l_k share it and
// 2^8 cannot overflow fp32 or bf16.
// Every mbarrier wait is bounded (see ptx_sm100.cuh); on a timeout every role leaves its
// loop, in-flight TMA loads and MMAs are drained, TMEM is freed and the kernel returns
// with CP_ERR_TIMEOUT recorded in the device status word.
#pragma once

#include <cuda.h>

#include "ptx_sm100.cuh"

namespace cpattn {

constexpr int kBM = 128;           // query rows per work unit (TMEM lanes)
constexpr int kBN = 128;           // keys per K/V tile
constexpr int kHalfN = 64;         // keys per softmax warpgroup and tile
constexpr int kStages = 2;         // Q slots, K stages, V stages
constexpr int kAttnThreads = 512;  // 16 warps: 2 softmax, 1 control, 1 epilogue warpgroup
constexpr int kProducerWarp = 8;   // Q and K loads
constexpr int kMmaWarp = 9;       // TMEM owner, QK issuer
constexpr int kVProducerWarp = 10; // V loads
constexpr int kPvWarp = 11;        // P.V issuer
constexpr int kEpilogueWarp0 = 12;
// setmaxnreg split of the 128 x 512 launch budget: softmax (8 warps), control (warps 8-11),
// epilogue (warps 12-15, enough to hold a whole O row: it releases O before storing it).
constexpr int kSoftmaxRegs = 136;
constexpr int kControlRegs = 48;
constexpr int kEpilogueRegs = 192;
constexpr int kLaunchRegs = 65536 / kAttnThreads;  // registers per thread at launch (128)
static_assert(2 * kSoftmaxRegs + kControlRegs + kEpilogueRegs == 4 * kLaunchRegs,
              "register split must use the launch budget");
static_assert(kSoftmaxRegs >= 128 && kEpilogueRegs >= 128 && kControlRegs <= 128,
              "softmax and epilogue warpgroups grow (setmaxnreg.inc), the control warps shrink");
constexpr int kTmemCols = 512;
constexpr int kTmemO = 256;        // first O column; O_k at kTmemO + 128 k
constexpr int kMaxChunks = 64;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// 2^x on the FMA pipe for one pair in kEmuEvery of a tile without masked keys (0: off):
// n = rint(x) by the 1.5*2^23 shift, f = x - n in [-1/2, 1/2], 2^f by a degree-3 minimax
// polynomial (relative error 7.5e-5; tests/exp2_poly_fit.py prints the
// coefficients), 2^n added to the exponent.
constexpr int kEmuEvery = 4;
constexpr float kExp2C0 = 0.9999280571937561f;
constexpr float kExp2C1 = 0.6932608485221863f;
constexpr float kExp2C2 = 0.24261115491390228f;
constexpr float kExp2C3 = 0.05517221987247467f;

struct AttnParams {
  int B, H, Sq;
  int n_chunks;
  int n_qt;                  // ceil(Sq / kBM) Q tiles
  int n_units;               // B * H * n_qt
  int tiles_per_unit;        // sum over blocks of ceil(len / kBN)
  float scale_log2;          // scale * log2(e)
  void* out;                 // block c at out + c*out_chunk_stride elements, row (b, s, h) at
                             // b*o_sb + s*o_ss + h*D (dense BSHD: o_sb = Sq*H*D, o_ss = H*D)
  int out_f32;               // 1: fp32 output, 0: bf16 output
  int out_v8;                // 1: every output row is 32-byte aligned (32-byte stores)
  long long out_chunk_stride;
  long long o_sb, o_ss;      // element strides of the output's batch and sequence dimensions
  int uly_p, uly_b;          // uly_p > 0: the attention ran on Ulysses head shards (batch
                             // uly_p*uly_b, H = heads per shard) and each row goes to its place
                             // in the sequence-sharded layout [uly_p][uly_b][Sq/uly_p][uly_p*H][D],
                             // its LSE to [uly_b][uly_p*H][Sq] (the inverse exchange, fused)
  float* lse;                // block c at lse + c*lse_chunk_stride, [B][H][Sq]; may be null
  long long lse_chunk_stride;
  long long out_elems, lse_elems;  // extents of out and lse (checked in debug builds)
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
  static constexpr int kQ = 0;                           // kStages Q slots
  static constexpr int kK = kQ + kStages * kTileBytes;   // kStages K stages
  static constexpr int kV = kK + kStages * kTileBytes;   // kStages V stages
  static constexpr int kStat = kV + kStages * kTileBytes;  // float2 [2 halves][2 parities][kBM]: (m, l)
  static constexpr int kBar = kStat + 2 * 2 * kBM * 8;
  static constexpr int kNumBars = 19;
  static constexpr int kUsed = kBar + kNumBars * 8 + 16;
  // Request enough that at most one CTA fits per SM (the kernel allocates all 512 TMEM
  // columns), plus 1 KB for aligning the base to the 128B-swizzle atom.
  static constexpr int kRequest = (kUsed + 1024) > 120 * 1024 ? (kUsed + 1024) : 120 * 1024;
};

// Barrier indices.  Tile t uses K stage, V stage and S buffer t % 2 (kStages = 2), so one
// commit per tile and issuer serves every consumer of that slot:
//   qk_done[t%2]  after S(t) = Q K(t)^T: S(t) is ready (softmax), K stage t%2 is free (K
//                 producer);
//   pv_done[t%2]  after O += P(t) V(t): V stage t%2 is free (V producer), S buffer t%2 is
//                 free for QK(t+2), O holds every product up to tile t (softmax rescale).
// p_ready is per S buffer.  Warp-level signals (p_ready, stat_ready, o_free) are arrived
// by one lane per warp after __syncwarp, so a barrier sees one arrival per warp.
enum : int {
  kQFull = 0, kQEmpty = 2, kKFull = 4, kVFull = 6, kQkDone = 8, kPvDone = 10, kPReady = 12,
  kODone = 14, kOFree = 15, kStatReady = 16, kDrain = 17, kDrainPV = 18
};

struct UnitCoord {
  int b, h, qt;
};

__device__ __forceinline__ UnitCoord decode_unit(int u, const AttnParams& p) {
  UnitCoord r;
  r.qt = u % p.n_qt;
  const int bh = u / p.n_qt;
  r.h = bh % p.H;
  r.b = bh / p.H;
  return r;
}

// Element offset of output row (b, s_row, h) of output block c, and the index of its LSE.
template <int D>
__device__ __forceinline__ long long out_row_offset(const AttnParams& p, int c, int b, int s_row, int h) {
  const long long base = static_cast<long long>(c) * p.out_chunk_stride;
  if (p.uly_p > 0) {
    const int shard = b / p.uly_b, b0 = b - shard * p.uly_b;  // head shard, true batch
    const int sp = p.Sq / p.uly_p;
    const int ps = s_row / sp, s0 = s_row - ps * sp;           // sequence shard, its row
    const long long hf = static_cast<long long>(p.uly_p) * p.H;
    return base + ((static_cast<long long>(ps) * p.uly_b + b0) * sp + s0) * hf * D +
           (static_cast<long long>(shard) * p.H + h) * D;
  }
  return base + b * p.o_sb + s_row * p.o_ss + static_cast<long long>(h) * D;
}

__device__ __forceinline__ long long lse_index(const AttnParams& p, int c, int b, int s_row, int h) {
  const long long base = static_cast<long long>(c) * p.lse_chunk_stride;
  if (p.uly_p > 0) {
    const int shard = b / p.uly_b, b0 = b - shard * p.uly_b;
    return base + (static_cast<long long>(b0) * p.uly_p * p.H + static_cast<long long>(shard) * p.H + h) * p.Sq +
           s_row;
  }
  return base + (static_cast<long long>(b) * p.H + h) * p.Sq + s_row;
}

// Keys of a tile with `valid` keys that fall in half k (0..64).
__device__ __forceinline__ int half_valid(int valid, int k) { return min(kHalfN, max(0, valid - k * kHalfN)); }

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

// Named barrier of the epilogue warpgroup (id 0 is __syncthreads).
constexpr int kBarEpilogue = 1;

// A 128-thread warpgroup waits for `bar`: only its first warp polls (fewer mbarrier polls
// in the MIO queue, for a group that waits most of the time), the others park at named
// barrier `id`.  `alive` carries an earlier
// failure of this thread into the decision, so that every warp of the group leaves
// together: a named barrier that one warp never reaches would never complete.
__device__ __forceinline__ bool group_wait(uint64_t* bar, uint32_t parity, int id, bool alive,
                                           volatile int* abort_flag, int* status, uint32_t sleep_ns = 0) {
  bool ok = alive;
  if ((threadIdx.x & 127) < 32 && ok) ok = mbar_wait(bar, parity, abort_flag, status, sleep_ns);
  return bar_and(id, 128, ok);
}

// One arrival for the whole warp, after every lane's earlier work (ordered by the caller's
// fences) is complete: __syncwarp orders the lanes, then lane 0 arrives.
__device__ __forceinline__ void warp_arrive(uint64_t* bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// Wait bounded by time only (used to drain in-flight work after an abort).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitLimitCycles) return;
  }
}

// ------------------------------------------------------------------------------- producers

// Warp 8, lane 0: the Q tile of every unit (two slots) and one K tile per K/V tile.
template <int D>
__device__ __forceinline__ void attn_producer_qk(const CUtensorMap* tm_q, const CUtensorMap* tm_k,
                                                 const AttnParams& p, uint8_t* smem, uint64_t* bars,
                                                 volatile int* abort_flag) {
  using L = AttnSmem<D>;
  if (p.tiles_per_unit == 0) return;
  uint32_t kc = 0;   // K tiles issued
  uint32_t n_q = 0;  // Q tiles issued
  bool ok = true;
  for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
    const UnitCoord uc = decode_unit(u, p);
    {
      const int qs = n_q % kStages;
      const uint32_t use = n_q / kStages;
      if (use > 0 && !mbar_wait(bars + kQEmpty + qs, (use - 1) & 1, abort_flag, p.status, 32)) break;
      mbar_arrive_expect_tx(bars + kQFull + qs, L::kTileBytes);
#pragma unroll
      for (int hf = 0; hf < D / 64; ++hf)
        tma_load_4d(smem + L::kQ + qs * L::kTileBytes + hf * L::kHalfBytes, tm_q, bars + kQFull + qs, hf * 64, uc.h,
                    uc.qt * kBM, uc.b);
      ++n_q;
    }
    Tile t;
    bool have = first_tile_from(p, 0, t);
    while (have) {
      const int st = kc % kStages;
      const uint32_t use = kc / kStages;
      if (use > 0 && !mbar_wait(bars + kQkDone + st, (use - 1) & 1, abort_flag, p.status, 32)) { ok = false; break; }
      // Test hook (p.fault == 1): skip the CTA's first K tile, so that the consumer's
      // bounded wait runs out and the kernel returns CP_ERR_TIMEOUT.
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
  // Drain: every issued load lands before the CTA may exit (normal path: already done).
  for (int st = 0; st < kStages; ++st) {
    const uint32_t uq = n_q / kStages + (st < static_cast<int>(n_q % kStages) ? 1u : 0u);
    const uint32_t uk = kc / kStages + (st < static_cast<int>(kc % kStages) ? 1u : 0u);
    if (uq > 0) drain_wait(bars + kQFull + st, (uq - 1) & 1);
    if (uk > 0) drain_wait(bars + kKFull + st, (uk - 1) & 1);
  }
}

// Warp 10, lane 0: one V tile per K/V tile.
template <int D>
__device__ __forceinline__ void attn_producer_v(const CUtensorMap* tm_v, const AttnParams& p, uint8_t* smem,
                                                uint64_t* bars, volatile int* abort_flag) {
  using L = AttnSmem<D>;
  if (p.tiles_per_unit == 0) return;
  uint32_t vc = 0;  // V tiles issued
  bool ok = true;
  for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
    const UnitCoord uc = decode_unit(u, p);
    Tile t;
    bool have = first_tile_from(p, 0, t);
    while (have) {
      const int st = vc % kStages;
      const uint32_t use = vc / kStages;
      if (use > 0 && !mbar_wait(bars + kPvDone + st, (use - 1) & 1, abort_flag, p.status, 32)) { ok = false; break; }
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

// ------------------------------------------------------------------------------- MMA issuer

// Warp 9, lane 0: S(t) = Q K(t)^T for every K/V tile t of the CTA (all its units), into
// S buffer t%2: D/16 k-steps of 16; step k sits in the 64-column half k/4 at byte 32*(k%4)
// (128B-swizzled K-major, 8-row groups 1 KB apart).  Buffer t%2 held P(t-2), so QK(t)
// waits for pv_done of tile t-2: MMAs of different threads are not ordered with each
// other.
template <int D>
__device__ __forceinline__ void attn_mma_qk(const AttnParams& p, uint8_t* smem, uint64_t* bars, uint32_t tmem,
                                            volatile int* abort_flag) {
  using L = AttnSmem<D>;
  if (p.tiles_per_unit == 0) return;
  constexpr uint32_t kIdescQK128 = idesc_bf16_f32(kBM, 128, 0);
  constexpr uint32_t kIdescQK64 = idesc_bf16_f32(kBM, 64, 0);
  const uint32_t sQ = smem_u32(smem + L::kQ);
  const uint32_t sK = smem_u32(smem + L::kK);
  uint32_t kc = 0;   // K tiles consumed
  uint32_t g = 0;    // tiles whose QK has been issued
  uint32_t n_q = 0;  // units started (Q slot use)
  for (int u = blockIdx.x; u < p.n_units; u += gridDim.x) {
    const int qs = n_q % kStages;
    if (!mbar_wait(bars + kQFull + qs, (n_q / kStages) & 1, abort_flag, p.status)) goto done;
    ++n_q;
    const uint64_t qd = sdesc_sw128(sQ + qs * L::kTileBytes, 16, 1024);
    Tile t;
    bool have = first_tile_from(p, 0, t);
    while (have) {
      Tile nxt;
      const bool more = next_tile(p, t, nxt);
      const int kst = kc % kStages;
      const int sb = g & 1;
      // K(t) lands long before buffer t%2 frees: test it first, off the critical path.
      if (!mbar_wait(bars + kKFull + kst, (kc / kStages) & 1, abort_flag, p.status)) goto done;
      if (g >= 2 && !mbar_wait(bars + kPvDone + sb, ((g >> 1) - 1) & 1, abort_flag, p.status)) goto done;
      tc_fence_after();
      const uint32_t d_tmem = tmem + sb * kBN;
      const uint64_t kd = sdesc_sw128(sK + kst * L::kTileBytes, 16, 1024);
      const uint32_t idesc = t.valid() > kHalfN ? kIdescQK128 : kIdescQK64;
#pragma unroll
      for (int k = 0; k < D / 16; ++k) {
        const uint32_t off = ((k >> 2) * L::kHalfBytes + (k & 3) * 32) >> 4;  // descriptor address units
        tc_mma_ss(d_tmem, qd + off, kd + off, idesc, k > 0);
      }
      tc_commit(bars + kQkDone + sb);  // kst == sb
      if (!more) tc_commit(bars + kQEmpty + qs);  // the unit's last QK: its Q slot frees
      ++kc;
      ++g;
      t = nxt;
      have = more;
    }
  }
done:
  // Drain: wait until every MMA this thread issued has completed.
  tc_commit(bars + kDrain);
  drain_wait(bars + kDrain, 0);
}

// Warp 11, lane 0: O_k (+)= P_k(t) V_k(t) once both softmax warpgroups have stored P(t).
// P_k = 64 keys as bf16 pairs in 32 columns of S buffer t%2; V MN-major, 16 keys per
// k-step = 2048 bytes, the two 64-wide D halves 16 KB apart (leading byte offset).
template <int D>
__device__ __forceinline__ void attn_mma_pv(const AttnParams& p, uint8_t* smem, uint64_t* bars, uint32_t tmem,
                                            volatile int* abort_flag) {
  using L = AttnSmem<D>;
  if (p.tiles_per_unit == 0) return;
  constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, D, 1);
  const uint32_t sV = smem_u32(smem + L::kV);
  uint32_t vc = 0;    // V tiles consumed
  uint32_t gp = 0;    // tiles whose P.V has been issued
  uint32_t nch = 0;   // segments finished (O phase)
  bool init0 = false, init1 = false;  // O_k already written in the current segment
  for (int u = blockIdx.x; u < p.n_units; u += gridDim.x) {
    Tile t;
    bool have = first_tile_from(p, 0, t);
    while (have) {
      const int vst = vc % kStages;
      const int sb = gp & 1;
      const uint32_t ppar = (gp >> 1) & 1;
      if (t.first()) init0 = init1 = false;
      if (!mbar_wait(bars + kVFull + vst, (vc / kStages) & 1, abort_flag, p.status)) goto done;
      if (!mbar_wait(bars + kPReady + sb, ppar, abort_flag, p.status)) goto done;
      if (t.first() && nch > 0 && !mbar_wait(bars + kOFree, (nch - 1) & 1, abort_flag, p.status)) goto done;
      tc_fence_after();
      const uint64_t vd = sdesc_sw128(sV + vst * L::kTileBytes, L::kHalfBytes, 1024);
      const uint32_t a0 = tmem + sb * kBN;
      {
        const uint32_t acc = init0 ? 1u : 0u;
#pragma unroll
        for (int ks = 0; ks < kHalfN / 16; ++ks)
          tc_mma_ts(tmem + kTmemO, a0 + ks * 8, vd + ks * (2048 >> 4), kIdescPV, acc | (ks > 0 ? 1u : 0u));
        init0 = true;
      }
      if (t.valid() > kHalfN) {
        const uint32_t acc = init1 ? 1u : 0u;
#pragma unroll
        for (int ks = 0; ks < kHalfN / 16; ++ks)
          tc_mma_ts(tmem + kTmemO + 128, a0 + kHalfN + ks * 8, vd + (4 + ks) * (2048 >> 4), kIdescPV,
                    acc | (ks > 0 ? 1u : 0u));
        init1 = true;
      }
      tc_commit(bars + kPvDone + sb);  // vst == sb
      if (t.last()) {
        tc_commit(bars + kODone);
        ++nch;
      }
      ++vc;
      ++gp;
      have = next_tile(p, t, t);
    }
  }
done:
  tc_commit(bars + kDrainPV);
  drain_wait(bars + kDrainPV, 0);
}

// ------------------------------------------------------------------------------- softmax

// Softmax of one tile's half (64 columns, MASK: keys at or past `valid` masked) for this
// thread's row, in one pass: load the 64 S values, row max, lazy max update, then
// P = 2^(S*scale*log2e - m) with packed fp32x2 FMAs, MUFU ex2 and packed sums, stored as
// bf16 pairs over the first 32 of the columns just read.  A rescale of O_k waits for the
// P.V of the previous tile (`pv_prev`, phase parity `pv_par`), which completes every
// earlier product;
// if that wait gives up, the rescale is skipped and false is returned (the kernel is
// aborting; the caller leaves at the next group wait).
template <int D, bool MASK>
__device__ __forceinline__ bool softmax_tile(uint32_t ts, uint32_t to, int valid, bool fresh, float sl2, float& m,
                                             float& l, uint64_t* pv_prev, uint32_t pv_par, volatile int* abort_flag,
                                             int* status) {
  uint32_t r[kHalfN];
  tmem_ld64(ts, r);
  if (MASK) {
#pragma unroll
    for (int i = 0; i < kHalfN; ++i)
      if (i >= valid) r[i] = __float_as_uint(-INFINITY);
  }
  float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
#pragma unroll
  for (int i = 0; i < kHalfN; i += 8) {
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
  for (int c = 0; c < kHalfN / 32; ++c) {
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
        const uint64_t t = add_f32x2(xc, shift);
        const uint64_t fr = add_f32x2(xc, add_f32x2(shift, f2_pack(-f2_lo(t), -f2_hi(t))));
        uint64_t q = fma_f32x2(fr, f2_pack(kExp2C3, kExp2C3), f2_pack(kExp2C2, kExp2C2));
        q = fma_f32x2(fr, q, f2_pack(kExp2C1, kExp2C1));
        q = fma_f32x2(fr, q, f2_pack(kExp2C0, kExp2C0));
        p0 = __uint_as_float(__float_as_uint(f2_lo(q)) + (__float_as_uint(f2_lo(t)) << 23));
        p1 = __uint_as_float(__float_as_uint(f2_hi(q)) + (__float_as_uint(f2_hi(t)) << 23));
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
    // Rows whose max grew by more than 8 rescale O_k by alpha (1 for the other rows of
    // the warp).  This tile's P.V is issued only after p_ready, i.e. after these stores.
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

// Write 32 columns (block cc) of this thread's output row (values already normalised):
// fp32 or bf16, with 32-byte stores when the output base is 32-byte aligned (p.out_v8),
// else 16-byte.
template <int D>
__device__ __forceinline__ void store_row(const AttnParams& p, size_t o_off, const uint32_t (&r)[32], int cc) {
  auto sc = [&](int i) { return __uint_as_float(r[i]); };
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
  const size_t o_off = static_cast<size_t>(out_row_offset<D>(p, c, uc.b, s_row, uc.h));
  if (in_bounds(static_cast<long long>(o_off), D, p.out_elems)) {
    if (p.out_f32) {
      float4* o = reinterpret_cast<float4*>(static_cast<float*>(p.out) + o_off);
      for (int i = 0; i < D / 4; ++i) o[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    } else {
      uint4* o = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + o_off);
      for (int i = 0; i < D / 8; ++i) o[i] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
#ifdef CP_DEBUG
  const long long li = lse_index(p, c, uc.b, s_row, uc.h);
  if (p.lse && in_bounds(li, 1, p.lse_elems)) p.lse[li] = -INFINITY;
#else
  if (p.lse) p.lse[lse_index(p, c, uc.b, s_row, uc.h)] = -INFINITY;
#endif
}

// Softmax warpgroup k (key half k): every tile of every block of every unit; at a
// segment's end it hands the row's (m_k, l_k) to the epilogue warpgroup.
template <int D>
__device__ __forceinline__ void attn_softmax(const AttnParams& p, uint8_t* smem, uint64_t* bars, uint32_t tmem,
                                             volatile int* abort_flag) {
  using L = AttnSmem<D>;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int kh = warp >> 2;       // key half
  const int quarter = warp & 3;   // TMEM lane quarter
  const int row = quarter * 32 + lane;
  const uint32_t lanes = static_cast<uint32_t>(quarter * 32) << 16;
  const uint32_t to = tmem + lanes + kTmemO + kh * 128;  // O_k
  float2* stat = reinterpret_cast<float2*>(smem + L::kStat) + kh * 2 * kBM;
  const float sl2 = p.scale_log2;
  uint32_t g = 0;     // tiles seen
  uint32_t nch = 0;   // segments finished
  bool alive = true;  // false once a wait of this thread gave up

  for (int u = blockIdx.x; u < p.n_units; u += gridDim.x) {
    const UnitCoord uc = decode_unit(u, p);
    const int s_row = uc.qt * kBM + row;
    float m = -INFINITY;  // running max of S*scale*log2e over this half's keys (stale by < 8)
    float l = 0.f;        // running sum of 2^(S*scale*log2e - m)
    bool fresh = true;    // no key of this half seen yet in the segment
    if (kh == 0 && p.fuse && p.first_c < 0 && s_row < p.Sq) write_empty_row<D>(p, 0, uc, s_row);  // no keys
    for (int c = 0; c < p.n_chunks; ++c) {
      const int n_kv = block_tiles(p, c);
      if (n_kv == 0) {  // no keys: O = 0, lse = -inf (fused: the block simply adds nothing)
        if (kh == 0 && !p.fuse && s_row < p.Sq) write_empty_row<D>(p, c, uc, s_row);
        continue;
      }
      if (!p.fuse || c == p.first_c) {
        m = -INFINITY;
        l = 0.f;
        fresh = true;
      }
      for (int j = 0; j < n_kv; ++j, ++g) {
        const Tile t = make_tile(p, c, j);
        const int sb = g & 1;
        if (!warp_wait(bars + kQkDone + sb, (g >> 1) & 1, abort_flag, p.status) || !alive) return;
        tc_fence_after();
        const int vh = half_valid(t.valid(), kh);
        if (vh > 0) {
          const uint32_t ts = tmem + lanes + sb * kBN + kh * kHalfN;
          // A rescale (never on a segment's first tile, so g >= 1) waits for PV(g-1).
          uint64_t* pv_prev = bars + kPvDone + ((g - 1) & 1);
          const uint32_t pv_par = ((g - 1) >> 1) & 1;
          const bool ok = vh == kHalfN
                              ? softmax_tile<D, false>(ts, to, vh, fresh, sl2, m, l, pv_prev, pv_par, abort_flag, p.status)
                              : softmax_tile<D, true>(ts, to, vh, fresh, sl2, m, l, pv_prev, pv_par, abort_flag, p.status);
          alive = alive && ok;
          fresh = false;
        }
        tc_fence_before();
        warp_arrive(bars + kPReady + sb);
      }
      if (p.fuse && c != p.last_c) continue;  // the segment goes on with the next block
      // Hand (m, l) to the epilogue.  First wait until it has finished the previous
      // segment (it releases O only after reading that segment's stats): without this
      // wait, one-tile segments let this warpgroup run two stat_ready phases ahead of the
      // epilogue, which a parity wait cannot tell apart.
      if (nch > 0 && (!warp_wait(bars + kOFree, (nch - 1) & 1, abort_flag, p.status) || !alive)) return;
      stat[(nch & 1) * kBM + row] = make_float2(m, l);
      warp_arrive(bars + kStatReady);
      ++nch;
    }
  }
}

// Epilogue warpgroup: for every segment, wait for its last P.V and both halves' (m, l),
// merge O_0 and O_1 32 columns at a time, write O and the LSE, then release O for the
// next segment's first P.V.
template <int D>
__device__ __forceinline__ void attn_epilogue(const AttnParams& p, uint8_t* smem, uint64_t* bars, uint32_t tmem,
                                              volatile int* abort_flag) {
  using L = AttnSmem<D>;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int quarter = warp & 3;
  const int row = quarter * 32 + lane;
  const uint32_t lanes = static_cast<uint32_t>(quarter * 32) << 16;
  const uint32_t to0 = tmem + lanes + kTmemO;
  const uint32_t to1 = to0 + 128;
  const float2* stat = reinterpret_cast<const float2*>(smem + L::kStat);
  uint32_t nch = 0;
  if (p.tiles_per_unit == 0) return;
  for (int u = blockIdx.x; u < p.n_units; u += gridDim.x) {
    const UnitCoord uc = decode_unit(u, p);
    const int s_row = uc.qt * kBM + row;
    const bool row_ok = s_row < p.Sq;
    for (int c0 = 0; c0 < p.n_chunks; ++c0) {
      if (block_tiles(p, c0) == 0) continue;
      if (p.fuse && c0 != p.last_c) continue;  // one merged output per unit
      const int c = p.fuse ? 0 : c0;             // output block index
      if (!group_wait(bars + kStatReady, nch & 1, kBarEpilogue, true, abort_flag, p.status, 64)) return;
      if (!group_wait(bars + kODone, nch & 1, kBarEpilogue, true, abort_flag, p.status, 64)) return;
      tc_fence_after();
      const float2 s0 = stat[(nch & 1) * kBM + row];
      const float2 s1 = stat[(2 + (nch & 1)) * kBM + row];
      // Half 0 always holds a key of a non-empty segment (l_0 >= 1); half 1 is empty when
      // every tile of the segment has at most 64 keys, and then O_1 was never written.
      const bool has1 = s1.y > 0.f;  // the same for every row
      const float mx = has1 ? fmaxf(s0.x, s1.x) : s0.x;
      const float w0 = ex2_approx(s0.x - mx);
      const float w1 = has1 ? ex2_approx(s1.x - mx) : 0.f;
      const float lsum = s0.y * w0 + s1.y * w1;
      const float inv = 1.f / lsum;
      const float c0f = w0 * inv, c1f = w1 * inv;
      const size_t o_off = static_cast<size_t>(out_row_offset<D>(p, c, uc.b, s_row, uc.h));
      // Read the whole merged O row into registers and release O before storing it: every
      // CTA reaches its block ends at about the same time, so a segment's stores run into
      // HBM bandwidth, and the next segment's first P.V must not wait for them.
      uint32_t r[D];
      if constexpr (D == 128)
        tmem_ld128(to0, r);
      else
        tmem_ld64(to0, r);
      const bool any1 = __any_sync(0xffffffffu, has1);
      if (any1) {
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t r1[32];
          tmem_ld32(to1 + cc * 32, r1);
#pragma unroll
          for (int i = 0; i < 32; ++i)
            r[cc * 32 + i] = __float_as_uint(
                fmaf(__uint_as_float(r[cc * 32 + i]), c0f, has1 ? __uint_as_float(r1[i]) * c1f : 0.f));
        }
      }
      tc_fence_before();
      warp_arrive(bars + kOFree);
      if (!any1) {
#pragma unroll
        for (int i = 0; i < D; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * c0f);
      }
      if (row_ok && in_bounds(static_cast<long long>(o_off), D, p.out_elems)) {
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) store_row<D>(p, o_off, *reinterpret_cast<const uint32_t(*)[32]>(r + cc * 32), cc);
      }
#ifdef CP_DEBUG
      const long long li = lse_index(p, c, uc.b, s_row, uc.h);
      if (row_ok && p.lse && in_bounds(li, 1, p.lse_elems)) p.lse[li] = (mx + log2f(lsum)) * 0.69314718055994530942f;
#else
      if (row_ok && p.lse) p.lse[lse_index(p, c, uc.b, s_row, uc.h)] = (mx + log2f(lsum)) * 0.69314718055994530942f;
#endif
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
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bars + kQFull + s, 1);   // TMA transaction count
      mbar_init(bars + kQEmpty + s, 1);  // MMA commit after the unit's last QK
      mbar_init(bars + kKFull + s, 1);
      mbar_init(bars + kVFull + s, 1);
      mbar_init(bars + kQkDone + s, 1);  // QK thread commit after S of a tile in slot s
      mbar_init(bars + kPvDone + s, 1);  // P.V thread commit after P.V of a tile in slot s
    }
    mbar_init(bars + kPReady + 0, 8);  // each of the 8 softmax warps stored its P
    mbar_init(bars + kPReady + 1, 8);
    mbar_init(bars + kODone, 1);       // MMA commit after a segment's last P.V
    mbar_init(bars + kOFree, 4);       // each epilogue warp has read its O rows
    mbar_init(bars + kStatReady, 8);   // each softmax warp wrote a segment's (m, l)
    mbar_init(bars + kDrain, 1);
    mbar_init(bars + kDrainPV, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == kProducerWarp && (threadIdx.x & 31) == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
  }
  if (warp == kVProducerWarp && (threadIdx.x & 31) == 0) tma_prefetch_desc(&tm_v);
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Launched as a programmatic dependent of the previous kernel in the stream: the setup
  // above overlaps that kernel's tail; no global memory is read or written before it has
  // completed and its writes are visible.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // Producer and MMA roles run on lane 0 of their warp; the other lanes wait at the
  // __syncwarp so that each warp is converged again for the teardown below.
  if (warp >= kEpilogueWarp0) {
    regs_set<kEpilogueRegs, kLaunchRegs>();
    attn_epilogue<D>(p, smem, bars, tmem, abort_flag);
  } else if (warp >= 8) {
    regs_set<kControlRegs, kLaunchRegs>();
    if (warp == kProducerWarp) {
      if ((threadIdx.x & 31) == 0) attn_producer_qk<D>(&tm_q, &tm_k, p, smem, bars, abort_flag);
    } else if (warp == kVProducerWarp) {
      if ((threadIdx.x & 31) == 0) attn_producer_v<D>(&tm_v, p, smem, bars, abort_flag);
    } else if (warp == kMmaWarp) {
      if ((threadIdx.x & 31) == 0) attn_mma_qk<D>(p, smem, bars, tmem, abort_flag);
    } else if (warp == kPvWarp) {
      if ((threadIdx.x & 31) == 0) attn_mma_pv<D>(p, smem, bars, tmem, abort_flag);
    }
    __syncwarp();
  } else {
    regs_set<kSoftmaxRegs, kLaunchRegs>();
    attn_softmax<D>(p, smem, bars, tmem, abort_flag);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace cpattn
