// cpattn.cu - the C ABI of libcpattn.so (declared in include/cpattn.h).
//
// Host side only: argument checks (all before any CUDA call, so a bad argument never
// launches anything), TMA descriptor encoding, and kernel launches on the caller's
// stream.  Every step of the computation runs in the kernels included below.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <algorithm>
#include <cstring>
#include <mutex>

#include "../../include/cpattn.h"
#include <nvtx3/nvToolsExt.h>

#include "attn_fwd_sm100.cuh"
#include "lse_merge.cuh"
#include "peer.cuh"
#include "ring_gather.cuh"
#include "ulysses_permute.cuh"

using namespace cpattn;

static_assert(kMaxChunks == CP_MAX_CHUNKS && kGatherMaxChunks == CP_MAX_CHUNKS, "chunk limit mismatch");
static_assert(kDevTimeout == CP_ERR_TIMEOUT && kDevBounds == CP_ERR_BOUNDS, "device status codes mismatch");
static_assert(kPeerMax == CP_PEER_MAX && kPeerMergeMax == CP_PEER_MAX, "peer limit mismatch");
static_assert(sizeof(cudaIpcMemHandle_t) == CP_IPC_HANDLE_BYTES, "IPC handle size mismatch");

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool init = false;
  int num_sms = 0;
  int* status = nullptr;  // device address of g_cp_status
  bool attn_attr_set[2] = {false, false};
};

std::mutex g_mutex;
DeviceInfo g_dev[kMaxDevices];
int g_fault_next = 0;  // test hook consumed by the next attention launch
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// An NVTX range around every public call, so that profilers show each call by name
// (header-only NVTX3: without an attached tool the push and pop cost a few instructions).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
// LSE arrays are read and written one float at a time.
inline bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

cp_status device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CP_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceInfo& d = g_dev[dev];
  if (!d.init) {
    if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return CP_ERR_CUDA;
    void* sym = nullptr;
    if (cudaGetSymbolAddress(&sym, g_cp_status) != cudaSuccess) return CP_ERR_CUDA;
    d.status = static_cast<int*>(sym);
    if (!g_encode) {
      cudaDriverEntryPointQueryResult q;
      void* fn = nullptr;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !fn)
        return CP_ERR_CUDA;
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    d.init = true;
  }
  *out = &d;
  return CP_OK;
}

// Element strides of a [B][S][H][D] tensor's batch and sequence dimensions (the head stride
// is D, the d stride 1).
struct BsStrides {
  long long sb, ss;
};

inline BsStrides dense(int S, int H, int D) {
  return {static_cast<long long>(S) * H * D, static_cast<long long>(H) * D};
}

// Encoded tensor maps, keyed on everything that goes into the encoding.  Encoding three
// maps costs microseconds of host time per call, which paces short launches; a map only
// describes an address range and a shape, so reusing one for the same key is exact.
struct MapKey {
  int dev;
  const void* base;
  int B, S, H, D;
  long long sb, ss;
  bool operator==(const MapKey& o) const {
    return dev == o.dev && base == o.base && B == o.B && S == o.S && H == o.H && D == o.D && sb == o.sb &&
           ss == o.ss;
  }
};
constexpr int kMapCacheSize = 64;
struct MapCacheEntry {
  MapKey key;
  CUtensorMap map;
  unsigned long long used = 0;  // 0: empty
};
std::mutex g_map_mutex;
MapCacheEntry g_map_cache[kMapCacheSize];
unsigned long long g_map_clock = 0;

// 4-D map over a bf16 [B][S][H][D] tensor with element strides `st` (batch, sequence):
// dims (D, H, S, B), box (64, 1, 128, 1), 128B swizzle.  Rows past S read as zeros.
cp_status make_bshd_map(CUtensorMap* m, const void* base, int B, int S, int H, int D, BsStrides st) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return CP_ERR_CUDA;
  if (B == 1) st.sb = st.ss * S;  // never used to address: any valid stride
  const MapKey key{dev, base, B, S, H, D, st.sb, st.ss};
  {
    std::lock_guard<std::mutex> lock(g_map_mutex);
    for (MapCacheEntry& e : g_map_cache)
      if (e.used && e.key == key) {
        e.used = ++g_map_clock;
        *m = e.map;
        return CP_OK;
      }
  }
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(S),
                        static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(st.ss) * 2,
                           static_cast<cuuint64_t>(st.sb) * 2};
  cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(kBM), 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return CP_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_map_mutex);
  MapCacheEntry* victim = &g_map_cache[0];
  for (MapCacheEntry& e : g_map_cache)
    if (e.used < victim->used) victim = &e;  // an empty entry (0) first, else the least recently used
  victim->key = key;
  victim->map = *m;
  victim->used = ++g_map_clock;
  return CP_OK;
}

cp_status check_attn_args(const void* q, const void* k, const void* v, const void* out, const float* lse, int B,
                          int H, int Sq, int Skv, int D, float scale, cp_dtype out_dtype) {
  if (B < 0 || H < 0 || Sq < 0 || Skv < 0) return CP_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return CP_ERR_UNSUPPORTED;
  if (out_dtype != CP_BF16 && out_dtype != CP_F32) return CP_ERR_INVALID_ARG;
  if (!(std::isfinite(scale) && scale > 0.f)) return CP_ERR_INVALID_ARG;
  if (B == 0 || H == 0 || Sq == 0) return CP_OK;
  if (!q || !out) return CP_ERR_INVALID_ARG;
  if (Skv > 0 && (!k || !v)) return CP_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out) || (Skv > 0 && (!aligned16(k) || !aligned16(v))) ||
      (lse && !aligned4(lse)))
    return CP_ERR_MISALIGNED;
  // 32-bit limits: TMA coordinates, unit counts.
  const long long n_qt = (Sq + kBM - 1) / kBM;
  if (static_cast<long long>(B) * H * n_qt >= (1LL << 31) || static_cast<long long>(Sq) + 2 * kBM >= (1LL << 31) ||
      static_cast<long long>(Skv) + kBN >= (1LL << 31))
    return CP_ERR_UNSUPPORTED;
  return CP_OK;
}

// Layout of the attention's operands when they are not dense BSHD tensors.
struct AttnLayout {
  BsStrides q, kv, o;   // element strides (batch, sequence) of Q, of K and V, of the output
  int uly_p = 0;        // > 0: output in the Ulysses sequence-sharded layout (see AttnParams)
  int uly_b = 0;
};

// The attention kernel launched as a programmatic dependent of the stream's previous kernel
// (its prologue overlaps that kernel's tail; it waits for it before touching memory).
template <typename Kernel>
void launch_pdl(Kernel kernel, int grid, int smem, cudaStream_t stream, const CUtensorMap& tq, const CUtensorMap& tk,
                const CUtensorMap& tv, const AttnParams& p) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kAttnThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, kernel, tq, tk, tv, p);
}

// Launch the attention kernel over n_chunks K/V blocks given by `bounds` (host array).
// `lay` == nullptr: Q, K, V and the output are dense BSHD tensors.
cp_status launch_attn(const void* q, const void* k, const void* v, const int* bounds, int n_chunks, void* out,
                      int out_f32, long long out_chunk_stride, float* lse, long long lse_chunk_stride, int B, int H,
                      int Sq, int Skv, int D, float scale, cudaStream_t stream, int fuse = 0,
                      const AttnLayout* lay = nullptr) {
  DeviceInfo* dev = nullptr;
  cp_status st = device_info(&dev);
  if (st != CP_OK) return st;
  AttnLayout dl;
  if (!lay) {
    dl.q = dense(Sq, H, D);
    dl.kv = dense(Skv, H, D);
    dl.o = dense(Sq, H, D);
    lay = &dl;
  }
  // Fused: every block feeds one running softmax, and the blocks are consecutive ranges of
  // one K/V tensor, so their union is tiled as one range.  A 128-key tile may then hold the
  // end of one block and the start of the next, and a block no longer ends in a short tile
  // (576-key ring-8 blocks would otherwise cost 5 tiles each instead of 4.5).
  int union_bounds[2];
  if (fuse && n_chunks > 1) {
    union_bounds[0] = bounds[0];
    union_bounds[1] = bounds[n_chunks];
    bounds = union_bounds;
    n_chunks = 1;
  }
  AttnParams p;
  std::memset(&p, 0, sizeof(p));
  p.B = B;
  p.H = H;
  p.Sq = Sq;
  p.n_chunks = n_chunks;
  p.n_qt = (Sq + kBM - 1) / kBM;
  p.n_units = B * H * p.n_qt;
  p.tiles_per_unit = 0;
  for (int i = 0; i < n_chunks; ++i) p.tiles_per_unit += (bounds[i + 1] - bounds[i] + kBN - 1) / kBN;
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.out = out;
  p.out_f32 = out_f32;
  p.out_chunk_stride = out_chunk_stride;
  p.o_sb = lay->o.sb;
  p.o_ss = lay->o.ss;
  p.uly_p = lay->uly_p;
  p.uly_b = lay->uly_b;
  {  // 32-byte stores need every row start 32-byte aligned
    const long long eb = out_f32 ? 4 : 2;
    const bool a32 = (reinterpret_cast<uintptr_t>(out) & 31u) == 0 && (out_chunk_stride * eb) % 32 == 0 &&
                     (lay->uly_p > 0 || ((lay->o.sb * eb) % 32 == 0 && (lay->o.ss * eb) % 32 == 0));
    p.out_v8 = a32 ? 1 : 0;
  }
  p.lse = lse;
  p.lse_chunk_stride = lse_chunk_stride;
  {  // output extents: one output (and [B][H][Sq] LSE) per written block
    const long long one_o = lay->uly_p > 0 ? static_cast<long long>(B) * Sq * H * D
                                           : (B - 1) * lay->o.sb + (Sq - 1) * lay->o.ss + static_cast<long long>(H) * D;
    const long long one_l = static_cast<long long>(B) * H * Sq;
    const int n_out = (fuse || out_chunk_stride == 0) ? 1 : n_chunks;
    p.out_elems = out_chunk_stride ? out_chunk_stride * (n_out - 1) + one_o : one_o;
    p.lse_elems = lse_chunk_stride ? lse_chunk_stride * (n_out - 1) + one_l : one_l;
  }
  p.status = dev->status;
  for (int i = 0; i <= n_chunks; ++i) p.bounds[i] = bounds[i];
  p.fuse = fuse;
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    p.fault = g_fault_next;
    g_fault_next = 0;
  }
  p.first_c = p.last_c = -1;
  for (int i = 0; i < n_chunks; ++i)
    if (bounds[i + 1] > bounds[i]) {
      if (p.first_c < 0) p.first_c = i;
      p.last_c = i;
    }

  CUtensorMap tq, tk, tv;
  // A map needs at least one row; with Skv == 0 every block is empty and K/V are never read.
  const int kv_rows = Skv > 0 ? Skv : 1;
  const void* kp = Skv > 0 ? k : q;
  const void* vp = Skv > 0 ? v : q;
  const BsStrides kvs = Skv > 0 ? lay->kv : lay->q;
  if (make_bshd_map(&tq, q, B, Sq, H, D, lay->q) != CP_OK ||
      make_bshd_map(&tk, kp, B, Skv > 0 ? kv_rows : Sq, H, D, kvs) != CP_OK ||
      make_bshd_map(&tv, vp, B, Skv > 0 ? kv_rows : Sq, H, D, kvs) != CP_OK)
    return CP_ERR_CUDA;

  const int grid = p.n_units < dev->num_sms ? p.n_units : dev->num_sms;
  if (D == 128) {
    using L = AttnSmem<128>;
    if (!dev->attn_attr_set[1]) {
      if (cudaFuncSetAttribute(attn_fwd_sm100_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               L::kRequest) != cudaSuccess)
        return CP_ERR_CUDA;
      dev->attn_attr_set[1] = true;
    }
    launch_pdl(attn_fwd_sm100_kernel<128>, grid, L::kRequest, stream, tq, tk, tv, p);
  } else {
    using L = AttnSmem<64>;
    if (!dev->attn_attr_set[0]) {
      if (cudaFuncSetAttribute(attn_fwd_sm100_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               L::kRequest) != cudaSuccess)
        return CP_ERR_CUDA;
      dev->attn_attr_set[0] = true;
    }
    launch_pdl(attn_fwd_sm100_kernel<64>, grid, L::kRequest, stream, tq, tk, tv, p);
  }
  return cudaGetLastError() == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

cp_status launch_merge(const float* partials, const float* lses, int n, void* out, float* out_lse, int B, int H,
                       int Sq, int D, cp_dtype out_dtype, cudaStream_t stream, int ulysses_p = 0, int ulysses_b = 0,
                       const MergePeers* peers = nullptr, int shard = 0) {
  const long long rows = static_cast<long long>(B) * H * Sq;
  const long long part_stride = rows * D;
  const long long lse_stride = rows;
  // ST query positions per block (all heads), about 64 rows per block.  Blocks of about 128
  // rows fit the FLUX merges in one wave whose blocks all stall on their LSE staging at once
  // (24 heads: 3.6 TB/s); with 64 the second wave's staging overlaps the first wave's
  // streaming (5.1 TB/s; 5.9 for the 3-head Ulysses shards).
  const int ST = H >= 64 ? 1 : 64 / H;
  const long long gx = (Sq + ST - 1) / ST;
  if (B > 65535 || gx >= (1LL << 31)) return CP_ERR_UNSUPPORTED;
  const size_t smem = static_cast<size_t>(n) * H * ST * sizeof(float);
  if (smem > 48 * 1024) return CP_ERR_UNSUPPORTED;
  const dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(B));
  const MergePeers none{};
  auto launch = [&](auto kernel) {
    kernel<<<grid, kMergeThreads, smem, stream>>>(partials, lses, n, out, out_lse, H, Sq, ST, part_stride, lse_stride,
                                                  ulysses_p, ulysses_b, peers ? *peers : none, shard);
  };
  const bool bf16 = out_dtype == CP_BF16;
  if (peers) {
    if (D == 128)
      bf16 ? launch(lse_merge_kernel<128, true, false, true>) : launch(lse_merge_kernel<128, false, false, true>);
    else
      bf16 ? launch(lse_merge_kernel<64, true, false, true>) : launch(lse_merge_kernel<64, false, false, true>);
  } else if (ulysses_p > 0) {
    if (D == 128)
      bf16 ? launch(lse_merge_kernel<128, true, true>) : launch(lse_merge_kernel<128, false, true>);
    else
      bf16 ? launch(lse_merge_kernel<64, true, true>) : launch(lse_merge_kernel<64, false, true>);
  } else {
    if (D == 128)
      bf16 ? launch(lse_merge_kernel<128, true, false>) : launch(lse_merge_kernel<128, false, false>);
    else
      bf16 ? launch(lse_merge_kernel<64, true, false>) : launch(lse_merge_kernel<64, false, false>);
  }
  return cudaGetLastError() == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

cp_status check_bounds(const int* chunk_bounds, int n_chunks, int Skv) {
  if (n_chunks < 1 || !chunk_bounds) return CP_ERR_INVALID_ARG;
  if (n_chunks > CP_MAX_CHUNKS) return CP_ERR_UNSUPPORTED;
  if (Skv < 0) return CP_ERR_INVALID_ARG;
  if (chunk_bounds[0] != 0 || chunk_bounds[n_chunks] != Skv) return CP_ERR_INVALID_ARG;
  for (int i = 0; i < n_chunks; ++i)
    if (chunk_bounds[i] > chunk_bounds[i + 1]) return CP_ERR_INVALID_ARG;
  return CP_OK;
}

inline size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

}  // namespace

extern "C" {

int cp_version(void) { return 101; }

const char* cp_status_string(cp_status s) {
  switch (s) {
    case CP_OK: return "CP_OK";
    case CP_ERR_INVALID_ARG: return "CP_ERR_INVALID_ARG: invalid argument";
    case CP_ERR_UNSUPPORTED: return "CP_ERR_UNSUPPORTED: unsupported size or head_dim";
    case CP_ERR_NOT_DIVISIBLE: return "CP_ERR_NOT_DIVISIBLE: sequence or heads not divisible by the degree";
    case CP_ERR_MISALIGNED: return "CP_ERR_MISALIGNED: device pointer not 16-byte aligned";
    case CP_ERR_CUDA: return "CP_ERR_CUDA: CUDA runtime or driver error";
    case CP_ERR_TIMEOUT: return "CP_ERR_TIMEOUT: a device-side wait ran out";
    case CP_ERR_BOUNDS: return "CP_ERR_BOUNDS: a debug build caught an index outside its buffer";
  }
  return "unknown cp_status";
}

cp_status cp_attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int H, int Sq,
                      int Skv, int D, float scale, cp_dtype out_dtype, void* stream) {
  NvtxRange nvtx_range("cp_attn_fwd");
  cp_status st = check_attn_args(q, k, v, out, lse, B, H, Sq, Skv, D, scale, out_dtype);
  if (st != CP_OK || B == 0 || H == 0 || Sq == 0) return st;
  const int bounds[2] = {0, Skv};
  return launch_attn(q, k, v, bounds, 1, out, out_dtype == CP_F32 ? 1 : 0, 0, lse, 0, B, H, Sq, Skv, D, scale,
                     static_cast<cudaStream_t>(stream));
}

cp_status cp_attn_fwd_strided(const void* q, const void* k, const void* v, void* out, float* lse, int B, int H,
                              int Sq, int Skv, int D, long long q_sb, long long q_ss, long long kv_sb, long long kv_ss,
                              long long o_sb, long long o_ss, float scale, cp_dtype out_dtype, void* stream) {
  NvtxRange nvtx_range("cp_attn_fwd_strided");
  cp_status st = check_attn_args(q, k, v, out, lse, B, H, Sq, Skv, D, scale, out_dtype);
  if (st != CP_OK || B == 0 || H == 0 || Sq == 0) return st;
  const long long row = static_cast<long long>(H) * D;
  const long long eb = out_dtype == CP_F32 ? 4 : 2;
  // Strides are positive; the batch stride matters only with more than one batch.
  auto stride_bad = [&](long long sb, long long ss) { return ss <= 0 || (B > 1 && sb <= 0); };
  if (stride_bad(q_sb, q_ss) || stride_bad(o_sb, o_ss) || (Skv > 0 && stride_bad(kv_sb, kv_ss)))
    return CP_ERR_INVALID_ARG;
  // TMA: bf16 input strides are multiples of 16 bytes (8 elements) and below 2^40 bytes.
  auto tma_bad = [&](long long sb, long long ss) { return ss % 8 != 0 || (B > 1 && sb % 8 != 0); };
  if (tma_bad(q_sb, q_ss) || (Skv > 0 && tma_bad(kv_sb, kv_ss))) return CP_ERR_MISALIGNED;
  if (q_ss >= (1LL << 39) || q_sb >= (1LL << 39) || kv_ss >= (1LL << 39) || kv_sb >= (1LL << 39))
    return CP_ERR_UNSUPPORTED;
  // Output rows start on 16-byte boundaries and do not overlap (one dimension nests in the other).
  if ((o_ss * eb) % 16 != 0 || (B > 1 && (o_sb * eb) % 16 != 0)) return CP_ERR_MISALIGNED;
  {
    long long s1 = o_ss, n1 = Sq, s2 = o_sb, n2 = B;
    if (B > 1 && s2 < s1) {
      std::swap(s1, s2);
      std::swap(n1, n2);
    }
    const bool inner_ok = n1 == 1 || s1 >= row;
    const bool outer_ok = n2 == 1 || s2 >= s1 * n1;
    if (!(B == 1 ? (Sq == 1 || o_ss >= row) : (inner_ok && outer_ok && (n1 > 1 || s2 >= row))))
      return CP_ERR_INVALID_ARG;
  }
  AttnLayout lay;
  lay.q = {q_sb, q_ss};
  lay.kv = {kv_sb, kv_ss};
  lay.o = {o_sb, o_ss};
  const int bounds[2] = {0, Skv};
  return launch_attn(q, k, v, bounds, 1, out, out_dtype == CP_F32 ? 1 : 0, 0, lse, 0, B, H, Sq, Skv, D, scale,
                     static_cast<cudaStream_t>(stream), 0, &lay);
}

cp_status cp_attn_merge(const float* partials, const float* lses, int n_chunks, void* out, float* out_lse, int B,
                        int H, int Sq, int D, cp_dtype out_dtype, void* stream) {
  NvtxRange nvtx_range("cp_attn_merge");
  if (B < 0 || H < 0 || Sq < 0) return CP_ERR_INVALID_ARG;
  if (n_chunks < 1 || n_chunks > CP_MAX_CHUNKS) return n_chunks < 1 ? CP_ERR_INVALID_ARG : CP_ERR_UNSUPPORTED;
  if (D != 64 && D != 128) return CP_ERR_UNSUPPORTED;
  if (out_dtype != CP_BF16 && out_dtype != CP_F32) return CP_ERR_INVALID_ARG;
  if (B == 0 || H == 0 || Sq == 0) return CP_OK;
  if (!partials || !lses || !out) return CP_ERR_INVALID_ARG;
  if (!aligned16(partials) || !aligned4(lses) || !aligned16(out) || (out_lse && !aligned4(out_lse)))
    return CP_ERR_MISALIGNED;
  return launch_merge(partials, lses, n_chunks, out, out_lse, B, H, Sq, D, out_dtype,
                      static_cast<cudaStream_t>(stream));
}

size_t cp_ring_sim_workspace_size(int n_chunks, int B, int H, int Sq, int D) {
  if (n_chunks <= 1 || B <= 0 || H <= 0 || Sq <= 0 || D <= 0) return 0;
  const size_t rows = static_cast<size_t>(B) * H * Sq;
  return round256(static_cast<size_t>(n_chunks) * rows * D * sizeof(float)) +
         round256(static_cast<size_t>(n_chunks) * rows * sizeof(float));
}

cp_status cp_attn_fwd_blocks(const void* q, const void* k, const void* v, const int* chunk_bounds, int n_chunks,
                             float* partials, float* lses, int B, int H, int Sq, int Skv, int D, float scale,
                             void* stream) {
  NvtxRange nvtx_range("cp_attn_fwd_blocks");
  cp_status st = check_bounds(chunk_bounds, n_chunks, Skv);
  if (st != CP_OK) return st;
  st = check_attn_args(q, k, v, partials, lses, B, H, Sq, Skv, D, scale, CP_F32);
  if (st != CP_OK || B == 0 || H == 0 || Sq == 0) return st;
  if (!lses) return CP_ERR_INVALID_ARG;
  const long long rows = static_cast<long long>(B) * H * Sq;
  return launch_attn(q, k, v, chunk_bounds, n_chunks, partials, 1, rows * D, lses, rows, B, H, Sq, Skv, D, scale,
                     static_cast<cudaStream_t>(stream));
}

cp_status cp_ring_sim(const void* q, const void* k, const void* v, const int* chunk_bounds, int n_chunks, void* out,
                      float* out_lse, int B, int H, int Sq, int Skv, int D, float scale, cp_dtype out_dtype,
                      void* workspace, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("cp_ring_sim");
  cp_status st = check_bounds(chunk_bounds, n_chunks, Skv);
  if (st != CP_OK) return st;
  st = check_attn_args(q, k, v, out, out_lse, B, H, Sq, Skv, D, scale, out_dtype);
  if (st != CP_OK || B == 0 || H == 0 || Sq == 0) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (n_chunks == 1)
    return launch_attn(q, k, v, chunk_bounds, 1, out, out_dtype == CP_F32 ? 1 : 0, 0, out_lse, 0, B, H, Sq, Skv, D,
                       scale, s);
  const size_t need = cp_ring_sim_workspace_size(n_chunks, B, H, Sq, D);
  if (!workspace || ws_bytes < need) return CP_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return CP_ERR_MISALIGNED;
  const long long rows = static_cast<long long>(B) * H * Sq;
  float* partials = static_cast<float*>(workspace);
  float* lses = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                         round256(static_cast<size_t>(n_chunks) * rows * D * sizeof(float)));
  st = launch_attn(q, k, v, chunk_bounds, n_chunks, partials, 1, rows * D, lses, rows, B, H, Sq, Skv, D, scale, s);
  if (st != CP_OK) return st;
  return launch_merge(partials, lses, n_chunks, out, out_lse, B, H, Sq, D, out_dtype, s);
}

}  // extern "C"

// Static scratch of cp_ring_sim_static: fp32 partials and LSEs of every K/V block, for
// callers that cannot allocate.  Host code only ever sees a stand-in for this symbol,
// so its device address is looked up per device (with that device current) and passed
// to the kernels as an ordinary pointer.
static __device__ __align__(256) unsigned char g_static_scratch[CP_STATIC_SCRATCH_BYTES];

namespace {
std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

cp_status static_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CP_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return CP_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return CP_OK;
}
}  // namespace

extern "C" {

cp_status cp_ring_sim_static(const void* q, const void* k, const void* v, const int* chunk_bounds, int n_chunks,
                             void* out, float* out_lse, int B, int H, int Sq, int Skv, int D, float scale,
                             cp_dtype out_dtype, void* stream) {
  NvtxRange nvtx_range("cp_ring_sim_static");
  cp_status st = check_bounds(chunk_bounds, n_chunks, Skv);
  if (st != CP_OK) return st;
  st = check_attn_args(q, k, v, out, out_lse, B, H, Sq, Skv, D, scale, out_dtype);
  if (st != CP_OK || B == 0 || H == 0 || Sq == 0) return st;
  const size_t need = cp_ring_sim_workspace_size(n_chunks, B, H, Sq, D);
  if (need > CP_STATIC_SCRATCH_BYTES) return CP_ERR_UNSUPPORTED;
  // The address look-up runs on every call, also one that needs no scratch (a single
  // block), so that whichever call comes first on a device does the set-up.
  void* scratch = nullptr;
  st = static_scratch(&scratch);
  if (st != CP_OK) return st;
  return cp_ring_sim(q, k, v, chunk_bounds, n_chunks, out, out_lse, B, H, Sq, Skv, D, scale, out_dtype, scratch,
                     need, stream);
}

size_t cp_usp_sim_workspace_size(int degree, int n_chunks, int B, int S, int H, int D, cp_dtype out_dtype) {
  if (degree < 1 || n_chunks < 1 || B <= 0 || S <= 0 || H <= 0 || D <= 0 || H % degree != 0) return 0;
  const size_t elems = static_cast<size_t>(B) * S * H * D;
  const size_t out_bytes = out_dtype == CP_F32 ? 4 : 2;
  return 3 * round256(elems * 2) + round256(elems * out_bytes) +
         round256(static_cast<size_t>(B) * H * S * sizeof(float)) +
         cp_ring_sim_workspace_size(n_chunks, degree * B, H / degree, S, D);
}

cp_status cp_usp_sim(const void* q, const void* k, const void* v, int degree, const int* chunk_bounds, int n_chunks,
                     void* out, float* out_lse, int B, int S, int H, int D, float scale, cp_dtype out_dtype,
                     void* workspace, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("cp_usp_sim");
  if (degree < 1 || B <= 0 || S <= 0 || H <= 0) return CP_ERR_INVALID_ARG;
  if (S % degree != 0 || H % degree != 0) return CP_ERR_NOT_DIVISIBLE;
  cp_status st = check_bounds(chunk_bounds, n_chunks, S);
  if (st != CP_OK) return st;
  st = check_attn_args(q, k, v, out, out_lse, B, H, S, S, D, scale, out_dtype);
  if (st != CP_OK) return st;
  const size_t need = cp_usp_sim_workspace_size(degree, n_chunks, B, S, H, D, out_dtype);
  if (!workspace || ws_bytes < need) return CP_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return CP_ERR_MISALIGNED;
  const size_t elems = static_cast<size_t>(B) * S * H * D;
  const int out_bytes = out_dtype == CP_F32 ? 4 : 2;
  char* w = static_cast<char*>(workspace);
  void* qh = w;
  void* kh = w + round256(elems * 2);
  void* vh = w + 2 * round256(elems * 2);
  void* oh = w + 3 * round256(elems * 2);
  float* lse_h = reinterpret_cast<float*>(w + 3 * round256(elems * 2) + round256(elems * out_bytes));
  char* ring_ws = reinterpret_cast<char*>(lse_h) + round256(static_cast<size_t>(B) * H * S * sizeof(float));
  const size_t ring_bytes = ws_bytes - static_cast<size_t>(ring_ws - w);
  // 1. First all-to-all: sequence-sharded Q, K, V -> head-sharded [P][B][S][H/P][D].
  const void* srcs[3] = {q, k, v};
  void* const dsts[3] = {qh, kh, vh};
  st = cp_ulysses_permute_n(srcs, dsts, 3, degree, B, S, H, D, 0, 2, stream);
  if (st != CP_OK) return st;
  // 2. Ring attention over the K/V blocks, every head shard at once (batch P*B, H/P heads).
  st = cp_ring_sim(qh, kh, vh, chunk_bounds, n_chunks, oh, out_lse ? lse_h : nullptr, degree * B, H / degree, S, S,
                   D, scale, out_dtype, ring_ws, ring_bytes, stream);
  if (st != CP_OK) return st;
  // 3. Second all-to-all: head-sharded O -> sequence-sharded, as the inputs.
  st = cp_ulysses_permute(oh, out, degree, B, S, H, D, 1, out_bytes, stream);
  if (st != CP_OK) return st;
  // 4. LSE [P][B][H/P][S] -> [B][H][S].
  if (out_lse) {
    const long long block = static_cast<long long>(H / degree) * S;
    const long long gx = (block + 255) / 256 < 1024 ? (block + 255) / 256 : 1024;
    if (static_cast<long long>(degree) * B > 65535) return CP_ERR_UNSUPPORTED;
    lse_regroup_kernel<<<dim3(static_cast<unsigned>(gx), static_cast<unsigned>(degree * B)), 256, 0,
                         static_cast<cudaStream_t>(stream)>>>(lse_h, out_lse, degree, B, block);
    if (cudaGetLastError() != cudaSuccess) return CP_ERR_CUDA;
  }
  return CP_OK;
}

cp_status cp_ring_sim_fused(const void* q, const void* k, const void* v, const int* chunk_bounds, int n_chunks,
                            void* out, float* out_lse, int B, int H, int Sq, int Skv, int D, float scale,
                            cp_dtype out_dtype, void* stream) {
  NvtxRange nvtx_range("cp_ring_sim_fused");
  cp_status st = check_bounds(chunk_bounds, n_chunks, Skv);
  if (st != CP_OK) return st;
  st = check_attn_args(q, k, v, out, out_lse, B, H, Sq, Skv, D, scale, out_dtype);
  if (st != CP_OK || B == 0 || H == 0 || Sq == 0) return st;
  return launch_attn(q, k, v, chunk_bounds, n_chunks, out, out_dtype == CP_F32 ? 1 : 0, 0, out_lse, 0, B, H, Sq, Skv,
                     D, scale, static_cast<cudaStream_t>(stream), 1);
}

cp_status cp_ring_sim_fused_ulysses(const void* q, const void* k, const void* v, int degree, const int* chunk_bounds,
                                    int n_chunks, void* out, float* out_lse, int B, int S, int H, int D, float scale,
                                    cp_dtype out_dtype, void* stream) {
  NvtxRange nvtx_range("cp_ring_sim_fused_ulysses");
  if (degree < 1 || B < 0 || S < 0 || H < 0) return CP_ERR_INVALID_ARG;
  if (S % degree != 0 || H % degree != 0) return CP_ERR_NOT_DIVISIBLE;
  cp_status st = check_bounds(chunk_bounds, n_chunks, S);
  if (st != CP_OK) return st;
  if (static_cast<long long>(degree) * B >= (1LL << 31)) return CP_ERR_UNSUPPORTED;
  const int Bp = degree * B, Hp = H / degree;
  st = check_attn_args(q, k, v, out, out_lse, Bp, Hp, S, S, D, scale, out_dtype);
  if (st != CP_OK || B == 0 || H == 0 || S == 0) return st;
  AttnLayout lay;
  lay.q = lay.kv = lay.o = dense(S, Hp, D);
  lay.uly_p = degree;
  lay.uly_b = B;
  return launch_attn(q, k, v, chunk_bounds, n_chunks, out, out_dtype == CP_F32 ? 1 : 0, 0, out_lse, 0, Bp, Hp, S, S,
                     D, scale, static_cast<cudaStream_t>(stream), 1, &lay);
}

cp_status cp_ring_anything_gather(const void* const* srcs, void* const* dsts, int n_tensors, const int* chunk_bounds,
                                  int n_chunks, int max_len, int B, int S, int H, int D, int elem_bytes,
                                  void* stream) {
  NvtxRange nvtx_range("cp_ring_anything_gather");
  cp_status st = check_bounds(chunk_bounds, n_chunks, S);
  if (st != CP_OK) return st;
  if (B < 0 || H < 0 || D < 0 || max_len < 0) return CP_ERR_INVALID_ARG;
  if (elem_bytes != 2 && elem_bytes != 4) return CP_ERR_UNSUPPORTED;
  if (n_tensors < 1 || !srcs || !dsts) return CP_ERR_INVALID_ARG;
  if (n_tensors > kGatherMaxTensors) return CP_ERR_UNSUPPORTED;
  GatherArgs a;
  std::memset(&a, 0, sizeof(a));
  int longest = 0;
  for (int c = 0; c < n_chunks; ++c) {
    a.bounds[c] = chunk_bounds[c];
    longest = std::max(longest, chunk_bounds[c + 1] - chunk_bounds[c]);
  }
  a.bounds[n_chunks] = chunk_bounds[n_chunks];
  if (max_len < longest) return CP_ERR_INVALID_ARG;
  if (B == 0 || H == 0 || D == 0 || max_len == 0) return CP_OK;
  const long long row_bytes = static_cast<long long>(H) * D * elem_bytes;
  const long long src_bytes = static_cast<long long>(B) * S * row_bytes;
  const long long dst_bytes = static_cast<long long>(n_chunks) * B * max_len * row_bytes;
  for (int t = 0; t < n_tensors; ++t) {
    if (!dsts[t] || (S > 0 && !srcs[t])) return CP_ERR_INVALID_ARG;
    if (!aligned16(dsts[t]) || (srcs[t] && !aligned16(srcs[t]))) return CP_ERR_MISALIGNED;
    a.src[t] = srcs[t];
    a.dst[t] = dsts[t];
  }
  // No destination may overlap a source or another destination.
  for (int t = 0; t < n_tensors; ++t) {
    const char* d0 = static_cast<const char*>(dsts[t]);
    for (int u = 0; u < n_tensors; ++u) {
      const char* s0 = static_cast<const char*>(srcs[u]);
      if (s0 && s0 < d0 + dst_bytes && d0 < s0 + src_bytes) return CP_ERR_INVALID_ARG;
      const char* e0 = static_cast<const char*>(dsts[u]);
      if (u != t && e0 < d0 + dst_bytes && d0 < e0 + dst_bytes) return CP_ERR_INVALID_ARG;
    }
  }
  const long long rows = static_cast<long long>(n_chunks) * B * max_len;  // destination rows per tensor
  if (rows * n_tensors >= (1LL << 31) || row_bytes >= (1LL << 31)) return CP_ERR_UNSUPPORTED;
  DeviceInfo* dev = nullptr;
  st = device_info(&dev);
  if (st != CP_OK) return st;
  a.n_chunks = n_chunks;
  a.B = B;
  a.S = S;
  a.max_len = max_len;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  auto launch = [&](auto tag) {
    using V = decltype(tag);
    const int row_vecs = static_cast<int>(row_bytes / sizeof(V));
    const long long groups = (rows + kGatherRows - 1) / kGatherRows;
    const dim3 grid((row_vecs + kGatherThreads - 1) / kGatherThreads,
                    static_cast<unsigned>(std::min<long long>(groups, 65535)), n_tensors);
    ring_anything_gather_kernel<V><<<grid, kGatherThreads, 0, cs>>>(a, row_vecs, static_cast<int>(rows));
  };
  if (row_bytes % 16 == 0)
    launch(uint4{});
  else if (row_bytes % 8 == 0)
    launch(uint2{});
  else if (row_bytes % 4 == 0)
    launch(uint32_t{});
  else
    launch(uint16_t{});
  return cudaGetLastError() == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

cp_status cp_ulysses_permute_n(const void* const* srcs, void* const* dsts, int n_tensors, int degree, int B, int S,
                               int H, int D, int direction, int elem_bytes, void* stream) {
  NvtxRange nvtx_range("cp_ulysses_permute_n");
  if (degree < 1 || B < 0 || S < 0 || H < 0 || D < 0) return CP_ERR_INVALID_ARG;
  if (direction != 0 && direction != 1) return CP_ERR_INVALID_ARG;
  if (elem_bytes != 2 && elem_bytes != 4) return CP_ERR_UNSUPPORTED;
  if (n_tensors < 1 || !srcs || !dsts) return CP_ERR_INVALID_ARG;
  if (n_tensors > kPermuteMaxTensors) return CP_ERR_UNSUPPORTED;
  if (S % degree != 0 || H % degree != 0) return CP_ERR_NOT_DIVISIBLE;
  if (B == 0 || S == 0 || H == 0 || D == 0) return CP_OK;
  const long long row_bytes = static_cast<long long>(H) * D * elem_bytes;
  const long long piece_bytes = row_bytes / degree;
  const long long total = static_cast<long long>(B) * S * row_bytes;
  PermuteArgs a;
  for (int t = 0; t < n_tensors; ++t) {
    if (!srcs[t] || !dsts[t]) return CP_ERR_INVALID_ARG;
    if (!aligned16(srcs[t]) || !aligned16(dsts[t])) return CP_ERR_MISALIGNED;
    a.src[t] = srcs[t];
    a.dst[t] = dsts[t];
  }
  // No destination may overlap any source or another destination.
  for (int t = 0; t < n_tensors; ++t) {
    const char* d0 = static_cast<const char*>(dsts[t]);
    for (int u = 0; u < n_tensors; ++u) {
      const char* s0 = static_cast<const char*>(srcs[u]);
      if (s0 < d0 + total && d0 < s0 + total) return CP_ERR_INVALID_ARG;
      const char* e0 = static_cast<const char*>(dsts[u]);
      if (u != t && e0 < d0 + total && d0 < e0 + total) return CP_ERR_INVALID_ARG;
    }
  }
  if (static_cast<long long>(n_tensors) * degree * B > 65535 || row_bytes / 2 >= (1LL << 31)) return CP_ERR_UNSUPPORTED;
  DeviceInfo* dev = nullptr;
  cp_status st = device_info(&dev);
  if (st != CP_OK) return st;
  const int Sp = S / degree;
  const int groups = (Sp + kPermuteRows - 1) / kPermuteRows;
  const unsigned gy = static_cast<unsigned>(groups < 65535 ? groups : 65535);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  auto launch = [&](auto tag) {
    using V = decltype(tag);
    const int row_vecs = static_cast<int>(row_bytes / sizeof(V));
    const int piece_vecs = static_cast<int>(piece_bytes / sizeof(V));
    const dim3 grid((row_vecs + kPermuteThreads - 1) / kPermuteThreads, gy, n_tensors * degree * B);
    ulysses_permute_kernel<V><<<grid, kPermuteThreads, 0, cs>>>(a, degree, B, Sp, row_vecs, piece_vecs, direction);
  };
  if (piece_bytes % 16 == 0)
    launch(uint4{});
  else if (piece_bytes % 8 == 0)
    launch(uint2{});
  else if (piece_bytes % 4 == 0)
    launch(uint32_t{});
  else
    launch(uint16_t{});
  return cudaGetLastError() == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

cp_status cp_attn_merge_ulysses(const float* partials, const float* lses, int n_chunks, void* out, float* out_lse,
                                int degree, int B, int S, int H, int D, cp_dtype out_dtype, void* stream) {
  NvtxRange nvtx_range("cp_attn_merge_ulysses");
  if (degree < 1 || B < 0 || S < 0 || H < 0) return CP_ERR_INVALID_ARG;
  if (S % degree != 0 || H % degree != 0) return CP_ERR_NOT_DIVISIBLE;
  if (n_chunks < 1 || n_chunks > CP_MAX_CHUNKS) return n_chunks < 1 ? CP_ERR_INVALID_ARG : CP_ERR_UNSUPPORTED;
  if (D != 64 && D != 128) return CP_ERR_UNSUPPORTED;
  if (out_dtype != CP_BF16 && out_dtype != CP_F32) return CP_ERR_INVALID_ARG;
  if (B == 0 || H == 0 || S == 0) return CP_OK;
  if (!partials || !lses || !out) return CP_ERR_INVALID_ARG;
  if (!aligned16(partials) || !aligned4(lses) || !aligned16(out) || (out_lse && !aligned4(out_lse)))
    return CP_ERR_MISALIGNED;
  if (static_cast<long long>(degree) * B > 65535) return CP_ERR_UNSUPPORTED;
  return launch_merge(partials, lses, n_chunks, out, out_lse, degree * B, H / degree, S, D, out_dtype,
                      static_cast<cudaStream_t>(stream), degree, B);
}

cp_status cp_ulysses_anything_permute_n(const void* const* srcs, void* const* dsts, int n_tensors, int degree,
                                        const int* seq_bounds, const int* head_bounds, int B, int S, int H, int D,
                                        int direction, int elem_bytes, void* stream) {
  NvtxRange nvtx_range("cp_ulysses_anything_permute_n");
  if (degree < 1 || B < 0 || S < 0 || H < 0 || D < 0 || !seq_bounds || !head_bounds) return CP_ERR_INVALID_ARG;
  if (degree > kPermuteMaxDegree) return CP_ERR_UNSUPPORTED;
  if (direction != 0 && direction != 1) return CP_ERR_INVALID_ARG;
  if (elem_bytes != 2 && elem_bytes != 4) return CP_ERR_UNSUPPORTED;
  if (n_tensors < 1 || !srcs || !dsts) return CP_ERR_INVALID_ARG;
  if (n_tensors > kPermuteMaxTensors) return CP_ERR_UNSUPPORTED;
  if (seq_bounds[0] != 0 || seq_bounds[degree] != S || head_bounds[0] != 0 || head_bounds[degree] != H)
    return CP_ERR_INVALID_ARG;
  for (int i = 0; i < degree; ++i)
    if (seq_bounds[i] > seq_bounds[i + 1] || head_bounds[i] > head_bounds[i + 1]) return CP_ERR_INVALID_ARG;
  if (B == 0 || S == 0 || H == 0 || D == 0) return CP_OK;
  PermuteArgs a;
  std::memset(&a, 0, sizeof(a));
  for (int t = 0; t < n_tensors; ++t) {
    if (!srcs[t] || !dsts[t]) return CP_ERR_INVALID_ARG;
    if (!aligned16(srcs[t]) || !aligned16(dsts[t])) return CP_ERR_MISALIGNED;
    a.src[t] = srcs[t];
    a.dst[t] = dsts[t];
  }
  // No destination may overlap any source or another destination.
  const long long total = static_cast<long long>(B) * S * H * D * elem_bytes;
  for (int t = 0; t < n_tensors; ++t) {
    const char* d0 = static_cast<const char*>(dsts[t]);
    for (int u = 0; u < n_tensors; ++u) {
      const char* s0 = static_cast<const char*>(srcs[u]);
      if (s0 < d0 + total && d0 < s0 + total) return CP_ERR_INVALID_ARG;
      const char* e0 = static_cast<const char*>(dsts[u]);
      if (u != t && e0 < d0 + total && d0 < e0 + total) return CP_ERR_INVALID_ARG;
    }
  }
  if (static_cast<long long>(n_tensors) * degree * B > 65535 || static_cast<long long>(H) * D >= (1LL << 31))
    return CP_ERR_UNSUPPORTED;
  DeviceInfo* dev = nullptr;
  cp_status st = device_info(&dev);
  if (st != CP_OK) return st;
  AnyBounds bd;
  std::memset(&bd, 0, sizeof(bd));
  int max_sp = 0;
  for (int i = 0; i <= degree; ++i) {
    bd.seq[i] = seq_bounds[i];
    bd.head[i] = head_bounds[i];
    if (i < degree && seq_bounds[i + 1] - seq_bounds[i] > max_sp) max_sp = seq_bounds[i + 1] - seq_bounds[i];
  }
  const int groups = (max_sp + kPermuteRows - 1) / kPermuteRows;
  const unsigned gy = static_cast<unsigned>(groups < 65535 ? groups : 65535);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const long long row_bytes = static_cast<long long>(D) * elem_bytes;  // a vector never crosses a head
  auto launch = [&](auto tag) {
    using V = decltype(tag);
    const int ve = static_cast<int>(sizeof(V)) / elem_bytes;
    const int row_vecs = H * D / ve;
    const dim3 grid((row_vecs + kPermuteThreads - 1) / kPermuteThreads, gy, n_tensors * degree * B);
    ulysses_anything_kernel<V><<<grid, kPermuteThreads, 0, cs>>>(a, bd, degree, B, S, H, D, ve, direction);
  };
  if (row_bytes % 16 == 0)
    launch(uint4{});
  else if (row_bytes % 8 == 0)
    launch(uint2{});
  else if (row_bytes % 4 == 0 && elem_bytes <= 4)
    launch(uint32_t{});
  else
    launch(uint16_t{});
  return cudaGetLastError() == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

cp_status cp_ulysses_anything_permute(const void* src, void* dst, int degree, const int* seq_bounds,
                                      const int* head_bounds, int B, int S, int H, int D, int direction, int elem_bytes,
                                      void* stream) {
  NvtxRange nvtx_range("cp_ulysses_anything_permute");
  // Pointers are checked by the batched form; nulls with empty sizes stay a no-op.
  return cp_ulysses_anything_permute_n(&src, &dst, 1, degree, seq_bounds, head_bounds, B, S, H, D, direction,
                                       elem_bytes, stream);
}

cp_status cp_ulysses_permute(const void* src, void* dst, int degree, int B, int S, int H, int D, int direction,
                             int elem_bytes, void* stream) {
  NvtxRange nvtx_range("cp_ulysses_permute");
  // Pointers are checked by the batched form; nulls with empty sizes stay a no-op.
  if (degree < 1 || B < 0 || S < 0 || H < 0 || D < 0) return CP_ERR_INVALID_ARG;
  if (direction != 0 && direction != 1) return CP_ERR_INVALID_ARG;
  if (elem_bytes != 2 && elem_bytes != 4) return CP_ERR_UNSUPPORTED;
  if (S % degree != 0 || H % degree != 0) return CP_ERR_NOT_DIVISIBLE;
  if (B == 0 || S == 0 || H == 0 || D == 0) return CP_OK;
  if (!src || !dst) return CP_ERR_INVALID_ARG;
  return cp_ulysses_permute_n(&src, &dst, 1, degree, B, S, H, D, direction, elem_bytes, stream);
}

cp_status cp_debug_set_fault(int mode) {
  if (mode < 0 || mode > 1) return CP_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_mutex);
  g_fault_next = mode;
  return CP_OK;
}

cp_status cp_ring_bounds(int S, int n, int anything, int* bounds_out) {
  if (S < 0 || n < 1 || !bounds_out) return CP_ERR_INVALID_ARG;
  if (!anything && S % n != 0) return CP_ERR_NOT_DIVISIBLE;
  const int base = S / n, extra = S % n;
  bounds_out[0] = 0;
  for (int i = 0; i < n; ++i) bounds_out[i + 1] = bounds_out[i] + base + (i < extra ? 1 : 0);
  return CP_OK;
}

cp_status cp_last_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return CP_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_cp_status, sizeof(int)) != cudaSuccess) return CP_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_cp_status, &zero, sizeof(int)) != cudaSuccess) return CP_ERR_CUDA;
  }
  return static_cast<cp_status>(v);
}

// ------------------------------------------------------------------ one process per GPU

cp_status cp_peer_alloc(size_t bytes, void** dptr, void* handle) {
  NvtxRange nvtx_range("cp_peer_alloc");
  if (bytes == 0 || !dptr || !handle) return CP_ERR_INVALID_ARG;
  *dptr = nullptr;
  void* p = nullptr;
  if (cudaMalloc(&p, bytes) != cudaSuccess) return CP_ERR_CUDA;
  cudaIpcMemHandle_t h;
  if (cudaMemset(p, 0, bytes) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess ||
      cudaIpcGetMemHandle(&h, p) != cudaSuccess) {
    cudaFree(p);
    return CP_ERR_CUDA;
  }
  std::memcpy(handle, &h, sizeof(h));
  *dptr = p;
  return CP_OK;
}

cp_status cp_peer_open(const void* handle, void** dptr) {
  NvtxRange nvtx_range("cp_peer_open");
  if (!handle || !dptr) return CP_ERR_INVALID_ARG;
  *dptr = nullptr;
  cudaIpcMemHandle_t h;
  std::memcpy(&h, handle, sizeof(h));
  void* p = nullptr;
  if (cudaIpcOpenMemHandle(&p, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) return CP_ERR_CUDA;
  *dptr = p;
  return CP_OK;
}

cp_status cp_peer_close(void* dptr) {
  if (!dptr) return CP_ERR_INVALID_ARG;
  return cudaIpcCloseMemHandle(dptr) == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

cp_status cp_peer_free(void* dptr) {
  if (!dptr) return CP_ERR_INVALID_ARG;
  return cudaFree(dptr) == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

cp_status cp_ulysses_push_n(const void* const* srcs, void* const* dsts, int n_tensors, int rank, int degree, int B,
                            int S, int H, int D, int direction, int elem_bytes, void* stream) {
  NvtxRange nvtx_range("cp_ulysses_push_n");
  if (degree < 1 || rank < 0 || rank >= degree || B < 0 || S < 0 || H < 0 || D < 0) return CP_ERR_INVALID_ARG;
  if (direction != 0 && direction != 1) return CP_ERR_INVALID_ARG;
  if (elem_bytes != 2 && elem_bytes != 4) return CP_ERR_UNSUPPORTED;
  if (n_tensors < 1 || !srcs || !dsts) return CP_ERR_INVALID_ARG;
  if (n_tensors > kPermuteMaxTensors || degree > kPeerMax) return CP_ERR_UNSUPPORTED;
  if (S % degree != 0 || H % degree != 0) return CP_ERR_NOT_DIVISIBLE;
  if (B == 0 || S == 0 || H == 0 || D == 0) return CP_OK;
  const long long row_bytes = static_cast<long long>(H) * D * elem_bytes;
  const long long piece_bytes = row_bytes / degree;
  const int Sp = S / degree;
  const long long total = static_cast<long long>(B) * Sp * row_bytes;  // bytes of every buffer
  PushArgs a;
  std::memset(&a, 0, sizeof(a));
  uintptr_t bits = static_cast<uintptr_t>(piece_bytes);  // the widest vector dividing every offset
  for (int t = 0; t < n_tensors; ++t) {
    if (!srcs[t]) return CP_ERR_INVALID_ARG;
    a.src[t] = srcs[t];
    bits |= reinterpret_cast<uintptr_t>(srcs[t]);
    for (int q = 0; q < degree; ++q) {
      void* d = dsts[t * degree + q];
      if (!d) return CP_ERR_INVALID_ARG;
      a.dst[t][q] = d;
      bits |= reinterpret_cast<uintptr_t>(d);
    }
  }
  if (bits % elem_bytes) return CP_ERR_MISALIGNED;
  // No destination may overlap a source or another destination.
  for (int t = 0; t < n_tensors * degree; ++t) {
    const char* d0 = static_cast<const char*>(dsts[t]);
    for (int u = 0; u < n_tensors; ++u) {
      const char* s0 = static_cast<const char*>(srcs[u]);
      if (s0 < d0 + total && d0 < s0 + total) return CP_ERR_INVALID_ARG;
    }
    for (int u = 0; u < n_tensors * degree; ++u) {
      const char* e0 = static_cast<const char*>(dsts[u]);
      if (u != t && e0 < d0 + total && d0 < e0 + total) return CP_ERR_INVALID_ARG;
    }
  }
  if (static_cast<long long>(n_tensors) * B > 65535 || row_bytes / 2 >= (1LL << 31)) return CP_ERR_UNSUPPORTED;
  DeviceInfo* dev = nullptr;
  cp_status st = device_info(&dev);
  if (st != CP_OK) return st;
  const int groups = (Sp + kPermuteRows - 1) / kPermuteRows;
  const unsigned gy = static_cast<unsigned>(groups < 65535 ? groups : 65535);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  auto launch = [&](auto tag) {
    using V = decltype(tag);
    const int piece_vecs = static_cast<int>(piece_bytes / sizeof(V));
    const int row_vecs = piece_vecs * degree;
    const dim3 grid((row_vecs + kPermuteThreads - 1) / kPermuteThreads, gy, n_tensors * B);
    ulysses_push_kernel<V><<<grid, kPermuteThreads, 0, cs>>>(a, rank, degree, B, Sp, piece_vecs, direction);
  };
  if (bits % 16 == 0)
    launch(uint4{});
  else if (bits % 8 == 0)
    launch(uint2{});
  else if (bits % 4 == 0)
    launch(uint32_t{});
  else
    launch(uint16_t{});
  return cudaGetLastError() == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

cp_status cp_ulysses_anything_push_n(const void* const* srcs, void* const* dsts, int n_tensors, int rank, int degree,
                                     const int* seq_bounds, const int* head_bounds, int B, int H, int D,
                                     int direction, int elem_bytes, void* stream) {
  NvtxRange nvtx_range("cp_ulysses_anything_push_n");
  if (degree < 1 || rank < 0 || rank >= degree || B < 0 || H < 0 || D < 0 || !seq_bounds || !head_bounds)
    return CP_ERR_INVALID_ARG;
  if (direction != 0 && direction != 1) return CP_ERR_INVALID_ARG;
  if (elem_bytes != 2 && elem_bytes != 4) return CP_ERR_UNSUPPORTED;
  if (n_tensors < 1 || !srcs || !dsts) return CP_ERR_INVALID_ARG;
  if (n_tensors > kPermuteMaxTensors || degree > kPeerMax) return CP_ERR_UNSUPPORTED;
  if (seq_bounds[0] != 0 || head_bounds[0] != 0 || head_bounds[degree] != H) return CP_ERR_INVALID_ARG;
  for (int i = 0; i < degree; ++i)
    if (seq_bounds[i] > seq_bounds[i + 1] || head_bounds[i] > head_bounds[i + 1]) return CP_ERR_INVALID_ARG;
  const int S = seq_bounds[degree];
  const int Sr = seq_bounds[rank + 1] - seq_bounds[rank];
  const int Hr = head_bounds[rank + 1] - head_bounds[rank];
  // Rows this rank reads: its sequence shard (forward) or every token of its head shard.
  if (B == 0 || H == 0 || D == 0 || (direction == 0 ? Sr : Hr) == 0) return CP_OK;
  AnyPushArgs a;
  std::memset(&a, 0, sizeof(a));
  uintptr_t bits = static_cast<uintptr_t>(D) * elem_bytes;  // a vector never crosses a head
  for (int t = 0; t < n_tensors; ++t) {
    if (!srcs[t]) return CP_ERR_INVALID_ARG;
    a.src[t] = srcs[t];
    bits |= reinterpret_cast<uintptr_t>(srcs[t]);
    for (int q = 0; q < degree; ++q) {
      void* d = dsts[t * degree + q];
      if (!d) return CP_ERR_INVALID_ARG;
      a.dst[t][q] = d;
      bits |= reinterpret_cast<uintptr_t>(d);
    }
  }
  if (bits % elem_bytes) return CP_ERR_MISALIGNED;
  // Byte extents: the source, and destination q of every tensor; none may overlap another.
  const long long row = static_cast<long long>(D) * elem_bytes;
  auto dst_bytes = [&](int q) {
    return direction == 0 ? static_cast<long long>(B) * S * (head_bounds[q + 1] - head_bounds[q]) * row
                          : static_cast<long long>(B) * (seq_bounds[q + 1] - seq_bounds[q]) * H * row;
  };
  const long long src_bytes = direction == 0 ? static_cast<long long>(B) * Sr * H * row
                                             : static_cast<long long>(B) * S * Hr * row;
  for (int t = 0; t < n_tensors * degree; ++t) {
    const char* d0 = static_cast<const char*>(dsts[t]);
    const long long dn = dst_bytes(t % degree);
    for (int u = 0; u < n_tensors; ++u) {
      const char* s0 = static_cast<const char*>(srcs[u]);
      if (dn > 0 && s0 < d0 + dn && d0 < s0 + src_bytes) return CP_ERR_INVALID_ARG;
    }
    for (int u = 0; u < n_tensors * degree; ++u) {
      const char* e0 = static_cast<const char*>(dsts[u]);
      const long long en = dst_bytes(u % degree);
      if (u != t && dn > 0 && en > 0 && e0 < d0 + dn && d0 < e0 + en) return CP_ERR_INVALID_ARG;
    }
  }
  if (static_cast<long long>(n_tensors) * B * degree > 65535 || static_cast<long long>(H) * D >= (1LL << 31))
    return CP_ERR_UNSUPPORTED;
  DeviceInfo* dev = nullptr;
  cp_status st = device_info(&dev);
  if (st != CP_OK) return st;
  int max_rows = Sr;
  for (int i = 0; i <= degree; ++i) {
    a.seq[i] = seq_bounds[i];
    a.head[i] = head_bounds[i];
    if (direction == 1 && i < degree && seq_bounds[i + 1] - seq_bounds[i] > max_rows)
      max_rows = seq_bounds[i + 1] - seq_bounds[i];
  }
  const int groups = (max_rows + kPermuteRows - 1) / kPermuteRows;
  const unsigned gy = static_cast<unsigned>(groups < 65535 ? groups : 65535);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  auto launch = [&](auto tag) {
    using V = decltype(tag);
    const int ve = static_cast<int>(sizeof(V)) / elem_bytes;
    const long long row_vecs = static_cast<long long>(direction == 0 ? H : Hr) * D / ve;
    const dim3 grid(static_cast<unsigned>((row_vecs + kPermuteThreads - 1) / kPermuteThreads), gy,
                    n_tensors * B * (direction == 0 ? 1 : degree));
    ulysses_anything_push_kernel<V><<<grid, kPermuteThreads, 0, cs>>>(a, rank, degree, B, H, D, ve, direction);
  };
  if (bits % 16 == 0)
    launch(uint4{});
  else if (bits % 8 == 0)
    launch(uint2{});
  else if (bits % 4 == 0)
    launch(uint32_t{});
  else
    launch(uint16_t{});
  return cudaGetLastError() == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

cp_status cp_attn_merge_push(const float* partials, const float* lses, int n_chunks, void* const* peer_outs,
                             int shard, int degree, int B, int S, int H, int D, cp_dtype out_dtype, void* stream) {
  NvtxRange nvtx_range("cp_attn_merge_push");
  if (degree < 1 || shard < 0 || shard >= degree || B < 0 || S < 0 || H < 0) return CP_ERR_INVALID_ARG;
  if (degree > kPeerMergeMax) return CP_ERR_UNSUPPORTED;
  if (S % degree != 0 || H % degree != 0) return CP_ERR_NOT_DIVISIBLE;
  if (n_chunks < 1 || n_chunks > CP_MAX_CHUNKS) return n_chunks < 1 ? CP_ERR_INVALID_ARG : CP_ERR_UNSUPPORTED;
  if (D != 64 && D != 128) return CP_ERR_UNSUPPORTED;
  if (out_dtype != CP_BF16 && out_dtype != CP_F32) return CP_ERR_INVALID_ARG;
  if (B == 0 || H == 0 || S == 0) return CP_OK;
  if (!partials || !lses || !peer_outs) return CP_ERR_INVALID_ARG;
  if (!aligned16(partials) || !aligned4(lses)) return CP_ERR_MISALIGNED;
  MergePeers peers{};
  for (int q = 0; q < degree; ++q) {
    if (!peer_outs[q]) return CP_ERR_INVALID_ARG;
    if (!aligned16(peer_outs[q])) return CP_ERR_MISALIGNED;
    peers.out[q] = peer_outs[q];
  }
  if (B > 65535) return CP_ERR_UNSUPPORTED;
  return launch_merge(partials, lses, n_chunks, nullptr, nullptr, B, H / degree, S, D, out_dtype,
                      static_cast<cudaStream_t>(stream), degree, B, &peers, shard);
}

cp_status cp_peer_barrier(void* const* signal_pads, int rank, int degree, unsigned int epoch,
                          unsigned int timeout_ms, void* stream) {
  NvtxRange nvtx_range("cp_peer_barrier");
  if (degree < 1 || rank < 0 || rank >= degree || !signal_pads) return CP_ERR_INVALID_ARG;
  if (degree > kPeerMax) return CP_ERR_UNSUPPORTED;
  SignalTable t;
  std::memset(&t, 0, sizeof(t));
  for (int q = 0; q < degree; ++q) {
    if (!signal_pads[q]) return CP_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(signal_pads[q]) & 3u) return CP_ERR_MISALIGNED;
    t.pad[q] = static_cast<uint32_t*>(signal_pads[q]);
  }
  DeviceInfo* dev = nullptr;
  cp_status st = device_info(&dev);
  if (st != CP_OK) return st;
  const uint64_t limit_ns = static_cast<uint64_t>(timeout_ms ? timeout_ms : 1000u) * 1000000ull;
  peer_barrier_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(t, rank, degree, epoch, limit_ns,
                                                                      dev->status);
  return cudaGetLastError() == cudaSuccess ? CP_OK : CP_ERR_CUDA;
}

cp_status cp_ring_fetch_block(void* dst, const void* src, int B, int rows, int H, int D, int dst_S, int dst_row0,
                              int src_S, int src_row0, int elem_bytes, void* stream) {
  NvtxRange nvtx_range("cp_ring_fetch_block");
  if (B < 0 || rows < 0 || H < 0 || D < 0 || dst_row0 < 0 || src_row0 < 0) return CP_ERR_INVALID_ARG;
  if (elem_bytes != 2 && elem_bytes != 4) return CP_ERR_UNSUPPORTED;
  if (dst_row0 + static_cast<long long>(rows) > dst_S || src_row0 + static_cast<long long>(rows) > src_S)
    return CP_ERR_INVALID_ARG;
  if (B == 0 || rows == 0 || H == 0 || D == 0) return CP_OK;
  if (!dst || !src) return CP_ERR_INVALID_ARG;
  const size_t row = static_cast<size_t>(H) * D * elem_bytes;
  char* d = static_cast<char*>(dst) + dst_row0 * row;
  const char* s = static_cast<const char*>(src) + src_row0 * row;
  const size_t dst_b = dst_S * row, src_b = src_S * row;
  if (s < d + (B - 1) * dst_b + rows * row && d < s + (B - 1) * src_b + rows * row) return CP_ERR_INVALID_ARG;
  return cudaMemcpy2DAsync(d, dst_b, s, src_b, rows * row, B, cudaMemcpyDefault, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? CP_OK
             : CP_ERR_CUDA;
}

}  // extern "C"
