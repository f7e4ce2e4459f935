/*
 * cpattn.h - C ABI of libcpattn.so: the single-GPU hot path of context-parallel
 * attention for diffusion transformers, hand-written for B200 (sm_100a).
 *
 * What is computed (sources are web pages on diffusers' context parallelism):
 *   - "Attention backends", section "Available backends": the default backend is
 *     scaled_dot_product_attention, i.e. non-causal softmax(Q K^T * scale) V over
 *     (batch, seq, heads, head_dim) tensors (section "Checks" uses (1, 10, 8, 64)).
 *   - "Context parallelism", section "Ring Attention": K/V blocks are attended one
 *     after another; section "Ring Anything Attention": blocks of unequal length.
 *   - "Parallelism" (API page), ContextParallelConfig.convert_to_fp32: each block's
 *     output and LSE are kept in float32 so that the ring accumulation is stable.
 *   - "Context parallelism", section "Ulysses Attention": an all-to-all regroups the
 *     data so that each GPU holds all tokens of a subset of heads, and a second one
 *     regroups the results by token.
 *
 * Conventions shared by every entry point:
 *   - Layout "BSHD": [B][S][H][D] row-major, D fastest, densely packed.
 *   - LSE layout: float32 [B][H][Sq], natural logarithm.
 *   - Every pointer argument except chunk_bounds/bounds_out is a DEVICE pointer on
 *     the current CUDA device, owned by the caller.  No entry point allocates device
 *     memory, with one exception: cp_peer_alloc, whose purpose is to allocate a buffer
 *     that other processes can map.  Separately, loading the library creates one
 *     file-scope device array of CP_STATIC_SCRATCH_BYTES (32 MiB) on every device that
 *     runs its code (the scratch of cp_ring_sim_static), held until the process exits.
 *     The library keeps no per-call state.  Device pointers must be 16-byte aligned,
 *     except LSE arrays (float32, read and written one element at a time: 4 bytes).
 *   - stream: a cudaStream_t passed as void*; NULL means the legacy default stream.
 *     All calls are asynchronous on that stream; inputs must stay alive until the
 *     stream has executed the call.
 *   - Arguments are checked on the host before anything is launched; a bad argument
 *     returns an error status and launches nothing.  No call aborts or throws.
 *   - Device-side failures (a bounded wait that ran out) are recorded in a device
 *     status word read by cp_last_device_status().
 *   - Inputs must be finite; NaN/Inf inputs are outside the contract (not checked).
 *   - Calls on the same stream are ordered; the library keeps no global state that
 *     two streams could race on, except the device status word.
 */
#ifndef CPATTN_H
#define CPATTN_H

#include <stddef.h>

/* Entry points are the library's only exported symbols (it is built with hidden visibility). */
#if defined(__GNUC__)
#define CP_API __attribute__((visibility("default")))
#else
#define CP_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  CP_OK = 0,
  CP_ERR_INVALID_ARG = -1,   /* null pointer, negative size, bad chunk bounds, small workspace, bad scale */
  CP_ERR_UNSUPPORTED = -2,   /* head_dim other than 64/128, too many chunks, size beyond 32-bit indexing */
  CP_ERR_NOT_DIVISIBLE = -3, /* S or H not divisible by the Ulysses degree; uneven split without "anything" */
  CP_ERR_MISALIGNED = -4,    /* a device pointer not 16-byte aligned (TMA and vector access need it) */
  CP_ERR_CUDA = -5,          /* a CUDA runtime/driver call failed (no device, launch failure, ...) */
  CP_ERR_TIMEOUT = -6,       /* a device-side bounded wait ran out; the kernel stopped and returned */
  CP_ERR_BOUNDS = -7         /* debug builds (-DCP_DEBUG): a kernel computed an index outside its
                                buffer and skipped that access */
} cp_status;

typedef enum { CP_BF16 = 0, CP_F32 = 1 } cp_dtype;

/* Largest number of K/V blocks a ring simulation or a merge accepts. */
#define CP_MAX_CHUNKS 64

/* Largest number of ranks in one peer exchange group, and the size of an IPC handle. */
#define CP_PEER_MAX 16
#define CP_IPC_HANDLE_BYTES 64

/*
 * cp_attn_fwd - non-causal attention over one K/V block, returning its LSE.
 *
 * Source: "Attention backends", "Available backends" (scaled_dot_product_attention);
 * "Parallelism", ContextParallelConfig.convert_to_fp32 (fp32 output + LSE per block).
 *   S_ij = scale * q_i . k_j;  O_i = sum_j softmax_j(S_ij) v_j;  lse_i = ln sum_j exp(S_ij)
 *
 * q:   bf16 [B][Sq][H][D];  k, v: bf16 [B][Skv][H][D]  (device, read only)
 * out: [B][Sq][H][D], bf16 (out_dtype CP_BF16) or fp32 (CP_F32)  (device, written)
 * lse: fp32 [B][H][Sq] natural log (device, written), or NULL if not wanted
 * D must be 64 or 128.  scale must be finite and > 0 (1/sqrt(D) is SDPA's default).
 * B, H or Sq equal to 0: nothing to do, CP_OK.  Skv == 0: out = 0, lse = -inf.
 * Computation: bf16 tensor-core products with fp32 accumulation; softmax in fp32;
 * probabilities rounded to bf16 for the P.V product; output rounded once at the end.
 */
CP_API cp_status cp_attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
                      int B, int H, int Sq, int Skv, int D, float scale,
                      cp_dtype out_dtype, void* stream);

/*
 * cp_attn_fwd_strided - cp_attn_fwd on tensors that are views inside larger ones.
 *
 * Source: "Context parallelism", "Ring Attention": each ring step attends the local
 * queries to one K/V block, which a caller often holds as a slice of a longer sequence
 * (rows [c, c + Skv) of a [B][S][H][D] tensor), or Q/K/V as slices of a packed QKV
 * tensor.  Same computation and output rules as cp_attn_fwd; only the addressing differs.
 *
 * Element (b, s, h, d) of q is at q + b*q_sb + s*q_ss + h*D + d (elements, not bytes);
 * k and v share kv_sb/kv_ss; the output row (b, s, h) is at out + b*o_sb + s*o_ss + h*D.
 * lse stays dense fp32 [B][H][Sq] (or NULL).
 *   - Strides are > 0 (batch strides are ignored when B == 1).
 *   - q/k/v strides are multiples of 8 elements (16 bytes, a TMA rule) and below 2^39;
 *     output strides times the element size are multiples of 16 bytes.
 *     Violations: CP_ERR_MISALIGNED (alignment) or CP_ERR_UNSUPPORTED (size).
 *   - Output rows (H*D elements each) must not overlap: one of the two output
 *     dimensions must nest inside the other (the smaller stride >= H*D, the larger >=
 *     the smaller times its extent); otherwise CP_ERR_INVALID_ARG.  Inputs may overlap.
 * Dense BSHD tensors (q_sb = Sq*H*D, q_ss = H*D, ...) give exactly cp_attn_fwd's result.
 */
CP_API cp_status cp_attn_fwd_strided(const void* q, const void* k, const void* v, void* out, float* lse,
                                     int B, int H, int Sq, int Skv, int D, long long q_sb, long long q_ss,
                                     long long kv_sb, long long kv_ss, long long o_sb, long long o_ss,
                                     float scale, cp_dtype out_dtype, void* stream);

/*
 * cp_attn_fwd_blocks - attention of q over every K/V block, without the merge.
 *
 * Source: "Context parallelism", "Ring Attention" / "Ring Anything Attention" (each
 * GPU attends its queries to one K/V block per ring step) and convert_to_fp32 (each
 * block's output and LSE in float32).  Block r holds K/V rows
 * [chunk_bounds[r], chunk_bounds[r+1]); all blocks run in one launch.
 *
 * chunk_bounds: HOST int[n_chunks+1], 0 = c_0 <= ... <= c_n = Skv (empty blocks allowed)
 * partials: fp32 [n_chunks][B][Sq][H][D], lses: fp32 [n_chunks][B][H][Sq] (device, written):
 *           exactly the inputs cp_attn_merge expects.  An empty block gives 0 and -inf.
 * Other arguments and rules as cp_attn_fwd; 1 <= n_chunks <= CP_MAX_CHUNKS.
 */
CP_API cp_status cp_attn_fwd_blocks(const void* q, const void* k, const void* v, const int* chunk_bounds,
                             int n_chunks, float* partials, float* lses, int B, int H, int Sq, int Skv,
                             int D, float scale, void* stream);

/*
 * cp_attn_merge - combine per-block attention results through their LSEs.
 *
 * Source: "Context parallelism", "Ring Attention" (results accumulate over K/V
 * blocks) and ContextParallelConfig.convert_to_fp32.  The pages print no formula;
 * the standard log-sum-exp merge is used:
 *   L = M + ln sum_i exp(lse_i - M),  M = max_i lse_i;   O = sum_i exp(lse_i - L) O_i
 * A block with lse_i = -inf (no keys) has weight 0; if all are -inf, O = 0, L = -inf.
 *
 * partials: fp32 [n_chunks][B][Sq][H][D];  lses: fp32 [n_chunks][B][H][Sq]
 * out: [B][Sq][H][D] in out_dtype;  out_lse: fp32 [B][H][Sq] or NULL
 * 1 <= n_chunks <= CP_MAX_CHUNKS; D must be 64 or 128.  out may not alias partials.
 */
CP_API cp_status cp_attn_merge(const float* partials, const float* lses, int n_chunks, void* out,
                        float* out_lse, int B, int H, int Sq, int D, cp_dtype out_dtype,
                        void* stream);

/* Bytes of device workspace cp_ring_sim needs: fp32 partials and LSEs of every block
 * (n_chunks * B*H*Sq*(D+1) * 4, each part rounded up to 256 B).  0 when n_chunks == 1. */
CP_API size_t cp_ring_sim_workspace_size(int n_chunks, int B, int H, int Sq, int D);

/*
 * cp_ring_sim - ring / ring-anything attention simulated on one GPU.
 *
 * Source: "Context parallelism", "Ring Attention" and "Ring Anything Attention".
 * Block r holds K/V rows [chunk_bounds[r], chunk_bounds[r+1]); blocks are attended
 * in ring order r = 0..n-1, each giving an fp32 partial and LSE in the workspace,
 * then the partials are merged: cp_attn_fwd_blocks followed by cp_attn_merge.  Padded rows of ring-anything are
 * cut away before attention on the pages, so blocks are simply their true rows.
 *
 * chunk_bounds: HOST int array of n_chunks+1 entries, 0 = c_0 <= c_1 <= ... <= c_n = Skv
 *               (empty blocks allowed).  Read during the call only.
 * workspace:    device buffer of at least cp_ring_sim_workspace_size(...) bytes,
 *               owned by the caller; contents on return are the per-block partials.
 * Other arguments as cp_attn_fwd.  n_chunks == 1 is plain cp_attn_fwd.
 */
CP_API cp_status cp_ring_sim(const void* q, const void* k, const void* v, const int* chunk_bounds,
                      int n_chunks, void* out, float* out_lse, int B, int H, int Sq, int Skv,
                      int D, float scale, cp_dtype out_dtype, void* workspace, size_t ws_bytes,
                      void* stream);

/*
 * cp_ring_sim_fused - cp_ring_sim with the LSE merge fused into the attention kernel.
 *
 * Source: "Context parallelism", "Ring Attention" / "Ring Anything Attention": a GPU's
 * queries meet the K/V blocks one after another and accumulate the result.  Here the
 * running (max, sum, output) of each query row is carried in TMEM from one block to the
 * next inside one launch, so no per-block partial is written and no merge pass runs; the
 * result equals merging the per-block partials (up to fp32 rounding order).  The blocks
 * are consecutive ranges of one K/V tensor feeding one running softmax, so the kernel tiles
 * their union: a 128-key tile may hold the end of one block and the start of the next.
 * Arguments as cp_ring_sim without the workspace; allocates nothing.  Output and LSE as
 * cp_attn_fwd; an all-empty split gives out = 0, lse = -inf.
 */
CP_API cp_status cp_ring_sim_fused(const void* q, const void* k, const void* v, const int* chunk_bounds,
                            int n_chunks, void* out, float* out_lse, int B, int H, int Sq, int Skv,
                            int D, float scale, cp_dtype out_dtype, void* stream);

/*
 * cp_ring_sim_fused_ulysses - Ulysses x ring attention after the first exchange: the fused
 * ring over K/V blocks on the head shards, writing the output in the sequence-sharded
 * layout (the second all-to-all folded into the kernel's epilogue).
 *
 * Source: "Context parallelism", "Unified Attention": an all-to-all regroups heads and
 * tokens, Ring Attention runs on the result, and the reverse all-to-all restores the
 * token layout.  Here the ring is cp_ring_sim_fused (the running max/sum/output carried
 * across blocks in TMEM, no partials) and each finished row is stored straight to its
 * place in the token-sharded output, so the head-sharded output is never written.
 * q, k, v:  bf16 head-sharded [degree][B][S][H/degree][D] (head shard p = heads
 *           [p*H/degree, (p+1)*H/degree)), as produced by cp_ulysses_permute direction 0.
 * chunk_bounds: HOST int[n_chunks+1] over [0, S], as cp_ring_sim with Skv = S.
 * out:      [degree][B][S/degree][H][D], bf16 or fp32 (out_dtype): the layout of
 *           cp_ulysses_permute direction 1 applied to the attention output.
 * out_lse:  fp32 [B][H][S] natural log, or NULL.
 * Errors: S or H not divisible by degree -> CP_ERR_NOT_DIVISIBLE; otherwise as
 * cp_ring_sim_fused.  Allocates nothing.  The result equals cp_usp_sim's up to fp32
 * rounding order (the merge runs inside the kernel).
 */
CP_API cp_status cp_ring_sim_fused_ulysses(const void* q, const void* k, const void* v, int degree,
                                           const int* chunk_bounds, int n_chunks, void* out, float* out_lse,
                                           int B, int S, int H, int D, float scale, cp_dtype out_dtype,
                                           void* stream);

/*
 * cp_ring_anything_gather - the Ring Anything pad -> all-gather buffer, built on one GPU.
 *
 * Source: "Context parallelism", "Ring Anything Attention": ranks whose K/V blocks have
 * different lengths pad their block to the longest, all-gather the padded blocks, and
 * slice each gathered block back to its true length before attention.  This call builds
 * the gathered buffer of every tensor from the unsharded one:
 *   dst[c][b][r][h][d] = src[b][chunk_bounds[c] + r][h][d]   for r < len_c,
 *   dst[c][b][r][h][d] = 0                                    for len_c <= r < max_len,
 * with len_c = chunk_bounds[c+1] - chunk_bounds[c].  Block c's true-length slice is the
 * [B][len_c][H][D] view at dst + c*B*max_len*H*D with batch stride max_len*H*D and sequence
 * stride H*D, which cp_attn_fwd_strided attends in place.  The copy is exact (bit for bit).
 * srcs:  n_tensors (1..8) device pointers, each [B][S][H][D] with elem_bytes-byte elements.
 * dsts:  n_tensors device pointers, each [n_chunks][B][max_len][H][D] (written); no
 *        destination may overlap a source or another destination (CP_ERR_INVALID_ARG).
 * chunk_bounds: HOST int[n_chunks+1] over [0, S] as cp_ring_sim; max_len >= the longest
 *        block (CP_ERR_INVALID_ARG otherwise).  elem_bytes 2 or 4.  Pointers 16-byte aligned.
 */
CP_API cp_status cp_ring_anything_gather(const void* const* srcs, void* const* dsts, int n_tensors,
                                         const int* chunk_bounds, int n_chunks, int max_len, int B, int S,
                                         int H, int D, int elem_bytes, void* stream);

/* Size in bytes of the workspace cp_usp_sim needs (0 for invalid sizes or H % degree != 0). */
CP_API size_t cp_usp_sim_workspace_size(int degree, int n_chunks, int B, int S, int H, int D,
                                        cp_dtype out_dtype);

/*
 * cp_usp_sim - unified sequence parallelism (Ulysses x ring) simulated on one GPU.
 *
 * Source: "Context parallelism", section "Unified Attention": an all-to-all regroups heads
 * and tokens, Ring Attention runs on the result, and the reverse all-to-all restores the
 * layout; the GPUs form a ulysses_degree x ring_degree grid.  Here: the Ulysses exchange of
 * cp_ulysses_permute (degree `degree`) on Q, K, V; cp_ring_sim over the K/V blocks
 * `chunk_bounds` on every head shard at once; the inverse exchange of O; the LSE regrouped
 * to the unsharded layout.  The result equals unsplit attention up to fp32 rounding order.
 * q, k, v:     bf16, sequence-sharded and stacked rank-major, [degree][B][S/degree][H][D]
 *              (shard p = tokens [p*S/degree, (p+1)*S/degree)), 16-byte aligned.
 * chunk_bounds: HOST int[n_chunks+1], the ring blocks over the whole sequence [0, S]
 *              (as cp_ring_sim, Skv = S).
 * out:         same layout as q, out_dtype (CP_BF16 or CP_F32).
 * out_lse:     fp32 [B][H][S] (natural log), or NULL.
 * workspace:   cp_usp_sim_workspace_size(...) bytes, 16-byte aligned, owned by the caller.
 * Errors: S or H not divisible by degree -> CP_ERR_NOT_DIVISIBLE; otherwise as cp_ring_sim
 * and cp_ulysses_permute.  Asynchronous on `stream`.
 */
CP_API cp_status cp_usp_sim(const void* q, const void* k, const void* v, int degree, const int* chunk_bounds,
                            int n_chunks, void* out, float* out_lse, int B, int S, int H, int D, float scale,
                            cp_dtype out_dtype, void* workspace, size_t ws_bytes, void* stream);

/* Size in bytes of the library's static device scratch used by cp_ring_sim_static. */
#define CP_STATIC_SCRATCH_BYTES (32u << 20)

/*
 * cp_ring_sim_static - cp_ring_sim for callers that cannot allocate device memory.
 *
 * The pages have no counterpart to this call.  It exists for callers of this library
 * that may not allocate device memory at the point where they attend: code that runs
 * inside another framework's memory pool or under a fixed memory budget, where a
 * cudaMalloc would bypass the pool's accounting or fail, and real-time loops where an
 * allocation's latency (and the synchronisation cudaMalloc/cudaFree can imply) is not
 * allowed.  It computes exactly what cp_ring_sim computes, with the same arguments
 * minus workspace/ws_bytes: the per-block fp32 partials and LSEs live in one
 * file-scope device array of CP_STATIC_SCRATCH_BYTES (32 MiB) that every GPU which
 * loads the library keeps until the process exits.  The call allocates nothing.
 *
 * - Sizes: if cp_ring_sim_workspace_size(n_chunks, B, H, Sq, D) exceeds
 *   CP_STATIC_SCRATCH_BYTES the call returns CP_ERR_UNSUPPORTED and launches nothing.
 * - Set-up: the first call on a device with non-empty sizes (B, H, Sq > 0) looks up
 *   the array's device address with that device current (cudaGetSymbolAddress), also
 *   when it needs no scratch (a single block); make that first call before any stream
 *   capture.  A failed look-up returns CP_ERR_CUDA.
 * - Sharing: every call on every stream of a device uses the same array.  Calls
 *   that overlap on the GPU (different streams, no ordering) race and corrupt each
 *   other's results; order them on one stream or with events.  The array keeps the
 *   last call's partials; nothing needs clearing, because every partial and LSE
 *   entry a call reads is written by that call first.
 */
CP_API cp_status cp_ring_sim_static(const void* q, const void* k, const void* v, const int* chunk_bounds,
                             int n_chunks, void* out, float* out_lse, int B, int H, int Sq, int Skv,
                             int D, float scale, cp_dtype out_dtype, void* stream);

/*
 * cp_attn_merge_ulysses - cp_attn_merge of Ulysses head-shard partials, fused with the
 * inverse exchange.
 *
 * Source: "Context parallelism", "Ulysses Attention" (the second all-to-all regroups the
 * results by token) after the LSE merge of the ring blocks (as cp_attn_merge).  The merged
 * rows are written straight to their sequence-sharded positions, so the head-sharded output
 * is never stored and re-read; the result is bit-identical to cp_attn_merge followed by
 * cp_ulysses_permute(direction 1).
 * partials: fp32 [n_chunks][degree*B][S][H/degree][D] (attention on the head shards, shard p
 *           = heads [p*H/degree, (p+1)*H/degree)); lses: fp32 [n_chunks][degree*B][H/degree][S].
 * out:      out_dtype, sequence-sharded [degree][B][S/degree][H][D] (cp_ulysses_permute's
 *           layout); out_lse: fp32 [B][H][S] (natural log), or NULL.
 * Errors: S or H not divisible by degree -> CP_ERR_NOT_DIVISIBLE; otherwise as cp_attn_merge.
 */
CP_API cp_status cp_attn_merge_ulysses(const float* partials, const float* lses, int n_chunks, void* out,
                                       float* out_lse, int degree, int B, int S, int H, int D, cp_dtype out_dtype,
                                       void* stream);

/*
 * cp_ulysses_anything_permute - the Ulysses exchange for shards of unequal size.
 *
 * Source: "Context parallelism", section "Ulysses Anything Attention": the sequence length
 * and the head count need not be divisible by ulysses_degree.  The pages give no layout;
 * the reading here: sequence shard p holds tokens [seq_bounds[p], seq_bounds[p+1]) of
 * every head and head shard q holds heads [head_bounds[q], head_bounds[q+1]) of every
 * token, as even as possible when made by cp_ring_bounds(count, degree, 1, ...) (the
 * first shards one longer).  Shards are packed back to back:
 *   sequence-sharded: shard p at element offset B*seq_bounds[p]*H*D, layout [B][S_p][H][D];
 *   head-sharded:     shard q at element offset B*S*head_bounds[q]*D, layout [B][S][H_q][D].
 * With equal shards these are exactly the stacked layouts of cp_ulysses_permute.
 * direction 0: sequence-sharded src -> head-sharded dst; 1: the inverse.  A pure copy,
 * bit-exact for any element type of elem_bytes (2 or 4) bytes.
 * seq_bounds, head_bounds: HOST int[degree+1], non-decreasing, from 0 to S and 0 to H;
 * empty shards are allowed.  src, dst: B*S*H*D elements each, 16-byte aligned, not
 * overlapping.  degree <= 64.
 * Errors: bad bounds, overlap -> CP_ERR_INVALID_ARG; degree > 64 or elem_bytes not 2/4
 * -> CP_ERR_UNSUPPORTED; misaligned -> CP_ERR_MISALIGNED.  Asynchronous on `stream`.
 */
CP_API cp_status cp_ulysses_anything_permute(const void* src, void* dst, int degree, const int* seq_bounds,
                                             const int* head_bounds, int B, int S, int H, int D, int direction,
                                             int elem_bytes, void* stream);

/*
 * cp_ulysses_anything_permute_n - cp_ulysses_anything_permute of n_tensors same-shaped
 * tensors in one launch (Q, K and V move together).
 *
 * srcs, dsts: HOST arrays of n_tensors device pointers (1 <= n_tensors <= 8), read during
 * the call only.  Other arguments and rules as cp_ulysses_anything_permute; no destination
 * may overlap any source or another destination (CP_ERR_INVALID_ARG).
 */
CP_API cp_status cp_ulysses_anything_permute_n(const void* const* srcs, void* const* dsts, int n_tensors, int degree,
                                               const int* seq_bounds, const int* head_bounds, int B, int S, int H,
                                               int D, int direction, int elem_bytes, void* stream);

/*
 * cp_ulysses_permute - the Ulysses all-to-all, simulated as one local copy.
 *
 * Source: "Context parallelism", "Ulysses Attention" and the variants table
 * (sequence length and head count must be divisible by ulysses_degree).
 * direction 0 (first exchange, sequence-sharded -> head-sharded):
 *   src [P][B][S/P][H][D]  ->  dst [P][B][S][H/P][D]
 *   dst[p][b][s][j][:] = src[s / (S/P)][b][s % (S/P)][p*(H/P) + j][:]
 * direction 1: the exact inverse (second exchange, head-sharded -> sequence-sharded).
 * P = degree >= 1.  elem_bytes: 2 (bf16/fp16) or 4 (fp32).  Bit-exact copy.
 * S % P != 0 or H % P != 0: CP_ERR_NOT_DIVISIBLE.  src and dst may not overlap.
 */
CP_API cp_status cp_ulysses_permute(const void* src, void* dst, int degree, int B, int S, int H, int D,
                             int direction, int elem_bytes, void* stream);

/*
 * cp_ulysses_permute_n - cp_ulysses_permute of n_tensors same-shaped tensors in one
 * launch (the Ulysses exchange moves Q, K and V together).
 *
 * srcs, dsts: HOST arrays of n_tensors device pointers (1 <= n_tensors <= 8), read during
 * the call only.  Other arguments and rules as cp_ulysses_permute; no destination may
 * overlap any source or another destination (CP_ERR_INVALID_ARG).
 */
CP_API cp_status cp_ulysses_permute_n(const void* const* srcs, void* const* dsts, int n_tensors, int degree,
                               int B, int S, int H, int D, int direction, int elem_bytes, void* stream);

/*
 * One process per GPU.  The calls below run the exchanges of "Context parallelism"
 * ("Ring Attention", "Ulysses Attention", "Unified Attention") between real GPUs: peer
 * buffers are plain device allocations shared with CUDA IPC; the Ulysses all-to-alls are
 * pushes by this library's kernels into the other ranks' buffers; a ring rank fetches the
 * other ranks' K/V blocks with the copy engines, so that the transfer overlaps the
 * attention kernel (which holds every SM); a signal-pad barrier with a bounded wait
 * orders the steps.  Process-group plumbing (who is rank q, exchanging the handles) is
 * the caller's.
 */

/*
 * cp_peer_alloc - a device buffer other processes can map.
 *
 * Allocates `bytes` (> 0) on the current device as its own allocation, zero-fills it
 * (synchronously), and writes its CUDA IPC handle, CP_IPC_HANDLE_BYTES bytes, to the
 * HOST buffer `handle`.  *dptr receives the device pointer (256-byte aligned); the caller
 * owns it and releases it with cp_peer_free once every process that opened it has closed
 * it.  Errors: bytes == 0 or a null pointer -> CP_ERR_INVALID_ARG; allocation or export
 * failure -> CP_ERR_CUDA (nothing is left allocated).
 */
CP_API cp_status cp_peer_alloc(size_t bytes, void** dptr, void* handle);

/*
 * cp_peer_open - map another process's cp_peer_alloc buffer into this process.
 *
 * handle: HOST, CP_IPC_HANDLE_BYTES bytes from cp_peer_alloc in another process (CUDA
 * does not open a handle in the process that made it).  Peer access is enabled on first
 * use.  *dptr receives the mapping; release it with cp_peer_close.  Errors: null ->
 * CP_ERR_INVALID_ARG; CUDA refused the handle -> CP_ERR_CUDA.
 */
CP_API cp_status cp_peer_open(const void* handle, void** dptr);

/* cp_peer_close - unmap a cp_peer_open mapping.  cp_peer_free - free a cp_peer_alloc buffer.
 * Both synchronous; null -> CP_ERR_INVALID_ARG; CUDA failure -> CP_ERR_CUDA. */
CP_API cp_status cp_peer_close(void* dptr);
CP_API cp_status cp_peer_free(void* dptr);

/*
 * cp_ulysses_push_n - this rank's half of a Ulysses all-to-all, pushed into peer buffers.
 *
 * Source: "Context parallelism", "Ulysses Attention".  P = degree ranks, Sp = S/P,
 * Hp = H/P; per rank, sequence shard X [B][Sp][H][D] and head shard Y [B][S][Hp][D].
 * direction 0 (first exchange): srcs[t] = this rank's X of tensor t;
 *   dsts[t*P + q] = rank q's Y buffer of tensor t (a cp_peer_open mapping, or local for q
 *   == rank); for every q: Y_q[b][rank*Sp + s][j][:] = X[b][s][q*Hp + j][:].
 * direction 1 (second exchange): srcs[t] = this rank's Y; dsts[t*P + p] = rank p's X;
 *   for every p: X_p[b][s][rank*Hp + j][:] = Y[b][p*Sp + s][j][:].
 * Once every rank has pushed (and a barrier has passed), the buffers hold exactly what
 * cp_ulysses_permute makes from the stacked shards.  A pure copy, bit-exact for any
 * element type of elem_bytes (2 or 4) bytes.  srcs: HOST array of n_tensors pointers
 * (1..8); dsts: HOST array of n_tensors*degree pointers; none overlapping another, all
 * aligned to the element size (the copy uses the widest vector, up to 16 bytes, that
 * divides every pointer and the piece of (H/P)*D elements).
 * 1 <= degree <= CP_PEER_MAX, 0 <= rank < degree.
 * The writes are performed at the other GPUs when the kernel completes; they are visible
 * to a peer's later work once a cp_peer_barrier issued after it on the same stream has
 * passed on both sides.
 * Errors: S or H not divisible -> CP_ERR_NOT_DIVISIBLE; null, overlap, bad rank ->
 * CP_ERR_INVALID_ARG; a pointer not aligned to the element -> CP_ERR_MISALIGNED; too
 * many tensors or ranks ->
 * CP_ERR_UNSUPPORTED.  Asynchronous on `stream`.
 */
CP_API cp_status cp_ulysses_push_n(const void* const* srcs, void* const* dsts, int n_tensors, int rank, int degree,
                                   int B, int S, int H, int D, int direction, int elem_bytes, void* stream);

/*
 * cp_ulysses_anything_push_n - cp_ulysses_push_n for shards of unequal size.
 *
 * Source: "Context parallelism", "Ulysses Anything Attention" (sequence length and head
 * count need not be divisible by ulysses_degree), with the layout of
 * cp_ulysses_anything_permute: sequence shard p holds tokens [seq_bounds[p],
 * seq_bounds[p+1]) and head shard q heads [head_bounds[q], head_bounds[q+1]); either may
 * be empty.  Per rank: X_p [B][S_p][H][D], Y_q [B][S][H_q][D], S = seq_bounds[degree].
 * direction 0: srcs[t] = this rank's X; dsts[t*P + q] = rank q's Y; for every q:
 *   Y_q[b][seq_bounds[rank] + s][j][:] = X[b][s][head_bounds[q] + j][:].
 * direction 1: srcs[t] = this rank's Y; dsts[t*P + p] = rank p's X; for every p:
 *   X_p[b][s][head_bounds[rank] + j][:] = Y[b][seq_bounds[p] + s][j][:].
 * seq_bounds, head_bounds: HOST int[degree+1], non-decreasing from 0 (head_bounds up to
 * H).  Every rank's push together gives exactly cp_ulysses_anything_permute's shards.
 * Other rules (pointers, alignment to the element, overlap, ordering by cp_peer_barrier,
 * errors) as cp_ulysses_push_n; bad bounds -> CP_ERR_INVALID_ARG.
 */
CP_API cp_status cp_ulysses_anything_push_n(const void* const* srcs, void* const* dsts, int n_tensors, int rank,
                                            int degree, const int* seq_bounds, const int* head_bounds, int B, int H,
                                            int D, int direction, int elem_bytes, void* stream);

/*
 * cp_attn_merge_push - LSE merge of this rank's head-shard partials, each merged row
 * stored straight into its owner's sequence shard over peer memory.
 *
 * Source: "Context parallelism", "Unified Attention" (ring attention on the Ulysses head
 * shards, then the second all-to-all) and "Ring Attention" (blocks merged through their
 * LSEs, as cp_attn_merge).  P = degree ranks of a Ulysses group; this rank holds head
 * shard `shard` (heads [shard*H/P, (shard+1)*H/P)) for all S tokens.
 * partials: fp32 [n_chunks][B][S][H/P][D]; lses: fp32 [n_chunks][B][H/P][S].
 * peer_outs: HOST array of P device pointers, peer_outs[p] = rank p's sequence shard
 * [B][S/P][H][D] (a cp_peer_open mapping, or local for p == shard): the merged row of
 * token s, head j goes to peer_outs[s/(S/P)][b][s%(S/P)][shard*H/P + j].  No LSE is
 * written.  The merge arithmetic is cp_attn_merge's, so the rows are bit-identical to it.
 * Ordering as cp_ulysses_push_n (a cp_peer_barrier after it).  Errors: as cp_attn_merge;
 * S or H not divisible -> CP_ERR_NOT_DIVISIBLE; bad shard -> CP_ERR_INVALID_ARG;
 * degree > CP_PEER_MAX -> CP_ERR_UNSUPPORTED.
 */
CP_API cp_status cp_attn_merge_push(const float* partials, const float* lses, int n_chunks, void* const* peer_outs,
                                    int shard, int degree, int B, int S, int H, int D, cp_dtype out_dtype,
                                    void* stream);

/*
 * cp_peer_barrier - all ranks of a group reach the same point of their streams.
 *
 * signal_pads: HOST array of degree pointers; signal_pads[q] = rank q's signal pad (at
 * least degree 32-bit words of a cp_peer_alloc buffer, zero at first use, 4-byte aligned;
 * this rank's own pad at index rank).  A one-warp kernel on `stream` first makes this
 * rank's earlier writes visible system-wide, stores `epoch` into word `rank` of every
 * pad, then waits until every word of its own pad has reached `epoch` (modulo 2^32:
 * epochs start at 1 and grow by one per barrier; every rank passes the same sequence).
 * The wait is bounded by timeout_ms of wall-clock time (the GPU's global timer; 0 means
 * 1000 ms): when it runs out the kernel records CP_ERR_TIMEOUT (read with
 * cp_last_device_status) and returns, the context stays usable, and the group is to be
 * treated as failed; whatever the stream runs after a timed-out barrier works on data
 * that may not have arrived.  Errors: bad rank or null -> CP_ERR_INVALID_ARG; misaligned
 * pad -> CP_ERR_MISALIGNED; degree > CP_PEER_MAX -> CP_ERR_UNSUPPORTED.
 */
CP_API cp_status cp_peer_barrier(void* const* signal_pads, int rank, int degree, unsigned int epoch,
                                 unsigned int timeout_ms, void* stream);

/*
 * cp_ring_fetch_block - copy rows [src_row0, src_row0+rows) of every batch of a
 * [B][src_S][H][D] tensor to rows [dst_row0, ...) of a [B][dst_S][H][D] tensor.
 *
 * Source: "Context parallelism", "Ring Attention" (each rank sees every K/V block) and
 * "Ring Anything Attention" (blocks of unequal length).  src may be another GPU's memory
 * (a cp_peer_open mapping): the copy engines move it, so it overlaps a running kernel.
 * Bit-exact.  elem_bytes 2 or 4.  Errors: rows outside either tensor, overlap, null ->
 * CP_ERR_INVALID_ARG; CUDA failure -> CP_ERR_CUDA.  Asynchronous on `stream`.
 */
CP_API cp_status cp_ring_fetch_block(void* dst, const void* src, int B, int rows, int H, int D, int dst_S,
                                     int dst_row0, int src_S, int src_row0, int elem_bytes, void* stream);

/*
 * cp_ring_bounds - host-only helper: block bounds for a ring of n over S rows.
 *
 * Source: "Context parallelism", variants table: Ring Attention needs S divisible by
 * ring_degree; "Ring Anything Attention" accepts any S.  anything == 0: even split,
 * CP_ERR_NOT_DIVISIBLE if S % n != 0.  anything != 0: the first S % n blocks get
 * ceil(S/n) rows, the rest floor(S/n) (the pages do not say how ring-anything splits;
 * this is the plainest reading).  bounds_out: HOST int[n+1].  No CUDA call.
 */
CP_API cp_status cp_ring_bounds(int S, int n, int anything, int* bounds_out);

/* Wait for `stream`, then return and clear the device status word: CP_OK, or
 * CP_ERR_TIMEOUT if a kernel's bounded wait ran out since the last call.  Returns
 * CP_ERR_CUDA if the stream reported an error. */
CP_API cp_status cp_last_device_status(void* stream);

/*
 * cp_debug_set_fault - test hook for the failure path (host only, no CUDA call).
 *
 * mode 1: the next attention launch (cp_attn_fwd, cp_attn_fwd_blocks, cp_ring_sim*) has its
 * TMA producer skip one K tile.  The consumer's bounded wait then runs out (about one
 * second), every warp leaves its loop, in-flight copies and MMAs are drained, TMEM is
 * freed and the kernel returns; cp_last_device_status() then reports CP_ERR_TIMEOUT and the
 * context stays usable.  The outputs of that launch are undefined.  mode 0 clears the hook.
 * Nothing traps or faults.
 */
CP_API cp_status cp_debug_set_fault(int mode);

/* Static string naming a status code. */
CP_API const char* cp_status_string(cp_status s);

/* Library ABI version (major*100 + minor). */
CP_API int cp_version(void);

#ifdef __cplusplus
}
#endif

#endif /* CPATTN_H */
