/*
 * rm_attn.h -- C ABI of librm_attn.so: the single-GPU (B200, sm_100a) hot path
 * of ring / striped / Ulysses context-parallel attention.
 *
 * Sources of the operations (web pages; section in brackets):
 *  - exact attention softmax(Q K^T / sqrt(d)) V
 *      [Mosaic: Sharding Attention Across GPUs..., "The Problem"]
 *  - computing it one KV chunk at a time and normalising at the end, with the
 *    softmax rescaling trick
 *      [Mosaic, "How Ring Attention Works"; Ring Attention & Friends,
 *       "Flash Attention - Tiling with the Softmax Rescaling Trick"]
 *  - LSE merge of partial results, contiguous / head_tail (zigzag) layouts,
 *    the backward that runs the ring in the opposite direction, the Ulysses
 *    all-to-all on the head dimension
 *      [ringmaster (axolotl-ringmaster 0.2.0), "Why", "Status", "Layout"]
 *  - striped layout (token t on rank t mod P)
 *      [Ring Attention & Friends, "Striped Attention"]
 *
 * Conventions shared by every entry point
 *  - Tokens-major layout [B, N, H, d] ("bshd"): the d axis is contiguous
 *    (stride 1); batch, token and head strides are given in ELEMENTS through
 *    rm_tensor.  LSE / delta vectors are dense fp32 [B, H, N] (N fastest).
 *  - "Rank-major order": a sequence of P*L tokens stored as rank 0's L local
 *    tokens, then rank 1's, ...  Local token j of rank r sits at global
 *    position pos(r, j):
 *        contiguous  pos = r*L + j
 *        zigzag      C = N/(2P); j < C: r*C + j;  else (2P-1-r)*C + (j-C)
 *        striped     pos = j*P + r
 *  - Causal masking: key u is visible to query t iff pos(u) <= pos(t).
 *  - Grouped-query attention: query head h reads KV head h / (Hq/Hkv).
 *  - scale <= 0 selects 1/sqrt(d) with d the true head dimension.
 *  - LSE is the natural log of the softmax normaliser; a row with no visible
 *    key has O = 0 and LSE = -inf.
 *  - Ownership: the caller owns every buffer, the workspace included; the
 *    library never allocates device memory and keeps no per-call state.
 *  - Asynchrony: every call only enqueues work on `stream` (a cudaStream_t,
 *    NULL = legacy default stream).  Argument errors are detected on the host
 *    before anything is launched and return RM_ERR_INVALID_ARG /
 *    RM_ERR_UNSUPPORTED / RM_ERR_WORKSPACE; launch failures return
 *    RM_ERR_CUDA.  Device-side bounded waits that expire record
 *    RM_ERR_TIMEOUT in a device status word read by rm_get_device_status.
 *    rm_last_error() gives a thread-local one-line reason for the last
 *    non-OK status.
 *  - Alignment: device pointers 16-byte aligned; every stride times the
 *    element size a multiple of 16 bytes (bf16 attention calls); other calls
 *    state their own rule.
 *  - Aliasing: outputs never alias inputs, except where an entry point says so.
 */
#ifndef RM_ATTN_H
#define RM_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Everything declared here is exported from librm_attn.so; the library is
 * built with hidden visibility otherwise. */
#if defined(__GNUC__)
#pragma GCC visibility push(default)
#endif

typedef enum {
  RM_OK = 0,
  RM_ERR_INVALID_ARG = 1,  /* bad pointer / shape / stride / enum            */
  RM_ERR_UNSUPPORTED = 2,  /* valid request this build does not implement    */
  RM_ERR_WORKSPACE = 3,    /* workspace missing or smaller than required     */
  RM_ERR_CUDA = 4,         /* a CUDA runtime / driver call failed            */
  RM_ERR_TIMEOUT = 5       /* a device-side bounded wait expired             */
} rm_status;

typedef enum { RM_F32 = 0, RM_BF16 = 1 } rm_dtype;

typedef enum {
  RM_LAYOUT_CONTIGUOUS = 0,
  RM_LAYOUT_ZIGZAG = 1,
  RM_LAYOUT_STRIPED = 2
} rm_layout;

/* Forward ring execution mode. */
typedef enum {
  RM_RING_FUSED = 0,    /* one persistent launch; running softmax state carried
                           across KV shards (the merge happens in registers) */
  RM_RING_STEPWISE = 1  /* per ring step one block launch per rank writing fp32
                           partials to the workspace, then rm_lse_merge */
} rm_ring_mode;

/* A strided [B, N, H, d] view; strides in elements, d stride is 1. */
typedef struct {
  void* ptr;
  int64_t stride_b;
  int64_t stride_n;
  int64_t stride_h;
} rm_tensor;

/* Token order of the ring entry points' operands.  RANK_MAJOR: rank 0's L
 * tokens, then rank 1's ... (what rm_layout_permute produces).  GLOBAL: the
 * tokens' own order; the kernels fetch every tile of a virtual rank straight
 * from it through the layout map (no permute pass).  GLOBAL needs bf16, the
 * fused mode, and for zigzag chunks of a multiple of 128 tokens
 * (N % (256 P) == 0); otherwise RM_ERR_UNSUPPORTED. */
typedef enum { RM_ORDER_RANK_MAJOR = 0, RM_ORDER_GLOBAL = 1 } rm_order;

/* One attention problem: B sequences of N tokens split over P virtual ranks
 * (L = N / P tokens each) laid out by `layout`; N < 2^31 (token positions
 * are 32-bit on the device).  d is the true head dimension.  bf16 supports
 * d in {24, 32, 64, 128} (24 is zero-padded to 32 on chip); fp32 supports
 * d % 4 == 0, d <= 128. */
typedef struct {
  rm_dtype dtype;
  int B;
  int Hq;
  int Hkv;
  int d;
  int64_t N;
  int P;
  rm_layout layout;
  int causal;
  float scale;        /* <= 0: 1/sqrt(d) */
  rm_ring_mode mode;  /* rm_ring_attn_fwd only */
  rm_order order;     /* rm_ring_attn_fwd / _bwd only: token order of every
                         [B, N, H, d] operand and of lse / delta */
  /* Packed or right-padded batches [ringmaster, "Status": dense causal
   * sequences or globally right-padded batches; packing by global position
   * boundaries].  A key is visible only inside its query's segment (and not
   * after it when causal); padding tokens see nothing and are seen by
   * nothing (their O is 0, their LSE -inf, their gradients 0).  At most one:
   *   cu_seqlens: device int32[num_segments + 1], global positions
   *               0 = cu[0] < cu[1] < ... < cu[num_segments] <= N; positions
   *               from cu[num_segments] on are padding; needs B == 1;
   *   seq_lens:   device int32[B], valid tokens of each batch entry (right
   *               padding).
   * NULL / 0: dense.  Taken by every entry point with a descriptor (block,
   * ring, USP, Mesh2D), bf16 and fp32; sequences of at most 16 tokens with
   * segments run on the general kernels instead of the short-sequence ones.
   * USP applies the caller's description to every head group (packing still
   * needs the caller's B == 1).  The values are read on the device:
   * malformed boundaries give wrong results but no out-of-range access. */
  const int32_t* cu_seqlens;
  int num_segments;
  const int32_t* seq_lens;
} rm_attn_desc;

/* ---- block level: one Q shard against one KV shard ---------------------- */

/* Attention of rank q_rank's query shard against rank kv_rank's KV shard
 * [Mosaic, "How Ring Attention Works": one step's partial result].
 *   q  [B, L, Hq, d] (desc->dtype), the L tokens of q_rank in local order
 *   k, v [B, L, Hkv, d], the L tokens of kv_rank in local order
 *   o  [B, L, Hq, d] written: fp32 if o_f32 != 0, else desc->dtype
 *   lse dense fp32 [B, Hq, L] written
 * Keys with pos > pos(query) are masked when desc->causal.  A shard pair with
 * no visible key writes O = 0, LSE = -inf.  L may have a ragged tail (any
 * L >= 1).  desc->mode is ignored. */
rm_status rm_attn_block_fwd(const rm_attn_desc* desc, int q_rank, int kv_rank,
                            rm_tensor q, rm_tensor k, rm_tensor v,
                            rm_tensor o, int o_f32, float* lse, void* stream);

/* Backward contribution of one (q_rank, kv_rank) pair [ringmaster, "Status":
 * the ring's backward; formulas are the derivative of the definition]:
 *   P_tu = exp(s_tu - lse_final_t);  dP = dO V^T;  dS = P o (dP - delta)
 *   dq_acc += scale dS K;  dk_acc += scale dS^T Q;  dv_acc += P^T dO
 * lse_final / delta: dense fp32 [B, Hq, L] of the query shard (the FINAL LSE
 * of the whole ring, and delta_t = dO_t . O_t of the final O).
 * dq_acc [B, L, Hq, d], dk_acc / dv_acc [B, L, Hkv, d]: fp32 accumulators,
 * read-modify-written (+=).  dK/dV of a KV head sum over its query heads. */
rm_status rm_attn_block_bwd(const rm_attn_desc* desc, int q_rank, int kv_rank,
                            rm_tensor q, rm_tensor k, rm_tensor v, rm_tensor dout,
                            const float* lse_final, const float* delta,
                            rm_tensor dq_acc, rm_tensor dk_acc, rm_tensor dv_acc,
                            void* stream);

/* delta[b, h, t] = sum_c dout[b, t, h, c] * o[b, t, h, c] (fp32 accumulate),
 * the row term of the softmax derivative computed from the FINAL output.
 * o / dout in `dtype`, [B, N, H, d], d % 4 == 0, pointers aligned to 4
 * elements and strides multiples of 4 elements; delta dense fp32 [B, H, N]. */
rm_status rm_attn_bwd_preprocess(rm_dtype dtype, int B, int64_t N, int H, int d,
                                 rm_tensor o, rm_tensor dout, float* delta,
                                 void* stream);

/* Backward finalize [ringmaster, "Status": the ring backward, whose dK / dV
 * travel round the ring with their KV shard and come back to its owner]:
 * fp32 [B, N, H, d] -> out_dtype [B, N, H, d] (bf16: round to nearest even;
 * fp32: a copy), both strided as rm_tensor (d contiguous), for a backward that
 * accumulated its gradients in fp32 (the block API's accumulators; the
 * multi-rank ring, whose dK / dV accumulators cross ranks in fp32).
 * The caller owns both buffers; in and out must not overlap.
 * Errors: RM_ERR_INVALID_ARG for another out_dtype, B < 0, N < 0, H < 1,
 * d < 4 or d % 4 != 0, a NULL pointer, or pointers / strides not aligned to
 * 4 elements (16 bytes of fp32 input; 8 bytes of bf16 output).  B * N == 0
 * launches nothing. */
rm_status rm_convert_f32(rm_dtype out_dtype, int B, int64_t N, int H, int d, rm_tensor in,
                         rm_tensor out, void* stream);

/* ---- LSE merge ---------------------------------------------------------- */

/* Merge n_parts partial results [ringmaster, "Layout": ring/merge.py, the
 * online-softmax LSE merge; formula is the exact identity of the LSE]:
 *   m = max_i lse_i;  LSE = m + ln sum_i exp(lse_i - m);
 *   O = sum_i exp(lse_i - LSE) O_i
 * Parts with lse = -inf get weight 0; if all are -inf, O = 0, LSE = -inf.
 *   o_parts[i]  fp32 [B, Nq, H, d] (strided)     lse_parts[i] fp32 [B, H, Nq]
 *   o_out       out_dtype [B, Nq, H, d]          lse_out      fp32 [B, H, Nq]
 * 1 <= n_parts <= 16; d % 4 == 0, d <= 128; o_parts 16-byte aligned with
 * strides that are multiples of 4 elements; o_out aligned to 4 elements with
 * strides that are multiples of 4 elements.
 * o_out may alias o_parts[0] exactly (in-place merge) when out_dtype is fp32;
 * lse_out may alias lse_parts[0]. */
rm_status rm_lse_merge(rm_dtype out_dtype, int B, int H, int64_t Nq, int d,
                       int n_parts, const rm_tensor* o_parts,
                       const float* const* lse_parts, rm_tensor o_out,
                       float* lse_out, void* stream);

/* ---- ring driver over P virtual ranks ----------------------------------- */

/* Workspace bytes rm_ring_attn_fwd (backward = 0) or rm_ring_attn_bwd
 * (backward = 1) needs for *desc; 0 is a valid answer. */
rm_status rm_ring_workspace_size(const rm_attn_desc* desc, int backward,
                                 size_t* bytes);

/* Ring forward [Mosaic, "How Ring Attention Works"]: for every rank r and
 * step k = 0..P-1, rank r attends to KV shard (r - k) mod P; the partials are
 * merged by the LSE merge.  q [B, N, Hq, d], k/v [B, N, Hkv, d] in rank-major
 * order; o [B, N, Hq, d] (desc->dtype) and lse fp32 [B, Hq, N] in rank-major
 * order.  Shard pairs (and tiles) that the causal mask empties are skipped.
 * ws: 256-byte aligned device buffer of rm_ring_workspace_size(desc, 0). */
rm_status rm_ring_attn_fwd(const rm_attn_desc* desc, rm_tensor q, rm_tensor k,
                           rm_tensor v, rm_tensor o, float* lse, void* ws,
                           size_t ws_bytes, void* stream);

/* Ring backward: delta from the final (o, dout), then every (query shard,
 * KV shard) pair's contribution accumulated in fp32, KV shards visiting the
 * ranks in reverse ring order; dq/dk/dv written in desc->dtype, in
 * desc->order.  o, lse: the outputs of rm_ring_attn_fwd.
 * ws: rm_ring_workspace_size(desc, 1) bytes, 256-byte aligned (delta; for
 * bf16 at head dims other than 128, which run on the CUDA-core kernels, also
 * fp32 dq/dk/dv that are then rounded to bf16).  Global token order in the
 * backward needs d = 128 (RM_ERR_UNSUPPORTED otherwise). */
rm_status rm_ring_attn_bwd(const rm_attn_desc* desc, rm_tensor q, rm_tensor k,
                           rm_tensor v, rm_tensor o, const float* lse,
                           rm_tensor dout, rm_tensor dq, rm_tensor dk,
                           rm_tensor dv, void* ws, size_t ws_bytes, void* stream);

/* Ring backward that allocates nothing.  The pages have no counterpart: this
 * is for callers that cannot allocate device memory -- e.g. a runtime that
 * reserved all of it for its own pool, or code that must not call cudaMalloc
 * because that would synchronise the device.  Same arguments and results as
 * rm_ring_attn_bwd, minus the workspace: the scratch comes from a fixed
 * 64 MiB device array inside the library, so rm_ring_workspace_size(desc, 1)
 * must be at most 64 MiB (else RM_ERR_WORKSPACE, nothing launched).
 * When the 64 MiB is reserved depends on how CUDA loads modules: with lazy
 * loading (CUDA_MODULE_LOADING=LAZY, the default of recent runtimes) the
 * first call in a context loads the library's device code and reserves it
 * then; with eager loading every context that loads the library reserves it
 * at once, whether or not it ever calls this function.  Either way it stays
 * reserved until the context ends.  So make the first call in each context
 * before any stream capture and before the caller hands the rest of device
 * memory to its own pool: under lazy loading that first call may otherwise
 * fail with RM_ERR_CUDA for lack of memory.  The array's device address is
 * looked up on every call in the current context, so a device reset or a
 * context switch between calls is safe.  All calls share the one array per
 * context: calls whose kernels overlap on the GPU (several streams, or
 * several threads) race and give wrong results -- serialise them.  Each call
 * writes the scratch it reads before reading it, so the previous call's
 * contents do not reach its results.
 * Calls no cudaMalloc / cudaFree / allocating library routine. */
rm_status rm_ring_attn_bwd_noalloc(const rm_attn_desc* desc, rm_tensor q, rm_tensor k,
                                   rm_tensor v, rm_tensor o, const float* lse,
                                   rm_tensor dout, rm_tensor dq, rm_tensor dk,
                                   rm_tensor dv, void* stream);

/* ---- USP: the Ulysses head all-to-all composed with the ring ------------- */

/* The split of `world` virtual devices into ulysses x ring [ringmaster,
 * "Why": USP on a 2-D mesh, with an auto-selector driven by the KV-head count
 * and the world size]: the largest Ulysses degree that divides `world` and
 * Hkv (the Ulysses cap) and is at most `node_size`; ring = world / ulysses.
 * Host only.  RM_ERR_INVALID_ARG for non-positive sizes or Hq % Hkv != 0. */
rm_status rm_usp_auto_select(int Hq, int Hkv, int world, int node_size, int* ulysses,
                             int* ring);

/* Workspace bytes of rm_usp_attn_fwd (backward = 0) or rm_usp_attn_bwd (1). */
rm_status rm_usp_workspace_size(const rm_attn_desc* desc, int ulysses, int backward,
                                size_t* bytes);

/* USP forward on one GPU: desc->P is the ring degree (the layout's rank
 * count) and `ulysses` the Ulysses degree, so P * ulysses virtual devices.
 * Each ring shard is cut into `ulysses` contiguous sub-shards; inside every
 * ring group the seq->head repack (rm_seq_head_repack) gives each Ulysses rank
 * the whole ring shard for Hq/ulysses query heads (and Hkv/ulysses KV heads);
 * the ring (rm_ring_attn_fwd, desc->mode / order) then runs for every head
 * group over the P ring ranks, and the head->seq repack returns O.
 * q/o [B, N, Hq, d], k/v [B, N, Hkv, d]: DENSE tensors in desc->order for the
 * P ring ranks; lse fp32 [B, Hq, N].  Needs Hq % ulysses == Hkv % ulysses ==
 * (N/P) % ulysses == 0.  ws: rm_usp_workspace_size(desc, ulysses, 0) bytes,
 * 256-byte aligned (the repacked operands and the ring's own workspace). */
rm_status rm_usp_attn_fwd(const rm_attn_desc* desc, int ulysses, rm_tensor q, rm_tensor k,
                          rm_tensor v, rm_tensor o, float* lse, void* ws, size_t ws_bytes,
                          void* stream);

/* USP backward: repack q, k, v, o, dout; rm_ring_attn_bwd per head group;
 * repack dq, dk, dv back.  Same layouts and requirements as the forward;
 * ws: rm_usp_workspace_size(desc, ulysses, 1) bytes. */
rm_status rm_usp_attn_bwd(const rm_attn_desc* desc, int ulysses, rm_tensor q, rm_tensor k,
                          rm_tensor v, rm_tensor o, const float* lse, rm_tensor dout,
                          rm_tensor dq, rm_tensor dk, rm_tensor dv, void* ws, size_t ws_bytes,
                          void* stream);

/* ---- Mesh2D ---------------------------------------------------------------
 * [Mosaic, "Beyond 1D: Mesh2D Attention": both Q and K are sharded; on a
 * grid of devices, device (i, j) computes the tile of QK^T between query
 * chunk i and key chunk j.]  Here the grid_q x grid_k tiles run in turn on
 * one GPU.  Query chunk i = global positions [i*N/grid_q, (i+1)*N/grid_q),
 * key / value chunk j = [j*N/grid_k, (j+1)*N/grid_k) (contiguous; the grid
 * may be rectangular).  Tile (i, j) is the block forward of that pair
 * (rm_attn_block_fwd with its own chunk lengths): an fp32 partial O and its
 * LSE.  The forward merges the partials of each query chunk with the LSE
 * merge (rm_lse_merge); the backward adds every tile's contributions, from
 * the final LSE and D = rowsum(dO o O), into dQ of chunk i and dK / dV of
 * chunk j (fp32 accumulators, then the output dtype, RNE for bf16).  Tiles
 * without a visible pair under the causal rule are skipped.
 *
 * desc: dtype, B, Hq, Hkv, d, N, causal, scale as for the ring; P, layout,
 * mode and order are ignored (operands in global token order); segments
 * (cu_seqlens / seq_lens) apply by global position.  grid_q, grid_k >= 1
 * must divide N; grid_k <= 16
 * (RM_ERR_UNSUPPORTED above).
 * q/o/dout/dq [B, N, Hq, d], k/v/dk/dv [B, N, Hkv, d] strided as rm_tensor;
 * lse fp32 [B, Hq, N].  Workspace (caller-owned, 256-byte aligned):
 * forward grid_k fp32 partial O [B, N, Hq, d] and LSE [B, Hq, N] slots;
 * backward delta [B, Hq, N] and fp32 dQ / dK / dV accumulators. */
rm_status rm_mesh2d_workspace_size(const rm_attn_desc* desc, int grid_q, int grid_k,
                                   int backward, size_t* bytes);
rm_status rm_mesh2d_attn_fwd(const rm_attn_desc* desc, int grid_q, int grid_k, rm_tensor q,
                             rm_tensor k, rm_tensor v, rm_tensor o, float* lse, void* ws,
                             size_t ws_bytes, void* stream);
rm_status rm_mesh2d_attn_bwd(const rm_attn_desc* desc, int grid_q, int grid_k, rm_tensor q,
                             rm_tensor k, rm_tensor v, rm_tensor o, const float* lse,
                             rm_tensor dout, rm_tensor dq, rm_tensor dk, rm_tensor dv, void* ws,
                             size_t ws_bytes, void* stream);

/* ---- bit-exact layout transforms ---------------------------------------- */

/* Global token order <-> rank-major order (see pos(r, j) above) of a dense
 * [B, N, H, d] tensor of `dtype`.  inverse = 0: out[b, r*L + j] = in[b, pos];
 * inverse = 1: out[b, pos] = in[b, r*L + j].  Bit copy.  N % P == 0 (and
 * N % 2P == 0 for zigzag).  in and out must not overlap. */
rm_status rm_layout_permute(rm_dtype dtype, int B, int64_t N, int H, int d,
                            rm_layout layout, int P, int inverse,
                            const void* in, void* out, void* stream);

/* Ulysses sequence <-> head repack as a local pack [ringmaster, "Why": the
 * all-to-all on the head dimension; P may not exceed the head count].
 * head_to_seq = 0 (seq -> head):
 *   in  [P][N_local][H][d]      (rank s's sequence shard of all heads)
 *   out [P][P*N_local][H/P][d]  out[r][s*N_local + t][h] = in[s][t][r*H/P + h]
 * head_to_seq = 1 is the inverse (in and out swap roles).  Bit copy; dense
 * tensors; H % P == 0.  in and out must not overlap. */
rm_status rm_seq_head_repack(rm_dtype dtype, int P, int64_t N_local, int H,
                             int d, int head_to_seq, const void* in, void* out,
                             void* stream);

/* ---- status ------------------------------------------------------------- */

/* Synchronises `stream`, then returns and clears the device status word of
 * the current device: RM_ERR_TIMEOUT if a bounded wait expired in any kernel
 * since the last call, RM_ERR_CUDA if the synchronisation failed or a kernel
 * found its shared memory misaligned (it then skipped its work), else RM_OK. */
rm_status rm_get_device_status(void* stream);

const char* rm_status_string(rm_status s);
const char* rm_last_error(void);

/* Test hook for the bounded-wait machinery: launches one CTA that waits on an
 * mbarrier nothing arrives at, giving up after `spin_limit` polls, and records
 * RM_ERR_TIMEOUT in the device status word.  Faults and hangs nothing. */
rm_status rm_debug_expire_wait(uint32_t spin_limit, void* stream);

/* Test hook for the polynomial exponential that the tensor-core forward uses
 * on the FMA pipe for part of its softmax at head dims up to 64 (the pages fix
 * no way of computing exp; this is an implementation choice of the kernel):
 * y[i] = that function's 2^x[i] for i < n.  x, y: device fp32 arrays of n
 * elements (caller-owned; they must not overlap).  Stated accuracy: relative
 * error at most 7.5e-5 for x in [-125, 127]; inputs below -125 (and -inf)
 * are clamped to -125.  RM_ERR_INVALID_ARG for n < 0 or null pointers. */
rm_status rm_debug_exp2_poly(const float* x, float* y, int64_t n, void* stream);

/* ---- launch timing ------------------------------------------------------ */

/* Opt-in per-kernel timing.  rm_profile_enable(1) clears earlier records and
 * starts bracketing every kernel launch of the library with two CUDA events
 * recorded on the launching stream; rm_profile_enable(0) stops (and also
 * clears).  rm_profile_count gives the number of launches recorded;
 * rm_profile_get(i, &name, &ms) waits for launch i to finish and returns the
 * kernel's name (static string) and its device time in milliseconds.  The
 * library owns the events; records are process-wide. */
rm_status rm_profile_enable(int on);
int rm_profile_count(void);
rm_status rm_profile_get(int i, const char** name, float* ms);

#if defined(__GNUC__)
#pragma GCC visibility pop
#endif

#ifdef __cplusplus
}
#endif

#endif /* RM_ATTN_H */
