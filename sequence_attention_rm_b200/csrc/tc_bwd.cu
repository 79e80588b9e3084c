// Backward attention on the sm_100a tensor cores (bf16 in, fp32 accumulate),
// head dim 128, as two kernels that need no reductions in global memory:
//
//  tc_bwd_dkdv_kernel (key-stationary).  One CTA owns one 128-key tile of one
//    KV head and keeps its dK and dV in TMEM while it walks, for every query
//    head of the GQA group and every rank in reverse-ring order (s, s+1, ...;
//    ringmaster, "Status": the backward runs the ring in the opposite
//    direction), the 128-query tiles that can see its keys:
//      S^T = K Q^T, dP^T = V dO^T             (TMEM, keys on lanes)
//      P^T = exp(S^T * scale - LSE),  dS^T = P^T o (dP^T - D)
//      dV += P^T dO,  dK += dS^T Q            (A = P^T, dS^T from TMEM)
//  tc_bwd_dq_kernel (query-stationary).  One CTA owns one 128-row query tile
//    of one head and walks the 128-key tiles it sees in ring order:
//      S = Q K^T, dP = dO V^T                 (TMEM, queries on lanes)
//      dS = exp(S * scale - LSE) o (dP - D)   (written over S as bf16)
//      dQ += dS K     (A = dS from TMEM)
//    and writes dQ once.
// S and dP are recomputed by both kernels (7 MMAs per pair instead of 5); in
// exchange dQ is never reduced through L2, whose fp32 reduce-add throughput
// (about 1.2 TB/s) bound the fused design, and the result is deterministic.
// Every contraction is M=128, N=128: a tcgen05.mma costs its issuing thread
// about 50 cycles, so the N=64 form (32 cycles of work) would leave the
// tensor pipe a third idle.
#include <cudaTypedefs.h>
#include <stdlib.h>

#include "tc_attn.h"
#include "tc_common.cuh"

namespace rm {

rm_status encode_operand_map(CUtensorMap* map, const rm_tensor& t, int B, int shards, int64_t L,
                             int H, int d, int box_cols, int box_rows, int view);
int operand_view(const AttnArgs& a, bool ring);
long long tc_wait_limit();

namespace {

using namespace tc;

constexpr int D = 128;  // head dim

struct BwdParams {
  int B, Hq, Hkv, P, layout, causal;
  int64_t N, L;
  int Pk;      // KV shards: P, except for one (query chunk, KV chunk) tile of a rectangular grid
  int64_t Lk;  // N / Pk
  float scale;       // softmax scale
  float scale_log2;  // scale * log2(e)
  int ring, q_rank, kv_rank;
  const float* lse;  // natural-log LSE
  const float* delta;
  int64_t lse_ld;
  void* dq;          // bf16 output (ring) or fp32 accumulator (block)
  int64_t dq_sb, dq_sn, dq_sh;
  void* dk;
  int64_t dk_sb, dk_sn, dk_sh;
  void* dv;
  int64_t dv_sb, dv_sn, dv_sh;
  int accumulate;
  int head_block;    // heads per grid block (see grid_place)
  int global_order;  // ring operands, outputs, LSE and D in global token order
  const int* cu_seqlens;  // packing boundaries (device) or null
  int num_segments;
  const int* seq_lens;    // right-padding lengths (device) or null
  int seg_div;            // batch entries per seq_lens entry
  unsigned int* status;
  long long wait_limit;
};

// Row addressing of a backward call: ring calls go through RingRows (rank-
// major or global order); a single shard has memory row = local row and TMA
// coordinates (row, 0).
struct BwdRows {
  RingRows rows;
  int ring;
  __device__ __forceinline__ void tma(int rank, int64_t j, int& crow, int& cshard) const {
    if (ring) {
      rows.tma(rank, j, crow, cshard);
    } else {
      crow = (int)j;
      cshard = 0;
    }
  }
  __device__ __forceinline__ int64_t row(int rank, int64_t j) const {
    return ring ? rows.row(rank, j) : j;
  }
};
__device__ __forceinline__ BwdRows bwd_rows(const BwdParams& p) {
  BwdRows r;
  r.rows.lay = make_layout(p.layout, p.N, p.P);
  r.rows.global = p.global_order;
  r.ring = p.ring;
  return r;
}

// K-major SW128 operand with rows of 128 B, 64-column boxes box_bytes apart:
// base descriptor, and the byte offset of K-step k (16 elements).
__device__ __forceinline__ uint64_t kdesc0(uint32_t base) {
  return smem_desc(base, 16, 1024, kSwizzle128B);
}
__device__ __forceinline__ uint32_t koff(int k, uint32_t box_bytes) {
  return (k * 16 / 64) * box_bytes + (k * 16 % 64) * 2;
}
// MN-major SW128 operand: rows of 128 B along the contiguous (M or N) axis, the
// K axis along rows; K-step k starts 16 rows later; 64-element blocks of the
// contiguous axis are box_bytes apart.
__device__ __forceinline__ uint64_t mndesc0(uint32_t base, uint32_t box_bytes) {
  return smem_desc(base, box_bytes, 1024, kSwizzle128B);
}
__device__ __forceinline__ uint32_t mnoff(int k) { return k * 16 * 128; }

// Writes 32 columns (acc * f) of one dK / dV / dQ row: bf16 output, or an fp32
// accumulator read-modify-written.
__device__ __forceinline__ void store_row(void* base, int accumulate, int c32,
                                          const uint32_t (&v)[32], float f, bool zero) {
  if (accumulate) {
    float* dst = reinterpret_cast<float*>(base) + c32 * 32;
#pragma unroll
    for (int x = 0; x < 32; ++x) dst[x] += zero ? 0.f : __uint_as_float(v[x]) * f;
  } else {
    uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(base) + c32 * 32);
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      float y[8];
#pragma unroll
      for (int z = 0; z < 8; ++z) y[z] = zero ? 0.f : __uint_as_float(v[8 * x + z]) * f;
      dst[x] = make_uint4(pack_bf16(y[0], y[1]), pack_bf16(y[2], y[3]), pack_bf16(y[4], y[5]),
                          pack_bf16(y[6], y[7]));
    }
  }
}

// ===========================================================================
// dK / dV (key-stationary)
// ===========================================================================
namespace kv {

constexpr int BK = 128;     // keys per CTA (TMEM lanes)
constexpr int BQ = 128;     // queries per tile (the N of S^T, dP^T)
constexpr int kHalf = BQ / 2;  // query columns per math warpgroup
constexpr int kQStages = 3;   // Q is read by S^T(i) and dK(i): the longer-lived operand
constexpr int kDOStages = 2;  // dO by dP^T(i) and dV(i)
constexpr int kThreads = 384;
// Warp w runs on SM sub-partition w % 4, so the math warps 0-7 put two warps
// on each; the TMA and MMA warps go to sub-partitions 3 and 2.  With them on
// 0 and 1 (warps 8 and 9), clock64 traces showed the two math warps beside
// the MMA warp finishing each tile ~900 cycles after the others, which then
// waited for them at the per-tile LSE / D staging barrier; warps 11 and 10
// measured 4.4% less kernel time (interleaved A/B on the 16k step).
constexpr int kWarpTma = 11;
constexpr int kWarpMma = 10;
constexpr int kRegsMath = 200;
constexpr int kRegsOther = 104;
static_assert(2 * 128 * kRegsMath + 128 * kRegsOther <= kThreads * 168, "register split");

constexpr int kKBox = BK * 128;             // 128 key rows x 128 B (64 cols)
constexpr int kKTile = 2 * kKBox;
constexpr int kQBox = BQ * 128;             // 128 query rows x 128 B
constexpr int kQTile = 2 * kQBox;
constexpr int kOffK = 0;
constexpr int kOffV = kOffK + kKTile;
constexpr int kOffQ = kOffV + kKTile;              // [kQStages]
constexpr int kOffDO = kOffQ + kQStages * kQTile;  // [kDOStages]
constexpr int kOffVec = kOffDO + kDOStages * kQTile; // [wg][2][lse2 | D][64] fp32
constexpr int kOffBar = kOffVec + 2 * 2 * 2 * kHalf * 4;
constexpr int kSmem = kOffBar + 256;  // the base must be 1024-aligned (checked)
static_assert(kSmem <= 232448, "shared memory");

// TMEM columns: dK, dV accumulators; S^T, released as soon as the math
// warpgroups have read it; dP^T, over which each warpgroup writes, in its own
// 64-column half, P^T (bf16, first 32 columns) and dS^T (bf16, last 32).
constexpr uint32_t kTdK = 0, kTdV = 128, kTS = 256, kTdP = 384;

// mbarrier slots (8 bytes each) in the 256-byte barrier area
constexpr int kBarKV = 0;
constexpr int kBarQFull = kBarKV + 1;
constexpr int kBarQEmpty = kBarQFull + kQStages;
constexpr int kBarDOFull = kBarQEmpty + kQStages;
constexpr int kBarDOEmpty = kBarDOFull + kDOStages;
constexpr int kBarS = kBarDOEmpty + kDOStages;
constexpr int kBarSFree = kBarS + 1;
constexpr int kBarDP = kBarSFree + 1;
constexpr int kBarP = kBarDP + 1;
constexpr int kBarDS = kBarP + 1;
constexpr int kBarVec = kBarDS + 1;
constexpr int kBarDone = kBarVec + 4;
constexpr int kBarTmem = kBarDone + 1;
static_assert((kBarTmem + 1) * 8 <= 256, "barrier area");

// TMEM column (from kTdP) of the bf16 A operand P^T / dS^T for K-step k (16
// queries): warpgroup k / 4 packed its 64 queries into 32 columns of its half.
__device__ __forceinline__ uint32_t p_col(int k) { return kHalf * (k >> 2) + 8 * (k & 3); }
__device__ __forceinline__ uint32_t ds_col(int k) { return p_col(k) + 32; }

// The CTA's walk: for every query head of the group, every rank in
// reverse-ring order, the query tiles that can see a key of the CTA: the
// queries at global positions [span_first, span_last].
struct Walk {
  LayoutMap lay;
  int s, g, group, nranks, qtiles, ring, q_rank, P, causal;
  int64_t span_first, span_last;
  __device__ __forceinline__ int rank_of(int step) const {
    return ring ? (s + step) % P : q_rank;
  }
  // query tiles [first_tile(r), end_tile(r)) of rank r
  __device__ __forceinline__ int first_tile(int r) const {
    return (int)(lay.visible_count(r, span_first - 1) / BQ);
  }
  __device__ __forceinline__ int end_tile(int r) const {
    return (int)((lay.visible_count(r, span_last) + BQ - 1) / BQ);
  }
  __device__ __forceinline__ int count() const {
    int n = 0;
    for (int step = 0; step < nranks; ++step) {
      const int r = rank_of(step);
      n += max(0, end_tile(r) - first_tile(r));
    }
    return n * group;
  }
  // A position in the walk, advanced one tile at a time (no rescans); end is
  // end_tile(r) of the current rank, computed when the rank changes.
  struct Cursor {
    int hh, step, r, t, end;
  };
  __device__ __forceinline__ void settle(Cursor& c) const {
    while (c.t >= c.end && c.hh < group) {
      if (++c.step == nranks) {
        c.step = 0;
        ++c.hh;
      }
      c.r = rank_of(c.step);
      c.t = first_tile(c.r);
      c.end = end_tile(c.r);
    }
  }
  __device__ __forceinline__ Cursor begin() const {
    Cursor c;
    c.hh = 0;
    c.step = 0;
    c.r = rank_of(0);
    c.t = first_tile(c.r);
    c.end = end_tile(c.r);
    settle(c);
    return c;
  }
  __device__ __forceinline__ void next(Cursor& c) const {
    ++c.t;
    settle(c);
  }
  __device__ __forceinline__ int head(const Cursor& c) const { return g * group + c.hh; }
};

// Warp roles (384 threads): warps 0-3 and 4-7 are two math warpgroups that
// split every 128-query tile by columns (queries 0-63 / 64-127) over all 128
// key lanes, then write dK (warps 0-3) and dV (warps 4-7); warp kWarpTma (11) TMA producer
// (K, V once; Q into a 3-stage ring, dO into a 2-stage ring); warp kWarpMma (10) MMA
// issuer.  All four contractions are M=128, N=128: S^T, dP^T from shared
// memory; dV and dK take P^T and dS^T from TMEM, so only Q and dO are read
// from shared memory for them.  The warpgroups copy S^T(i) into registers and
// release its columns at once, so the tensor pipe runs, per tile i,
//   dV(i) [needs P^T(i)], dK(i) [needs dS^T(i)], dP^T(i+1), S^T(i+2)
// and the exponentials of tile i+1 overlap all four; the in-order pipe makes
// the single dP^T buffer safe (dP^T(i+1) is issued after dK(i) read dS^T(i)).
// kChunkedKeys: the KV side is one contiguous chunk of a rectangular grid (Pk != P).
template <bool kChunkedKeys>
__global__ void __launch_bounds__(kThreads, 1)
    tc_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                       const BwdParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  if (smem_u32(smem) & 1023u) {  // SW128 tiles need a 1024-byte aligned base
    if (threadIdx.x == 0) report_status(p.status, kStatusSmemAlign);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* bar_kv = bars + kBarKV;
  uint64_t* bar_q_full = bars + kBarQFull;    // [kQStages]
  uint64_t* bar_q_empty = bars + kBarQEmpty;  // [kQStages]
  uint64_t* bar_do_full = bars + kBarDOFull;    // [kDOStages]
  uint64_t* bar_do_empty = bars + kBarDOEmpty;  // [kDOStages]
  uint64_t* bar_s_full = bars + kBarS;        // S^T of the tile in TMEM
  uint64_t* bar_s_free = bars + kBarSFree;    // S^T read by the warpgroups (256 arrivals)
  uint64_t* bar_dp_full = bars + kBarDP;      // dP^T of the tile in TMEM
  uint64_t* bar_p_full = bars + kBarP;        // P^T written (256 arrivals)
  uint64_t* bar_ds_full = bars + kBarDS;      // dS^T written (256 arrivals)
  uint64_t* bar_vec = bars + kBarVec;         // [wg][2] LSE / D staged (128 arrivals)
  uint64_t* bar_done = bars + kBarDone;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kBarTmem);
  float* vec = reinterpret_cast<float*>(smem + kOffVec);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  Walk W;
  W.lay = make_layout(p.layout, p.N, p.P);
  const int64_t L = p.L;                   // queries per shard
  const int64_t Lk = kChunkedKeys ? p.Lk : L;  // keys per shard
  // global position of key i of shard s (a tile of a rectangular grid:
  // contiguous chunks of Lk keys)
  auto kpos = [&](int s, int64_t i) -> int64_t {
    return kChunkedKeys ? (int64_t)s * Lk + i : W.lay.pos(s, i);
  };
  // grid: (key tile in order of decreasing work x KV head, KV head block, batch)
  const int b = blockIdx.z;
  int c, gh;
  if (!grid_place(p.head_block, p.Hkv, c, gh)) return;
  int xt;
  {
    const int T = (int)((Lk + BK - 1) / BK);
    if (!p.ring) {
      W.s = p.kv_rank;
      xt = c;
    } else if (p.causal) {
      W.lay.ordered_tile(T, BK, c, false, W.s, xt);
    } else {
      W.s = c / T;
      xt = c - W.s * T;
    }
  }
  W.g = gh;
  W.group = p.Hq / p.Hkv;
  W.nranks = p.ring ? p.P : 1;
  W.qtiles = (int)((L + BQ - 1) / BQ);
  W.ring = p.ring;
  W.q_rank = p.q_rank;
  W.P = p.P;
  W.causal = p.causal;
  const int64_t i0 = (int64_t)xt * BK;  // first key (local index in shard s)
  const Segs sg{p.cu_seqlens, p.num_segments, p.seq_lens, p.N, p.seg_div};
  {  // queries that may see a key of the CTA (the bounds are monotone in the key)
    int64_t f, l;
    sg.key_span(b, kpos(W.s, i0), p.causal, W.span_first, l);
    sg.key_span(b, kpos(W.s, LayoutMap::min64(i0 + BK - 1, Lk - 1)), p.causal, f, W.span_last);
  }
  const int s = W.s, g = W.g;
  const long long limit = p.wait_limit;
  const BwdRows R = bwd_rows(p);

  if (threadIdx.x == 0) {
    mbar_init(bar_kv, 1);
    for (int x = 0; x < kQStages; ++x) {
      mbar_init(bar_q_full + x, 1);
      mbar_init(bar_q_empty + x, 1);
    }
    for (int x = 0; x < kDOStages; ++x) {
      mbar_init(bar_do_full + x, 1);
      mbar_init(bar_do_empty + x, 1);
    }
    mbar_init(bar_s_full, 1);
    mbar_init(bar_s_free, 256);
    mbar_init(bar_dp_full, 1);
    mbar_init(bar_p_full, 256);
    mbar_init(bar_ds_full, 256);
    for (int x = 0; x < 4; ++x) mbar_init(bar_vec + x, 128);
    mbar_init(bar_done, 1);
    fence_barrier_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int n = W.count();

  if (warp >= 8) {
    regs_dec<kRegsOther>();
    if (warp == kWarpTma && lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      prefetch_tmap(&tmDO);
      int kr, ks;
      R.tma(s, i0, kr, ks);
      mbar_arrive_expect_tx(bar_kv, 2 * kKTile);
      for (int x = 0; x < 2; ++x) {
        tma_load_5d(smem + kOffK + x * kKBox, &tmK, bar_kv, x * 64, g, kr, ks, b);
        tma_load_5d(smem + kOffV + x * kKBox, &tmV, bar_kv, x * 64, g, kr, ks, b);
      }
      int nq = 0, ndo = 0;  // Q / dO tiles issued
      Walk::Cursor cur = W.begin();
      for (int i = 0; i < n; ++i, W.next(cur)) {
        const int sq = i % kQStages, sd = i % kDOStages;
        const int h = W.head(cur), t = cur.t;
        int qr, qs;
        R.tma(cur.r, (int64_t)t * BQ, qr, qs);
        if (i >= kQStages &&
            !mbar_wait(bar_q_empty + sq, ((i / kQStages) - 1) & 1, limit, p.status))
          break;
        mbar_arrive_expect_tx(bar_q_full + sq, kQTile);
        for (int x = 0; x < 2; ++x)
          tma_load_5d(smem + kOffQ + sq * kQTile + x * kQBox, &tmQ, bar_q_full + sq, x * 64, h,
                      qr, qs, b);
        ++nq;
        if (i >= kDOStages &&
            !mbar_wait(bar_do_empty + sd, ((i / kDOStages) - 1) & 1, limit, p.status))
          break;
        mbar_arrive_expect_tx(bar_do_full + sd, kQTile);
        for (int x = 0; x < 2; ++x)
          tma_load_5d(smem + kOffDO + sd * kQTile + x * kQBox, &tmDO, bar_do_full + sd, x * 64, h,
                      qr, qs, b);
        ++ndo;
      }
      // drain: every load issued has landed before the CTA exits
      mbar_wait(bar_kv, 0, limit, p.status);
      for (int st = 0; st < kQStages && st < nq; ++st) {
        const int uses = (nq - st + kQStages - 1) / kQStages;
        mbar_wait(bar_q_full + st, (uses - 1) & 1, limit, p.status);
      }
      for (int st = 0; st < kDOStages && st < ndo; ++st) {
        const int uses = (ndo - st + kDOStages - 1) / kDOStages;
        mbar_wait(bar_do_full + st, (uses - 1) & 1, limit, p.status);
      }
    } else if (warp == kWarpMma && lane == 0) {
      constexpr uint32_t idST = idesc_bf16(BK, BQ, 0, 0);  // S^T, dP^T
      constexpr uint32_t idKV = idesc_bf16(BK, D, 0, 1);   // dV, dK (A in TMEM, B MN-major)
      const uint64_t kAd = kdesc0(smem_u32(smem + kOffK)), vAd = kdesc0(smem_u32(smem + kOffV));
      const uint64_t qBd = kdesc0(smem_u32(smem + kOffQ)), doBd = kdesc0(smem_u32(smem + kOffDO));
      const uint64_t qMNd = mndesc0(smem_u32(smem + kOffQ), kQBox);
      const uint64_t doMNd = mndesc0(smem_u32(smem + kOffDO), kQBox);
      auto issue_s = [&](int i) -> bool {  // S^T(i) = K Q(i)^T
        const int qst = i % kQStages;
        if (!mbar_wait(bar_q_full + qst, (i / kQStages) & 1, limit, p.status)) return false;
        fence_after_sync();
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          mma_ss(tmem + kTS, desc_add(kAd, koff(k, kKBox)),
                 desc_add(qBd, qst * kQTile + koff(k, kQBox)), idST, k > 0);
        mma_commit(bar_s_full);
        return true;
      };
      auto issue_dp = [&](int i) -> bool {  // dP^T(i) = V dO(i)^T
        const int sd = i % kDOStages;
        if (!mbar_wait(bar_do_full + sd, (i / kDOStages) & 1, limit, p.status)) return false;
        fence_after_sync();
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          mma_ss(tmem + kTdP, desc_add(vAd, koff(k, kKBox)),
                 desc_add(doBd, sd * kQTile + koff(k, kQBox)), idST, k > 0);
        mma_commit(bar_dp_full);
        return true;
      };
      bool ok = n == 0 || (mbar_wait(bar_kv, 0, limit, p.status) && issue_s(0) && issue_dp(0));
      if (ok && n > 1) ok = mbar_wait(bar_s_free, 0, limit, p.status) && issue_s(1);
      for (int i = 0; ok && i < n; ++i) {
        const int qst = i % kQStages, sd = i % kDOStages;
        if (!mbar_wait(bar_p_full, i & 1, limit, p.status)) break;
        fence_after_sync();
#pragma unroll
        for (int k = 0; k < BQ / 16; ++k)  // dV += P^T dO
          mma_ts(tmem + kTdV, tmem + kTdP + p_col(k), desc_add(doMNd, sd * kQTile + mnoff(k)),
                 idKV, (i == 0 && k == 0) ? 0u : 1u);
        mma_commit(bar_do_empty + sd);
        if (!mbar_wait(bar_ds_full, i & 1, limit, p.status)) break;
        fence_after_sync();
#pragma unroll
        for (int k = 0; k < BQ / 16; ++k)  // dK += dS^T Q
          mma_ts(tmem + kTdK, tmem + kTdP + ds_col(k), desc_add(qMNd, qst * kQTile + mnoff(k)),
                 idKV, (i == 0 && k == 0) ? 0u : 1u);
        mma_commit(bar_q_empty + qst);
        if (i + 1 < n && !issue_dp(i + 1)) break;
        if (i + 2 < n &&
            !(mbar_wait(bar_s_free, (i + 1) & 1, limit, p.status) && issue_s(i + 2)))
          break;
      }
      mma_commit(bar_done);
      mbar_wait(bar_done, 0, limit, p.status);  // every MMA done before TMEM is freed
    }
  } else {
    regs_inc<kRegsMath>();
    const int X = warp >> 2;                 // this warpgroup's query columns: [64X, 64X + 64)
    const int lane_base = (warp & 3) * 32;
    const uint32_t tl = (uint32_t)lane_base << 16;
    const int krow = lane_base + lane;       // key row of the tile (TMEM lane)
    const int64_t key = i0 + krow;
    const bool key_live = key < Lk;
    // local queries [span_lo, span_hi) of rank span_rank see this key
    int span_rank = -1, span_lo = 0, span_hi = 0;
    const int tid = threadIdx.x & 127;
    const uint32_t cS = kTS + kHalf * X, cdP = kTdP + kHalf * X;
    bool ok = true;
    // LSE*log2(e) (tid < 64) or D (tid >= 64) of column 64X + (tid & 63) of the tile at c
    auto fetch = [&](const Walk::Cursor& c, int idx) -> float {
      if (idx >= n) return 0.f;
      const int64_t j = (int64_t)c.t * BQ + kHalf * X + (tid & 63);
      if (j >= L) return 0.f;
      const int64_t off = ((int64_t)b * p.Hq + W.head(c)) * p.lse_ld + R.row(c.r, j);
      return tid < 64 ? p.lse[off] * kLog2e : p.delta[off];
    };
    Walk::Cursor cur = W.begin();
    Walk::Cursor ahead = cur;
    W.next(ahead);
    float next = fetch(cur, 0);
    for (int i = 0; i < n; ++i) {
      const int y = i & 1;  // staging buffer
      float* vbuf = vec + (X * 2 + y) * 2 * kHalf;
      vbuf[tid] = next;
      mbar_arrive(bar_vec + X * 2 + y);
      next = fetch(ahead, i + 1);  // in flight during this tile
      const int r = cur.r, t = cur.t;
      if (r != span_rank) {  // recomputed per rank rather than held across the walk
        span_rank = r;
        span_lo = span_hi = 0;
        if (key_live) {
          int64_t f, l;  // global positions of the queries that see this key
          sg.key_span(b, kpos(s, key), p.causal, f, l);
          span_lo = (int)W.lay.visible_count(r, f - 1);
          span_hi = (int)W.lay.visible_count(r, l);
        }
      }
      // visible query columns [lo, hi) of this key in this warpgroup's half
      const int j0 = t * BQ + kHalf * X;
      const int lo = min(max(span_lo - j0, 0), kHalf);
      const int hi = min(max(span_hi - j0, 0), kHalf);
      const bool full = __all_sync(0xffffffffu, lo == 0 && hi == kHalf);
      W.next(cur);
      W.next(ahead);
      if (!__all_sync(0xffffffffu, mbar_wait(bar_vec + X * 2 + y, (i >> 1) & 1, limit, p.status)) ||
          !__all_sync(0xffffffffu, mbar_wait(bar_s_full, i & 1, limit, p.status))) {
        ok = false;
        break;
      }
      fence_after_sync();
      const float4* lse4 = reinterpret_cast<const float4*>(vbuf);
      const float4* dd4 = reinterpret_cast<const float4*>(vbuf + kHalf);
      float pt[kHalf];
      {
        uint32_t v[kHalf];
        tmem_ld32(tmem + tl + cS, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
        tmem_ld32(tmem + tl + cS + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
        tmem_wait_ld();
        fence_before_sync();
        mbar_arrive(bar_s_free);  // S^T(i) is in registers: S^T(i+1) may overwrite it
#pragma unroll
        for (int e = 0; e < kHalf; e += 4) {
          const float4 l4 = lse4[e / 4];
          pt[e + 0] = ex2(fmaf(__uint_as_float(v[e + 0]), p.scale_log2, -l4.x));
          pt[e + 1] = ex2(fmaf(__uint_as_float(v[e + 1]), p.scale_log2, -l4.y));
          pt[e + 2] = ex2(fmaf(__uint_as_float(v[e + 2]), p.scale_log2, -l4.z));
          pt[e + 3] = ex2(fmaf(__uint_as_float(v[e + 3]), p.scale_log2, -l4.w));
        }
      }
      if (!full) {
#pragma unroll
        for (int col = 0; col < kHalf; ++col) pt[col] = (col >= lo && col < hi) ? pt[col] : 0.f;
      }
      if (!__all_sync(0xffffffffu, mbar_wait(bar_dp_full, i & 1, limit, p.status))) {
        ok = false;
        break;
      }
      fence_after_sync();
      {
        uint32_t v[kHalf];
        tmem_ld32(tmem + tl + cdP, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
        tmem_ld32(tmem + tl + cdP + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
        tmem_wait_ld();
        // P^T over the first 32 columns of this half (its dP^T is in registers)
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) pk[e] = pack_bf16(pt[2 * e], pt[2 * e + 1]);
        tmem_st32(tmem + tl + cdP, pk);
        tmem_wait_st();
        fence_before_sync();
        mbar_arrive(bar_p_full);
        // dS^T = P^T o (dP^T - D) over the last 32 columns
#pragma unroll
        for (int e = 0; e < kHalf; e += 4) {
          const float4 d4 = dd4[e / 4];
          pk[e / 2] = pack_bf16(pt[e] * (__uint_as_float(v[e]) - d4.x),
                                pt[e + 1] * (__uint_as_float(v[e + 1]) - d4.y));
          pk[e / 2 + 1] = pack_bf16(pt[e + 2] * (__uint_as_float(v[e + 2]) - d4.z),
                                    pt[e + 3] * (__uint_as_float(v[e + 3]) - d4.w));
        }
        tmem_st32(tmem + tl + cdP + 32, pk);
        tmem_wait_st();
        fence_before_sync();
        mbar_arrive(bar_ds_full);
      }
    }
    // ---------------- epilogue: dK (warps 0-3), dV (warps 4-7); lane = key ----------------
    if (__all_sync(0xffffffffu, ok && mbar_wait(bar_done, 0, limit, p.status))) {
      fence_after_sync();
      const uint32_t tcol = X == 0 ? kTdK : kTdV;
      const float f = X == 0 ? p.scale : 1.0f;
      const int es = p.accumulate ? 4 : 2;
      const int64_t row = R.row(s, key);
      char* base = X == 0 ? reinterpret_cast<char*>(p.dk) +
                                (b * p.dk_sb + row * p.dk_sn + (int64_t)g * p.dk_sh) * es
                          : reinterpret_cast<char*>(p.dv) +
                                (b * p.dv_sb + row * p.dv_sn + (int64_t)g * p.dv_sh) * es;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + tl + tcol + c * 32, v);
        tmem_wait_ld();
        if (key_live) store_row(base, p.accumulate, c, v, f, n == 0);
      }
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == kWarpMma) {
    fence_after_sync();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace kv

// ===========================================================================
// dQ (query-stationary)
// ===========================================================================
namespace dq {

constexpr int BM = 128;     // query rows per CTA (TMEM lanes)
constexpr int BN = 128;     // keys per KV tile (the N of S, dP)
constexpr int kHalf = BN / 2;  // key columns per math warpgroup
constexpr int kKStages = 3;    // K is read by S(j) and dQ(j): the longer-lived operand
constexpr int kVStages = 2;    // V only by dP(j)
constexpr int kThreads = 384;
constexpr int kWarpTma = 8;
constexpr int kWarpMma = 9;
constexpr int kRegsMath = 200;
constexpr int kRegsOther = 104;
static_assert(2 * 128 * kRegsMath + 128 * kRegsOther <= kThreads * 168, "register split");

constexpr int kQBox = BM * 128;             // 128 query rows x 128 B
constexpr int kQTile = 2 * kQBox;           // d = 128
constexpr int kKBox = BN * 128;             // 128 key rows x 128 B
constexpr int kKTile = 2 * kKBox;
constexpr int kOffQ = 0;
constexpr int kOffDO = kOffQ + kQTile;
constexpr int kOffK = kOffDO + kQTile;      // [kKStages]
constexpr int kOffV = kOffK + kKStages * kKTile;  // [kVStages]
constexpr int kOffBar = kOffV + kVStages * kKTile;
constexpr int kSmem = kOffBar + 256;  // the base must be 1024-aligned (checked)
static_assert(kSmem <= 232448, "shared memory");

// TMEM columns: S double-buffered (dS written over it as bf16), dP, dQ.
constexpr uint32_t kTS = 0, kTdP = 256, kTdQ = 384;

// mbarrier slots (8 bytes each) in the 256-byte barrier area
constexpr int kBarQ = 0;
constexpr int kBarKFull = kBarQ + 1;
constexpr int kBarKEmpty = kBarKFull + kKStages;
constexpr int kBarVFull = kBarKEmpty + kKStages;
constexpr int kBarVEmpty = kBarVFull + kVStages;
constexpr int kBarS = kBarVEmpty + kVStages;  // [2]
constexpr int kBarDP = kBarS + 2;
constexpr int kBarDS = kBarDP + 1;
constexpr int kBarDone = kBarDS + 1;
constexpr int kBarTmem = kBarDone + 1;
static_assert((kBarTmem + 1) * 8 <= 256, "barrier area");

// TMEM column of the bf16 A operand dS for K-step k (16 keys): warpgroup k / 4
// packed its 64 keys into the first 32 columns of its half.
__device__ __forceinline__ uint32_t a_col(int k) { return kHalf * (k >> 2) + 8 * (k & 3); }

// Warp roles (384 threads): warps 0-3 and 4-7 are two math warpgroups that
// split every 128-key tile by columns (keys 0-63 / 64-127) over the 128 query
// rows (one thread per row: dS = P o (dP - D), written over S as bf16), then
// write dQ; warp 8 TMA producer (Q, dO once; K tiles into a 3-stage ring, V
// tiles into a 2-stage ring);
// warp 9 MMA issuer.  S is double-buffered in TMEM, dP single-buffered; the
// tensor pipe runs, per tile j,
//   dQ(j) [needs dS(j)], dP(j+1), S(j+2)
// so the exponentials of tile j+1 overlap dQ(j) and dP(j+1).
// kChunkedKeys: the KV side is one contiguous chunk of a rectangular grid (Pk != P).
template <bool kChunkedKeys>
__global__ void __launch_bounds__(kThreads, 1)
    tc_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                     const BwdParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  if (smem_u32(smem) & 1023u) {  // SW128 tiles need a 1024-byte aligned base
    if (threadIdx.x == 0) report_status(p.status, kStatusSmemAlign);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* bar_q = bars + kBarQ;
  uint64_t* bar_k_full = bars + kBarKFull;    // [kKStages]
  uint64_t* bar_k_empty = bars + kBarKEmpty;  // [kKStages]
  uint64_t* bar_v_full = bars + kBarVFull;    // [kVStages]
  uint64_t* bar_v_empty = bars + kBarVEmpty;  // [kVStages]
  uint64_t* bar_s_full = bars + kBarS;          // [2] S of a tile in TMEM buffer
  uint64_t* bar_dp_full = bars + kBarDP;        // dP of the tile in TMEM
  uint64_t* bar_ds_full = bars + kBarDS;        // dS written (256 arrivals)
  uint64_t* bar_done = bars + kBarDone;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kBarTmem);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const LayoutMap lay = make_layout(p.layout, p.N, p.P);
  const int64_t L = p.L;
  // grid: (query tile in order of decreasing work x query head, head block, batch)
  const int b = blockIdx.z;
  int c, h;
  if (!grid_place(p.head_block, p.Hq, c, h)) return;
  int r, u;
  {
    const int T = (int)((L + BM - 1) / BM);
    if (!p.ring) {
      r = p.q_rank;
      u = p.causal ? T - 1 - c : c;  // later rows see more keys: start them first
    } else if (p.causal) {
      lay.ordered_tile(T, BM, c, true, r, u);
    } else {
      r = c / T;
      u = c - r * T;
    }
  }
  const int64_t row0 = (int64_t)u * BM;
  const int g = h / (p.Hq / p.Hkv);
  const int64_t last_row = LayoutMap::min64(row0 + BM - 1, L - 1);
  const int64_t t_last = lay.pos(r, last_row);
  const Segs sg{p.cu_seqlens, p.num_segments, p.seq_lens, p.N, p.seg_div};
  // global span of the keys any row of the CTA may see (the bounds are
  // monotone in the row, so its first and last rows give them)
  int64_t span_first, span_last;
  {
    int64_t f, l;
    sg.query_span(b, lay.pos(r, LayoutMap::min64(row0, L - 1)), p.causal, span_first, l);
    sg.query_span(b, t_last, p.causal, f, span_last);
  }
  const int nsteps = p.ring ? p.P : 1;
  const long long limit = p.wait_limit;
  const BwdRows R = bwd_rows(p);
  auto shard_of = [&](int step) { return p.ring ? ((r - step) % p.P + p.P) % p.P : p.kv_rank; };
  // keys of shard s at global positions <= t: the layout's count, or for a
  // tile of a rectangular grid (contiguous chunks of Lk keys) the chunk's
  auto kvis = [&](int s, int64_t t) -> int64_t {
    return !kChunkedKeys ? lay.visible_count(s, t)
                       : LayoutMap::clamp64(t - (int64_t)s * p.Lk + 1, 0, p.Lk);
  };
  // key tiles [tile_begin(s), tile_end(s)) of shard s hold every key the CTA may see
  auto tile_begin = [&](int s) -> int { return (int)(kvis(s, span_first - 1) / BN); };
  auto tile_end = [&](int s) -> int { return (int)((kvis(s, span_last) + BN - 1) / BN); };
  int n = 0;  // key tiles of the whole walk
  for (int step = 0; step < nsteps; ++step) {
    const int s = shard_of(step);
    n += max(0, tile_end(s) - tile_begin(s));
  }

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int x = 0; x < kKStages; ++x) {
      mbar_init(bar_k_full + x, 1);
      mbar_init(bar_k_empty + x, 1);
    }
    for (int x = 0; x < kVStages; ++x) {
      mbar_init(bar_v_full + x, 1);
      mbar_init(bar_v_empty + x, 1);
    }
    mbar_init(bar_s_full + 0, 1);
    mbar_init(bar_s_full + 1, 1);
    mbar_init(bar_dp_full, 1);
    mbar_init(bar_ds_full, 256);
    mbar_init(bar_done, 1);
    fence_barrier_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 8) {
    regs_dec<kRegsOther>();
    if (warp == kWarpTma && lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      prefetch_tmap(&tmDO);
      int qr, qs;
      R.tma(r, row0, qr, qs);
      mbar_arrive_expect_tx(bar_q, 2 * kQTile);
      for (int x = 0; x < 2; ++x) {
        tma_load_5d(smem + kOffQ + x * kQBox, &tmQ, bar_q, x * 64, h, qr, qs, b);
        tma_load_5d(smem + kOffDO + x * kQBox, &tmDO, bar_q, x * 64, h, qr, qs, b);
      }
      int nk = 0, nv = 0;  // K / V tiles issued
      bool ok = true;
      for (int step = 0; step < nsteps && ok; ++step) {
        const int s = shard_of(step);
        const int te = tile_end(s);
        for (int t = tile_begin(s); t < te; ++t) {
          const int sk = nk % kKStages, sv = nv % kVStages;
          int kr, ks;
          R.tma(s, (int64_t)t * BN, kr, ks);
          if (nk >= kKStages &&
              !mbar_wait(bar_k_empty + sk, ((nk / kKStages) - 1) & 1, limit, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar_k_full + sk, kKTile);
          for (int x = 0; x < 2; ++x)
            tma_load_5d(smem + kOffK + sk * kKTile + x * kKBox, &tmK, bar_k_full + sk, x * 64, g,
                        kr, ks, b);
          ++nk;
          if (nv >= kVStages &&
              !mbar_wait(bar_v_empty + sv, ((nv / kVStages) - 1) & 1, limit, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar_v_full + sv, kKTile);
          for (int x = 0; x < 2; ++x)
            tma_load_5d(smem + kOffV + sv * kKTile + x * kKBox, &tmV, bar_v_full + sv, x * 64, g,
                        kr, ks, b);
          ++nv;
        }
      }
      // drain: every load issued has landed before the CTA exits
      mbar_wait(bar_q, 0, limit, p.status);
      for (int st = 0; st < kKStages && nk > st; ++st) {
        const int uses = (nk - st + kKStages - 1) / kKStages;
        mbar_wait(bar_k_full + st, (uses - 1) & 1, limit, p.status);
      }
      for (int st = 0; st < kVStages && nv > st; ++st) {
        const int uses = (nv - st + kVStages - 1) / kVStages;
        mbar_wait(bar_v_full + st, (uses - 1) & 1, limit, p.status);
      }
    } else if (warp == kWarpMma && lane == 0) {
      constexpr uint32_t idSD = idesc_bf16(BM, BN, 0, 0);  // S, dP
      constexpr uint32_t idQ = idesc_bf16(BM, D, 0, 1);    // dQ += dS K (A in TMEM, B MN-major)
      const uint64_t qAd = kdesc0(smem_u32(smem + kOffQ)), doAd = kdesc0(smem_u32(smem + kOffDO));
      const uint64_t kBd = kdesc0(smem_u32(smem + kOffK)), vBd = kdesc0(smem_u32(smem + kOffV));
      const uint64_t kMNd = mndesc0(smem_u32(smem + kOffK), kKBox);
      auto issue_s = [&](int j) -> bool {  // S(j) = Q K(j)^T into buffer j & 1
        const int sk = j % kKStages;
        if (!mbar_wait(bar_k_full + sk, (j / kKStages) & 1, limit, p.status)) return false;
        fence_after_sync();
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          mma_ss(tmem + kTS + (j & 1) * BN, desc_add(qAd, koff(k, kQBox)),
                 desc_add(kBd, sk * kKTile + koff(k, kKBox)), idSD, k > 0);
        mma_commit(bar_s_full + (j & 1));
        return true;
      };
      auto issue_dp = [&](int j) -> bool {  // dP(j) = dO V(j)^T
        const int sv = j % kVStages;
        if (!mbar_wait(bar_v_full + sv, (j / kVStages) & 1, limit, p.status)) return false;
        fence_after_sync();
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          mma_ss(tmem + kTdP, desc_add(doAd, koff(k, kQBox)),
                 desc_add(vBd, sv * kKTile + koff(k, kKBox)), idSD, k > 0);
        mma_commit(bar_dp_full);
        mma_commit(bar_v_empty + sv);
        return true;
      };
      bool ok = n == 0 || (mbar_wait(bar_q, 0, limit, p.status) && issue_s(0) && issue_dp(0));
      if (ok && n > 1) ok = issue_s(1);
      for (int j = 0; ok && j < n; ++j) {
        const int sk = j % kKStages;
        if (!mbar_wait(bar_ds_full, j & 1, limit, p.status)) break;
        fence_after_sync();
#pragma unroll
        for (int k = 0; k < BN / 16; ++k)  // dQ += dS K
          mma_ts(tmem + kTdQ, tmem + kTS + (j & 1) * BN + a_col(k),
                 desc_add(kMNd, sk * kKTile + mnoff(k)), idQ, (j == 0 && k == 0) ? 0u : 1u);
        mma_commit(bar_k_empty + sk);
        if (j + 1 < n && !issue_dp(j + 1)) break;
        if (j + 2 < n && !issue_s(j + 2)) break;
      }
      mma_commit(bar_done);
      mbar_wait(bar_done, 0, limit, p.status);
    }
  } else {
    regs_inc<kRegsMath>();
    const int X = warp >> 2;                 // this warpgroup's key columns: [64X, 64X + 64)
    const int lane_base = (warp & 3) * 32;
    const uint32_t tl = (uint32_t)lane_base << 16;
    const int64_t row = row0 + lane_base + lane;
    const bool live = row < L;
    const int64_t tq = live ? lay.pos(r, row) : -1;
    const int64_t qrow = R.row(r, row);
    float lse2 = 0.f, dd = 0.f;
    if (live) {
      const int64_t off = ((int64_t)b * p.Hq + h) * p.lse_ld + qrow;
      lse2 = p.lse[off] * kLog2e;
      dd = p.delta[off];
    }
    int j = 0;
    bool ok = true;
    for (int step = 0; step < nsteps && ok; ++step) {
      const int s = shard_of(step);
      const int te = tile_end(s);
      // keys [row_lo, row_hi) of shard s are visible to this row
      int64_t row_lo = 0, row_hi = 0;
      if (live) {
        int64_t f, l;
        sg.query_span(b, tq, p.causal, f, l);
        row_lo = kvis(s, f - 1);
        row_hi = kvis(s, l);
      }
      for (int t = tile_begin(s); t < te; ++t, ++j) {
        const uint32_t cS = kTS + (j & 1) * BN + kHalf * X, cdP = kTdP + kHalf * X;
        // visible keys of this warpgroup's half: [c_lo, c_hi)
        const int64_t c0 = (int64_t)t * BN + kHalf * X;
        const int64_t c_lo = row_lo - c0, c_hi = row_hi - c0;
        const bool full = __all_sync(0xffffffffu, c_lo <= 0 && c_hi >= kHalf);
        if (!__all_sync(0xffffffffu, mbar_wait(bar_s_full + (j & 1), (j >> 1) & 1, limit, p.status))) {
          ok = false;
          break;
        }
        fence_after_sync();
        float pt[kHalf];
#pragma unroll
        for (int c = 0; c < kHalf / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tmem + tl + cS + 32 * c, v);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; e += 2) {  // exponents two at a time (packed fp32 FMA)
            const float2 x2 = __ffma2_rn(make_float2(__uint_as_float(v[e]), __uint_as_float(v[e + 1])),
                                         make_float2(p.scale_log2, p.scale_log2),
                                         make_float2(-lse2, -lse2));
            pt[32 * c + e] = ex2(x2.x);
            pt[32 * c + e + 1] = ex2(x2.y);
          }
        }
        if (!full) {
#pragma unroll
          for (int col = 0; col < kHalf; ++col) pt[col] = (col >= c_lo && col < c_hi) ? pt[col] : 0.f;
        }
        if (!__all_sync(0xffffffffu, mbar_wait(bar_dp_full, j & 1, limit, p.status))) {
          ok = false;
          break;
        }
        fence_after_sync();
        // dS over the 64 columns in two halves, written over S (already read)
#pragma unroll
        for (int c = 0; c < kHalf / 32; ++c) {
          uint32_t v[32], ds[16];
          tmem_ld32(tmem + tl + cdP + 32 * c, v);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; e += 2) {  // packed fp32 subtract and multiply
            const float2 s2 = __fmul2_rn(make_float2(pt[32 * c + e], pt[32 * c + e + 1]),
                                         __fadd2_rn(make_float2(__uint_as_float(v[e]), __uint_as_float(v[e + 1])),
                                                    make_float2(-dd, -dd)));
            ds[e / 2] = pack_bf16(s2.x, s2.y);
          }
          tmem_st16(tmem + tl + cS + 16 * c, ds);
        }
        tmem_wait_st();
        fence_before_sync();
        mbar_arrive(bar_ds_full);
      }
    }
    // ---------------- epilogue: dQ = scale * acc, columns [64X, 64X + 64) ----------------
    if (__all_sync(0xffffffffu, ok && mbar_wait(bar_done, 0, limit, p.status))) {
      fence_after_sync();
      const int es = p.accumulate ? 4 : 2;
      char* base = reinterpret_cast<char*>(p.dq) +
                   (b * p.dq_sb + qrow * p.dq_sn + (int64_t)h * p.dq_sh) * es;
#pragma unroll
      for (int c = 2 * X; c < 2 * X + 2; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + tl + kTdQ + c * 32, v);
        tmem_wait_ld();
        if (live) store_row(base, p.accumulate, c, v, p.scale, n == 0);
      }
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == kWarpMma) {
    fence_after_sync();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace dq

}  // namespace

rm_status tc_bwd(const AttnArgs& a, int q_rank, int kv_rank, cudaStream_t stream) {
  if (a.B == 0 || a.N == 0) return RM_OK;
  if (a.d != D) return RM_ERR_UNSUPPORTED;
  const bool ring = q_rank < 0;
  const int64_t L = a.N / a.P;
  const int Pk = ring ? a.P : kv_shards(a);
  const int64_t Lk = a.N / Pk;
  const int shards = ring ? a.P : 1;
  BwdParams p;
  p.B = a.B;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.P = a.P;
  p.layout = a.layout;
  p.causal = a.causal;
  p.N = a.N;
  p.L = L;
  p.Pk = Pk;
  p.Lk = Lk;
  p.scale = a.scale;
  p.scale_log2 = a.scale * kLog2e;
  p.ring = ring ? 1 : 0;
  p.q_rank = q_rank;
  p.kv_rank = kv_rank;
  p.lse = a.lse_in;
  p.delta = a.delta;
  p.lse_ld = a.lse_ld;
  p.dq = a.dq.ptr;
  p.dq_sb = a.dq.stride_b;
  p.dq_sn = a.dq.stride_n;
  p.dq_sh = a.dq.stride_h;
  p.dk = a.dk.ptr;
  p.dk_sb = a.dk.stride_b;
  p.dk_sn = a.dk.stride_n;
  p.dk_sh = a.dk.stride_h;
  p.dv = a.dv.ptr;
  p.dv_sb = a.dv.stride_b;
  p.dv_sn = a.dv.stride_n;
  p.dv_sh = a.dv.stride_h;
  p.accumulate = a.accumulate;
  p.global_order = ring ? a.global_order : 0;
  p.cu_seqlens = a.cu_seqlens;
  p.num_segments = a.num_segments;
  p.seq_lens = a.seq_lens;
  p.seg_div = a.seg_div > 1 ? a.seg_div : 1;
  const int view = operand_view(a, ring);
  p.status = a.status;
  p.wait_limit = tc_wait_limit();
  if (a.B > 65535) return RM_ERR_UNSUPPORTED;  // grid.z
  {  // dK, dV
    CUtensorMap mq, mk, mv, mdo;
    if (encode_operand_map(&mq, a.q, a.B, shards, L, a.Hq, a.d, 64, kv::BQ, view) != RM_OK ||
        encode_operand_map(&mk, a.k, a.B, shards, Lk, a.Hkv, a.d, 64, kv::BK, view) != RM_OK ||
        encode_operand_map(&mv, a.v, a.B, shards, Lk, a.Hkv, a.d, 64, kv::BK, view) != RM_OK ||
        encode_operand_map(&mdo, a.dout, a.B, shards, L, a.Hq, a.d, 64, kv::BQ, view) != RM_OK)
      return RM_ERR_CUDA;
    // a key-tile CTA streams Q and dO of every query head of its group
    p.head_block = head_block((int64_t)(a.Hq / a.Hkv) * a.N * D * 2 * 2, a.Hkv);
    dim3 grid((unsigned)(ceil_div(Lk, kv::BK) * shards * p.head_block),
              (unsigned)ceil_div(a.Hkv, p.head_block), (unsigned)a.B);
    auto kernel = Pk != a.P ? kv::tc_bwd_dkdv_kernel<true> : kv::tc_bwd_dkdv_kernel<false>;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kv::kSmem) !=
        cudaSuccess)
      return RM_ERR_CUDA;
    ProfScope ps("tc_bwd_dkdv_kernel", stream);
    kernel<<<grid, kv::kThreads, kv::kSmem, stream>>>(mq, mk, mv, mdo, p);
    if (cudaGetLastError() != cudaSuccess) return RM_ERR_CUDA;
  }
  {  // dQ
    CUtensorMap mq, mk, mv, mdo;
    if (encode_operand_map(&mq, a.q, a.B, shards, L, a.Hq, a.d, 64, dq::BM, view) != RM_OK ||
        encode_operand_map(&mk, a.k, a.B, shards, Lk, a.Hkv, a.d, 64, dq::BN, view) != RM_OK ||
        encode_operand_map(&mv, a.v, a.B, shards, Lk, a.Hkv, a.d, 64, dq::BN, view) != RM_OK ||
        encode_operand_map(&mdo, a.dout, a.B, shards, L, a.Hq, a.d, 64, dq::BM, view) != RM_OK)
      return RM_ERR_CUDA;
    // a query-tile CTA streams K and V of its KV head (shared by the group)
    const int group = a.Hq / a.Hkv;
    p.head_block = head_block((int64_t)a.N * D * 2 * 2 / group, a.Hq);
    dim3 grid((unsigned)(ceil_div(L, dq::BM) * shards * p.head_block),
              (unsigned)ceil_div(a.Hq, p.head_block), (unsigned)a.B);
    auto kernel = Pk != a.P ? dq::tc_bwd_dq_kernel<true> : dq::tc_bwd_dq_kernel<false>;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dq::kSmem) !=
        cudaSuccess)
      return RM_ERR_CUDA;
    ProfScope ps("tc_bwd_dq_kernel", stream);
    kernel<<<grid, dq::kThreads, dq::kSmem, stream>>>(mq, mk, mv, mdo, p);
    if (cudaGetLastError() != cudaSuccess) return RM_ERR_CUDA;
  }
  return RM_OK;
}

}  // namespace rm
