// Backward attention on the sm_100a tensor cores (bf16 in, fp32 accumulate),
// head dim 128.
//
// One CTA owns one 128-key tile of one KV head (ringmaster, "Status": the
// backward runs the ring in the opposite direction -- the KV shard visits the
// ranks s, s+1, ..., and every rank's queries add their contribution).  It walks, for every
// query head of the GQA group and every rank in reverse-ring order, the
// 64-query tiles that can see its keys, recomputing the probabilities from the
// final LSE:
//   S^T  = K Q^T            (TMEM, keys on lanes)
//   dP^T = V dO^T           (TMEM)
//   P^T  = exp(S^T * scale - LSE),  dS^T = P^T o (dP^T - D)
//   dV  += P^T dO           (A = P^T from TMEM)
//   dK  += dS^T Q           (A = dS^T from TMEM)
//   dQ^T = K^T dS^T         (TMEM, head-dim on lanes) -> fp32 reductions to dQ
// dK and dV stay in TMEM for the whole walk, so they need no atomics; dQ is
// accumulated with coalesced fp32 reductions (consecutive lanes hold
// consecutive head-dim columns of one query row).
//
// Warp roles (384 threads):
//   warps 0-3  per-key math (P^T, dS^T), then the dK epilogue
//   warps 4-7  dQ^T readout and reduction, then the dV epilogue
//   warp  8    TMA producer: K, V once; Q, dO tiles into a 2-stage ring
//   warp  9    MMA issuer
// TMEM: dK [0,128) dV [128,256) S^T x2 [256,384) dP^T [384,448) dQ^T [448,512)
#include <cudaTypedefs.h>
#include <stdlib.h>

#include "tc_attn.h"
#include "tc_common.cuh"

namespace rm {

rm_status encode_operand_map(CUtensorMap* map, const rm_tensor& t, int B, int shards, int64_t L,
                             int H, int d, int box_cols, int box_rows);
long long tc_wait_limit();

namespace {

using namespace tc;

constexpr int D = 128;      // head dim
constexpr int BK = 128;     // keys per CTA (TMEM lanes)
constexpr int BQ = 64;      // queries per tile
constexpr int kThreads = 384;
constexpr int kWarpTma = 8;
constexpr int kWarpMma = 9;
constexpr int kRegsMath = 216;
constexpr int kRegsOther = 64;
static_assert(2 * 128 * kRegsMath + 128 * kRegsOther <= kThreads * 168, "register split");

// shared memory (bytes from a 1024-aligned base)
constexpr int kKBox = BK * 128;             // 128 key rows x 128 B (64 cols)
constexpr int kKTile = 2 * kKBox;           // d = 128: two boxes
constexpr int kQBox = BQ * 128;             // 64 query rows x 128 B
constexpr int kQTile = 2 * kQBox;
constexpr int kOffK = 0;
constexpr int kOffV = kOffK + kKTile;
constexpr int kOffQ = kOffV + kKTile;       // [2] stages
constexpr int kOffDO = kOffQ + 2 * kQTile;  // [2] stages
constexpr int kOffDS = kOffDO + 2 * kQTile; // dS^T bf16 [128 keys][64 queries], SW128
constexpr int kDSBytes = BK * 128;
constexpr int kOffVec = kOffDS + kDSBytes;  // LSE*log2e and D for 2 stages: [2][2][64] fp32
constexpr int kOffBar = kOffVec + 2 * 2 * BQ * 4;
constexpr int kSmem = kOffBar + 256 + 1024;

constexpr uint32_t kTdK = 0, kTdV = 128, kTS = 256, kTdP = 384, kTdQ = 448;

struct BwdParams {
  int B, Hq, Hkv, P, layout, causal;
  int64_t N, L;
  float scale;        // softmax scale
  float scale_log2;   // scale * log2(e)
  int ring, q_rank, kv_rank;
  const float* lse;   // natural-log LSE
  const float* delta;
  int64_t lse_ld;
  float* dq;          // fp32, strided
  int64_t dq_sb, dq_sn, dq_sh;
  void* dk;           // bf16 output (ring) or fp32 accumulator (block)
  int64_t dk_sb, dk_sn, dk_sh;
  void* dv;
  int64_t dv_sb, dv_sn, dv_sh;
  int accumulate;
  unsigned int* status;
  long long wait_limit;
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// K-major SW128 operand with rows of 128 B, two 64-column boxes box_bytes apart.
__device__ __forceinline__ uint64_t kdesc(uint32_t base, int k, uint32_t box_bytes) {
  const int col = k * 16;
  return smem_desc(base + (col / 64) * box_bytes + (col % 64) * 2, 16, 1024, kSwizzle128B);
}
// MN-major SW128 operand: rows of 128 B along the contiguous (M or N) axis, the
// K axis along rows; K-step k starts 16 rows later; 64-element blocks of the
// contiguous axis are box_bytes apart.
__device__ __forceinline__ uint64_t mndesc(uint32_t base, int k, uint32_t box_bytes) {
  return smem_desc(base + k * 16 * 128, box_bytes, 1024, kSwizzle128B);
}

__global__ void __launch_bounds__(kThreads, 1)
    tc_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                  const BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* bar_kv = bars + 0;
  uint64_t* bar_q_full = bars + 1;   // [2]
  uint64_t* bar_q_empty = bars + 3;  // [2]
  uint64_t* bar_s_full = bars + 5;   // [2] S^T buffers
  uint64_t* bar_dp_full = bars + 7;
  uint64_t* bar_p_full = bars + 8;   // P^T in TMEM (128 arrivals)
  uint64_t* bar_ds_full = bars + 9;  // dS^T in TMEM and smem (128 arrivals)
  uint64_t* bar_ds_empty = bars + 10;
  uint64_t* bar_dq_full = bars + 11;
  uint64_t* bar_dq_empty = bars + 12;  // dQ^T read out (128 arrivals)
  uint64_t* bar_done = bars + 13;
  uint64_t* bar_vec = bars + 14;      // [2] LSE / D staged (128 arrivals)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
  float* vec = reinterpret_cast<float*>(smem + kOffVec);  // [stage][0: lse2, 1: D][64]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const LayoutMap lay = make_layout(p.layout, p.N, p.P);
  const int64_t L = p.L;
  const int s = p.ring ? (int)(blockIdx.z % p.P) : p.kv_rank;
  const int b = p.ring ? (int)(blockIdx.z / p.P) : (int)blockIdx.z;
  const int g = blockIdx.y;
  const int group = p.Hq / p.Hkv;
  const int64_t i0 = (int64_t)blockIdx.x * BK;  // first key (local index in shard s)
  const int64_t tk_first = lay.pos(s, i0);
  const int nranks = p.ring ? p.P : 1;
  const int qtiles = (int)((L + BQ - 1) / BQ);
  const long long limit = p.wait_limit;

  // first query tile of rank r that can see key i0 (later tiles all can)
  auto first_tile = [&](int r) -> int {
    if (!p.causal) return 0;
    const int64_t before = lay.visible_count(r, tk_first - 1);  // queries with pos < tk_first
    return (int)(before / BQ);
  };
  auto rank_of = [&](int step) { return p.ring ? (s + step) % p.P : p.q_rank; };

  if (threadIdx.x == 0) {
    mbar_init(bar_kv, 1);
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar_q_full + x, 1);
      mbar_init(bar_q_empty + x, 1);
      mbar_init(bar_s_full + x, 1);
    }
    mbar_init(bar_dp_full, 1);
    mbar_init(bar_p_full, 128);
    mbar_init(bar_ds_full, 128);
    mbar_init(bar_ds_empty, 1);
    mbar_init(bar_dq_full, 1);
    mbar_init(bar_dq_empty, 128);
    mbar_init(bar_done, 1);
    mbar_init(bar_vec + 0, 128);
    mbar_init(bar_vec + 1, 128);
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

  // total number of query tiles this CTA walks
  int n = 0;
  for (int hh = 0; hh < group; ++hh)
    for (int step = 0; step < nranks; ++step) n += qtiles - first_tile(rank_of(step));

  if (warp >= 8) {
    regs_dec<kRegsOther>();
    if (warp == kWarpTma && lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      prefetch_tmap(&tmDO);
      const int ks = p.ring ? s : 0;
      mbar_arrive_expect_tx(bar_kv, 2 * kKTile);
      for (int x = 0; x < 2; ++x) {
        tma_load_5d(smem + kOffK + x * kKBox, &tmK, bar_kv, x * 64, g, (int)i0, ks, b);
        tma_load_5d(smem + kOffV + x * kKBox, &tmV, bar_kv, x * 64, g, (int)i0, ks, b);
      }
      int i = 0;
      bool ok = true;
      for (int hh = 0; hh < group && ok; ++hh) {
        const int h = g * group + hh;
        for (int step = 0; step < nranks && ok; ++step) {
          const int r = rank_of(step);
          const int qs = p.ring ? r : 0;
          for (int t = first_tile(r); t < qtiles; ++t, ++i) {
            const int st = i & 1;
            if (i >= 2 && !mbar_wait(bar_q_empty + st, ((i >> 1) - 1) & 1, limit, p.status)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(bar_q_full + st, 2 * kQTile);
            for (int x = 0; x < 2; ++x) {
              tma_load_5d(smem + kOffQ + st * kQTile + x * kQBox, &tmQ, bar_q_full + st, x * 64, h,
                          t * BQ, qs, b);
              tma_load_5d(smem + kOffDO + st * kQTile + x * kQBox, &tmDO, bar_q_full + st, x * 64,
                          h, t * BQ, qs, b);
            }
          }
        }
      }
      mbar_wait(bar_kv, 0, limit, p.status);
      for (int st = 0; st < 2 && i > st; ++st) {
        const int uses = (i - st + 1) / 2;
        mbar_wait(bar_q_full + st, (uses - 1) & 1, limit, p.status);
      }
    } else if (warp == kWarpMma && lane == 0) {
      constexpr uint32_t idST = idesc_bf16(BK, BQ, 0, 0);   // S^T, dP^T
      constexpr uint32_t idKV = idesc_bf16(BK, D, 0, 1);    // dV, dK (A from TMEM)
      constexpr uint32_t idDQ = idesc_bf16(D, BQ, 1, 1);    // dQ^T = K^T dS^T
      const uint32_t kA = smem_u32(smem + kOffK), vA = smem_u32(smem + kOffV);
      const uint32_t qB = smem_u32(smem + kOffQ), doB = smem_u32(smem + kOffDO);
      const uint32_t dsB = smem_u32(smem + kOffDS);
      auto issue_st = [&](int i) {  // S^T(i) and dP^T(i) into their TMEM buffers
        const int st = i & 1;
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          mma_ss(tmem + kTS + st * BQ, kdesc(kA, k, kKBox), kdesc(qB + st * kQTile, k, kQBox),
                 idST, k > 0);
        mma_commit(bar_s_full + st);
      };
      auto issue_dp = [&](int i) {
        const int st = i & 1;
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          mma_ss(tmem + kTdP, kdesc(vA, k, kKBox), kdesc(doB + st * kQTile, k, kQBox), idST,
                 k > 0);
        mma_commit(bar_dp_full);
      };
      bool ok = mbar_wait(bar_kv, 0, limit, p.status);
      if (ok && n > 0) {
        ok = mbar_wait(bar_q_full + 0, 0, limit, p.status);
        if (ok) {
          fence_after_sync();
          issue_st(0);
          issue_dp(0);
        }
      }
      for (int i = 0; ok && i < n; ++i) {
        const int st = i & 1;
        if (i + 1 < n) {
          if (!mbar_wait(bar_q_full + ((i + 1) & 1), ((i + 1) >> 1) & 1, limit, p.status)) break;
          fence_after_sync();
          issue_st(i + 1);
        }
        if (!mbar_wait(bar_p_full, i & 1, limit, p.status)) break;
        fence_after_sync();
#pragma unroll
        for (int k = 0; k < BQ / 16; ++k)  // dV += P^T dO
          mma_ts(tmem + kTdV, tmem + kTS + st * BQ + k * 8, mndesc(doB + st * kQTile, k, kQBox),
                 idKV, (i == 0 && k == 0) ? 0u : 1u);
        if (!mbar_wait(bar_ds_full, i & 1, limit, p.status)) break;
        fence_after_sync();
#pragma unroll
        for (int k = 0; k < BQ / 16; ++k)  // dK += dS^T Q
          mma_ts(tmem + kTdK, tmem + kTdP + k * 8, mndesc(qB + st * kQTile, k, kQBox), idKV,
                 (i == 0 && k == 0) ? 0u : 1u);
        mma_commit(bar_q_empty + st);
        if (i > 0 && !mbar_wait(bar_dq_empty, (i - 1) & 1, limit, p.status)) break;
        fence_after_sync();
#pragma unroll
        for (int k = 0; k < BK / 16; ++k)  // dQ^T = K^T dS^T
          mma_ss(tmem + kTdQ, mndesc(kA, k, kKBox), mndesc(dsB, k, kDSBytes), idDQ, k > 0);
        mma_commit(bar_dq_full);
        mma_commit(bar_ds_empty);
        if (i + 1 < n) issue_dp(i + 1);
      }
      mma_commit(bar_done);
    }
  } else {
    regs_inc<kRegsMath>();
    const int lane_base = (warp & 3) * 32;
    const uint32_t tl = (uint32_t)lane_base << 16;
    if (warp < 4) {
      // ---------------- per-key math ----------------
      const int64_t key = i0 + lane_base + lane;
      const bool key_live = key < L;
      const int64_t tk = key_live ? lay.pos(s, key) : INT64_MAX;
      int i = 0;
      bool ok = true;
      for (int hh = 0; hh < group && ok; ++hh) {
        const int h = g * group + hh;
        for (int step = 0; step < nranks && ok; ++step) {
          const int r = rank_of(step);
          const int64_t q0 = p.ring ? (int64_t)r * L : 0;
          // queries of rank r before this key (causal: they do not see it)
          const int64_t hidden = !p.causal ? 0 : (key_live ? lay.visible_count(r, tk - 1) : L);
          for (int t = first_tile(r); t < qtiles; ++t, ++i) {
            const int st = i & 1;
            const int64_t j0 = (int64_t)t * BQ;
            // stage LSE * log2(e) and D of the 64 queries (0 past the shard end)
            {
              const int c = threadIdx.x & 63;
              const int which = threadIdx.x >> 6;  // 0: lse, 1: delta
              const int64_t j = j0 + c;
              float v = 0.f;
              if (j < L) {
                const int64_t idx = ((int64_t)b * p.Hq + h) * p.lse_ld + q0 + j;
                v = which == 0 ? p.lse[idx] * kLog2e : p.delta[idx];
              }
              vec[(st * 2 + which) * BQ + c] = v;
              mbar_arrive(bar_vec + st);
              if (!__all_sync(0xffffffffu, mbar_wait(bar_vec + st, (i >> 1) & 1, limit, p.status))) {
                ok = false;
                break;
              }
            }
            const float* lse2 = vec + (st * 2 + 0) * BQ;
            const float* dd = vec + (st * 2 + 1) * BQ;
            // visible query columns: [lo, hi)
            const int lo = (int)LayoutMap::clamp64(hidden - j0, 0, BQ);
            const int hi = key_live ? (int)LayoutMap::min64(L - j0, BQ) : 0;
            if (!__all_sync(0xffffffffu, mbar_wait(bar_s_full + st, (i >> 1) & 1, limit, p.status))) {
              ok = false;
              break;
            }
            fence_after_sync();
            float pt[BQ];
            {
              uint32_t v[32];
#pragma unroll
              for (int c = 0; c < BQ / 32; ++c) {
                tmem_ld32(tmem + tl + kTS + st * BQ + c * 32, v);
                tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < 32; ++x) {
                  const int col = c * 32 + x;
                  const float e = ex2(fmaf(__uint_as_float(v[x]), p.scale_log2, -lse2[col]));
                  pt[col] = (col >= lo && col < hi) ? e : 0.f;
                }
              }
              uint32_t pk[32];
#pragma unroll
              for (int x = 0; x < BQ / 2; ++x) pk[x] = pack_bf16(pt[2 * x], pt[2 * x + 1]);
              tmem_st32(tmem + tl + kTS + st * BQ, pk);
              tmem_wait_st();
            }
            fence_before_sync();
            mbar_arrive(bar_p_full);
            if (!__all_sync(0xffffffffu, mbar_wait(bar_dp_full, i & 1, limit, p.status))) {
              ok = false;
              break;
            }
            fence_after_sync();
            uint32_t dsk[BQ / 2];
            {
              uint32_t v[32];
#pragma unroll
              for (int c = 0; c < BQ / 32; ++c) {
                tmem_ld32(tmem + tl + kTdP + c * 32, v);
                tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < 32; x += 2) {
                  const int col = c * 32 + x;
                  const float d0 = pt[col] * (__uint_as_float(v[x]) - dd[col]);
                  const float d1 = pt[col + 1] * (__uint_as_float(v[x + 1]) - dd[col + 1]);
                  dsk[col / 2] = pack_bf16(d0, d1);
                }
              }
              tmem_st32(tmem + tl + kTdP, dsk);
            }
            // dS^T row into smem for the dQ^T MMA (SW128: 16-byte chunk c of
            // row k lands at chunk c ^ (k & 7) of its 128-byte row)
            if (!__all_sync(0xffffffffu, i == 0 || mbar_wait(bar_ds_empty, (i - 1) & 1, limit, p.status))) {
              ok = false;
              break;
            }
            {
              const int krow = lane_base + lane;
              uint4* row = reinterpret_cast<uint4*>(smem + kOffDS + krow * 128);
#pragma unroll
              for (int c = 0; c < 8; ++c)
                row[c ^ (krow & 7)] = make_uint4(dsk[4 * c], dsk[4 * c + 1], dsk[4 * c + 2], dsk[4 * c + 3]);
            }
            fence_proxy_async_smem();
            tmem_wait_st();
            fence_before_sync();
            mbar_arrive(bar_ds_full);
          }
        }
      }
      // ---------------- dK epilogue ----------------
      if (__all_sync(0xffffffffu, ok && mbar_wait(bar_done, 0, limit, p.status))) {
        fence_after_sync();
        const int64_t krow = (p.ring ? (int64_t)s * L : 0) + key;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tmem + tl + kTdK + c * 32, v);
          tmem_wait_ld();
          if (!key_live) continue;
          if (p.accumulate) {
            float* dst = reinterpret_cast<float*>(p.dk) + b * p.dk_sb + krow * p.dk_sn +
                         (int64_t)g * p.dk_sh + c * 32;
#pragma unroll
            for (int x = 0; x < 32; ++x) dst[x] += n > 0 ? __uint_as_float(v[x]) * p.scale : 0.f;
          } else {
            uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.dk) +
                                                  b * p.dk_sb + krow * p.dk_sn + (int64_t)g * p.dk_sh +
                                                  c * 32);
#pragma unroll
            for (int x = 0; x < 4; ++x) {
              float f[8];
#pragma unroll
              for (int y = 0; y < 8; ++y) f[y] = n > 0 ? __uint_as_float(v[8 * x + y]) * p.scale : 0.f;
              dst[x] = make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]),
                                  pack_bf16(f[6], f[7]));
            }
          }
        }
      }
    } else {
      // ---------------- dQ^T readout: lane = head-dim column ----------------
      const int col = lane_base + lane;
      int i = 0;
      bool ok = true;
      for (int hh = 0; hh < group && ok; ++hh) {
        const int h = g * group + hh;
        for (int step = 0; step < nranks && ok; ++step) {
          const int r = rank_of(step);
          const int64_t q0 = p.ring ? (int64_t)r * L : 0;
          for (int t = first_tile(r); t < qtiles; ++t, ++i) {
            if (!__all_sync(0xffffffffu, mbar_wait(bar_dq_full, i & 1, limit, p.status))) {
              ok = false;
              break;
            }
            fence_after_sync();
            uint32_t v0[32], v1[32];
            tmem_ld32(tmem + tl + kTdQ, v0);
            tmem_ld32(tmem + tl + kTdQ + 32, v1);
            tmem_wait_ld();
            fence_before_sync();
            mbar_arrive(bar_dq_empty);
            const int64_t j0 = (int64_t)t * BQ;
            float* base = p.dq + b * p.dq_sb + (int64_t)h * p.dq_sh + (q0 + j0) * p.dq_sn + col;
            const int nq = (int)LayoutMap::min64(L - j0, BQ);
#pragma unroll
            for (int x = 0; x < 32; ++x)
              if (x < nq) atomicAdd(base + x * p.dq_sn, __uint_as_float(v0[x]) * p.scale);
#pragma unroll
            for (int x = 0; x < 32; ++x)
              if (32 + x < nq) atomicAdd(base + (32 + x) * p.dq_sn, __uint_as_float(v1[x]) * p.scale);
          }
        }
      }
      // ---------------- dV epilogue: lane = key ----------------
      if (__all_sync(0xffffffffu, ok && mbar_wait(bar_done, 0, limit, p.status))) {
        fence_after_sync();
        const int64_t key = i0 + lane_base + lane;
        const bool key_live = key < L;
        const int64_t krow = (p.ring ? (int64_t)s * L : 0) + key;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tmem + tl + kTdV + c * 32, v);
          tmem_wait_ld();
          if (!key_live) continue;
          if (p.accumulate) {
            float* dst = reinterpret_cast<float*>(p.dv) + b * p.dv_sb + krow * p.dv_sn +
                         (int64_t)g * p.dv_sh + c * 32;
#pragma unroll
            for (int x = 0; x < 32; ++x) dst[x] += n > 0 ? __uint_as_float(v[x]) : 0.f;
          } else {
            uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.dv) +
                                                  b * p.dv_sb + krow * p.dv_sn + (int64_t)g * p.dv_sh +
                                                  c * 32);
#pragma unroll
            for (int x = 0; x < 4; ++x) {
              float f[8];
#pragma unroll
              for (int y = 0; y < 8; ++y) f[y] = n > 0 ? __uint_as_float(v[8 * x + y]) : 0.f;
              dst[x] = make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]),
                                  pack_bf16(f[6], f[7]));
            }
          }
        }
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

}  // namespace

rm_status tc_bwd(const AttnArgs& a, int q_rank, int kv_rank, cudaStream_t stream) {
  if (a.B == 0 || a.N == 0) return RM_OK;
  if (a.d != D) return RM_ERR_UNSUPPORTED;
  const bool ring = q_rank < 0;
  const int64_t L = a.N / a.P;
  const int shards = ring ? a.P : 1;
  CUtensorMap mq, mk, mv, mdo;
  if (encode_operand_map(&mq, a.q, a.B, shards, L, a.Hq, a.d, 64, BQ) != RM_OK ||
      encode_operand_map(&mk, a.k, a.B, shards, L, a.Hkv, a.d, 64, BK) != RM_OK ||
      encode_operand_map(&mv, a.v, a.B, shards, L, a.Hkv, a.d, 64, BK) != RM_OK ||
      encode_operand_map(&mdo, a.dout, a.B, shards, L, a.Hq, a.d, 64, BQ) != RM_OK)
    return RM_ERR_CUDA;
  BwdParams p;
  p.B = a.B;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.P = a.P;
  p.layout = a.layout;
  p.causal = a.causal;
  p.N = a.N;
  p.L = L;
  p.scale = a.scale;
  p.scale_log2 = a.scale * kLog2e;
  p.ring = ring ? 1 : 0;
  p.q_rank = q_rank;
  p.kv_rank = kv_rank;
  p.lse = a.lse_in;
  p.delta = a.delta;
  p.lse_ld = a.lse_ld;
  p.dq = reinterpret_cast<float*>(a.dq.ptr);
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
  p.status = a.status;
  p.wait_limit = tc_wait_limit();
  dim3 grid((unsigned)ceil_div(L, BK), (unsigned)a.Hkv, (unsigned)(ring ? a.B * a.P : a.B));
  if (cudaFuncSetAttribute(tc_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) !=
      cudaSuccess)
    return RM_ERR_CUDA;
  tc_bwd_kernel<<<grid, kThreads, kSmem, stream>>>(mq, mk, mv, mdo, p);
  return cudaGetLastError() == cudaSuccess ? RM_OK : RM_ERR_CUDA;
}

}  // namespace rm
