// Forward attention on the sm_100a tensor cores (bf16 in, fp32 accumulate).
//
// One CTA owns two 128-row query tiles, A and B, that read the same KV head:
// two query heads of one GQA group on the same rows when the group size is
// even, else two consecutive row tiles of one head.  It walks the KV tiles
// the tiles may see -- in ring mode over every KV shard in ring order
// (r, r-1, ...; Mosaic, "How Ring Attention Works") -- and keeps the running
// softmax state (m, l, O) across tiles and shards, so the LSE merge of the
// per-shard partials happens implicitly in the rescaling (Ring Attention &
// Friends, "Tiling with the Softmax Rescaling Trick").
//
// Warp roles (384 threads, three warpgroups):
//   warps 0-3  softmax for tile A (one thread per TMEM lane = query row)
//   warps 4-7  softmax for tile B
//   warp  8    TMA producer: Q once, then K / V tiles into a 2-stage ring
//   warp  9    MMA issuer (one thread): S = Q K^T into TMEM, O += P V with P
//              read from TMEM (written over S by the softmax warps)
//   warps 10-11 idle
// Register split: the block launches at 168 registers a thread (64512 in
// all); the softmax warpgroups grow to 216 and the third shrinks to 64:
// 2*128*216 + 128*64 = 63488 <= 64512.
// TMEM (512 columns): S_A [0,128), S_B [128,256), O_A, O_B after them.
// While softmax A works on S_A(j), the tensor core runs PV_B(j-1) / S_B(j),
// and vice versa.
//
// Causal masking: positions are increasing in the local index for every
// layout, so the keys of shard s visible to a query form a prefix of the
// shard; tiles past the last row's prefix are never loaded, and only tiles
// that cut a row's prefix apply an element mask.
#include <cudaTypedefs.h>
#include <stdlib.h>

#include <mutex>

#include "tc_attn.h"
#include "exp2_poly.cuh"
#include "tc_common.cuh"

namespace rm {

namespace {

using namespace tc;

constexpr int kBM = 128;  // query rows per tile (TMEM lanes)
constexpr int kBN = 128;  // keys per KV tile
constexpr int kStages = 2;
constexpr int kThreads = 384;
constexpr int kRegsSoftmax = 216;
constexpr int kRegsOther = 64;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsOther <= kThreads * 168, "register split");
constexpr int kWarpTma = 8;
constexpr int kWarpMma = 9;
constexpr long long kDefaultWaitLimit = 4000000000LL;  // clock cycles (~2 s)

template <int DP>
struct FwdCfg {
  static constexpr int kBoxCols = DP >= 64 ? 64 : DP;  // elements per TMA box row (<= 128 B)
  static constexpr int kBoxes = DP / kBoxCols;         // boxes per 128-row tile
  static constexpr int kRowBytes = kBoxCols * 2;
  static constexpr uint32_t kSwz = kRowBytes == 128 ? kSwizzle128B : kSwizzle64B;
  static constexpr int kBoxBytes = kBM * kRowBytes;
  static constexpr int kTileBytes = kBM * DP * 2;
  static constexpr int kQ0 = 0;
  static constexpr int kQ1 = kTileBytes;
  static constexpr int kK = 2 * kTileBytes;
  static constexpr int kV = kK + kStages * kTileBytes;
  static constexpr int kBar = kV + kStages * kTileBytes;
  static constexpr int kSmem = kBar + 256 + 1024;  // barriers + 1 KB alignment slack
  static constexpr uint32_t kS0 = 0, kS1 = 128, kO0 = 256, kO1 = 256 + DP;
  static_assert(kO1 + DP <= 512, "TMEM budget");
};

struct FwdParams {
  int B, Hq, Hkv, d, P, layout, causal;
  int Pk;     // KV shards: P, except for one (query chunk, KV chunk) tile of a rectangular grid
  int64_t Lk;  // N / Pk
  int64_t N, L;
  float scale_log2;  // softmax scale * log2(e)
  int ring, q_rank, kv_rank;
  int head_pairs;
  int head_block;  // head units per grid block (see grid_place)
  int global_order;  // ring operands, O and LSE in global token order
  const int* cu_seqlens;  // packing boundaries (device) or null
  int num_segments;
  const int* seq_lens;    // right-padding lengths (device) or null
  int seg_div;            // batch entries per seq_lens entry
  void* o;
  int64_t o_sb, o_sn, o_sh;
  int o_f32;
  float* lse;
  int64_t lse_ld;
  unsigned int* status;
  long long wait_limit;
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// K-major operand tile (Q or K): descriptor for UMMA K-step k (16 elements).
template <int DP>
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile_addr, int k) {
  using C = FwdCfg<DP>;
  const int col = k * 16;
  const uint32_t addr = tile_addr + (col / C::kBoxCols) * C::kBoxBytes + (col % C::kBoxCols) * 2;
  return smem_desc(addr, 16, 8 * C::kRowBytes, C::kSwz);
}
// Byte offset of K-step k (columns [16k, 16k + 16)) within a K-major tile:
// kmajor_desc(tile, k) and kmajor_desc(tile, 0) differ by kmajor_off(k) >> 4
// in the address field of the low word.
template <int DP>
__host__ __device__ constexpr uint32_t kmajor_off(int k) {
  using C = FwdCfg<DP>;
  return (uint32_t)((k * 16 / C::kBoxCols) * C::kBoxBytes + (k * 16 % C::kBoxCols) * 2);
}
// A descriptor from its low word and a high word that does not depend on the
// address (the stride / swizzle fields).
__device__ __forceinline__ uint64_t desc_of(uint32_t hi, uint32_t lo) {
  return ((uint64_t)hi << 32) | lo;
}
// V tile as the MN-major B operand of O += P V: K-step k covers kv rows
// [16k, 16k+16); the d axis is split over boxes kBoxBytes apart.
template <int DP>
__device__ __forceinline__ uint64_t v_desc(uint32_t tile_addr, int k) {
  using C = FwdCfg<DP>;
  return smem_desc(tile_addr + k * 16 * C::kRowBytes, C::kBoxBytes, 8 * C::kRowBytes, C::kSwz);
}

// Pairs (of the 16 in each 32-column chunk of a row) whose exponentials use
// exp2_fma2 instead of the SFU: for d <= 64 the SFU outweighs the tensor
// work (on the d = 24 tabular rows 6 of 16 pairs measured 4.6% faster than
// none; with the MMA thread's cheaper descriptors 4 measured 5.0% faster than
// 6, and 8 slower); for d = 128 every split measured slower, so all go to
// the SFU.
template <int DP>
constexpr int kEmuPairs = DP >= 128 ? 0 : 4;

// P of a tile is handed to the PV MMA in kPParts parts (each kBN / kPParts
// keys, its own barrier), so O += P V starts on the first keys while the
// softmax is still exponentiating the rest.
constexpr int kPParts = 2;

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

template <int DP>
__global__ void __launch_bounds__(kThreads, 1)
    tc_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using C = FwdCfg<DP>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBar);
  static_assert(kStages == 2, "the barrier slots below assume a 2-stage K/V ring");
  uint64_t* bar_q = bars + 0;
  uint64_t* bar_k_full = bars + 1;    // [kStages]
  uint64_t* bar_v_full = bars + 3;    // [kStages]
  uint64_t* bar_kv_empty = bars + 5;  // [kStages]
  uint64_t* bar_s_full = bars + 7;    // [2] per query tile
  uint64_t* bar_p_full = bars + 9;    // [2] per query tile
  uint64_t* bar_o_done = bars + 11;
  uint64_t* bar_drain = bars + 12;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 13);
  // [2][kPParts - 1]: P of the first parts of a tile written (the last part is bar_p_full)
  uint64_t* bar_p_part = bars + 14;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const LayoutMap lay = make_layout(p.layout, p.N, p.P);
  // keys of shard s at global positions <= t: the layout's count, or for a
  // tile of a rectangular grid (contiguous chunks of Lk keys) the chunk's
  auto kvis = [&](int s, int64_t t) -> int64_t {
    return p.Pk == p.P ? lay.visible_count(s, t)
                       : LayoutMap::clamp64(t - (int64_t)s * p.Lk + 1, 0, p.Lk);
  };
  const int64_t L = p.L;
  // grid: (row unit in order of decreasing work x head unit, head block, batch);
  // a head unit is a head pair (heads 2x, 2x+1) or one head
  const int b = blockIdx.z;
  const int urows = p.head_pairs ? kBM : 2 * kBM;  // query rows of one unit
  int c, hu;
  if (!grid_place(p.head_block, p.head_pairs ? p.Hq / 2 : p.Hq, c, hu)) return;
  int r, unit;
  {
    const int T = (int)((L + urows - 1) / urows);
    if (!p.ring) {
      r = p.q_rank;
      unit = p.causal ? T - 1 - c : c;  // later rows see more keys: start them first
    } else if (p.causal) {
      lay.ordered_tile(T, urows, c, true, r, unit);
    } else {
      r = c / T;
      unit = c - r * T;
    }
  }
  int hA, hB;
  int64_t rowA, rowB;
  if (p.head_pairs) {
    hA = 2 * hu;
    hB = hA + 1;
    rowA = rowB = (int64_t)unit * kBM;
  } else {
    hA = hB = hu;
    rowA = (int64_t)unit * 2 * kBM;
    rowB = rowA + kBM;
  }
  const int g = hA / (p.Hq / p.Hkv);
  RingRows rows;
  rows.lay = lay;
  rows.global = p.global_order;
  // TMA (row, shard) coordinates of local row j of rank `rank` (a single
  // shard: row j of the one shard)
  auto tma_rs = [&](int rank, int64_t j, int& crow, int& cshard) {
    if (p.ring) {
      rows.tma(rank, j, crow, cshard);
    } else {
      crow = (int)j;
      cshard = 0;
    }
  };
  const int64_t last_row = min((p.head_pairs ? rowA : rowB) + kBM - 1, L - 1);
  const int64_t t_last = lay.pos(r, last_row);
  const Segs sg{p.cu_seqlens, p.num_segments, p.seq_lens, p.N, p.seg_div};
  // global span of the keys any row of the CTA may see (bounds are monotone
  // in the row, so its first and last rows give them)
  int64_t span_first, span_last;
  {
    int64_t f, l;
    sg.query_span(b, lay.pos(r, min(rowA, L - 1)), p.causal, span_first, l);
    sg.query_span(b, t_last, p.causal, f, span_last);
  }
  const int nsteps = p.ring ? p.P : 1;
  const long long limit = p.wait_limit;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar_k_full + s, 1);
      mbar_init(bar_v_full + s, 1);
      mbar_init(bar_kv_empty + s, 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar_s_full + x, 1);
      for (int q = 0; q + 1 < kPParts; ++q) mbar_init(bar_p_part + x * (kPParts - 1) + q, 128);
      mbar_init(bar_p_full + x, 128);
    }
    mbar_init(bar_o_done, 1);
    mbar_init(bar_drain, 1);
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

  // KV shard of ring step `step`, and how many of its keys the CTA may see.
  auto shard_of = [&](int step) { return p.ring ? ((r - step) % p.P + p.P) % p.P : p.kv_rank; };
  // key tiles [tile_begin(s), tile_end(s)) of shard s hold every key the CTA may see
  auto tile_begin = [&](int s) -> int {
    return (int)(kvis(s, span_first - 1) / kBN);
  };
  auto tile_end = [&](int s) -> int {
    return (int)((kvis(s, span_last) + kBN - 1) / kBN);
  };

  if (warp >= 8) {
    regs_dec<kRegsOther>();
  if (warp == kWarpTma) {
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      int qrA, qsA, qrB, qsB;  // TMA (row, shard) coordinates of the two query tiles
      tma_rs(r, rowA, qrA, qsA);
      tma_rs(r, rowB, qrB, qsB);
      mbar_arrive_expect_tx(bar_q, 2 * C::kTileBytes);
#pragma unroll
      for (int x = 0; x < C::kBoxes; ++x) {
        tma_load_5d(smem + C::kQ0 + x * C::kBoxBytes, &tmQ, bar_q, x * C::kBoxCols, hA, qrA, qsA, b);
        tma_load_5d(smem + C::kQ1 + x * C::kBoxBytes, &tmQ, bar_q, x * C::kBoxCols, hB, qrB, qsB, b);
      }
      int j = 0;
      bool ok = true;
      for (int step = 0; step < nsteps && ok; ++step) {
        const int s = shard_of(step);
        const int te = tile_end(s);
        for (int t = tile_begin(s); t < te; ++t, ++j) {
          const int st = j & 1;
          int kr, ks;
          tma_rs(s, (int64_t)t * kBN, kr, ks);
          if (j >= kStages && !mbar_wait(bar_kv_empty + st, ((j >> 1) - 1) & 1, limit, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar_k_full + st, C::kTileBytes);
#pragma unroll
          for (int x = 0; x < C::kBoxes; ++x)
            tma_load_5d(smem + C::kK + st * C::kTileBytes + x * C::kBoxBytes, &tmK,
                        bar_k_full + st, x * C::kBoxCols, g, kr, ks, b);
          mbar_arrive_expect_tx(bar_v_full + st, C::kTileBytes);
#pragma unroll
          for (int x = 0; x < C::kBoxes; ++x)
            tma_load_5d(smem + C::kV + st * C::kTileBytes + x * C::kBoxBytes, &tmV,
                        bar_v_full + st, x * C::kBoxCols, g, kr, ks, b);
        }
      }
      // drain: the last load issued into each stage has landed before exit
      for (int st = 0; st < kStages && j > st; ++st) {
        const int uses = (j - st + 1) / 2;  // loads issued into stage st
        mbar_wait(bar_k_full + st, (uses - 1) & 1, limit, p.status);
        mbar_wait(bar_v_full + st, (uses - 1) & 1, limit, p.status);
      }
    }
  } else if (warp == kWarpMma) {
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(kBM, kBN, 0, 0);
      constexpr uint32_t idO = idesc_bf16(kBM, DP, 0, 1);
      const uint32_t q0 = smem_u32(smem + C::kQ0), q1 = smem_u32(smem + C::kQ1);
      const uint32_t kbase = smem_u32(smem + C::kK), vbase = smem_u32(smem + C::kV);
      int n = 0;
      for (int step = 0; step < nsteps; ++step) {
        const int s = shard_of(step);
        n += max(0, tile_end(s) - tile_begin(s));
      }
      // descriptors as a constant high word and a low word per tile: a K-step
      // adds a constant to the low word (the address field does not carry:
      // shared memory is below 256 KB)
      const uint32_t hiK = (uint32_t)(kmajor_desc<DP>(q0, 0) >> 32);
      const uint32_t hiV = (uint32_t)(v_desc<DP>(vbase, 0) >> 32);
      const uint32_t loK0 = (uint32_t)kmajor_desc<DP>(kbase, 0);
      const uint32_t loV0 = (uint32_t)v_desc<DP>(vbase, 0);
      auto issue_s = [&](uint32_t qaddr, uint32_t scol, int st) {
        const uint32_t lq = (uint32_t)kmajor_desc<DP>(qaddr, 0);
        const uint32_t lk = loK0 + st * (C::kTileBytes >> 4);
#pragma unroll
        for (int k = 0; k < DP / 16; ++k)
          mma_ss(tmem + scol, desc_of(hiK, lq + (kmajor_off<DP>(k) >> 4)),
                 desc_of(hiK, lk + (kmajor_off<DP>(k) >> 4)), idS, k > 0);
      };
      // O += P V over the keys of one part of the tile (kBN / kPParts keys):
      // each part starts as soon as the softmax has written it
      auto issue_pv_part = [&](uint32_t scol, uint32_t ocol, int st, bool first, int part) {
        const uint32_t lv = loV0 + st * (C::kTileBytes >> 4);
        constexpr int kSteps = kBN / 16 / kPParts;
#pragma unroll
        for (int kk = 0; kk < kSteps; ++kk) {
          const int k = part * kSteps + kk;
          mma_ts(tmem + ocol, tmem + scol + k * 8, desc_of(hiV, lv + ((k * 16 * C::kRowBytes) >> 4)),
                 idO, (first && k == 0) ? 0u : 1u);
        }
      };
      auto issue_pv = [&](int x, uint32_t scol, uint32_t ocol, int st, int j) -> bool {
#pragma unroll
        for (int part = 0; part < kPParts; ++part) {
          uint64_t* bar = part + 1 < kPParts ? bar_p_part + x * (kPParts - 1) + part
                                             : bar_p_full + x;
          if (!mbar_wait(bar, j & 1, limit, p.status)) return false;
          fence_after_sync();
          issue_pv_part(scol, ocol, st, j == 0, part);
        }
        return true;
      };
      bool ok = mbar_wait(bar_q, 0, limit, p.status);
      if (ok && n > 0) {
        ok = mbar_wait(bar_k_full + 0, 0, limit, p.status);
        if (ok) {
          fence_after_sync();
          issue_s(q0, C::kS0, 0);
          mma_commit(bar_s_full + 0);
          issue_s(q1, C::kS1, 0);
          mma_commit(bar_s_full + 1);
        }
      }
      for (int j = 0; ok && j < n; ++j) {
        const int st = j & 1;
        const int nx = (j + 1) & 1;
        if (!mbar_wait(bar_v_full + st, (j >> 1) & 1, limit, p.status)) break;
        if (!issue_pv(0, C::kS0, C::kO0, st, j)) break;
        if (j + 1 < n) {
          if (!mbar_wait(bar_k_full + nx, ((j + 1) >> 1) & 1, limit, p.status)) break;
          fence_after_sync();
          issue_s(q0, C::kS0, nx);
          mma_commit(bar_s_full + 0);
        }
        if (!issue_pv(1, C::kS1, C::kO1, st, j)) break;
        mma_commit(bar_kv_empty + st);
        if (j + 1 < n) {
          issue_s(q1, C::kS1, nx);
          mma_commit(bar_s_full + 1);
        }
      }
      mma_commit(bar_o_done);
      // every MMA issued above has completed before TMEM is released
      mma_commit(bar_drain);
      mbar_wait(bar_drain, 0, limit, p.status);
    }
  }
  } else {
    regs_inc<kRegsSoftmax>();
    // ---------------- softmax warpgroups ----------------
    const int X = warp >> 2;
    const int lane_base = (warp & 3) * 32;
    const int64_t row = (X ? rowB : rowA) + lane_base + lane;
    const int h = X ? hB : hA;
    const bool live = row < L;
    const int64_t tq = live ? lay.pos(r, row) : -1;
    const uint32_t tS = tmem + ((uint32_t)lane_base << 16) + (X ? C::kS1 : C::kS0);
    const uint32_t tO = tmem + ((uint32_t)lane_base << 16) + (X ? C::kO1 : C::kO0);
    uint64_t* s_full = bar_s_full + X;
    uint64_t* p_part = bar_p_part + X * (kPParts - 1);
    uint64_t* p_full = bar_p_full + X;
    float m = -INFINITY;  // running max of the scaled scores, log2 units
    float l = 0.f;        // running row sum (relative to m)
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
        // all lanes leave together, so the warp-collective tcgen05.ld / st
        // below always run converged
        if (!__all_sync(0xffffffffu, mbar_wait(s_full, j & 1, limit, p.status))) {
          ok = false;
          break;
        }
        fence_after_sync();
        float sc[kBN];
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tS + c * 32, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) sc[c * 32 + i] = __uint_as_float(v[i]);
        }
        tmem_wait_ld();
        const int64_t c_lo = row_lo - (int64_t)t * kBN, c_hi = row_hi - (int64_t)t * kBN;
        if (c_lo > 0 || c_hi < kBN) {
#pragma unroll
          for (int c = 0; c < kBN; ++c)
            if (c < c_lo || c >= c_hi) sc[c] = -INFINITY;
        }
        // row max: 8 independent chains of three-input max (a single two-input
        // chain is 128 dependent steps)
        float mx8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float a = max3f(sc[e], sc[e + 8], sc[e + 16]);
#pragma unroll
          for (int j = 3; j + 1 < kBN / 8; j += 2) a = max3f(a, sc[e + 8 * j], sc[e + 8 * j + 8]);
          mx8[e] = (kBN / 8) % 2 == 0 ? fmaxf(a, sc[e + kBN - 8]) : a;
        }
        const float mx = max3f(max3f(mx8[0], mx8[1], mx8[2]), max3f(mx8[3], mx8[4], mx8[5]),
                               fmaxf(mx8[6], mx8[7]));
        const float m_tile = mx * p.scale_log2;
        // Lazy rescale: the reference max only moves when it grows by more
        // than 8 (a factor 256), so O is rescaled rarely; p <= 256 otherwise.
        const bool grow = m_tile > m + 8.0f;
        const float m_new = grow ? m_tile : m;
        const bool need = grow && j > 0 && m != -INFINITY;
        if (__any_sync(0xffffffffu, need)) {
          const float f = need ? ex2(m - m_new) : 1.0f;
#pragma unroll
          for (int c = 0; c < DP / 32; ++c) {
            uint32_t v[32];
            tmem_ld32(tO + c * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * f);
            tmem_st32(tO + c * 32, v);
          }
        }
        if (grow) {
          l *= (m == -INFINITY) ? 0.f : ex2(m - m_new);
          m = m_new;
        }
        const float m_use = (m == -INFINITY) ? 0.f : m;
        // scores to exponents two at a time (packed fp32 FMA), partial row
        // sums two at a time in two independent chains (packed fp32 add)
        const float2 scale2 = make_float2(p.scale_log2, p.scale_log2);
        const float2 neg_m2 = make_float2(-m_use, -m_use);
        float2 l2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float2 x2 = __ffma2_rn(make_float2(sc[c * 32 + 2 * i], sc[c * 32 + 2 * i + 1]),
                                         scale2, neg_m2);
            const float2 p2 = i >= 16 - kEmuPairs<DP> ? exp2_fma2(x2)
                                                      : make_float2(ex2(x2.x), ex2(x2.y));
            l2[i & 1] = __fadd2_rn(l2[i & 1], p2);
            pk[i] = pack_bf16(p2.x, p2.y);
          }
          tmem_st16(tS + c * 16, pk);
          constexpr int kChunksPerPart = kBN / 32 / kPParts;
          if ((c + 1) % kChunksPerPart == 0 && c + 1 < kBN / 32) {
            // a part of P is written: the PV MMA may start on its keys
            tmem_wait_st();
            fence_before_sync();
            mbar_arrive(p_part + (c + 1) / kChunksPerPart - 1);
          }
        }
        l += (l2[0].x + l2[0].y) + (l2[1].x + l2[1].y);
        tmem_wait_st();
        fence_before_sync();
        mbar_arrive(p_full);
      }
    }
    // ---------------- epilogue: O / l, LSE ----------------
    if (__all_sync(0xffffffffu, ok && mbar_wait(bar_o_done, 0, limit, p.status))) {
      fence_after_sync();
      if (m == -INFINITY) l = 0.f;  // no visible key: only exp2_fma2's 2^-125 floors in l
      const float inv = l > 0.f ? 1.0f / l : 0.f;
      const float lse = l > 0.f ? (((m == -INFINITY) ? 0.f : m) + __log2f(l)) * kLn2 : -INFINITY;
      const int64_t orow = p.ring ? rows.row(r, row) : row;
      char* obase = reinterpret_cast<char*>(p.o) +
                    (b * p.o_sb + orow * p.o_sn + (int64_t)h * p.o_sh) * (p.o_f32 ? 4 : 2);
#pragma unroll
      for (int c = 0; c < DP / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tO + c * 32, v);
        tmem_wait_ld();
        if (live) {
          if (p.o_f32) {
            float4* dst = reinterpret_cast<float4*>(obase) + c * 8;
#pragma unroll
            for (int i = 0; i < 8; ++i)
              if (c * 32 + 4 * i < p.d)
                dst[i] = make_float4(__uint_as_float(v[4 * i]) * inv, __uint_as_float(v[4 * i + 1]) * inv,
                                     __uint_as_float(v[4 * i + 2]) * inv,
                                     __uint_as_float(v[4 * i + 3]) * inv);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(obase) + c * 4;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              if (c * 32 + 8 * i >= p.d) continue;  // d = 24 stores 3 of the 4 vectors
              uint4 u;
              u.x = pack_bf16(__uint_as_float(v[8 * i + 0]) * inv, __uint_as_float(v[8 * i + 1]) * inv);
              u.y = pack_bf16(__uint_as_float(v[8 * i + 2]) * inv, __uint_as_float(v[8 * i + 3]) * inv);
              u.z = pack_bf16(__uint_as_float(v[8 * i + 4]) * inv, __uint_as_float(v[8 * i + 5]) * inv);
              u.w = pack_bf16(__uint_as_float(v[8 * i + 6]) * inv, __uint_as_float(v[8 * i + 7]) * inv);
              dst[i] = u;
            }
          }
        }
      }
      if (live) p.lse[((int64_t)b * p.Hq + h) * p.lse_ld + orow] = lse;
    }
  }
  fence_before_sync();
  __syncthreads();
  if (warp == kWarpMma) {
    fence_after_sync();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

}  // namespace

// A TMA view of a [B, N or L, H, d] bf16 operand with 5 coordinates
// (col, head, row, shard, batch).  view 0: [B, P', L, H, d] (P' = shards, 1
// for a single shard), row j of shard r at memory row r * L + j -- rank-major
// ring operands or one shard.  view 1 (global striped): the same dimensions
// with the row / shard strides swapped, row j of shard r at j * P + r.  view 2
// (global zigzag): [B, 2P, C, H, d], row j of chunk q at q * C + j.  Boxes of
// box_rows rows and box_cols columns; columns past d (head-dim padding) and
// rows past the row dimension are zero-filled by the TMA unit.
rm_status encode_operand_map(CUtensorMap* map, const rm_tensor& t, int B, int shards, int64_t L,
                             int H, int d, int box_cols, int box_rows, int view) {
  auto fn = encode_fn();
  if (!fn) return RM_ERR_CUDA;
  const int64_t sn = t.stride_n * 2;
  const int64_t sh = (H > 1 ? t.stride_h : d) * 2;
  const int64_t sb = (B > 1 ? t.stride_b : (int64_t)shards * L * t.stride_n) * 2;
  int64_t rows = L, nshard = shards, s_row = sn, s_shard = L * sn;
  if (view == 1) {  // striped: row j of shard r is global row j * P + r
    s_row = (int64_t)shards * sn;
    s_shard = sn;
  } else if (view == 2) {  // zigzag: 2P chunks of C = L / 2 rows
    rows = L / 2;
    nshard = 2 * (int64_t)shards;
    s_shard = rows * sn;
  }
  cuuint64_t dims[5] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)rows, (cuuint64_t)nshard,
                        (cuuint64_t)B};
  cuuint64_t strides[4] = {(cuuint64_t)sh, (cuuint64_t)s_row,
                           (cuuint64_t)(s_shard > 0 ? s_shard : 16), (cuuint64_t)(sb > 0 ? sb : 16)};
  cuuint32_t box[5] = {(cuuint32_t)box_cols, 1, (cuuint32_t)box_rows, 1, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const CUtensorMapSwizzle swz =
      box_cols * 2 == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  CUresult rc = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, t.ptr, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return rc == CUDA_SUCCESS ? RM_OK : RM_ERR_CUDA;
}

// The operand view (see encode_operand_map) of a ring or single-shard call.
int operand_view(const AttnArgs& a, bool ring) {
  if (!ring || !a.global_order) return 0;
  return a.layout == RM_LAYOUT_STRIPED ? 1 : a.layout == RM_LAYOUT_ZIGZAG ? 2 : 0;
}

rm_status encode_copy_map(CUtensorMap* map, const void* ptr, int esize, const int64_t (&dims)[5],
                          const int64_t (&strides)[4], const int (&box)[5]) {
  auto fn = encode_fn();
  if (!fn) return RM_ERR_CUDA;
  CUtensorMapDataType type;
  if (esize == 1) type = CU_TENSOR_MAP_DATA_TYPE_UINT8;
  else if (esize == 2) type = CU_TENSOR_MAP_DATA_TYPE_UINT16;
  else if (esize == 4) type = CU_TENSOR_MAP_DATA_TYPE_UINT32;
  else return RM_ERR_UNSUPPORTED;
  cuuint64_t gdim[5], gstr[4];
  cuuint32_t bx[5], estr[5] = {1, 1, 1, 1, 1};
  for (int i = 0; i < 5; ++i) {
    gdim[i] = (cuuint64_t)dims[i];
    bx[i] = (cuuint32_t)box[i];
  }
  for (int i = 0; i < 4; ++i) gstr[i] = (cuuint64_t)strides[i];
  CUresult rc = fn(map, type, 5, const_cast<void*>(ptr), gdim, gstr, bx, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return rc == CUDA_SUCCESS ? RM_OK : RM_ERR_CUDA;
}

bool tc_supported_head_dim(int d) { return d == 24 || d == 32 || d == 64 || d == 128; }

int tc_padded_head_dim(int d) { return d <= 32 ? 32 : d; }

long long tc_wait_limit() {
  static long long lim = [] {
    const char* e = getenv("RM_WAIT_LIMIT_CYCLES");
    long long v = e ? atoll(e) : 0;
    return v > 0 ? v : kDefaultWaitLimit;
  }();
  return lim;
}

template <int DP>
static rm_status launch_fwd(const AttnArgs& a, int q_rank, int kv_rank, cudaStream_t stream) {
  using C = FwdCfg<DP>;
  const bool ring = q_rank < 0;
  const int64_t L = a.N / a.P;
  const int Pk = ring ? a.P : kv_shards(a);
  const int64_t Lk = a.N / Pk;
  const int shards = ring ? a.P : 1;
  CUtensorMap mq, mk, mv;
  const int view = operand_view(a, ring);
  if (encode_operand_map(&mq, a.q, a.B, shards, L, a.Hq, a.d, C::kBoxCols, kBM, view) != RM_OK ||
      encode_operand_map(&mk, a.k, a.B, shards, Lk, a.Hkv, a.d, C::kBoxCols, kBN, view) != RM_OK ||
      encode_operand_map(&mv, a.v, a.B, shards, Lk, a.Hkv, a.d, C::kBoxCols, kBN, view) != RM_OK)
    return RM_ERR_CUDA;
  FwdParams p;
  p.B = a.B;
  p.d = a.d;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.P = a.P;
  p.Pk = Pk;
  p.Lk = Lk;
  p.layout = a.layout;
  p.causal = a.causal;
  p.N = a.N;
  p.L = L;
  p.scale_log2 = a.scale * kLog2e;
  p.ring = ring ? 1 : 0;
  p.q_rank = q_rank;
  p.kv_rank = kv_rank;
  p.head_pairs = ((a.Hq / a.Hkv) % 2 == 0) ? 1 : 0;
  p.global_order = ring ? a.global_order : 0;
  p.cu_seqlens = a.cu_seqlens;
  p.num_segments = a.num_segments;
  p.seq_lens = a.seq_lens;
  p.seg_div = a.seg_div > 1 ? a.seg_div : 1;
  p.o = a.o.ptr;
  p.o_sb = a.o.stride_b;
  p.o_sn = a.o.stride_n;
  p.o_sh = a.o.stride_h;
  p.o_f32 = a.o_f32;
  p.lse = a.lse;
  p.lse_ld = a.lse_ld;
  p.status = a.status;
  p.wait_limit = tc_wait_limit();
  const int units = p.head_pairs ? ceil_div(L, kBM) : ceil_div(L, 2 * kBM);
  if (a.B > 65535) return RM_ERR_UNSUPPORTED;  // grid.z
  const int hunits = p.head_pairs ? a.Hq / 2 : a.Hq;
  // a CTA streams K and V of its KV head, shared by the query heads of the group
  p.head_block = head_block((int64_t)a.N * a.d * 2 * 2 * a.Hkv / hunits, hunits);
  dim3 grid((unsigned)(units * shards * p.head_block), (unsigned)ceil_div(hunits, p.head_block),
            (unsigned)a.B);
  if (cudaFuncSetAttribute(tc_fwd_kernel<DP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::kSmem) != cudaSuccess)
    return RM_ERR_CUDA;
  ProfScope ps("tc_fwd_kernel", stream);
  tc_fwd_kernel<DP><<<grid, kThreads, C::kSmem, stream>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? RM_OK : RM_ERR_CUDA;
}

rm_status tc_fwd(const AttnArgs& a, int q_rank, int kv_rank, cudaStream_t stream) {
  if (a.B == 0 || a.N == 0) return RM_OK;
  switch (tc_padded_head_dim(a.d)) {
    case 32: return launch_fwd<32>(a, q_rank, kv_rank, stream);
    case 64: return launch_fwd<64>(a, q_rank, kv_rank, stream);
    case 128: return launch_fwd<128>(a, q_rank, kv_rank, stream);
  }
  return RM_ERR_UNSUPPORTED;
}

}  // namespace rm
