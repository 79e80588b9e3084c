// Shared device/host helpers of librm_attn.so (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/rm_attn.h"

namespace rm {

// ---- token layouts --------------------------------------------------------
// Global position of local token j of rank r (ringmaster "Layout":
// contiguous shard / head_tail balancer; Ring Attention & Friends, "Striped
// Attention").  L = N / P tokens per rank; C = N / (2P) zigzag chunk.
struct LayoutMap {
  int layout;   // rm_layout
  int P;
  int64_t L;
  int64_t C;

  __host__ __device__ __forceinline__ int64_t pos(int r, int64_t j) const {
    if (layout == RM_LAYOUT_CONTIGUOUS) return (int64_t)r * L + j;
    if (layout == RM_LAYOUT_STRIPED) return j * P + r;
    return j < C ? (int64_t)r * C + j : (int64_t)(2 * P - 1 - r) * C + (j - C);
  }

  // pos(r, j) is strictly increasing in j for every layout (the second
  // zigzag chunk, from (2P-1-r)*C, lies above the first, which ends at
  // (r+1)*C - 1), so under the causal rule the keys of shard s visible to a
  // query at global position t are a prefix of the shard: local keys
  // [0, visible_count(s, t)).
  __host__ __device__ __forceinline__ int64_t visible_count(int s, int64_t t) const {
    if (layout == RM_LAYOUT_CONTIGUOUS) return clamp64(t - (int64_t)s * L + 1, 0, L);
    if (layout == RM_LAYOUT_STRIPED) return t < s ? 0 : min64((t - s) / P + 1, L);
    int64_t n1 = clamp64(t - (int64_t)s * C + 1, 0, C);
    int64_t n2 = clamp64(t - (int64_t)(2 * P - 1 - s) * C + 1, 0, C);
    return n1 + n2;
  }

  // The (rank r, tile t) at place c when all P * T tiles of `tile` local rows
  // (T = ceil(L / tile)) are ordered by the global position of their rows:
  // ascending, or descending with `descending`.  Under the causal rule this
  // is the order of decreasing (key tiles, ascending) or decreasing (query
  // tiles, descending) work, which launches the longest CTAs first.  Tiles
  // of different ranks never interleave in position except under the
  // striped layout, where tile t of every rank precedes tile t + 1.
  __host__ __device__ __forceinline__ void ordered_tile(int T, int tile, int c, bool descending,
                                                        int& r, int& t) const {
    if (descending) c = P * T - 1 - c;
    if (layout == RM_LAYOUT_STRIPED) {
      t = c / P;
      r = c - t * P;
    } else if (layout == RM_LAYOUT_ZIGZAG && C % tile == 0) {
      const int tc = (int)(C / tile);  // tiles per chunk; chunk q of the sequence is on rank
      const int q = c / tc;            // q (first half) or 2P - 1 - q (second half)
      r = q < P ? q : 2 * P - 1 - q;
      t = (q < P ? 0 : tc) + (c - q * tc);
    } else {  // contiguous, or zigzag chunks that do not hold whole tiles
      r = c / T;
      t = c - r * T;
    }
  }

  __host__ __device__ __forceinline__ static int64_t min64(int64_t a, int64_t b) {
    return a < b ? a : b;
  }
  __host__ __device__ __forceinline__ static int64_t clamp64(int64_t x, int64_t lo, int64_t hi) {
    return x < lo ? lo : (x > hi ? hi : x);
  }
};

// Segments of packed / right-padded batches (see rm_attn_desc).  range():
// the [start, end) global positions of the segment holding position t of
// batch entry b; a padding token gets the empty range start = t + 1, end = t.
// query_span / key_span: the first and last global position a query may see /
// that may see a key (last < first when there is none).  Every bound is
// non-decreasing in t, so the bounds of a run of consecutive local rows are
// those of its first and last row.
struct Segs {
  const int* cu;    // packing boundaries, or null
  int nseg;
  const int* lens;  // right padding lengths, or null
  int64_t N;
  // batch entries per lens entry: a call whose batch entries are the
  // lens_div head groups of each caller batch entry (USP) reads lens[b / lens_div]
  int lens_div = 1;
  __device__ __forceinline__ void range(int b, int64_t t, int64_t& start, int64_t& end) const {
    if (cu) {
      if (t >= cu[nseg]) {
        start = t + 1;
        end = t;
        return;
      }
      int lo = 0, hi = nseg;  // cu[lo] <= t < cu[hi]
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (cu[mid] <= t) lo = mid;
        else hi = mid;
      }
      start = cu[lo];
      end = cu[hi];
    } else if (lens) {
      const int64_t len = lens[lens_div > 1 ? b / lens_div : b];
      if (t < len) {
        start = 0;
        end = len;
      } else {
        start = t + 1;
        end = t;
      }
    } else {
      start = 0;
      end = N;
    }
  }
  __device__ __forceinline__ void query_span(int b, int64_t t, bool causal, int64_t& first,
                                             int64_t& last) const {
    int64_t a, e;
    range(b, t, a, e);
    first = a;
    last = causal ? (t < e - 1 ? t : e - 1) : e - 1;
  }
  __device__ __forceinline__ void key_span(int b, int64_t u, bool causal, int64_t& first,
                                           int64_t& last) const {
    int64_t a, e;
    range(b, u, a, e);
    first = causal ? (u > a ? u : a) : a;
    last = e - 1;
  }
};

// Where the ring kernels find local row j of virtual rank r.  Rank-major
// operands: memory row r * L + j, TMA coordinates (row j, shard r) of the
// [B, P, L, H, d] view.  Global-order operands: memory row pos(r, j); TMA
// coordinates in a view that matches the layout -- striped: [B, P, L, H, d]
// with the row and shard strides swapped (row j of shard r is global row
// j * P + r), so the coordinates stay (j, r); zigzag: [B, 2P chunks, C, H, d],
// coordinates (j mod C, chunk r or 2P - 1 - r), which needs tiles that do not
// straddle a chunk (C a multiple of the tile).
struct RingRows {
  LayoutMap lay;
  int global;
  __host__ __device__ __forceinline__ int64_t row(int r, int64_t j) const {
    return global ? lay.pos(r, j) : (int64_t)r * lay.L + j;
  }
  __host__ __device__ __forceinline__ void tma(int r, int64_t j, int& crow, int& cshard) const {
    if (global && lay.layout == RM_LAYOUT_ZIGZAG) {
      const bool second = j >= lay.C;
      crow = (int)(second ? j - lay.C : j);
      cshard = second ? 2 * lay.P - 1 - r : r;
    } else {
      crow = (int)j;
      cshard = r;
    }
  }
};

// Grid order of the tensor-core attention kernels: blockIdx.x = c * G + i
// walks the tile places c (in order of decreasing work) of a block of G heads
// (or head units), blockIdx.y is the head block; G is chosen so that the
// operands streamed by G heads' CTAs stay in L2 together.  Returns false for
// the padding CTAs of a ragged last block.
__device__ __forceinline__ bool grid_place(int G, int heads, int& c, int& head) {
  c = (int)(blockIdx.x / G);
  head = (int)blockIdx.y * G + (int)(blockIdx.x - c * G);
  return head < heads;
}
// G for heads whose CTAs each stream `bytes_per_head` bytes: about as many
// heads as fit in 48 MB (well inside the 126 MB L2), at least 1, evened out
// so that the last block is nearly full.
inline int head_block(int64_t bytes_per_head, int heads) {
  int64_t g = ((int64_t)48 << 20) / (bytes_per_head > 0 ? bytes_per_head : 1);
  if (g < 1) g = 1;
  if (g > heads) g = heads;
  const int64_t blocks = (heads + g - 1) / g;  // then spread the heads evenly over the blocks
  return (int)((heads + blocks - 1) / blocks);
}

__host__ __device__ inline LayoutMap make_layout(int layout, int64_t N, int P) {
  LayoutMap m;
  m.layout = layout;
  m.P = P;
  m.L = N / P;
  m.C = N / (2 * P);
  return m;
}

// Key side of a (query shard, KV shard) call: the layout's own shards, or,
// for one tile of a rectangular grid (Pk != P, contiguous layout), contiguous
// chunks of N / Pk keys.
struct KeyShards {
  LayoutMap lay;  // equal shards
  int chunked;    // 1: chunks of L keys
  int64_t L;      // keys per shard
  __host__ __device__ __forceinline__ int64_t pos(int s, int64_t i) const {
    return chunked ? (int64_t)s * L + i : lay.pos(s, i);
  }
  __host__ __device__ __forceinline__ int64_t visible_count(int s, int64_t t) const {
    return chunked ? LayoutMap::clamp64(t - (int64_t)s * L + 1, 0, L) : lay.visible_count(s, t);
  }
};
__host__ __device__ inline KeyShards key_shards(const LayoutMap& lay, int64_t N, int Pk) {
  KeyShards k;
  k.lay = lay;
  k.chunked = Pk != lay.P;
  k.L = N / Pk;
  return k;
}

// ---- device status word (bounded-wait expiry) ------------------------------
enum : uint32_t { kStatusTimeout = 1u, kStatusSmemAlign = 2u };

// Host: address of the status word on the current device.
unsigned int* status_word();

__device__ __forceinline__ void report_timeout(unsigned int* status) {
  if (status) atomicOr(status, kStatusTimeout);
}
__device__ __forceinline__ void report_status(unsigned int* status, uint32_t bit) {
  if (status) atomicOr(status, bit);
}

// ---- small math helpers -----------------------------------------------------
__device__ __forceinline__ float bf16_to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

inline int ceil_div(int64_t a, int64_t b) { return (int)((a + b - 1) / b); }

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

}  // namespace rm
