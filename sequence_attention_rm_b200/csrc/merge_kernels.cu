// Row-wise HBM-bound kernels: the LSE merge of partial (O, LSE) results, the
// backward preprocess (delta = rowsum(dO * O)) and the fp32 -> output-dtype
// finalize.  A "row" is one (b, t, h) vector of d values; a group of
// d/4 lanes (rounded up to a power of two) owns a row and moves it with
// 16-byte fp32 vectors.  The preprocess and finalize enumerate rows (b, h, t)
// with t fastest so that the per-row delta scalars of neighbouring warps
// share sectors; the merge kernels state their own row order.
#include <climits>

#include "common.cuh"
#include "internal.h"

namespace rm {

namespace {

struct RowGroup {
  int lanes;      // lanes per row (power of two, <= 32)
  int rows_per_warp;
};

inline RowGroup row_group(int d) {
  int need = (d + 3) / 4;
  int lanes = 1;
  while (lanes < need) lanes <<= 1;
  return RowGroup{lanes, 32 / lanes};
}

__device__ __forceinline__ void store4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
__device__ __forceinline__ void store4(__nv_bfloat16* p, float4 v) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
  __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = u;
}
__device__ __forceinline__ float4 load4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
  uint2 u = *reinterpret_cast<const uint2*>(p);
  __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&u.x);
  __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&u.y);
  float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
  return make_float4(fa.x, fa.y, fb.x, fb.y);
}

// ---- LSE merge --------------------------------------------------------------
// SAME: every partial and the output have the same element strides, so one
// row offset serves all of them (no per-part 64-bit address arithmetic).
// Row order.  With the head stride inner ([B, N, H, d] tensors), rows are
// enumerated in tiles of kTileT consecutive t of one head, the tiles of a t
// range head after head: row = ((b * NB + tb) * H + h) * kTileT + ti, t =
// kTileT * tb + ti.  A block's warps read the LSE scalars of whole 32-byte
// sectors, and neighbouring blocks cover the H * kTileT rows of a contiguous
// run of O.  Measured on the 8-way merge of 8 fp32 [1, 131072, 16, 128]
// partials (interleaved A/B, same process): 6.53-6.56 TB/s with t fastest
// over the whole sequence, 6.62 with 8-token tiles, 6.67 with 16, 6.70-6.77
// with 32.  The two-part in-place merge runs the same in every tiled order
// (5.83-5.86 TB/s); rows in plain memory order (h fastest), which give every
// row's LSE scalar a sector of its own, made it slower (4.5-5.5 TB/s with 1
// to 8 adjacent heads per warp pass).
// With the head stride outer, t fastest is the memory order: kTileT = 1
// there, i.e. row = (b * H + h) * Nq + t with one tile range.
constexpr int kTileT = 32;

template <typename OutT, int NPARTS, bool SAME, bool TILED>
__global__ void __launch_bounds__(256) lse_merge_kernel(MergeArgs a, int lanes, int rows_per_warp) {
  const int lane = threadIdx.x & 31;
  const int sub = lane / lanes;      // row slot within the warp
  const int col = (lane % lanes) * 4;
  const int64_t warp0 = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int nparts = NPARTS > 0 ? NPARTS : a.n_parts;
  // (ti, h, tb, b) of the row, radices (TT, H, NB, B).  The row index is
  // split once; each pass then adds the grid stride with carries, so the
  // loop divides nothing.  Rows with t >= Nq (the last tile's tail) are idle.
  constexpr int TT = TILED ? kTileT : 1;
  const int64_t NB = TILED ? (a.Nq + TT - 1) / TT : a.Nq;
  const int64_t rows = (int64_t)a.B * a.H * NB * TT;
  const int64_t step = nwarps * rows_per_warp;
  int64_t row = warp0 * rows_per_warp + sub;
  // t fastest (not TILED): the radices are (1, Nq, H, B) with the roles of
  // h and tb swapped, handled by the same carry chain
  const int64_t R1 = TILED ? a.H : NB, R2 = TILED ? NB : a.H;
  int ti = (int)(row % TT);
  int64_t x1 = (row / TT) % R1;
  int64_t x2 = (row / TT / R1) % R2;
  int b = (int)(row / TT / R1 / R2);
  const int st_ti = (int)(step % TT);
  const int64_t st_1 = (step / TT) % R1;
  const int64_t st_2 = (step / TT / R1) % R2;
  const int st_b = (int)(step / TT / R1 / R2);
  for (; row < rows; row += step) {
    const int h = (int)(TILED ? x1 : x2);
    const int64_t t = TILED ? x2 * TT + ti : x1;
    const bool live = t < a.Nq;
    if (live) {
      const int64_t bh = (int64_t)b * a.H + h;
      const int64_t lidx = bh * a.lse_ld + t;
      const bool active = col < a.d;
      const int64_t off0 = b * a.o_sb[0] + t * a.o_sn[0] + h * a.o_sh[0] + col;
      // every load of the row is issued before any of them is used (the O loads
      // do not wait for the LSE values), so one row costs one memory latency
      float4 x[kMaxMergeParts];
      float l[kMaxMergeParts];
  #pragma unroll
      for (int i = 0; i < kMaxMergeParts; ++i) {
        if (i < nparts) {
          if (active)
            x[i] = load4(a.o_ptr[i] +
                         (SAME ? off0 : b * a.o_sb[i] + t * a.o_sn[i] + h * a.o_sh[i] + col));
          l[i] = a.lse_ptr[i][lidx];
        }
      }
      float m = -INFINITY;
  #pragma unroll
      for (int i = 0; i < kMaxMergeParts; ++i)
        if (i < nparts) m = fmaxf(m, l[i]);
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      float lse;
      if (m == -INFINITY) {
        lse = -INFINITY;
      } else {
        float w[kMaxMergeParts];
        float sum = 0.f;
  #pragma unroll
        for (int i = 0; i < kMaxMergeParts; ++i) {
          if (i < nparts) {
            w[i] = expf(l[i] - m);  // exp(-inf) = 0 for empty partials
            sum += w[i];
          }
        }
        const float inv = 1.0f / sum;
        lse = m + logf(sum);
        if (active) {
  #pragma unroll
          for (int i = 0; i < kMaxMergeParts; ++i) {
            if (i < nparts && w[i] != 0.f) {
              const float c = w[i] * inv;
              acc.x = fmaf(c, x[i].x, acc.x);
              acc.y = fmaf(c, x[i].y, acc.y);
              acc.z = fmaf(c, x[i].z, acc.z);
              acc.w = fmaf(c, x[i].w, acc.w);
            }
          }
        }
      }
      if (active) {
        OutT* out = reinterpret_cast<OutT*>(a.out) +
                    (SAME ? off0 : b * a.out_sb + t * a.out_sn + h * a.out_sh + col);
        store4(out, acc);
      }
      if ((lane % lanes) == 0) a.lse_out[lidx] = lse;
    }
    ti += st_ti;
    int carry = ti >= TT;
    if (carry) ti -= TT;
    x1 += st_1 + carry;
    carry = x1 >= R1;
    if (carry) x1 -= R1;
    x2 += st_2 + carry;
    carry = x2 >= R2;
    if (carry) x2 -= R2;
    b += st_b + carry;
  }
}

// Two parts, d = 128 (one 32-lane warp per row), the running-state merge of
// the stepwise and multi-rank rings: a warp takes 32 consecutive t of one
// (b, h).  Lane i reads the two LSE values of row t0 + i (one
// coalesced load per part), computes the row's weights and new LSE once and
// writes the LSE back (in place is safe: the lane that writes it read it);
// the warp then streams the 32 rows U at a time, weights passed by shuffle,
// all 2U loads of a pass issued before any is used.  The per-row kernel
// repeats the exp / log chain in every lane between one row's loads and the
// next (5.82 -> 5.95-5.99 TB/s with the same grid; rows in memory order or 8
// rows per pass measured no better).  Same arithmetic as lse_merge_kernel, so
// the same bits.
constexpr int kMerge2Rows = 4;  // rows per pass

template <typename OutT, int U>
__global__ void __launch_bounds__(256) merge2_rows_kernel(MergeArgs a) {
  const int lane = threadIdx.x & 31;
  const int col = lane * 4;
  const int64_t NC = (a.Nq + 31) / 32;  // 32-token chunks per (b, h)
  const int64_t chunks = (int64_t)a.B * a.H * NC;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const float skip = __int_as_float(0x7fffffff);  // NaN: the part has weight 0
  for (int64_t c = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); c < chunks;
       c += nwarps) {
    const int64_t bh = c / NC;
    const int64_t t0 = (c - bh * NC) * 32;
    const int h = (int)(bh % a.H), b = (int)(bh / a.H);
    const int rows = (int)(a.Nq - t0 < 32 ? a.Nq - t0 : 32);
    float c0 = skip, c1 = skip;
    if (lane < rows) {
      const int64_t lidx = bh * a.lse_ld + t0 + lane;
      const float l0 = a.lse_ptr[0][lidx], l1 = a.lse_ptr[1][lidx];
      const float m = fmaxf(l0, l1);
      float lse = -INFINITY;
      if (m != -INFINITY) {
        const float w0 = expf(l0 - m);  // exp(-inf) = 0 for an empty partial
        const float w1 = expf(l1 - m);
        const float sum = 0.f + w0 + w1;
        const float inv = 1.0f / sum;
        lse = m + logf(sum);
        if (w0 != 0.f) c0 = w0 * inv;
        if (w1 != 0.f) c1 = w1 * inv;
      }
      a.lse_out[lidx] = lse;
    }
    const float* p0 = a.o_ptr[0] + b * a.o_sb[0] + t0 * a.o_sn[0] + h * a.o_sh[0] + col;
    const float* p1 = a.o_ptr[1] + b * a.o_sb[1] + t0 * a.o_sn[1] + h * a.o_sh[1] + col;
    OutT* po = reinterpret_cast<OutT*>(a.out) + b * a.out_sb + t0 * a.out_sn + h * a.out_sh + col;
    for (int r0 = 0; r0 < rows; r0 += U) {
      float4 x0[U], x1[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (r0 + u < rows) {
          x0[u] = load4(p0 + (int64_t)(r0 + u) * a.o_sn[0]);
          x1[u] = load4(p1 + (int64_t)(r0 + u) * a.o_sn[1]);
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const float k0 = __shfl_sync(0xffffffffu, c0, (r0 + u) & 31);
        const float k1 = __shfl_sync(0xffffffffu, c1, (r0 + u) & 31);
        if (r0 + u < rows) {
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
          if (k0 == k0) {
            acc.x = fmaf(k0, x0[u].x, acc.x);
            acc.y = fmaf(k0, x0[u].y, acc.y);
            acc.z = fmaf(k0, x0[u].z, acc.z);
            acc.w = fmaf(k0, x0[u].w, acc.w);
          }
          if (k1 == k1) {
            acc.x = fmaf(k1, x1[u].x, acc.x);
            acc.y = fmaf(k1, x1[u].y, acc.y);
            acc.z = fmaf(k1, x1[u].z, acc.z);
            acc.w = fmaf(k1, x1[u].w, acc.w);
          }
          store4(po + (int64_t)(r0 + u) * a.out_sn, acc);
        }
      }
    }
  }
}

// ---- backward preprocess ----------------------------------------------------
template <typename InT>
__global__ void __launch_bounds__(256) bwd_preprocess_kernel(int B, int64_t N, int H, int d,
                                                             rm_tensor o, rm_tensor dout,
                                                             float* __restrict__ delta,
                                                             float* __restrict__ zero_fill,
                                                             int lanes, int rows_per_warp) {
  const int lane = threadIdx.x & 31;
  const int sub = lane / lanes;
  const int col = (lane % lanes) * 4;
  const int64_t warp0 = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  // a warp takes whole tokens (b, t): its lane groups read the H head rows of
  // the token, which are contiguous in memory, so the tensor is read in order;
  // delta is written at its [B, H, N] index
  const int64_t tokens = (int64_t)B * N;
  for (int64_t bt = warp0; bt < tokens; bt += nwarps) {
    const int64_t t = bt % N;
    const int64_t b = bt / N;
    const InT* orow = reinterpret_cast<const InT*>(o.ptr) + b * o.stride_b + t * o.stride_n;
    const InT* drow = reinterpret_cast<const InT*>(dout.ptr) + b * dout.stride_b + t * dout.stride_n;
    for (int h0 = 0; h0 < H; h0 += rows_per_warp) {
      const int h = h0 + sub;
      float v = 0.f;
      if (h < H && col < d) {
        const float4 x = load4(orow + (int64_t)h * o.stride_h + col);
        const float4 y = load4(drow + (int64_t)h * dout.stride_h + col);
        v = x.x * y.x + x.y * y.y + x.z * y.z + x.w * y.w;
        if (zero_fill)
          store4(zero_fill + ((b * H + h) * N + t) * d + col, make_float4(0.f, 0.f, 0.f, 0.f));
      }
      for (int off = lanes >> 1; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      if (h < H && (lane % lanes) == 0) delta[(b * H + h) * N + t] = v;
    }
  }
}

// bf16 operands with 16-byte rows (d % 8 == 0): 8 elements per lane, LANES
// lanes per head row, so a warp pass covers 32 / LANES rows of a token; the
// loads of kAhead passes are issued before any row is reduced.  The grid is
// sized to the blocks that fit on the device at once (one wave).
template <int LANES>
__global__ void __launch_bounds__(256) bwd_delta_bf16_kernel(int B, int64_t N, int H, int d,
                                                             rm_tensor o, rm_tensor dout,
                                                             float* __restrict__ delta) {
  constexpr int kRows = 32 / LANES;  // head rows per warp pass
  constexpr int kAhead = 4;
  const int lane = threadIdx.x & 31;
  const int sub = lane / LANES;
  const int col = (lane % LANES) * 8;
  const int64_t warp0 = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int64_t tokens = (int64_t)B * N;
  for (int64_t bt = warp0; bt < tokens; bt += nwarps) {
    const int64_t t = bt % N;
    const int64_t b = bt / N;
    const __nv_bfloat16* orow =
        reinterpret_cast<const __nv_bfloat16*>(o.ptr) + b * o.stride_b + t * o.stride_n;
    const __nv_bfloat16* drow =
        reinterpret_cast<const __nv_bfloat16*>(dout.ptr) + b * dout.stride_b + t * dout.stride_n;
    for (int h0 = 0; h0 < H; h0 += kRows * kAhead) {
      uint4 x[kAhead], y[kAhead];
#pragma unroll
      for (int j = 0; j < kAhead; ++j) {
        const int h = h0 + j * kRows + sub;
        x[j] = y[j] = make_uint4(0u, 0u, 0u, 0u);
        if (h < H && col < d) {
          x[j] = *reinterpret_cast<const uint4*>(orow + (int64_t)h * o.stride_h + col);
          y[j] = *reinterpret_cast<const uint4*>(drow + (int64_t)h * dout.stride_h + col);
        }
      }
#pragma unroll
      for (int j = 0; j < kAhead; ++j) {
        const int h = h0 + j * kRows + sub;
        const uint32_t xa[4] = {x[j].x, x[j].y, x[j].z, x[j].w};
        const uint32_t ya[4] = {y[j].x, y[j].y, y[j].z, y[j].w};
        float v = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          v = fmaf(__uint_as_float(xa[e] << 16), __uint_as_float(ya[e] << 16), v);
          v = fmaf(__uint_as_float(xa[e] & 0xffff0000u), __uint_as_float(ya[e] & 0xffff0000u), v);
        }
#pragma unroll
        for (int off = LANES >> 1; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (h < H && (lane % LANES) == 0) delta[(b * H + h) * N + t] = v;
      }
    }
  }
}

// ---- fp32 -> output dtype ---------------------------------------------------
template <typename OutT>
__global__ void __launch_bounds__(256) convert_f32_kernel(int B, int64_t N, int H, int d,
                                                          rm_tensor in, rm_tensor out, int lanes,
                                                          int rows_per_warp) {
  const int lane = threadIdx.x & 31;
  const int sub = lane / lanes;
  const int col = (lane % lanes) * 4;
  const int64_t rows = (int64_t)B * N * H;
  const int64_t warp0 = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t base = warp0 * rows_per_warp; base < rows; base += nwarps * rows_per_warp) {
    const int64_t row = base + sub;  // (b, t, h) with h fastest
    if (row >= rows || col >= d) continue;
    const int h = (int)(row % H);
    const int64_t bt = row / H;
    const int64_t t = bt % N;
    const int b = (int)(bt / N);
    float4 x = load4(reinterpret_cast<const float*>(in.ptr) + b * in.stride_b + t * in.stride_n +
                     h * in.stride_h + col);
    store4(reinterpret_cast<OutT*>(out.ptr) + b * out.stride_b + t * out.stride_n +
               h * out.stride_h + col,
           x);
  }
}

// Blocks of a 256-thread kernel resident on one SM at once, from the
// occupancy calculator (registers decide it), cached per device and kernel.
template <auto Kernel>
int resident_blocks() {
  static int per_sm[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  int& k = per_sm[dev & 63];
  if (k <= 0 &&
      (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&k, Kernel, 256, 0) != cudaSuccess || k <= 0))
    k = 4;
  return k;
}

// Grid of a grid-stride row kernel: enough 8-warp blocks for every warp to
// get a row group, capped at one wave of resident blocks (a second, partial
// wave would leave SMs idle at the end while the rest stream).
int grid_for_rows(int64_t rows, int rows_per_warp, int blocks_per_sm) {
  int64_t warps = (rows + rows_per_warp - 1) / rows_per_warp;
  int64_t blocks = (warps + 7) / 8;
  int64_t cap = (int64_t)num_sms() * blocks_per_sm;
  if (blocks > cap) blocks = cap;
  return (int)(blocks < 1 ? 1 : blocks);
}

template <typename OutT, int NPARTS, bool SAME, bool TILED>
void launch_merge_kernel(const MergeArgs& a, RowGroup g, int64_t rows, cudaStream_t s) {
  constexpr auto kern = lse_merge_kernel<OutT, NPARTS, SAME, TILED>;
  const int grid = grid_for_rows(rows, g.rows_per_warp, resident_blocks<kern>());
  kern<<<grid, 256, 0, s>>>(a, g.lanes, g.rows_per_warp);
}

template <typename OutT, bool SAME, bool TILED>
cudaError_t merge_dispatch(const MergeArgs& a, RowGroup g, int64_t rows, cudaStream_t s) {
  switch (a.n_parts) {
    case 2: launch_merge_kernel<OutT, 2, SAME, TILED>(a, g, rows, s); break;
    case 4: launch_merge_kernel<OutT, 4, SAME, TILED>(a, g, rows, s); break;
    case 8: launch_merge_kernel<OutT, 8, SAME, TILED>(a, g, rows, s); break;
    default: launch_merge_kernel<OutT, 0, SAME, TILED>(a, g, rows, s); break;
  }
  return cudaGetLastError();
}

template <typename OutT, bool SAME>
cudaError_t merge_order(const MergeArgs& a, RowGroup g, int64_t rows, cudaStream_t s) {
  bool heads_inner = a.out_sh <= a.out_sn;
  for (int i = 0; i < a.n_parts; ++i) heads_inner = heads_inner && a.o_sh[i] <= a.o_sn[i];
  return heads_inner ? merge_dispatch<OutT, SAME, true>(a, g, rows, s)
                     : merge_dispatch<OutT, SAME, false>(a, g, rows, s);
}

}  // namespace

cudaError_t launch_lse_merge(const MergeArgs& a, int out_bf16, cudaStream_t stream) {
  const int64_t rows = (int64_t)a.B * a.H * a.Nq;
  if (rows == 0) return cudaSuccess;
  RowGroup g = row_group(a.d);
  bool same = a.out_sb == a.o_sb[0] && a.out_sn == a.o_sn[0] && a.out_sh == a.o_sh[0];
  for (int i = 1; i < a.n_parts; ++i)
    same = same && a.o_sb[i] == a.o_sb[0] && a.o_sn[i] == a.o_sn[0] && a.o_sh[i] == a.o_sh[0];
  ProfScope ps("lse_merge", stream);
  if (a.n_parts == 2 && a.d == 128) {
    // one chunk per warp, blocks scheduled as SMs free up: on the 2-part
    // in-place merge of [1, 131072, 16, 128] fp32 this ran at 6.35-6.38 TB/s
    // against 5.93-5.98 for a single wave of resident blocks that loop over
    // the chunks (whose SMs finish unevenly)
    const int64_t chunks = (int64_t)a.B * a.H * ((a.Nq + 31) / 32);
    const int grid = (int)((chunks + 7) / 8 < INT_MAX ? (chunks + 7) / 8 : INT_MAX);
    if (out_bf16) {
      merge2_rows_kernel<__nv_bfloat16, kMerge2Rows><<<grid, 256, 0, stream>>>(a);
    } else {
      merge2_rows_kernel<float, kMerge2Rows><<<grid, 256, 0, stream>>>(a);
    }
    return cudaGetLastError();
  }
  if (same)
    return out_bf16 ? merge_order<__nv_bfloat16, true>(a, g, rows, stream)
                    : merge_order<float, true>(a, g, rows, stream);
  return out_bf16 ? merge_order<__nv_bfloat16, false>(a, g, rows, stream)
                  : merge_order<float, false>(a, g, rows, stream);
}

template <int LANES>
cudaError_t launch_delta_bf16(int B, int64_t N, int H, int d, rm_tensor o, rm_tensor dout,
                              float* delta, cudaStream_t stream) {
  const int k = resident_blocks<bwd_delta_bf16_kernel<LANES>>();
  const int64_t warps = (int64_t)B * N;  // one token per warp pass
  const int64_t need = (warps + 7) / 8;
  const int64_t cap = (int64_t)num_sms() * k;
  const int grid = (int)(need < cap ? need : cap);
  bwd_delta_bf16_kernel<LANES><<<grid, 256, 0, stream>>>(B, N, H, d, o, dout, delta);
  return cudaGetLastError();
}

cudaError_t launch_bwd_preprocess(int in_bf16, int B, int64_t N, int H, int d, rm_tensor o,
                                  rm_tensor dout, float* delta, float* zero_fill,
                                  cudaStream_t stream) {
  const int64_t rows = (int64_t)B * H * N;
  if (rows == 0) return cudaSuccess;
  auto rows16 = [](const rm_tensor& x) {
    return ((uintptr_t)x.ptr % 16) == 0 && x.stride_b % 8 == 0 && x.stride_n % 8 == 0 &&
           x.stride_h % 8 == 0;
  };
  if (in_bf16 && !zero_fill && d % 8 == 0 && d <= 128 && rows16(o) && rows16(dout)) {
    ProfScope ps("bwd_preprocess", stream);
    const int need = d / 8;
    if (need > 8) return launch_delta_bf16<16>(B, N, H, d, o, dout, delta, stream);
    if (need > 4) return launch_delta_bf16<8>(B, N, H, d, o, dout, delta, stream);
    if (need > 2) return launch_delta_bf16<4>(B, N, H, d, o, dout, delta, stream);
    return launch_delta_bf16<2>(B, N, H, d, o, dout, delta, stream);
  }
  RowGroup g = row_group(d);
  ProfScope ps("bwd_preprocess", stream);
  if (in_bf16) {
    constexpr auto kern = bwd_preprocess_kernel<__nv_bfloat16>;
    // one token per warp pass
    const int grid = grid_for_rows((int64_t)B * N, 1, resident_blocks<kern>());
    kern<<<grid, 256, 0, stream>>>(B, N, H, d, o, dout, delta, zero_fill, g.lanes,
                                   g.rows_per_warp);
  } else {
    constexpr auto kern = bwd_preprocess_kernel<float>;
    const int grid = grid_for_rows((int64_t)B * N, 1, resident_blocks<kern>());
    kern<<<grid, 256, 0, stream>>>(B, N, H, d, o, dout, delta, zero_fill, g.lanes,
                                   g.rows_per_warp);
  }
  return cudaGetLastError();
}

cudaError_t launch_convert_f32(int out_bf16, int B, int64_t N, int H, int d, rm_tensor in,
                               rm_tensor out, cudaStream_t stream) {
  const int64_t rows = (int64_t)B * N * H;
  if (rows == 0) return cudaSuccess;
  RowGroup g = row_group(d);
  ProfScope ps("convert_f32", stream);
  if (out_bf16) {
    constexpr auto kern = convert_f32_kernel<__nv_bfloat16>;
    const int grid = grid_for_rows(rows, g.rows_per_warp, resident_blocks<kern>());
    kern<<<grid, 256, 0, stream>>>(B, N, H, d, in, out, g.lanes, g.rows_per_warp);
  } else {
    constexpr auto kern = convert_f32_kernel<float>;
    const int grid = grid_for_rows(rows, g.rows_per_warp, resident_blocks<kern>());
    kern<<<grid, 256, 0, stream>>>(B, N, H, d, in, out, g.lanes, g.rows_per_warp);
  }
  return cudaGetLastError();
}

}  // namespace rm
