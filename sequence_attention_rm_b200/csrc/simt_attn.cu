// Exact-fp32 attention on CUDA cores (fp32 inputs; the tensor-core path is
// bf16).  TF32 tensor cores could not hold 1e-5 parity, so fp32 problems are
// computed with fp32 FMA: each query (or key) row is owned by 4 lanes, each
// holding d/4 of its columns; K/V (or Q/dO) tiles of 32 rows are staged in
// shared memory and read as broadcasts.  The backward kernels also take bf16
// operands (widened to fp32 as they are read): the bf16 backward at head dims
// other than 128, which the tensor-core backward does not cover.
//
// Forward: online softmax over the KV tiles of every KV shard the row sees
// (Ring Attention & Friends, "Tiling with the Softmax Rescaling Trick"), the
// shards taken in ring order (r, r-1, ...; Mosaic, "How Ring Attention Works").
// Backward: two passes, one owning query rows (dQ), one owning key rows
// (dK, dV), each recomputing P = exp(s - LSE_final); no atomics.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace rm {

namespace {

constexpr int kRows = 32;     // rows per CTA
constexpr int kTile = 32;     // staged rows per tile
constexpr int kThreads = kRows * 4;

template <int DMAX>
struct Slice {
  float v[DMAX / 4];
};

// column of slot c for lane `sub` of the row's 4 lanes
__device__ __forceinline__ int col_of(int c, int sub) { return c * 4 + sub; }

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <int DMAX, typename InT>
__device__ __forceinline__ void load_slice(Slice<DMAX>& s, const InT* row, int d, int sub) {
#pragma unroll
  for (int c = 0; c < DMAX / 4; ++c) {
    int col = col_of(c, sub);
    s.v[c] = col < d ? to_f32(row[col]) : 0.f;
  }
}

__device__ __forceinline__ float row_sum4(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  x += __shfl_xor_sync(0xffffffffu, x, 2);
  return x;
}

// Stage rows [row0, row0 + kTile) of a [rows, d] operand (row stride `ld`
// elements from `base`) into smem [kTile][DMAX]; rows >= nrows are zeroed.
template <int DMAX, typename InT>
__device__ __forceinline__ void stage(float (*dst)[DMAX], const InT* base, int64_t ld,
                                      int64_t row0, int64_t nrows, int d) {
  for (int i = threadIdx.x; i < kTile * DMAX; i += blockDim.x) {
    int rr = i / DMAX, col = i % DMAX;
    int64_t row = row0 + rr;
    dst[rr][col] = (row < nrows && col < d) ? to_f32(base[row * ld + col]) : 0.f;
  }
}

// The CTA's range of local keys: the union [min lo, max hi) of the ranges its
// rows contribute (`mine`: this thread contributes [lo, hi)); empty ranges
// give [0, 0).  Every thread of the CTA must call it.
__device__ __forceinline__ void cta_key_range(unsigned long long* shared, bool mine, int64_t lo,
                                              int64_t hi, int64_t& cta_lo, int64_t& cta_hi) {
  __syncthreads();  // the previous step's readers are done with `shared`
  if (threadIdx.x == 0) {
    shared[0] = ~0ull;
    shared[1] = 0ull;
  }
  __syncthreads();
  if (mine) {
    atomicMin(&shared[0], (unsigned long long)lo);
    atomicMax(&shared[1], (unsigned long long)hi);
  }
  __syncthreads();
  cta_hi = (int64_t)shared[1];
  cta_lo = cta_hi > 0 ? (int64_t)shared[0] : 0;
}

// ---------------------------------------------------------------------------
template <int DMAX>
__global__ void __launch_bounds__(kThreads) simt_fwd_kernel(AttnArgs a, int q_rank, int kv_rank) {
  __shared__ float ks[kTile][DMAX];
  __shared__ float vs[kTile][DMAX];
  const LayoutMap lay = make_layout(a.layout, a.N, a.P);
  const int64_t L = lay.L;
  const bool ring = q_rank < 0;
  const KeyShards kmap = key_shards(lay, a.N, ring ? a.P : kv_shards(a));
  const int r = ring ? (int)(blockIdx.z % a.P) : q_rank;
  const int b = ring ? (int)(blockIdx.z / a.P) : (int)blockIdx.z;
  const int h = blockIdx.y;
  const int g = h / (a.Hq / a.Hkv);
  const int row_in_cta = threadIdx.x >> 2, sub = threadIdx.x & 3;
  const int64_t j = (int64_t)blockIdx.x * kRows + row_in_cta;  // local query index
  const bool live = j < L;
  const int64_t qrow = (ring ? (int64_t)r * L : 0) + j;
  const int64_t tq = live ? lay.pos(r, j) : 0;
  // global positions [qf, ql] of the keys this row may see (causal rule and
  // segment of a packed or right-padded batch)
  const Segs sg{a.cu_seqlens, a.num_segments, a.seq_lens, a.N, a.seg_div > 1 ? a.seg_div : 1};
  int64_t qf = 0, ql = -1;
  if (live) sg.query_span(b, tq, a.causal, qf, ql);
  __shared__ unsigned long long cta_range[2];

  Slice<DMAX> q, acc;
  const float* qp = reinterpret_cast<const float*>(a.q.ptr) + b * a.q.stride_b + qrow * a.q.stride_n +
                    h * a.q.stride_h;
  if (live) load_slice<DMAX>(q, qp, a.d, sub);
  else
#pragma unroll
    for (int c = 0; c < DMAX / 4; ++c) q.v[c] = 0.f;
#pragma unroll
  for (int c = 0; c < DMAX / 4; ++c) acc.v[c] = 0.f;
  float m = -INFINITY, l = 0.f;

  const int nsteps = ring ? a.P : 1;
  for (int step = 0; step < nsteps; ++step) {
    const int s = ring ? ((r - step) % a.P + a.P) % a.P : kv_rank;
    // local keys [row_lo, row_hi) of shard s this row may see (positions are
    // increasing in the local index), and their union over the CTA's rows
    const int64_t row_lo = live ? kmap.visible_count(s, qf - 1) : 0;
    const int64_t row_hi = live ? kmap.visible_count(s, ql) : 0;
    int64_t cta_lo, cta_hi;
    cta_key_range(cta_range, sub == 0 && row_hi > row_lo, row_lo, row_hi, cta_lo, cta_hi);
    const int64_t kv0 = ring ? (int64_t)s * L : 0;
    const float* kb = reinterpret_cast<const float*>(a.k.ptr) + b * a.k.stride_b + g * a.k.stride_h +
                      kv0 * a.k.stride_n;
    const float* vb = reinterpret_cast<const float*>(a.v.ptr) + b * a.v.stride_b + g * a.v.stride_h +
                      kv0 * a.v.stride_n;
    for (int64_t i0 = cta_lo; i0 < cta_hi; i0 += kTile) {
      __syncthreads();
      stage<DMAX>(ks, kb, a.k.stride_n, i0, kmap.L, a.d);
      stage<DMAX>(vs, vb, a.v.stride_n, i0, kmap.L, a.d);
      __syncthreads();
      float sc[kTile];
      float tmax = -INFINITY;
#pragma unroll
      for (int kk = 0; kk < kTile; ++kk) {
        float part = 0.f;
#pragma unroll
        for (int c = 0; c < DMAX / 4; ++c) part = fmaf(q.v[c], ks[kk][col_of(c, sub)], part);
        float sv = row_sum4(part) * a.scale;
        sc[kk] = (i0 + kk >= row_lo && i0 + kk < row_hi) ? sv : -INFINITY;
        tmax = fmaxf(tmax, sc[kk]);
      }
      if (tmax == -INFINITY) continue;  // nothing visible in this tile for this row
      const float m_new = fmaxf(m, tmax);
      const float corr = expf(m - m_new);  // 0 when m == -inf
      l *= corr;
#pragma unroll
      for (int c = 0; c < DMAX / 4; ++c) acc.v[c] *= corr;
#pragma unroll
      for (int kk = 0; kk < kTile; ++kk) {
        const float p = expf(sc[kk] - m_new);
        l += p;
#pragma unroll
        for (int c = 0; c < DMAX / 4; ++c) acc.v[c] = fmaf(p, vs[kk][col_of(c, sub)], acc.v[c]);
      }
      m = m_new;
    }
  }
  if (!live) return;
  const float inv = l > 0.f ? 1.0f / l : 0.f;
  const float lse = l > 0.f ? m + logf(l) : -INFINITY;
  const int64_t orow = (ring ? (int64_t)r * L : 0) + j;
  // fp32 problems write fp32 outputs whether or not o_f32 is requested
  float* op = reinterpret_cast<float*>(a.o.ptr) + b * a.o.stride_b + orow * a.o.stride_n +
              h * a.o.stride_h;
#pragma unroll
  for (int c = 0; c < DMAX / 4; ++c)
    if (col_of(c, sub) < a.d) op[col_of(c, sub)] = acc.v[c] * inv;
  if (sub == 0) a.lse[((int64_t)b * a.Hq + h) * a.lse_ld + orow] = lse;
}

// ---------------------------------------------------------------------------
// dQ pass: one CTA owns 32 query rows of (b, h, rank r).
template <int DMAX, typename InT>
__global__ void __launch_bounds__(kThreads) simt_bwd_dq_kernel(AttnArgs a, int q_rank, int kv_rank) {
  __shared__ float ks[kTile][DMAX];
  __shared__ float vs[kTile][DMAX];
  const LayoutMap lay = make_layout(a.layout, a.N, a.P);
  const int64_t L = lay.L;
  const bool ring = q_rank < 0;
  const KeyShards kmap = key_shards(lay, a.N, ring ? a.P : kv_shards(a));
  const int r = ring ? (int)(blockIdx.z % a.P) : q_rank;
  const int b = ring ? (int)(blockIdx.z / a.P) : (int)blockIdx.z;
  const int h = blockIdx.y;
  const int g = h / (a.Hq / a.Hkv);
  const int row_in_cta = threadIdx.x >> 2, sub = threadIdx.x & 3;
  const int64_t j = (int64_t)blockIdx.x * kRows + row_in_cta;
  const bool live = j < L;
  const int64_t qrow = (ring ? (int64_t)r * L : 0) + j;
  const int64_t tq = live ? lay.pos(r, j) : 0;
  const Segs sg{a.cu_seqlens, a.num_segments, a.seq_lens, a.N, a.seg_div > 1 ? a.seg_div : 1};
  int64_t qf = 0, ql = -1;
  if (live) sg.query_span(b, tq, a.causal, qf, ql);
  __shared__ unsigned long long cta_range[2];

  Slice<DMAX> q, dO, dq;
#pragma unroll
  for (int c = 0; c < DMAX / 4; ++c) { q.v[c] = 0.f; dO.v[c] = 0.f; dq.v[c] = 0.f; }
  float lse = 0.f, D = 0.f;
  if (live) {
    load_slice<DMAX>(q, reinterpret_cast<const InT*>(a.q.ptr) + b * a.q.stride_b +
                            qrow * a.q.stride_n + h * a.q.stride_h, a.d, sub);
    load_slice<DMAX>(dO, reinterpret_cast<const InT*>(a.dout.ptr) + b * a.dout.stride_b +
                             qrow * a.dout.stride_n + h * a.dout.stride_h, a.d, sub);
    lse = a.lse_in[((int64_t)b * a.Hq + h) * a.lse_ld + qrow];
    D = a.delta[((int64_t)b * a.Hq + h) * a.lse_ld + qrow];
  }
  const int nsteps = ring ? a.P : 1;
  for (int step = 0; step < nsteps; ++step) {
    const int s = ring ? ((r - step) % a.P + a.P) % a.P : kv_rank;
    const int64_t row_lo = live ? kmap.visible_count(s, qf - 1) : 0;
    const int64_t row_hi = live ? kmap.visible_count(s, ql) : 0;
    int64_t cta_lo, cta_hi;
    cta_key_range(cta_range, sub == 0 && row_hi > row_lo, row_lo, row_hi, cta_lo, cta_hi);
    const int64_t kv0 = ring ? (int64_t)s * L : 0;
    const InT* kb = reinterpret_cast<const InT*>(a.k.ptr) + b * a.k.stride_b + g * a.k.stride_h +
                      kv0 * a.k.stride_n;
    const InT* vb = reinterpret_cast<const InT*>(a.v.ptr) + b * a.v.stride_b + g * a.v.stride_h +
                      kv0 * a.v.stride_n;
    for (int64_t i0 = cta_lo; i0 < cta_hi; i0 += kTile) {
      __syncthreads();
      stage<DMAX>(ks, kb, a.k.stride_n, i0, kmap.L, a.d);
      stage<DMAX>(vs, vb, a.v.stride_n, i0, kmap.L, a.d);
      __syncthreads();
#pragma unroll 2
      for (int kk = 0; kk < kTile; ++kk) {
        float ps = 0.f, pd = 0.f;
#pragma unroll
        for (int c = 0; c < DMAX / 4; ++c) {
          ps = fmaf(q.v[c], ks[kk][col_of(c, sub)], ps);
          pd = fmaf(dO.v[c], vs[kk][col_of(c, sub)], pd);
        }
        const float sv = row_sum4(ps) * a.scale;
        const float dp = row_sum4(pd);
        if (i0 + kk >= row_lo && i0 + kk < row_hi) {
          const float p = expf(sv - lse);
          const float ds = p * (dp - D) * a.scale;
#pragma unroll
          for (int c = 0; c < DMAX / 4; ++c) dq.v[c] = fmaf(ds, ks[kk][col_of(c, sub)], dq.v[c]);
        }
      }
    }
  }
  if (!live) return;
  float* dqp = reinterpret_cast<float*>(a.dq.ptr) + b * a.dq.stride_b + qrow * a.dq.stride_n +
               h * a.dq.stride_h;
#pragma unroll
  for (int c = 0; c < DMAX / 4; ++c)
    if (col_of(c, sub) < a.d) dqp[col_of(c, sub)] = (a.accumulate ? dqp[col_of(c, sub)] : 0.f) + dq.v[c];
}

// dK/dV pass: one CTA owns 32 key rows of (b, kv head g, shard s); it walks
// the query heads of the group and the query ranks that use the shard.
template <int DMAX, typename InT>
__global__ void __launch_bounds__(kThreads) simt_bwd_dkdv_kernel(AttnArgs a, int q_rank, int kv_rank) {
  __shared__ float qs[kTile][DMAX];
  __shared__ float dos[kTile][DMAX];
  __shared__ float lses[kTile], ds_[kTile];
  __shared__ int64_t tpos[kTile];
  const LayoutMap lay = make_layout(a.layout, a.N, a.P);
  const int64_t L = lay.L;
  const bool ring = q_rank < 0;
  const KeyShards kmap = key_shards(lay, a.N, ring ? a.P : kv_shards(a));
  const int s = ring ? (int)(blockIdx.z % a.P) : kv_rank;
  const int b = ring ? (int)(blockIdx.z / a.P) : (int)blockIdx.z;
  const int g = blockIdx.y;
  const int group = a.Hq / a.Hkv;
  const int row_in_cta = threadIdx.x >> 2, sub = threadIdx.x & 3;
  const int64_t i = (int64_t)blockIdx.x * kRows + row_in_cta;  // local key index
  const bool live = i < kmap.L;
  const int64_t krow = (ring ? (int64_t)s * L : 0) + i;
  const int64_t tk = live ? kmap.pos(s, i) : 0;
  const int64_t i_first = (int64_t)blockIdx.x * kRows;
  const int64_t t_first = kmap.pos(s, i_first);
  // global positions [kf, kl] of the queries that see this key
  const Segs sg{a.cu_seqlens, a.num_segments, a.seq_lens, a.N, a.seg_div > 1 ? a.seg_div : 1};
  int64_t kf = 0, kl = -1;
  if (live) sg.key_span(b, tk, a.causal, kf, kl);

  Slice<DMAX> k, v, dk, dv;
#pragma unroll
  for (int c = 0; c < DMAX / 4; ++c) { k.v[c] = 0.f; v.v[c] = 0.f; dk.v[c] = 0.f; dv.v[c] = 0.f; }
  if (live) {
    load_slice<DMAX>(k, reinterpret_cast<const InT*>(a.k.ptr) + b * a.k.stride_b +
                            krow * a.k.stride_n + g * a.k.stride_h, a.d, sub);
    load_slice<DMAX>(v, reinterpret_cast<const InT*>(a.v.ptr) + b * a.v.stride_b +
                            krow * a.v.stride_n + g * a.v.stride_h, a.d, sub);
  }
  const int nranks = ring ? a.P : 1;
  for (int hh = 0; hh < group; ++hh) {
    const int h = g * group + hh;
    for (int step = 0; step < nranks; ++step) {
      // reverse ring: shard s visits ranks s, s+1, ...
      const int r = ring ? (s + step) % a.P : q_rank;
      const int64_t q0 = ring ? (int64_t)r * L : 0;
      const InT* qb = reinterpret_cast<const InT*>(a.q.ptr) + b * a.q.stride_b + h * a.q.stride_h +
                        q0 * a.q.stride_n;
      const InT* dob = reinterpret_cast<const InT*>(a.dout.ptr) + b * a.dout.stride_b +
                         h * a.dout.stride_h + q0 * a.dout.stride_n;
      const float* lse_b = a.lse_in + ((int64_t)b * a.Hq + h) * a.lse_ld + q0;
      const float* del_b = a.delta + ((int64_t)b * a.Hq + h) * a.lse_ld + q0;
      for (int64_t j0 = 0; j0 < L; j0 += kTile) {
        const int64_t j_last = min(j0 + kTile, L) - 1;
        if (a.causal && lay.pos(r, j_last) < t_first) continue;  // whole tile sees none of our keys
        __syncthreads();
        stage<DMAX>(qs, qb, a.q.stride_n, j0, L, a.d);
        stage<DMAX>(dos, dob, a.dout.stride_n, j0, L, a.d);
        for (int x = threadIdx.x; x < kTile; x += blockDim.x) {
          const int64_t jj = j0 + x;
          lses[x] = jj < L ? lse_b[jj] : 0.f;
          ds_[x] = jj < L ? del_b[jj] : 0.f;
          tpos[x] = jj < L ? lay.pos(r, jj) : -1;
        }
        __syncthreads();
#pragma unroll 2
        for (int qq = 0; qq < kTile; ++qq) {
          float ps = 0.f, pd = 0.f;
#pragma unroll
          for (int c = 0; c < DMAX / 4; ++c) {
            ps = fmaf(k.v[c], qs[qq][col_of(c, sub)], ps);
            pd = fmaf(v.v[c], dos[qq][col_of(c, sub)], pd);
          }
          const float sv = row_sum4(ps) * a.scale;
          const float dp = row_sum4(pd);
          const bool vis = live && tpos[qq] >= kf && tpos[qq] <= kl;
          if (vis) {
            const float p = expf(sv - lses[qq]);
            const float dsv = p * (dp - ds_[qq]) * a.scale;
#pragma unroll
            for (int c = 0; c < DMAX / 4; ++c) {
              dv.v[c] = fmaf(p, dos[qq][col_of(c, sub)], dv.v[c]);
              dk.v[c] = fmaf(dsv, qs[qq][col_of(c, sub)], dk.v[c]);
            }
          }
        }
      }
    }
  }
  if (!live) return;
  float* dkp = reinterpret_cast<float*>(a.dk.ptr) + b * a.dk.stride_b + krow * a.dk.stride_n +
               g * a.dk.stride_h;
  float* dvp = reinterpret_cast<float*>(a.dv.ptr) + b * a.dv.stride_b + krow * a.dv.stride_n +
               g * a.dv.stride_h;
#pragma unroll
  for (int c = 0; c < DMAX / 4; ++c) {
    if (col_of(c, sub) < a.d) {
      const int col = col_of(c, sub);
      dkp[col] = (a.accumulate ? dkp[col] : 0.f) + dk.v[c];
      dvp[col] = (a.accumulate ? dvp[col] : 0.f) + dv.v[c];
    }
  }
}

}  // namespace

cudaError_t launch_simt_fwd(const AttnArgs& a, int q_rank, int kv_rank, cudaStream_t stream) {
  const int64_t L = a.N / a.P;
  if (L == 0 || a.B == 0 || a.Hq == 0) return cudaSuccess;
  dim3 grid((unsigned)ceil_div(L, kRows), (unsigned)a.Hq,
            (unsigned)(q_rank < 0 ? a.B * a.P : a.B));
  ProfScope ps("simt_fwd", stream);
  if (a.d <= 32) simt_fwd_kernel<32><<<grid, kThreads, 0, stream>>>(a, q_rank, kv_rank);
  else if (a.d <= 64) simt_fwd_kernel<64><<<grid, kThreads, 0, stream>>>(a, q_rank, kv_rank);
  else simt_fwd_kernel<128><<<grid, kThreads, 0, stream>>>(a, q_rank, kv_rank);
  return cudaGetLastError();
}

namespace {
template <typename InT>
cudaError_t launch_simt_bwd_t(const AttnArgs& a, int q_rank, int kv_rank, cudaStream_t stream) {
  const int64_t L = a.N / a.P;
  const unsigned z = (unsigned)(q_rank < 0 ? a.B * a.P : a.B);
  dim3 gq((unsigned)ceil_div(L, kRows), (unsigned)a.Hq, z);
  dim3 gk((unsigned)ceil_div(q_rank < 0 ? L : a.N / kv_shards(a), kRows), (unsigned)a.Hkv, z);
  if (a.d <= 32) {
    simt_bwd_dq_kernel<32, InT><<<gq, kThreads, 0, stream>>>(a, q_rank, kv_rank);
    simt_bwd_dkdv_kernel<32, InT><<<gk, kThreads, 0, stream>>>(a, q_rank, kv_rank);
  } else if (a.d <= 64) {
    simt_bwd_dq_kernel<64, InT><<<gq, kThreads, 0, stream>>>(a, q_rank, kv_rank);
    simt_bwd_dkdv_kernel<64, InT><<<gk, kThreads, 0, stream>>>(a, q_rank, kv_rank);
  } else {
    simt_bwd_dq_kernel<128, InT><<<gq, kThreads, 0, stream>>>(a, q_rank, kv_rank);
    simt_bwd_dkdv_kernel<128, InT><<<gk, kThreads, 0, stream>>>(a, q_rank, kv_rank);
  }
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_simt_bwd(const AttnArgs& a, int q_rank, int kv_rank, int in_bf16,
                            cudaStream_t stream) {
  const int64_t L = a.N / a.P;
  if (L == 0 || a.B == 0 || a.Hq == 0) return cudaSuccess;
  ProfScope ps("simt_bwd", stream);
  return in_bf16 ? launch_simt_bwd_t<__nv_bfloat16>(a, q_rank, kv_rank, stream)
                 : launch_simt_bwd_t<float>(a, q_rank, kv_rank, stream);
}

}  // namespace rm
