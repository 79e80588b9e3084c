// Attention over very short sequences (L <= 16 tokens, d <= 64): the
// "local" backend of the Mosaic page (attention over a 5-token feature axis
// of a tabular tensor).  A 128-row tensor-core tile would be >95% padding
// here and the problem is HBM-bound, so the work is spread as thinly as it
// goes: one thread per (sequence, query token, head), heads fastest, so the
// threads of a warp read consecutive head rows of one token (coalesced) and
// share each key / value row through L1.  A thread keeps its query row in
// registers (pre-scaled into log2 units), scores the L keys, takes the
// softmax with the SFU exp2, accumulates O and writes O and the LSE.
// Rows are read as 16-byte vectors when every stride and the base pointers
// allow it (VEC), else element by element.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace rm {

namespace {

constexpr int kMaxL = 16;
constexpr int kMaxD = 64;
constexpr int kThreads = 256;

__device__ __forceinline__ float ex2(float x) {  // the SFU exp2
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

template <typename T, int DMAX, bool VEC>
__device__ __forceinline__ void load_row(const T* __restrict__ p, int d, float f, float (&out)[DMAX]) {
  if constexpr (VEC && sizeof(T) == 2) {
    const uint4* p4 = reinterpret_cast<const uint4*>(p);
#pragma unroll
    for (int i = 0; i < DMAX / 8; ++i) {
      if (8 * i < d) {
        const uint4 u = __ldg(p4 + i);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          out[8 * i + 2 * j] = __uint_as_float(w[j] << 16) * f;
          out[8 * i + 2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u) * f;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) out[8 * i + j] = 0.f;
      }
    }
  } else if constexpr (VEC) {  // fp32
    const float4* p4 = reinterpret_cast<const float4*>(p);
#pragma unroll
    for (int i = 0; i < DMAX / 4; ++i) {
      if (4 * i < d) {
        const float4 u = __ldg(p4 + i);
        out[4 * i] = u.x * f;
        out[4 * i + 1] = u.y * f;
        out[4 * i + 2] = u.z * f;
        out[4 * i + 3] = u.w * f;
      } else {
        out[4 * i] = out[4 * i + 1] = out[4 * i + 2] = out[4 * i + 3] = 0.f;
      }
    }
  } else {
#pragma unroll
    for (int c = 0; c < DMAX; ++c) out[c] = c < d ? to_f32<T>(p[c]) * f : 0.f;
  }
}

template <typename T, int DMAX, bool VEC>
__global__ void __launch_bounds__(kThreads) small_seq_attn_kernel(AttnArgs a, int q_rank,
                                                                 int kv_rank) {
  const LayoutMap lay = make_layout(a.layout, a.N, a.P);
  const int L = (int)lay.L;
  const int d = a.d;
  const int group = a.Hq / a.Hkv;
  const float qscale = a.scale * kLog2e;  // scores in log2 units
  const int64_t total = (int64_t)a.B * L * a.Hq;
  for (int64_t idx = (int64_t)blockIdx.x * kThreads + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * kThreads) {
    const int h = (int)(idx % a.Hq);
    const int64_t bt = idx / a.Hq;
    const int t = (int)(bt % L);
    const int64_t b = bt / L;
    const int g = h / group;
    const T* qrow = reinterpret_cast<const T*>(a.q.ptr) + b * a.q.stride_b +
                    (int64_t)t * a.q.stride_n + (int64_t)h * a.q.stride_h;
    const T* kb = reinterpret_cast<const T*>(a.k.ptr) + b * a.k.stride_b + (int64_t)g * a.k.stride_h;
    const T* vb = reinterpret_cast<const T*>(a.v.ptr) + b * a.v.stride_b + (int64_t)g * a.v.stride_h;
    float q[DMAX];
    load_row<T, DMAX, VEC>(qrow, d, qscale, q);
    const int64_t tq = lay.pos(q_rank, t);
    float s[kMaxL];
    float m = -INFINITY;
#pragma unroll
    for (int u = 0; u < kMaxL; ++u) {
      s[u] = -INFINITY;
      if (u < L && (!a.causal || lay.pos(kv_rank, u) <= tq)) {
        float kr[DMAX];
        load_row<T, DMAX, VEC>(kb + (int64_t)u * a.k.stride_n, d, 1.0f, kr);
        float acc = 0.f;
#pragma unroll
        for (int c = 0; c < DMAX; ++c) acc = fmaf(q[c], kr[c], acc);
        s[u] = acc;
        m = fmaxf(m, acc);
      }
    }
    float z = 0.f;
    float o[DMAX];
#pragma unroll
    for (int c = 0; c < DMAX; ++c) o[c] = 0.f;
#pragma unroll
    for (int u = 0; u < kMaxL; ++u) {
      if (u < L && s[u] != -INFINITY) {
        const float p = ex2(s[u] - m);
        z += p;
        float vr[DMAX];
        load_row<T, DMAX, VEC>(vb + (int64_t)u * a.v.stride_n, d, 1.0f, vr);
#pragma unroll
        for (int c = 0; c < DMAX; ++c) o[c] = fmaf(p, vr[c], o[c]);
      }
    }
    const float inv = z > 0.f ? 1.0f / z : 0.f;
    const int64_t off = b * a.o.stride_b + (int64_t)t * a.o.stride_n + (int64_t)h * a.o.stride_h;
    if (a.o_f32) {
      float* orow = reinterpret_cast<float*>(a.o.ptr) + off;
#pragma unroll
      for (int c = 0; c < DMAX; ++c)
        if (c < d) orow[c] = o[c] * inv;
    } else {
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.o.ptr) + off;
      if (VEC && d % 8 == 0) {
#pragma unroll
        for (int i = 0; i < DMAX / 8; ++i)
          if (8 * i < d) {
            uint4 u;
            u.x = pack2_bf16(o[8 * i] * inv, o[8 * i + 1] * inv);
            u.y = pack2_bf16(o[8 * i + 2] * inv, o[8 * i + 3] * inv);
            u.z = pack2_bf16(o[8 * i + 4] * inv, o[8 * i + 5] * inv);
            u.w = pack2_bf16(o[8 * i + 6] * inv, o[8 * i + 7] * inv);
            reinterpret_cast<uint4*>(orow)[i] = u;
          }
      } else {
#pragma unroll
        for (int c = 0; c < DMAX; ++c)
          if (c < d) orow[c] = __float2bfloat16_rn(o[c] * inv);
      }
    }
    a.lse[(b * a.Hq + h) * a.lse_ld + t] = z > 0.f ? (m + __log2f(z)) * kLn2 : -INFINITY;
  }
}

template <typename T, int DMAX, bool VEC>
cudaError_t launch(const AttnArgs& a, int q_rank, int kv_rank, int64_t total, cudaStream_t stream) {
  const int64_t need = (total + kThreads - 1) / kThreads;
  const int64_t cap = (int64_t)num_sms() * 16;
  const int blocks = (int)(need < cap ? need : cap);
  small_seq_attn_kernel<T, DMAX, VEC><<<blocks, kThreads, 0, stream>>>(a, q_rank, kv_rank);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_t(const AttnArgs& a, int q_rank, int kv_rank, int64_t total, bool vec,
                     cudaStream_t stream) {
  if (a.d <= 32)
    return vec ? launch<T, 32, true>(a, q_rank, kv_rank, total, stream)
               : launch<T, 32, false>(a, q_rank, kv_rank, total, stream);
  return vec ? launch<T, 64, true>(a, q_rank, kv_rank, total, stream)
             : launch<T, 64, false>(a, q_rank, kv_rank, total, stream);
}

}  // namespace

bool small_seq_supported(int64_t L, int d) { return L >= 1 && L <= kMaxL && d <= kMaxD; }

cudaError_t launch_small_seq_fwd(const AttnArgs& a, int q_rank, int kv_rank, int bf16,
                                 cudaStream_t stream) {
  const int64_t L = a.N / a.P;
  const int64_t total = (int64_t)a.B * L * a.Hq;
  if (total == 0) return cudaSuccess;
  // 16-byte rows: vector width in elements divides d, every stride and the bases
  const int w = bf16 ? 8 : 4, es = bf16 ? 2 : 4;
  auto ok = [&](const rm_tensor& x) {
    return ((uintptr_t)x.ptr % 16) == 0 && x.stride_b % w == 0 && x.stride_n % w == 0 &&
           x.stride_h % w == 0;
  };
  const bool vec = a.d % w == 0 && ok(a.q) && ok(a.k) && ok(a.v) && (a.d * es) % 16 == 0 &&
                   (a.o_f32 || (a.o.stride_b % 8 == 0 && a.o.stride_n % 8 == 0 &&
                                a.o.stride_h % 8 == 0 && (uintptr_t)a.o.ptr % 16 == 0));
  ProfScope ps("small_seq_fwd", stream);
  return bf16 ? launch_t<__nv_bfloat16>(a, q_rank, kv_rank, total, vec, stream)
              : launch_t<float>(a, q_rank, kv_rank, total, vec, stream);
}

}  // namespace rm
