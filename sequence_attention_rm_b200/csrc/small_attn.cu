// Attention over very short sequences (L <= 16 tokens, d <= 64): the
// "local" backend of the Mosaic page (attention over a 5-token feature axis
// of a tabular tensor).  A 128-row tensor-core tile would be >95% padding
// here and the problem is HBM-bound, so one warp owns one (sequence, head):
// it stages q, k, v of the sequence in shared memory as fp32, computes the
// L x L scores, the softmax and O with fp32 FMAs, and writes O and the LSE.
// Consecutive warps take consecutive heads of one sequence, so a CTA reads
// contiguous token rows.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace rm {

namespace {

constexpr int kMaxL = 16;
constexpr int kMaxD = 64;
constexpr int kWarps = 2;  // 2 x (3 x 16 x 65 + 16 x 17) floats = 27 KB static smem

template <typename T>
__global__ void __launch_bounds__(kWarps * 32) small_seq_attn_kernel(AttnArgs a, int q_rank,
                                                                    int kv_rank) {
  __shared__ float sq[kWarps][kMaxL][kMaxD + 1];
  __shared__ float sk[kWarps][kMaxL][kMaxD + 1];
  __shared__ float sv[kWarps][kMaxL][kMaxD + 1];
  __shared__ float sp[kWarps][kMaxL][kMaxL + 1];
  const int wi = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const LayoutMap lay = make_layout(a.layout, a.N, a.P);
  const int L = (int)lay.L;
  const int d = a.d;
  const int64_t pair = (int64_t)blockIdx.x * kWarps + wi;  // (b, h) with h fastest
  if (pair >= (int64_t)a.B * a.Hq) return;
  const int h = (int)(pair % a.Hq);
  const int64_t b = pair / a.Hq;
  const int g = h / (a.Hq / a.Hkv);
  const T* qb = reinterpret_cast<const T*>(a.q.ptr) + b * a.q.stride_b + (int64_t)h * a.q.stride_h;
  const T* kb = reinterpret_cast<const T*>(a.k.ptr) + b * a.k.stride_b + (int64_t)g * a.k.stride_h;
  const T* vb = reinterpret_cast<const T*>(a.v.ptr) + b * a.v.stride_b + (int64_t)g * a.v.stride_h;
  for (int e = lane; e < L * d; e += 32) {
    const int t = e / d, c = e % d;
    sq[wi][t][c] = to_f32<T>(qb[t * a.q.stride_n + c]);
    sk[wi][t][c] = to_f32<T>(kb[t * a.k.stride_n + c]);
    sv[wi][t][c] = to_f32<T>(vb[t * a.v.stride_n + c]);
  }
  __syncwarp();
  // one lane per query row: scores, max, normaliser
  float lse = -INFINITY;
  if (lane < L) {
    const int64_t tq = lay.pos(q_rank, lane);
    float s[kMaxL];
    float m = -INFINITY;
#pragma unroll
    for (int u = 0; u < kMaxL; ++u) {
      s[u] = -INFINITY;
      if (u < L && (!a.causal || lay.pos(kv_rank, u) <= tq)) {
        float acc = 0.f;
        for (int c = 0; c < d; ++c) acc = fmaf(sq[wi][lane][c], sk[wi][u][c], acc);
        s[u] = acc * a.scale;
        m = fmaxf(m, s[u]);
      }
    }
    float z = 0.f;
#pragma unroll
    for (int u = 0; u < kMaxL; ++u) {
      const float e = (m == -INFINITY) ? 0.f : expf(s[u] - m);
      s[u] = e;
      z += e;
    }
    const float inv = z > 0.f ? 1.0f / z : 0.f;
#pragma unroll
    for (int u = 0; u < kMaxL; ++u) sp[wi][lane][u] = s[u] * inv;
    lse = z > 0.f ? m + logf(z) : -INFINITY;
  }
  __syncwarp();
  // O[t][c] = sum_u p[t][u] v[u][c], spread over the lanes
  char* ob = reinterpret_cast<char*>(a.o.ptr);
  for (int e = lane; e < L * d; e += 32) {
    const int t = e / d, c = e % d;
    float acc = 0.f;
    for (int u = 0; u < L; ++u) acc = fmaf(sp[wi][t][u], sv[wi][u][c], acc);
    const int64_t off = b * a.o.stride_b + (int64_t)t * a.o.stride_n + (int64_t)h * a.o.stride_h + c;
    if (a.o_f32) reinterpret_cast<float*>(ob)[off] = acc;
    else reinterpret_cast<__nv_bfloat16*>(ob)[off] = __float2bfloat16_rn(acc);
  }
  if (lane < L) a.lse[(b * a.Hq + h) * a.lse_ld + lane] = lse;
}

}  // namespace

bool small_seq_supported(int64_t L, int d) { return L >= 1 && L <= kMaxL && d <= kMaxD; }

cudaError_t launch_small_seq_fwd(const AttnArgs& a, int q_rank, int kv_rank, int bf16,
                                 cudaStream_t stream) {
  const int64_t pairs = (int64_t)a.B * a.Hq;
  if (pairs == 0) return cudaSuccess;
  const int64_t blocks = (pairs + kWarps - 1) / kWarps;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  ProfScope ps("small_seq_fwd", stream);
  if (bf16)
    small_seq_attn_kernel<__nv_bfloat16><<<(unsigned)blocks, kWarps * 32, 0, stream>>>(a, q_rank, kv_rank);
  else
    small_seq_attn_kernel<float><<<(unsigned)blocks, kWarps * 32, 0, stream>>>(a, q_rank, kv_rank);
  return cudaGetLastError();
}

}  // namespace rm
