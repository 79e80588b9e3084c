// Attention over very short sequences (L <= 16 tokens, d <= 64): the
// "local" backend of the Mosaic page (attention over a 5-token feature axis
// of a tabular tensor).  A 128-row tensor-core tile would be >95% padding
// here and the problem is HBM-bound, so one thread owns one (sequence, query
// token, head): it keeps its query row in registers, scores the L keys,
// takes the softmax with the SFU exp2, accumulates O and writes O and the
// LSE.  Two kernels:
//  - small_seq_tma_kernel (bf16 operands and output, d in {24, 32, 64}):
//    persistent and warp-specialised; a producer warp copies whole batches
//    of sequences into a shared-memory ring (bulk or TMA copies) and the
//    consumer threads read rows from shared memory, with mixed-precision
//    bf16 FMAs (see the comment above the kernel);
//  - small_seq_attn_kernel (fp32 operands, fp32 partial outputs): rows read
//    from global memory, heads fastest so that the threads of a warp read
//    consecutive head rows of one token and share key / value rows through
//    L1; 16-byte vectors when every stride and the base pointers allow it
//    (VEC), else element by element.
#include <math.h>

#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace rm {

rm_status encode_copy_map(CUtensorMap* map, const void* ptr, int esize, const int64_t (&dims)[5],
                          const int64_t (&strides)[4], const int (&box)[5]);
long long tc_wait_limit();

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

// bf16 operands with 16-byte rows: a warp-specialised persistent kernel.
// Batches of SB whole sequences flow through a ring of shared-memory stages:
// a producer warp issues, per batch, three asynchronous copies -- the Q, K
// and V rows of the batch -- onto the stage's "full" mbarrier, running up to
// kStagedStages batches ahead; eight consumer warps attend and release the
// stage on its "empty" mbarrier.  Dense operands take one bulk copy each (a
// batch is one run of memory); strided views take TMA boxes (D, H, L, SB) of
// their [B, L, H, D] maps, which read as zero past the last sequence.  So
// staging costs no per-element index arithmetic and no block-wide barrier.
// SB is chosen so that SB * L * Hq <= 256: each consumer thread owns one
// fixed (sequence, query token, head) slot of every batch, decoded once,
// scores its keys from shared memory with packed fp32 FMAs, and writes its O
// row (16-byte stores) and its LSE (a batch's LSE values are one contiguous
// range of the [B, H, L] output, so a warp's stores share few sectors).
// Only when L * Hq > 256 (then SB = 1) does a thread take several slots.
struct StagedLayout {
  int SB;
  uint32_t q_bytes, kv_bytes;  // box bytes of a full batch (the TMA transaction sizes)
  uint32_t off_k, off_v;       // within a stage
  uint32_t stage_bytes;
  uint32_t off_bar, total;
};

constexpr int kStagedStages = 3;
constexpr int kConsumerWarps = kThreads / 32;
constexpr int kStagedThreads = kThreads + 32;     // consumers + one producer warp
constexpr uint32_t kStagedSmemPerSm = 220 * 1024;  // shared memory the blocks of one SM share

__host__ __device__ inline uint32_t round128(uint32_t x) { return (x + 127u) & ~127u; }

__host__ __device__ inline StagedLayout staged_layout(int SB, int L, int Hq, int Hkv, int d) {
  StagedLayout g;
  g.SB = SB;
  g.q_bytes = (uint32_t)SB * L * Hq * d * 2;
  g.kv_bytes = (uint32_t)SB * L * Hkv * d * 2;
  g.off_k = round128(g.q_bytes);
  g.off_v = g.off_k + round128(g.kv_bytes);
  g.stage_bytes = g.off_v + round128(g.kv_bytes);
  g.off_bar = kStagedStages * g.stage_bytes;
  g.total = g.off_bar + 16 * kStagedStages;  // full and empty barrier per stage
  return g;
}

// One contiguous run of global memory into shared memory through the bulk
// copy unit, completing `bytes` on the mbarrier (16-byte aligned addresses,
// size a multiple of 16; no multicast).
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(tc::smem_u32(smem_dst)),
      "l"(gsrc), "r"(bytes), "r"(tc::smem_u32(bar))
      : "memory");
}

// acc + a.lo * b.lo + a.hi * b.hi for two bf16 pairs a, b (32-bit words), with
// fp32 accumulation: the mixed-precision FMA takes the bf16 halves directly
// (a bf16 x bf16 product is exact in fp32), so nothing is unpacked.
__device__ __forceinline__ float dot2_bf16(uint32_t a, uint32_t b, float acc) {
  float r;
  asm("{\n\t.reg .b16 al, ah, bl, bh;\n\t"
      "mov.b32 {al, ah}, %1;\n\t"
      "mov.b32 {bl, bh}, %2;\n\t"
      "fma.rn.f32.bf16 %0, al, bl, %3;\n\t"
      "fma.rn.f32.bf16 %0, ah, bh, %0;\n\t}"
      : "=f"(r)
      : "r"(a), "r"(b), "f"(acc));
  return r;
}
// (o.x, o.y) += p * (v.lo, v.hi), p a bf16 in the low half of a 16-bit word
__device__ __forceinline__ void axpy2_bf16(uint16_t p, uint32_t v, float2& o) {
  asm("{\n\t.reg .b16 vl, vh;\n\t"
      "mov.b32 {vl, vh}, %2;\n\t"
      "fma.rn.f32.bf16 %0, %3, vl, %0;\n\t"
      "fma.rn.f32.bf16 %1, %3, vh, %1;\n\t}"
      : "+f"(o.x), "+f"(o.y)
      : "r"(v), "h"(p));
}

// Registers per thread the launch bounds allow: two blocks per SM up to
// D = 32, one block at D = 64.
template <int D>
constexpr int staged_blocks_per_sm() { return D <= 32 ? 2 : 1; }

template <int D, int LMAX>
__global__ void __launch_bounds__(kStagedThreads, staged_blocks_per_sm<D>())
    small_seq_tma_kernel(const __grid_constant__ CUtensorMap mq,
                         const __grid_constant__ CUtensorMap mk,
                         const __grid_constant__ CUtensorMap mv, AttnArgs a, int q_rank,
                         int kv_rank, StagedLayout g, int contiguous, long long wait_limit) {
  extern __shared__ __align__(128) unsigned char smem[];
  using namespace tc;
  constexpr int S = kStagedStages;
  const int L = (int)(a.N / a.P);
  const int Hq = a.Hq, Hkv = a.Hkv;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + g.off_bar);
  uint64_t* empty = full + S;
  const int64_t nbatch = ((int64_t)a.B + g.SB - 1) / g.SB;
  const int64_t mine =
      nbatch > blockIdx.x ? (nbatch - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if ((smem_u32(smem) & 127u) != 0) {  // TMA boxes need a 128-byte aligned destination
    if (threadIdx.x == 0) report_status(a.status, kStatusSmemAlign);
    return;
  }
  if (threadIdx.x == 0) {
    for (int st = 0; st < S; ++st) {
      mbar_init(full + st, 1);
      mbar_init(empty + st, kConsumerWarps);
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ---- producer ----------------------------------------------------------
    if (lane != 0) return;
    int64_t issued = 0;
    for (; issued < mine; ++issued) {
      const int st = (int)(issued % S);
      if (issued >= S &&
          !mbar_wait(empty + st, (uint32_t)((issued / S - 1) & 1), wait_limit, a.status))
        break;
      unsigned char* dst = smem + st * g.stage_bytes;
      const int bc = (int)((blockIdx.x + issued * gridDim.x) * g.SB);
      if (contiguous) {
        // the batch's rows of each operand are one run: sb sequences of L*H*D
        const int sb = a.B - bc < g.SB ? a.B - bc : g.SB;
        const uint32_t qb = g.q_bytes / g.SB * sb, kvb = g.kv_bytes / g.SB * sb;
        mbar_arrive_expect_tx(full + st, qb + 2 * kvb);
        const size_t qoff = (size_t)bc * a.q.stride_b * 2, koff = (size_t)bc * a.k.stride_b * 2;
        bulk_load(dst, reinterpret_cast<const char*>(a.q.ptr) + qoff, qb, full + st);
        bulk_load(dst + g.off_k, reinterpret_cast<const char*>(a.k.ptr) + koff, kvb, full + st);
        bulk_load(dst + g.off_v, reinterpret_cast<const char*>(a.v.ptr) + koff, kvb, full + st);
      } else {
        mbar_arrive_expect_tx(full + st, g.q_bytes + 2 * g.kv_bytes);
        tma_load_5d(dst, &mq, full + st, 0, 0, 0, bc, 0);
        tma_load_5d(dst + g.off_k, &mk, full + st, 0, 0, 0, bc, 0);
        tma_load_5d(dst + g.off_v, &mv, full + st, 0, 0, 0, bc, 0);
      }
    }
    if (issued < mine) {
      // a timeout: the copies already issued may still be landing; wait for
      // the latest one of every stage (bounded) before leaving
      for (int64_t j = issued - 1; j >= 0 && j >= issued - S; --j)
        mbar_wait(full + (int)(j % S), (uint32_t)((j / S) & 1), wait_limit, a.status);
    }
    return;
  }

  // ---- consumers -------------------------------------------------------------
  const LayoutMap lay = make_layout(a.layout, a.N, a.P);
  const int group = Hq / Hkv;
  const float qscale = a.scale * kLog2e;  // scores in log2 units
  const int slots = g.SB * L * Hq;        // (s, t, h) slots of a full batch, h fastest
  // this thread's first slot, decoded once
  const int h0 = threadIdx.x % Hq;
  const int t0 = (threadIdx.x / Hq) % L;
  const int s0 = threadIdx.x / (Hq * L);
  for (int64_t k = 0; k < mine; ++k) {
    const int st = (int)(k % S);
    const bool ok = mbar_wait(full + st, (uint32_t)((k / S) & 1), wait_limit, a.status);
    if (!__all_sync(0xffffffffu, ok)) return;  // a timeout ends the warp as a whole
    const unsigned char* base = smem + st * g.stage_bytes;
    const __nv_bfloat16* qs = reinterpret_cast<const __nv_bfloat16*>(base);
    const __nv_bfloat16* ks = reinterpret_cast<const __nv_bfloat16*>(base + g.off_k);
    const __nv_bfloat16* vs = reinterpret_cast<const __nv_bfloat16*>(base + g.off_v);
    const int64_t b0 = (blockIdx.x + k * gridDim.x) * g.SB;
    const int sb = (int)((int64_t)a.B - b0 < g.SB ? (int64_t)a.B - b0 : g.SB);
    for (int idx = threadIdx.x; idx < slots; idx += kThreads) {
      int h = h0, t = t0, s = s0;
      if (idx != (int)threadIdx.x) {
        h = idx % Hq;
        t = (idx / Hq) % L;
        s = idx / (Hq * L);
      }
      if (s >= sb) break;  // the last batch may hold fewer sequences
      const int kvh = h / group;
      uint32_t q[D / 2];  // raw bf16 pairs
      {
        const uint4* q4 = reinterpret_cast<const uint4*>(qs + ((size_t)(s * L + t) * Hq + h) * D);
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
          const uint4 w = q4[i];
          q[4 * i] = w.x;
          q[4 * i + 1] = w.y;
          q[4 * i + 2] = w.z;
          q[4 * i + 3] = w.w;
        }
      }
      const int64_t tq = lay.pos(q_rank, t);
      const __nv_bfloat16* kseq = ks + ((size_t)s * L * Hkv + kvh) * D;  // key 0 of sequence s
      const __nv_bfloat16* vseq = vs + ((size_t)s * L * Hkv + kvh) * D;
      float sc[LMAX];
      float m = -INFINITY;
#pragma unroll
      for (int u = 0; u < LMAX; ++u) {
        sc[u] = -INFINITY;
        if (u < L && (!a.causal || lay.pos(kv_rank, u) <= tq)) {
          const uint4* k4 = reinterpret_cast<const uint4*>(kseq + (size_t)u * Hkv * D);
          float acc0 = 0.f, acc1 = 0.f;  // two chains
#pragma unroll
          for (int i = 0; i < D / 8; ++i) {
            const uint4 w = k4[i];
            acc0 = dot2_bf16(q[4 * i], w.x, acc0);
            acc1 = dot2_bf16(q[4 * i + 1], w.y, acc1);
            acc0 = dot2_bf16(q[4 * i + 2], w.z, acc0);
            acc1 = dot2_bf16(q[4 * i + 3], w.w, acc1);
          }
          sc[u] = (acc0 + acc1) * qscale;
          m = fmaxf(m, sc[u]);
        }
      }
      // O accumulates bf16(p) * V in fp32 (the probabilities enter the
      // product in bf16, as they do in the tensor-core kernels' P V); the
      // normaliser z sums the fp32 p
      float z = 0.f;
      float2 o[D / 2];
#pragma unroll
      for (int c = 0; c < D / 2; ++c) o[c] = make_float2(0.f, 0.f);
#pragma unroll
      for (int u = 0; u < LMAX; ++u) {
        if (u < L && sc[u] != -INFINITY) {
          const float p = ex2(sc[u] - m);
          z += p;
          const __nv_bfloat16 pb = __float2bfloat16_rn(p);
          const uint16_t ph = *reinterpret_cast<const uint16_t*>(&pb);
          const uint4* v4 = reinterpret_cast<const uint4*>(vseq + (size_t)u * Hkv * D);
#pragma unroll
          for (int i = 0; i < D / 8; ++i) {
            const uint4 w = v4[i];
            axpy2_bf16(ph, w.x, o[4 * i]);
            axpy2_bf16(ph, w.y, o[4 * i + 1]);
            axpy2_bf16(ph, w.z, o[4 * i + 2]);
            axpy2_bf16(ph, w.w, o[4 * i + 3]);
          }
        }
      }
      const float inv = z > 0.f ? 1.0f / z : 0.f;
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.o.ptr) + (b0 + s) * a.o.stride_b +
                            (int64_t)t * a.o.stride_n + (int64_t)h * a.o.stride_h;
#pragma unroll
      for (int i = 0; i < D / 8; ++i) {
        uint4 w;
        w.x = pack2_bf16(o[4 * i].x * inv, o[4 * i].y * inv);
        w.y = pack2_bf16(o[4 * i + 1].x * inv, o[4 * i + 1].y * inv);
        w.z = pack2_bf16(o[4 * i + 2].x * inv, o[4 * i + 2].y * inv);
        w.w = pack2_bf16(o[4 * i + 3].x * inv, o[4 * i + 3].y * inv);
        reinterpret_cast<uint4*>(orow)[i] = w;
      }
      a.lse[((b0 + s) * Hq + h) * a.lse_ld + t] = z > 0.f ? (m + __log2f(z)) * kLn2 : -INFINITY;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty + st);  // this warp is done with the stage
  }
}

// The [B, L, H, D] operand x as a TMA map with box (D, H, L, SB).
rm_status staged_map(CUtensorMap* m, const rm_tensor& x, int64_t B, int L, int H, int d, int SB) {
  const int64_t dims[5] = {d, H, L, B, 1};
  const int64_t strides[4] = {x.stride_h * 2, x.stride_n * 2, x.stride_b * 2, x.stride_b * 2};
  const int box[5] = {d, H, L, SB, 1};
  return encode_copy_map(m, x.ptr, 2, dims, strides, box);
}

template <int D>
cudaError_t launch_staged(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                          const AttnArgs& a, int q_rank, int kv_rank, const StagedLayout& g,
                          int contiguous, int64_t nbatch, cudaStream_t stream) {
  // the key loops unroll to 8 or 16 keys
  auto kern = a.N / a.P <= 8 ? small_seq_tma_kernel<D, 8> : small_seq_tma_kernel<D, kMaxL>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)g.total);
  if (e != cudaSuccess) return e;
  const int per_sm = (int)(kStagedSmemPerSm / g.total) < staged_blocks_per_sm<D>()
                         ? (int)(kStagedSmemPerSm / g.total)
                         : staged_blocks_per_sm<D>();
  const int64_t cap = (int64_t)num_sms() * (per_sm < 1 ? 1 : per_sm);
  const unsigned grid = (unsigned)(nbatch < cap ? nbatch : cap);
  kern<<<grid, kStagedThreads, g.total, stream>>>(mq, mk, mv, a, q_rank, kv_rank, g, contiguous,
                                                  tc_wait_limit());
  return cudaGetLastError();
}

// Launches the staged kernel if the problem fits it; false (nothing
// launched) otherwise, and the caller takes the one-thread-per-row kernel.
bool try_launch_staged(const AttnArgs& a, int q_rank, int kv_rank, int64_t L, cudaStream_t stream,
                       cudaError_t* err) {
  if (a.B < 1 || a.Hq > 256 || a.Hkv > 256 || L > kMaxL || (a.d != 24 && a.d != 32 && a.d != 64))
    return false;
  // TMA strides: nonzero multiples of 16 bytes; 16-byte aligned bases
  for (const rm_tensor* x : {&a.q, &a.k, &a.v})
    if (x->stride_b <= 0 || x->stride_n <= 0 || x->stride_h <= 0 || ((uintptr_t)x->ptr & 15))
      return false;
  // one slot per consumer thread, and every stage within a third of the
  // shared memory the SM's blocks share
  int SB = (int)(kThreads / (L * a.Hq));
  if (SB < 1) SB = 1;
  if (SB > 256) SB = 256;
  while (SB > 1 && staged_layout(SB, (int)L, a.Hq, a.Hkv, a.d).total > kStagedSmemPerSm / 2) --SB;
  const StagedLayout g = staged_layout(SB, (int)L, a.Hq, a.Hkv, a.d);
  if (g.total > kStagedSmemPerSm) return false;
  CUtensorMap mq, mk, mv;
  if (staged_map(&mq, a.q, a.B, (int)L, a.Hq, a.d, SB) != RM_OK ||
      staged_map(&mk, a.k, a.B, (int)L, a.Hkv, a.d, SB) != RM_OK ||
      staged_map(&mv, a.v, a.B, (int)L, a.Hkv, a.d, SB) != RM_OK)
    return false;
  // every batch of each operand one contiguous run (dense [B, L, H, d])
  auto dense = [&](const rm_tensor& x, int H) {
    return x.stride_h == a.d && x.stride_n == (int64_t)H * a.d && x.stride_b == L * H * a.d;
  };
  const int contiguous = dense(a.q, a.Hq) && dense(a.k, a.Hkv) && dense(a.v, a.Hkv) &&
                         a.k.stride_b == a.v.stride_b;
  const int64_t nbatch = ((int64_t)a.B + SB - 1) / SB;
  if (a.d == 24)
    *err = launch_staged<24>(mq, mk, mv, a, q_rank, kv_rank, g, contiguous, nbatch, stream);
  else if (a.d == 32)
    *err = launch_staged<32>(mq, mk, mv, a, q_rank, kv_rank, g, contiguous, nbatch, stream);
  else
    *err = launch_staged<64>(mq, mk, mv, a, q_rank, kv_rank, g, contiguous, nbatch, stream);
  return true;
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
  cudaError_t err = cudaSuccess;
  if (bf16 && vec && !a.o_f32 && try_launch_staged(a, q_rank, kv_rank, L, stream, &err))
    return err;
  return bf16 ? launch_t<__nv_bfloat16>(a, q_rank, kv_rank, total, vec, stream)
              : launch_t<float>(a, q_rank, kv_rank, total, vec, stream);
}

}  // namespace rm
