// C ABI of librm_attn.so: argument validation, workspace carving and kernel
// dispatch.  Every entry point validates on the host and returns before any
// launch on a bad argument; no entry point allocates device memory.
#include <math.h>
#include <stdint.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <mutex>
#include <string>

#include "common.cuh"
#include "internal.h"
#include "tc_attn.h"

namespace rm {

__device__ unsigned int g_device_status;  // bit kStatusTimeout: a bounded wait expired

namespace {
thread_local std::string t_last_error;

rm_status fail(rm_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
rm_status fail(rm_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return s;
}

rm_status cuda_fail(cudaError_t e, const char* where) {
  return fail(RM_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int g_sms[kMaxDevices];

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  return dev < 0 || dev >= kMaxDevices ? 0 : dev;
}

int esize_of(rm_dtype t) { return t == RM_BF16 ? 2 : 4; }

// Inner batch entries per caller batch entry, for the segment arrays.  USP
// runs its ring with every (batch entry, head group) as a batch entry of its
// own, so u inner entries share one seq_lens entry, and a packed batch (which
// the caller gives with B == 1) reaches the ring with B == u.  USP sets it for
// the duration of its inner calls on the calling thread; 1 everywhere else.
thread_local int t_seg_div = 1;
struct SegDivScope {
  int prev;
  explicit SegDivScope(int u) : prev(t_seg_div) { t_seg_div = u; }
  ~SegDivScope() { t_seg_div = prev; }
};

rm_status check_desc(const rm_attn_desc* d) {
  if (!d) return fail(RM_ERR_INVALID_ARG, "desc is NULL");
  if (d->dtype != RM_F32 && d->dtype != RM_BF16) return fail(RM_ERR_INVALID_ARG, "bad dtype");
  if (d->B < 0 || d->N < 0 || d->P < 1 || d->Hq < 1 || d->Hkv < 1)
    return fail(RM_ERR_INVALID_ARG, "bad sizes (B=%d N=%lld P=%d Hq=%d Hkv=%d)", d->B,
                (long long)d->N, d->P, d->Hq, d->Hkv);
  if (d->N > INT32_MAX) return fail(RM_ERR_INVALID_ARG, "N must be < 2^31");
  if (d->Hq % d->Hkv) return fail(RM_ERR_INVALID_ARG, "Hq %% Hkv != 0");
  if (d->layout != RM_LAYOUT_CONTIGUOUS && d->layout != RM_LAYOUT_ZIGZAG &&
      d->layout != RM_LAYOUT_STRIPED)
    return fail(RM_ERR_INVALID_ARG, "bad layout");
  if (d->N % d->P) return fail(RM_ERR_INVALID_ARG, "N %% P != 0");
  if (d->layout == RM_LAYOUT_ZIGZAG && d->N % (2 * (int64_t)d->P))
    return fail(RM_ERR_INVALID_ARG, "zigzag needs N %% 2P == 0");
  if (d->mode != RM_RING_FUSED && d->mode != RM_RING_STEPWISE)
    return fail(RM_ERR_INVALID_ARG, "bad ring mode");
  if (d->order != RM_ORDER_RANK_MAJOR && d->order != RM_ORDER_GLOBAL)
    return fail(RM_ERR_INVALID_ARG, "bad token order");
  if (d->cu_seqlens && d->seq_lens)
    return fail(RM_ERR_INVALID_ARG, "cu_seqlens and seq_lens are exclusive");
  if (d->cu_seqlens && (d->num_segments < 1 || d->B != t_seg_div))
    return fail(RM_ERR_INVALID_ARG, "packing needs num_segments >= 1 and B == 1");
  if (!(d->scale == d->scale) || isinf(d->scale)) return fail(RM_ERR_INVALID_ARG, "bad scale");
  if (d->dtype == RM_BF16) {
    if (!tc_supported_head_dim(d->d))
      return fail(RM_ERR_UNSUPPORTED, "bf16 head dim %d not in {24, 32, 64, 128}", d->d);
  } else {
    if (d->d < 4 || d->d > 128 || d->d % 4)
      return fail(RM_ERR_UNSUPPORTED, "fp32 head dim %d: need d %% 4 == 0, d <= 128", d->d);
  }
  return RM_OK;
}

// The ring entry points with global-order operands: the tensor-core kernels
// fetch rank tiles through the layout (contiguous: global = rank-major).
rm_status check_order(const rm_attn_desc* d, int backward) {
  if (d->order != RM_ORDER_GLOBAL || d->layout == RM_LAYOUT_CONTIGUOUS || d->P == 1) return RM_OK;
  if (d->dtype != RM_BF16)
    return fail(RM_ERR_UNSUPPORTED, "global token order needs bf16 (the tensor-core path)");
  if (backward && d->d != 128)
    return fail(RM_ERR_UNSUPPORTED,
                "global token order in the backward needs head dim 128 (the tensor-core path)");
  if (!backward && d->mode != RM_RING_FUSED)
    return fail(RM_ERR_UNSUPPORTED, "global token order needs the fused ring mode");
  if (d->layout == RM_LAYOUT_ZIGZAG && (d->N / (2 * (int64_t)d->P)) % 128)
    return fail(RM_ERR_UNSUPPORTED,
                "global token order with zigzag needs chunks of a multiple of 128 tokens");
  return RM_OK;
}

float eff_scale(const rm_attn_desc* d) {
  return d->scale > 0.f ? d->scale : 1.0f / sqrtf((float)d->d);
}

// A strided [B, rows, H, d] operand: pointer and strides must keep every row
// `align` bytes aligned (16 for TMA operands; 4 elements for the row kernels).
rm_status check_tensor(const char* name, rm_tensor t, int esize, int64_t rows, int heads, int d,
                       int align = 16) {
  if (rows == 0) return RM_OK;
  if (!t.ptr) return fail(RM_ERR_INVALID_ARG, "%s: NULL pointer", name);
  if ((uintptr_t)t.ptr % align)
    return fail(RM_ERR_INVALID_ARG, "%s: pointer not %d-byte aligned", name, align);
  if (t.stride_b < 0 || t.stride_n <= 0 || t.stride_h < 0)
    return fail(RM_ERR_INVALID_ARG, "%s: negative / zero stride", name);
  if ((t.stride_b * esize) % align || (t.stride_n * esize) % align || (t.stride_h * esize) % align)
    return fail(RM_ERR_INVALID_ARG, "%s: strides * element size must be multiples of %d bytes",
                name, align);
  if (heads > 1 && t.stride_h < d)
    return fail(RM_ERR_INVALID_ARG, "%s: head stride smaller than d (overlapping heads)", name);
  return RM_OK;
}

#define RM_TRY(x)                   \
  do {                              \
    rm_status _s = (x);             \
    if (_s != RM_OK) return _s;     \
  } while (0)

#define RM_CUDA(x, where)                               \
  do {                                                  \
    cudaError_t _e = (x);                               \
    if (_e != cudaSuccess) return cuda_fail(_e, where); \
  } while (0)

size_t align_up(size_t x) { return (x + 255) & ~(size_t)255; }

// Workspace layout (byte offsets from ws).
struct FwdWs {
  size_t o_parts, lse_parts, total;
};
FwdWs fwd_ws(const rm_attn_desc* d) {
  FwdWs w{0, 0, 0};
  if (d->mode != RM_RING_STEPWISE) return w;
  const size_t rows = (size_t)d->B * d->N * d->Hq;
  w.o_parts = 0;
  w.lse_parts = align_up(rows * d->d * 4 * (size_t)d->P);
  w.total = w.lse_parts + align_up(rows * 4 * (size_t)d->P);
  return w;
}
// The bf16 backward at head dims other than 128 runs on the SIMT kernels
// (bf16 operands read as fp32) into fp32 dQ / dK / dV, then rounds them.
bool bf16_simt_bwd(const rm_attn_desc* d) { return d->dtype == RM_BF16 && d->d != 128; }

struct BwdWs {
  size_t delta, dq, dk, dv, total;  // dq / dk / dv: fp32 [B, N, H, d], bf16 SIMT backward only
};
BwdWs bwd_ws(const rm_attn_desc* d) {
  BwdWs w;
  memset(&w, 0, sizeof(w));
  const size_t rows_q = (size_t)d->B * d->N * d->Hq, rows_kv = (size_t)d->B * d->N * d->Hkv;
  w.delta = 0;
  // the tensor-core and fp32 backward paths write dQ / dK / dV themselves:
  // delta is all they keep
  w.total = align_up(rows_q * 4);
  if (bf16_simt_bwd(d)) {
    w.dq = w.total;
    w.dk = w.dq + align_up(rows_q * d->d * 4);
    w.dv = w.dk + align_up(rows_kv * d->d * 4);
    w.total = w.dv + align_up(rows_kv * d->d * 4);
  }
  return w;
}

rm_tensor dense_bnhd(void* p, int64_t N, int H, int d) {
  rm_tensor t;
  t.ptr = p;
  t.stride_b = N * H * d;
  t.stride_n = (int64_t)H * d;
  t.stride_h = d;
  return t;
}

rm_tensor offset_rows(rm_tensor t, int64_t rows, int esize) {
  t.ptr = (char*)t.ptr + rows * t.stride_n * esize;
  return t;
}

}  // namespace

// Records a one-line reason for the calling thread's next rm_last_error().
void set_last_error(const char* msg) { t_last_error = msg; }

int num_sms() {
  int dev = current_device();
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_sms[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    g_sms[dev] = n;
  }
  return g_sms[dev];
}

// The status word's device address in the current context.  It is looked up
// on every call, not cached: a __device__ variable's address belongs to the
// context that loaded the module, and a caller may switch contexts or reset
// the device between calls (the lookup is a table search once the module is
// loaded).
unsigned int* status_word() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
  return (unsigned int*)p;
}

}  // namespace rm

using namespace rm;

extern "C" {

const char* rm_status_string(rm_status s) {
  switch (s) {
    case RM_OK: return "RM_OK";
    case RM_ERR_INVALID_ARG: return "RM_ERR_INVALID_ARG";
    case RM_ERR_UNSUPPORTED: return "RM_ERR_UNSUPPORTED";
    case RM_ERR_WORKSPACE: return "RM_ERR_WORKSPACE";
    case RM_ERR_CUDA: return "RM_ERR_CUDA";
    case RM_ERR_TIMEOUT: return "RM_ERR_TIMEOUT";
  }
  return "RM_ERR_UNKNOWN";
}

const char* rm_last_error(void) { return t_last_error.c_str(); }

rm_status rm_get_device_status(void* stream) {
  cudaStream_t st = (cudaStream_t)stream;
  RM_CUDA(cudaStreamSynchronize(st), "rm_get_device_status: stream sync");
  unsigned int* p = status_word();
  if (!p) return fail(RM_ERR_CUDA, "rm_get_device_status: no status word");
  unsigned int v = 0;
  RM_CUDA(cudaMemcpyAsync(&v, p, sizeof(v), cudaMemcpyDeviceToHost, st), "status read");
  RM_CUDA(cudaMemsetAsync(p, 0, sizeof(v), st), "status clear");
  RM_CUDA(cudaStreamSynchronize(st), "status sync");
  if (v & kStatusTimeout) return fail(RM_ERR_TIMEOUT, "a device-side bounded wait expired");
  if (v & kStatusSmemAlign)
    return fail(RM_ERR_CUDA, "a kernel found its dynamic shared memory not 1024-byte aligned");
  return RM_OK;
}

rm_status rm_debug_exp2_poly(const float* x, float* y, int64_t n, void* stream) {
  if (n < 0 || (n > 0 && (!x || !y)))
    return fail(RM_ERR_INVALID_ARG, "rm_debug_exp2_poly: bad pointers or size");
  RM_CUDA(launch_debug_exp2_poly(x, y, n, (cudaStream_t)stream), "exp2 poly launch");
  return RM_OK;
}

rm_status rm_debug_expire_wait(uint32_t spin_limit, void* stream) {
  unsigned int* p = status_word();
  if (!p) return fail(RM_ERR_CUDA, "no status word");
  RM_CUDA(launch_debug_expire_wait(spin_limit, p, (cudaStream_t)stream), "debug wait launch");
  return RM_OK;
}

rm_status rm_layout_permute(rm_dtype dtype, int B, int64_t N, int H, int d, rm_layout layout,
                            int P, int inverse, const void* in, void* out, void* stream) {
  if (dtype != RM_F32 && dtype != RM_BF16) return fail(RM_ERR_INVALID_ARG, "bad dtype");
  if (B < 0 || N < 0 || H < 1 || d < 1 || P < 1) return fail(RM_ERR_INVALID_ARG, "bad sizes");
  if (layout != RM_LAYOUT_CONTIGUOUS && layout != RM_LAYOUT_ZIGZAG && layout != RM_LAYOUT_STRIPED)
    return fail(RM_ERR_INVALID_ARG, "bad layout");
  if (N % P) return fail(RM_ERR_INVALID_ARG, "N %% P != 0");
  if (layout == RM_LAYOUT_ZIGZAG && N % (2 * (int64_t)P))
    return fail(RM_ERR_INVALID_ARG, "zigzag needs N %% 2P == 0");
  if (inverse != 0 && inverse != 1) return fail(RM_ERR_INVALID_ARG, "inverse must be 0 or 1");
  const int64_t bytes = (int64_t)B * N * H * d * esize_of(dtype);
  if (bytes == 0) return RM_OK;
  if (!in || !out) return fail(RM_ERR_INVALID_ARG, "NULL pointer");
  if ((const char*)in < (const char*)out + bytes && (const char*)out < (const char*)in + bytes)
    return fail(RM_ERR_INVALID_ARG, "in and out overlap");
  RM_CUDA(launch_layout_permute(esize_of(dtype), B, N, H, d, layout, P, inverse, in, out,
                                (cudaStream_t)stream),
          "layout_permute launch");
  return RM_OK;
}

rm_status rm_seq_head_repack(rm_dtype dtype, int P, int64_t N_local, int H, int d,
                             int head_to_seq, const void* in, void* out, void* stream) {
  if (dtype != RM_F32 && dtype != RM_BF16) return fail(RM_ERR_INVALID_ARG, "bad dtype");
  if (P < 1 || N_local < 0 || H < 1 || d < 1) return fail(RM_ERR_INVALID_ARG, "bad sizes");
  if (H % P) return fail(RM_ERR_INVALID_ARG, "H %% P != 0 (Ulysses degree exceeds heads)");
  if (head_to_seq != 0 && head_to_seq != 1)
    return fail(RM_ERR_INVALID_ARG, "head_to_seq must be 0 or 1");
  const int64_t bytes = (int64_t)P * N_local * H * d * esize_of(dtype);
  if (bytes == 0) return RM_OK;
  if (!in || !out) return fail(RM_ERR_INVALID_ARG, "NULL pointer");
  if ((const char*)in < (const char*)out + bytes && (const char*)out < (const char*)in + bytes)
    return fail(RM_ERR_INVALID_ARG, "in and out overlap");
  RM_CUDA(launch_seq_head_repack(esize_of(dtype), P, N_local, H, d, head_to_seq, in, out,
                                 (cudaStream_t)stream),
          "seq_head_repack launch");
  return RM_OK;
}

rm_status rm_convert_f32(rm_dtype out_dtype, int B, int64_t N, int H, int d, rm_tensor in,
                         rm_tensor out, void* stream) {
  if (out_dtype != RM_F32 && out_dtype != RM_BF16) return fail(RM_ERR_INVALID_ARG, "bad dtype");
  if (B < 0 || N < 0 || H < 1 || d < 4 || d % 4) return fail(RM_ERR_INVALID_ARG, "bad sizes");
  const int64_t rows = (int64_t)B * N;
  if (rows == 0) return RM_OK;
  RM_TRY(check_tensor("in", in, 4, rows, H, d, 16));
  RM_TRY(check_tensor("out", out, esize_of(out_dtype), rows, H, d, out_dtype == RM_BF16 ? 8 : 16));
  RM_CUDA(launch_convert_f32(out_dtype == RM_BF16, B, N, H, d, in, out, (cudaStream_t)stream),
          "convert launch");
  return RM_OK;
}

rm_status rm_lse_merge(rm_dtype out_dtype, int B, int H, int64_t Nq, int d, int n_parts,
                       const rm_tensor* o_parts, const float* const* lse_parts, rm_tensor o_out,
                       float* lse_out, void* stream) {
  if (out_dtype != RM_F32 && out_dtype != RM_BF16) return fail(RM_ERR_INVALID_ARG, "bad dtype");
  if (B < 0 || H < 1 || Nq < 0 || d < 4 || d > 128 || d % 4)
    return fail(RM_ERR_INVALID_ARG, "bad sizes (need d %% 4 == 0, 4 <= d <= 128)");
  if (n_parts < 1 || n_parts > kMaxMergeParts)
    return fail(RM_ERR_INVALID_ARG, "n_parts must be in [1, %d]", kMaxMergeParts);
  if (!o_parts || !lse_parts) return fail(RM_ERR_INVALID_ARG, "NULL part arrays");
  const int64_t rows = (int64_t)B * Nq;
  if (rows == 0) return RM_OK;
  MergeArgs a;
  memset(&a, 0, sizeof(a));
  a.B = B;
  a.H = H;
  a.d = d;
  a.Nq = Nq;
  a.n_parts = n_parts;
  a.lse_ld = Nq;
  for (int i = 0; i < n_parts; ++i) {
    RM_TRY(check_tensor("o_parts[i]", o_parts[i], 4, rows, H, d, 16));
    if (!lse_parts[i] || ((uintptr_t)lse_parts[i] & 3))
      return fail(RM_ERR_INVALID_ARG, "lse_parts[%d] NULL or misaligned", i);
    a.o_ptr[i] = (const float*)o_parts[i].ptr;
    a.o_sb[i] = o_parts[i].stride_b;
    a.o_sn[i] = o_parts[i].stride_n;
    a.o_sh[i] = o_parts[i].stride_h;
    a.lse_ptr[i] = lse_parts[i];
  }
  RM_TRY(check_tensor("o_out", o_out, esize_of(out_dtype), rows, H, d, 4 * esize_of(out_dtype)));
  if (out_dtype == RM_BF16 && o_out.ptr == o_parts[0].ptr)
    return fail(RM_ERR_INVALID_ARG, "in-place merge needs an fp32 output");
  if (!lse_out || ((uintptr_t)lse_out & 3)) return fail(RM_ERR_INVALID_ARG, "lse_out NULL/misaligned");
  a.out = o_out.ptr;
  a.out_sb = o_out.stride_b;
  a.out_sn = o_out.stride_n;
  a.out_sh = o_out.stride_h;
  a.lse_out = lse_out;
  RM_CUDA(launch_lse_merge(a, out_dtype == RM_BF16, (cudaStream_t)stream), "lse_merge launch");
  return RM_OK;
}

rm_status rm_attn_bwd_preprocess(rm_dtype dtype, int B, int64_t N, int H, int d, rm_tensor o,
                                 rm_tensor dout, float* delta, void* stream) {
  if (dtype != RM_F32 && dtype != RM_BF16) return fail(RM_ERR_INVALID_ARG, "bad dtype");
  if (B < 0 || N < 0 || H < 1 || d < 4 || d > 128 || d % 4)
    return fail(RM_ERR_INVALID_ARG, "bad sizes (need d %% 4 == 0, 4 <= d <= 128)");
  const int64_t rows = (int64_t)B * N;
  if (rows == 0) return RM_OK;
  RM_TRY(check_tensor("o", o, esize_of(dtype), rows, H, d, 4 * esize_of(dtype)));
  RM_TRY(check_tensor("dout", dout, esize_of(dtype), rows, H, d, 4 * esize_of(dtype)));
  if (!delta || ((uintptr_t)delta & 3)) return fail(RM_ERR_INVALID_ARG, "delta NULL/misaligned");
  RM_CUDA(launch_bwd_preprocess(dtype == RM_BF16, B, N, H, d, o, dout, delta, nullptr,
                                (cudaStream_t)stream),
          "bwd_preprocess launch");
  return RM_OK;
}

static rm_status check_qkv(const rm_attn_desc* desc, int64_t rows, rm_tensor q, rm_tensor k,
                           rm_tensor v) {
  const int es = esize_of(desc->dtype);
  const int64_t r = (int64_t)desc->B * rows;
  RM_TRY(check_tensor("q", q, es, r, desc->Hq, desc->d));
  RM_TRY(check_tensor("k", k, es, r, desc->Hkv, desc->d));
  RM_TRY(check_tensor("v", v, es, r, desc->Hkv, desc->d));
  return RM_OK;
}

static AttnArgs attn_args(const rm_attn_desc* desc, int64_t lse_ld) {
  AttnArgs a;
  memset(&a, 0, sizeof(a));
  a.B = desc->B;
  a.Hq = desc->Hq;
  a.Hkv = desc->Hkv;
  a.d = desc->d;
  a.N = desc->N;
  a.P = desc->P;
  a.layout = desc->layout;
  a.causal = desc->causal ? 1 : 0;
  a.scale = eff_scale(desc);
  a.lse_ld = lse_ld;
  a.global_order = (desc->order == RM_ORDER_GLOBAL && desc->layout != RM_LAYOUT_CONTIGUOUS &&
                    desc->P > 1) ? 1 : 0;
  a.cu_seqlens = desc->cu_seqlens;
  a.num_segments = desc->cu_seqlens ? desc->num_segments : 0;
  a.seq_lens = desc->seq_lens;
  a.seg_div = t_seg_div;
  a.status = status_word();
  return a;
}

// One (q_rank, kv_rank) forward with shard-local operands; LSE rows lse_ld apart.
// Pk > 0: the KV side has Pk contiguous chunks (a tile of a rectangular grid).
static rm_status block_fwd(const rm_attn_desc* desc, int q_rank, int kv_rank, rm_tensor q,
                           rm_tensor k, rm_tensor v, rm_tensor o, int o_f32, float* lse,
                           int64_t lse_ld, cudaStream_t st, int Pk = 0) {
  AttnArgs a = attn_args(desc, lse_ld);
  a.q = q; a.k = k; a.v = v; a.o = o; a.o_f32 = o_f32; a.lse = lse;
  a.Pk = Pk;
  if (small_seq_supported(desc->N / desc->P, desc->d) && !desc->cu_seqlens && !desc->seq_lens &&
      kv_shards(a) == desc->P) {
    RM_CUDA(launch_small_seq_fwd(a, q_rank, kv_rank, desc->dtype == RM_BF16, st),
            "short-sequence fwd launch");
    return RM_OK;
  }
  if (desc->dtype == RM_F32) {
    RM_CUDA(launch_simt_fwd(a, q_rank, kv_rank, st), "simt fwd launch");
    return RM_OK;
  }
  return tc_fwd(a, q_rank, kv_rank, st);
}

rm_status rm_attn_block_fwd(const rm_attn_desc* desc, int q_rank, int kv_rank, rm_tensor q,
                            rm_tensor k, rm_tensor v, rm_tensor o, int o_f32, float* lse,
                            void* stream) {
  RM_TRY(check_desc(desc));
  if (q_rank < 0 || q_rank >= desc->P || kv_rank < 0 || kv_rank >= desc->P)
    return fail(RM_ERR_INVALID_ARG, "rank out of range");
  const int64_t L = desc->N / desc->P;
  if (desc->B == 0 || L == 0) return RM_OK;
  RM_TRY(check_qkv(desc, L, q, k, v));
  const int f32_out = (o_f32 || desc->dtype == RM_F32) ? 1 : 0;
  RM_TRY(check_tensor("o", o, f32_out ? 4 : 2, (int64_t)desc->B * L, desc->Hq, desc->d));
  if (!lse || ((uintptr_t)lse & 3)) return fail(RM_ERR_INVALID_ARG, "lse NULL/misaligned");
  return block_fwd(desc, q_rank, kv_rank, q, k, v, o, f32_out, lse, L, (cudaStream_t)stream);
}

rm_status rm_attn_block_bwd(const rm_attn_desc* desc, int q_rank, int kv_rank, rm_tensor q,
                            rm_tensor k, rm_tensor v, rm_tensor dout, const float* lse_final,
                            const float* delta, rm_tensor dq_acc, rm_tensor dk_acc,
                            rm_tensor dv_acc, void* stream) {
  RM_TRY(check_desc(desc));
  if (q_rank < 0 || q_rank >= desc->P || kv_rank < 0 || kv_rank >= desc->P)
    return fail(RM_ERR_INVALID_ARG, "rank out of range");
  const int64_t L = desc->N / desc->P;
  if (desc->B == 0 || L == 0) return RM_OK;
  RM_TRY(check_qkv(desc, L, q, k, v));
  const int64_t rows = (int64_t)desc->B * L;
  RM_TRY(check_tensor("dout", dout, esize_of(desc->dtype), rows, desc->Hq, desc->d));
  RM_TRY(check_tensor("dq_acc", dq_acc, 4, rows, desc->Hq, desc->d));
  RM_TRY(check_tensor("dk_acc", dk_acc, 4, rows, desc->Hkv, desc->d));
  RM_TRY(check_tensor("dv_acc", dv_acc, 4, rows, desc->Hkv, desc->d));
  if (!lse_final || !delta) return fail(RM_ERR_INVALID_ARG, "lse_final / delta NULL");
  cudaStream_t st = (cudaStream_t)stream;
  AttnArgs a = attn_args(desc, L);
  a.q = q; a.k = k; a.v = v; a.dout = dout; a.lse_in = lse_final; a.delta = delta;
  a.dq = dq_acc; a.dk = dk_acc; a.dv = dv_acc;
  a.accumulate = 1;
  if (desc->dtype == RM_F32 || bf16_simt_bwd(desc)) {
    RM_CUDA(launch_simt_bwd(a, q_rank, kv_rank, desc->dtype == RM_BF16, st), "simt bwd launch");
    return RM_OK;
  }
  return tc_bwd(a, q_rank, kv_rank, st);
}

rm_status rm_ring_workspace_size(const rm_attn_desc* desc, int backward, size_t* bytes) {
  RM_TRY(check_desc(desc));
  RM_TRY(check_order(desc, backward));
  if (!bytes) return fail(RM_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = backward ? bwd_ws(desc).total : fwd_ws(desc).total;
  return RM_OK;
}

rm_status rm_ring_attn_fwd(const rm_attn_desc* desc, rm_tensor q, rm_tensor k, rm_tensor v,
                           rm_tensor o, float* lse, void* ws, size_t ws_bytes, void* stream) {
  RM_TRY(check_desc(desc));
  RM_TRY(check_order(desc, 0));
  if (desc->B == 0 || desc->N == 0) return RM_OK;
  RM_TRY(check_qkv(desc, desc->N, q, k, v));
  const int es = esize_of(desc->dtype);
  RM_TRY(check_tensor("o", o, es, (int64_t)desc->B * desc->N, desc->Hq, desc->d));
  if (!lse || ((uintptr_t)lse & 3)) return fail(RM_ERR_INVALID_ARG, "lse NULL/misaligned");
  const FwdWs w = fwd_ws(desc);
  if (w.total && (!ws || ws_bytes < w.total || ((uintptr_t)ws & 255)))
    return fail(RM_ERR_WORKSPACE, "workspace needs %zu bytes, 256-byte aligned", w.total);
  if (desc->mode == RM_RING_STEPWISE && desc->P > kMaxMergeParts)
    return fail(RM_ERR_UNSUPPORTED, "stepwise mode supports P <= %d", kMaxMergeParts);
  cudaStream_t st = (cudaStream_t)stream;
  const int64_t L = desc->N / desc->P;
  if (desc->mode == RM_RING_FUSED && desc->P == 1 && small_seq_supported(desc->N, desc->d) &&
      !desc->cu_seqlens && !desc->seq_lens)
    return block_fwd(desc, 0, 0, q, k, v, o, desc->dtype == RM_F32, lse, desc->N, st);
  if (desc->mode == RM_RING_FUSED) {
    AttnArgs a = attn_args(desc, desc->N);
    a.q = q; a.k = k; a.v = v; a.o = o; a.o_f32 = desc->dtype == RM_F32; a.lse = lse;
    if (desc->dtype == RM_F32) {
      RM_CUDA(launch_simt_fwd(a, -1, -1, st), "simt ring fwd launch");
      return RM_OK;
    }
    return tc_fwd(a, -1, -1, st);
  }
  // Stepwise: at ring step k rank r attends to shard (r - k) mod P; the fp32
  // partial O of step k fills slot k ([B, N, Hq, d], rank-major) and its LSE
  // slot k ([B, Hq, N]); then every rank merges its P partials.
  const size_t rows_q = (size_t)desc->B * desc->N * desc->Hq;
  float* o_slots = (float*)((char*)ws + w.o_parts);
  float* lse_slots = (float*)((char*)ws + w.lse_parts);
  for (int step = 0; step < desc->P; ++step) {
    rm_tensor o_k = dense_bnhd(o_slots + (size_t)step * rows_q * desc->d, desc->N, desc->Hq,
                               desc->d);
    float* lse_k = lse_slots + (size_t)step * rows_q;
    for (int r = 0; r < desc->P; ++r) {
      const int s = ((r - step) % desc->P + desc->P) % desc->P;
      RM_TRY(block_fwd(desc, r, s, offset_rows(q, (int64_t)r * L, es),
                       offset_rows(k, (int64_t)s * L, es), offset_rows(v, (int64_t)s * L, es),
                       offset_rows(o_k, (int64_t)r * L, 4), 1, lse_k + (int64_t)r * L, desc->N,
                       st));
    }
  }
  MergeArgs m;
  memset(&m, 0, sizeof(m));
  m.B = desc->B;
  m.H = desc->Hq;
  m.d = desc->d;
  m.Nq = desc->N;  // all ranks at once: rank-major rows, every row has P partials
  m.n_parts = desc->P;
  m.lse_ld = desc->N;
  for (int step = 0; step < desc->P; ++step) {
    m.o_ptr[step] = o_slots + (size_t)step * rows_q * desc->d;
    m.o_sb[step] = desc->N * desc->Hq * desc->d;
    m.o_sn[step] = (int64_t)desc->Hq * desc->d;
    m.o_sh[step] = desc->d;
    m.lse_ptr[step] = lse_slots + (size_t)step * rows_q;
  }
  m.out = o.ptr;
  m.out_sb = o.stride_b;
  m.out_sn = o.stride_n;
  m.out_sh = o.stride_h;
  m.lse_out = lse;
  RM_CUDA(launch_lse_merge(m, desc->dtype == RM_BF16, st), "ring merge launch");
  return RM_OK;
}

rm_status rm_ring_attn_bwd(const rm_attn_desc* desc, rm_tensor q, rm_tensor k, rm_tensor v,
                           rm_tensor o, const float* lse, rm_tensor dout, rm_tensor dq,
                           rm_tensor dk, rm_tensor dv, void* ws, size_t ws_bytes, void* stream) {
  RM_TRY(check_desc(desc));
  RM_TRY(check_order(desc, 1));
  if (desc->B == 0 || desc->N == 0) return RM_OK;
  RM_TRY(check_qkv(desc, desc->N, q, k, v));
  const int es = esize_of(desc->dtype);
  const int64_t rows = (int64_t)desc->B * desc->N;
  RM_TRY(check_tensor("o", o, es, rows, desc->Hq, desc->d));
  RM_TRY(check_tensor("dout", dout, es, rows, desc->Hq, desc->d));
  RM_TRY(check_tensor("dq", dq, es, rows, desc->Hq, desc->d));
  RM_TRY(check_tensor("dk", dk, es, rows, desc->Hkv, desc->d));
  RM_TRY(check_tensor("dv", dv, es, rows, desc->Hkv, desc->d));
  if (!lse) return fail(RM_ERR_INVALID_ARG, "lse NULL");
  const BwdWs w = bwd_ws(desc);
  if (!ws || ws_bytes < w.total || ((uintptr_t)ws & 255))
    return fail(RM_ERR_WORKSPACE, "workspace needs %zu bytes, 256-byte aligned", w.total);
  cudaStream_t st = (cudaStream_t)stream;
  float* delta = (float*)((char*)ws + w.delta);
  AttnArgs a = attn_args(desc, desc->N);
  a.q = q; a.k = k; a.v = v; a.dout = dout; a.lse_in = lse; a.delta = delta;
  a.accumulate = 0;
  if (desc->dtype == RM_F32) {
    // every SIMT thread owns complete sums: dq / dk / dv are written directly
    RM_CUDA(launch_bwd_preprocess(0, desc->B, desc->N, desc->Hq, desc->d, o, dout, delta, nullptr,
                                  st),
            "bwd preprocess launch");
    a.dq = dq; a.dk = dk; a.dv = dv;
    RM_CUDA(launch_simt_bwd(a, -1, -1, 0, st), "simt ring bwd launch");
    return RM_OK;
  }
  if (bf16_simt_bwd(desc)) {
    // SIMT kernels on the bf16 operands into fp32 dQ / dK / dV, rounded (RNE)
    // into the caller's tensors
    RM_CUDA(launch_bwd_preprocess(1, desc->B, desc->N, desc->Hq, desc->d, o, dout, delta, nullptr,
                                  st),
            "bwd preprocess launch");
    char* base = (char*)ws;
    a.dq = dense_bnhd(base + w.dq, desc->N, desc->Hq, desc->d);
    a.dk = dense_bnhd(base + w.dk, desc->N, desc->Hkv, desc->d);
    a.dv = dense_bnhd(base + w.dv, desc->N, desc->Hkv, desc->d);
    RM_CUDA(launch_simt_bwd(a, -1, -1, 1, st), "simt ring bwd launch");
    RM_CUDA(launch_convert_f32(1, desc->B, desc->N, desc->Hq, desc->d, a.dq, dq, st), "dQ convert");
    RM_CUDA(launch_convert_f32(1, desc->B, desc->N, desc->Hkv, desc->d, a.dk, dk, st),
            "dK convert");
    RM_CUDA(launch_convert_f32(1, desc->B, desc->N, desc->Hkv, desc->d, a.dv, dv, st),
            "dV convert");
    return RM_OK;
  }
  // delta from the final O, then the dK/dV and dQ kernels write their outputs
  RM_CUDA(launch_bwd_preprocess(1, desc->B, desc->N, desc->Hq, desc->d, o, dout, delta, nullptr,
                                st),
          "bwd preprocess launch");
  a.dq = dq; a.dk = dk; a.dv = dv;
  return tc_bwd(a, -1, -1, st);
}

// ---- USP ------------------------------------------------------------------

rm_status rm_usp_auto_select(int Hq, int Hkv, int world, int node_size, int* ulysses,
                             int* ring) {
  if (Hq < 1 || Hkv < 1 || world < 1 || node_size < 1 || !ulysses || !ring)
    return fail(RM_ERR_INVALID_ARG, "bad USP selector arguments");
  if (Hq % Hkv) return fail(RM_ERR_INVALID_ARG, "Hq %% Hkv != 0");
  int best = 1;
  for (int u = 1; u <= world; ++u)
    if (world % u == 0 && Hkv % u == 0 && u <= node_size) best = u;
  *ulysses = best;
  *ring = world / best;
  return RM_OK;
}

namespace {

// The ring problem of one USP call: every (batch, head group) is a sequence
// of its own, with Hq/u query and Hkv/u KV heads.
rm_status usp_desc(const rm_attn_desc* desc, int u, rm_attn_desc* out) {
  RM_TRY(check_desc(desc));
  if (u < 1) return fail(RM_ERR_INVALID_ARG, "ulysses degree must be >= 1");
  if (desc->Hq % u || desc->Hkv % u)
    return fail(RM_ERR_INVALID_ARG, "ulysses degree %d must divide Hq (%d) and Hkv (%d)", u,
                desc->Hq, desc->Hkv);
  if ((desc->N / desc->P) % u)
    return fail(RM_ERR_INVALID_ARG, "ulysses degree %d must divide the ring shard (%lld tokens)",
                u, (long long)(desc->N / desc->P));
  *out = *desc;
  out->B = desc->B * u;
  out->Hq = desc->Hq / u;
  out->Hkv = desc->Hkv / u;
  return RM_OK;
}

struct UspWs {
  size_t q, kv, ring_off, ring_bytes, total;  // q / kv: bytes of one repacked operand
};

rm_status usp_ws(const rm_attn_desc* desc, int u, int backward, UspWs* w) {
  rm_attn_desc d2;
  RM_TRY(usp_desc(desc, u, &d2));
  const size_t es = esize_of(desc->dtype);
  w->q = align_up((size_t)desc->B * desc->N * desc->Hq * desc->d * es);
  w->kv = align_up((size_t)desc->B * desc->N * desc->Hkv * desc->d * es);
  // forward: q, o, k, v; backward: q, o, dout, dq and k, v, dk, dv
  w->ring_off = backward ? 4 * w->q + 4 * w->kv : 2 * w->q + 2 * w->kv;
  size_t rb = 0;
  {
    SegDivScope scope(u);
    RM_TRY(rm_ring_workspace_size(&d2, backward, &rb));
  }
  w->ring_bytes = rb;
  w->total = w->ring_off + align_up(rb);
  return RM_OK;
}

bool dense(const rm_tensor& t, int64_t N, int H, int d) {
  return t.stride_h == d && t.stride_n == (int64_t)H * d && t.stride_b == N * H * d;
}

// seq->head (or back) of every batch entry of a dense [B, N, H, d] tensor:
// batch b viewed as [u, N/u, H, d] <-> [u, N, H/u, d] at the same offset.
rm_status usp_repack(const rm_attn_desc* desc, int u, int H, int head_to_seq, const void* in,
                     void* out, cudaStream_t st) {
  const int es = esize_of(desc->dtype);
  const int64_t per = desc->N * H * desc->d * es;
  for (int b = 0; b < desc->B; ++b)
    RM_CUDA(launch_seq_head_repack(es, u, desc->N / u, H, desc->d, head_to_seq,
                                   (const char*)in + b * per, (char*)out + b * per, st),
            "usp repack launch");
  return RM_OK;
}

rm_tensor dense_t(void* p, const rm_attn_desc& d2, int H) {
  rm_tensor t;
  t.ptr = p;
  t.stride_h = d2.d;
  t.stride_n = (int64_t)H * d2.d;
  t.stride_b = d2.N * H * d2.d;
  return t;
}

}  // namespace

rm_status rm_usp_workspace_size(const rm_attn_desc* desc, int ulysses, int backward,
                                size_t* bytes) {
  if (!bytes) return fail(RM_ERR_INVALID_ARG, "bytes is NULL");
  UspWs w;
  RM_TRY(usp_ws(desc, ulysses, backward, &w));
  *bytes = w.total;
  return RM_OK;
}

rm_status rm_usp_attn_fwd(const rm_attn_desc* desc, int ulysses, rm_tensor q, rm_tensor k,
                          rm_tensor v, rm_tensor o, float* lse, void* ws, size_t ws_bytes,
                          void* stream) {
  rm_attn_desc d2;
  RM_TRY(usp_desc(desc, ulysses, &d2));
  if (desc->B == 0 || desc->N == 0) return RM_OK;
  const int64_t N = desc->N;
  if (!dense(q, N, desc->Hq, desc->d) || !dense(o, N, desc->Hq, desc->d) ||
      !dense(k, N, desc->Hkv, desc->d) || !dense(v, N, desc->Hkv, desc->d))
    return fail(RM_ERR_INVALID_ARG, "USP operands must be dense [B, N, H, d]");
  if (!q.ptr || !k.ptr || !v.ptr || !o.ptr || !lse) return fail(RM_ERR_INVALID_ARG, "NULL pointer");
  UspWs w;
  RM_TRY(usp_ws(desc, ulysses, 0, &w));
  if (!ws || ws_bytes < w.total || ((uintptr_t)ws & 255))
    return fail(RM_ERR_WORKSPACE, "workspace needs %zu bytes, 256-byte aligned", w.total);
  cudaStream_t st = (cudaStream_t)stream;
  char* base = (char*)ws;
  void *yq = base, *yo = base + w.q, *yk = base + 2 * w.q, *yv = base + 2 * w.q + w.kv;
  const int u = ulysses;
  RM_TRY(usp_repack(desc, u, desc->Hq, 0, q.ptr, yq, st));
  RM_TRY(usp_repack(desc, u, desc->Hkv, 0, k.ptr, yk, st));
  RM_TRY(usp_repack(desc, u, desc->Hkv, 0, v.ptr, yv, st));
  // lse [B, Hq, N] is [B*u, Hq/u, N]: the ring writes it in place.  Segment
  // boundaries are global positions, which the head exchange keeps.
  {
    SegDivScope scope(u);
    RM_TRY(rm_ring_attn_fwd(&d2, dense_t(yq, d2, d2.Hq), dense_t(yk, d2, d2.Hkv),
                            dense_t(yv, d2, d2.Hkv), dense_t(yo, d2, d2.Hq), lse,
                            base + w.ring_off, w.ring_bytes, stream));
  }
  return usp_repack(desc, u, desc->Hq, 1, yo, o.ptr, st);
}

rm_status rm_usp_attn_bwd(const rm_attn_desc* desc, int ulysses, rm_tensor q, rm_tensor k,
                          rm_tensor v, rm_tensor o, const float* lse, rm_tensor dout,
                          rm_tensor dq, rm_tensor dk, rm_tensor dv, void* ws, size_t ws_bytes,
                          void* stream) {
  rm_attn_desc d2;
  RM_TRY(usp_desc(desc, ulysses, &d2));
  if (desc->B == 0 || desc->N == 0) return RM_OK;
  const int64_t N = desc->N;
  const int hq = desc->Hq, hkv = desc->Hkv, d = desc->d;
  if (!dense(q, N, hq, d) || !dense(o, N, hq, d) || !dense(dout, N, hq, d) ||
      !dense(dq, N, hq, d) || !dense(k, N, hkv, d) || !dense(v, N, hkv, d) ||
      !dense(dk, N, hkv, d) || !dense(dv, N, hkv, d))
    return fail(RM_ERR_INVALID_ARG, "USP operands must be dense [B, N, H, d]");
  if (!q.ptr || !k.ptr || !v.ptr || !o.ptr || !dout.ptr || !dq.ptr || !dk.ptr || !dv.ptr || !lse)
    return fail(RM_ERR_INVALID_ARG, "NULL pointer");
  UspWs w;
  RM_TRY(usp_ws(desc, ulysses, 1, &w));
  if (!ws || ws_bytes < w.total || ((uintptr_t)ws & 255))
    return fail(RM_ERR_WORKSPACE, "workspace needs %zu bytes, 256-byte aligned", w.total);
  cudaStream_t st = (cudaStream_t)stream;
  char* base = (char*)ws;
  void *yq = base, *yo = base + w.q, *ydo = base + 2 * w.q, *ydq = base + 3 * w.q;
  char* kvb = base + 4 * w.q;
  void *yk = kvb, *yv = kvb + w.kv, *ydk = kvb + 2 * w.kv, *ydv = kvb + 3 * w.kv;
  const int u = ulysses;
  RM_TRY(usp_repack(desc, u, hq, 0, q.ptr, yq, st));
  RM_TRY(usp_repack(desc, u, hkv, 0, k.ptr, yk, st));
  RM_TRY(usp_repack(desc, u, hkv, 0, v.ptr, yv, st));
  RM_TRY(usp_repack(desc, u, hq, 0, o.ptr, yo, st));
  RM_TRY(usp_repack(desc, u, hq, 0, dout.ptr, ydo, st));
  {
    SegDivScope scope(u);
    RM_TRY(rm_ring_attn_bwd(&d2, dense_t(yq, d2, d2.Hq), dense_t(yk, d2, d2.Hkv),
                            dense_t(yv, d2, d2.Hkv), dense_t(yo, d2, d2.Hq), lse,
                            dense_t(ydo, d2, d2.Hq), dense_t(ydq, d2, d2.Hq),
                            dense_t(ydk, d2, d2.Hkv), dense_t(ydv, d2, d2.Hkv), base + w.ring_off,
                            w.ring_bytes, stream));
  }
  RM_TRY(usp_repack(desc, u, hq, 1, ydq, dq.ptr, st));
  RM_TRY(usp_repack(desc, u, hkv, 1, ydk, dk.ptr, st));
  return usp_repack(desc, u, hkv, 1, ydv, dv.ptr, st);
}

// ---- Mesh2D ---------------------------------------------------------------

namespace {

// The tile problem of a Mesh2D call: query chunks are the P = grid_q
// contiguous shards of the block API, KV chunks its Pk = grid_k ones.
rm_status mesh2d_desc(const rm_attn_desc* desc, int grid_q, int grid_k, rm_attn_desc* out) {
  if (!desc) return fail(RM_ERR_INVALID_ARG, "desc is NULL");
  if (grid_q < 1 || grid_k < 1) return fail(RM_ERR_INVALID_ARG, "grid sizes must be >= 1");
  if (grid_k > kMaxMergeParts)
    return fail(RM_ERR_UNSUPPORTED, "grid_k must be <= %d (merge parts)", kMaxMergeParts);
  if (desc->N % grid_q) return fail(RM_ERR_INVALID_ARG, "grid_q must divide N");
  *out = *desc;
  out->P = grid_q;
  out->layout = RM_LAYOUT_CONTIGUOUS;
  out->mode = RM_RING_STEPWISE;
  out->order = RM_ORDER_RANK_MAJOR;
  RM_TRY(check_desc(out));
  if (desc->N % grid_k) return fail(RM_ERR_INVALID_ARG, "grid_k must divide N");
  return RM_OK;
}

struct MeshWs {
  size_t o_parts, lse_parts;    // forward: grid_k fp32 partial O and LSE slots
  size_t delta, dq, dk, dv;     // backward: delta and fp32 accumulators
  size_t total;
};
MeshWs mesh2d_ws(const rm_attn_desc* d, int grid_k, int backward) {
  MeshWs w;
  memset(&w, 0, sizeof(w));
  const size_t rows_q = (size_t)d->B * d->N * d->Hq, rows_kv = (size_t)d->B * d->N * d->Hkv;
  if (!backward) {
    w.lse_parts = align_up(rows_q * d->d * 4 * (size_t)grid_k);
    w.total = w.lse_parts + align_up(rows_q * 4 * (size_t)grid_k);
  } else {
    w.dq = align_up(rows_q * 4);
    w.dk = w.dq + align_up(rows_q * d->d * 4);
    w.dv = w.dk + align_up(rows_kv * d->d * 4);
    w.total = w.dv + align_up(rows_kv * d->d * 4);
  }
  return w;
}

// Whether tile (i, j) holds a visible pair: under the causal rule the first
// key of chunk j must not lie after the last query of chunk i.
bool mesh2d_tile_live(const rm_attn_desc* d, int grid_q, int grid_k, int i, int j) {
  if (!d->causal) return true;
  return (int64_t)j * (d->N / grid_k) <= (int64_t)(i + 1) * (d->N / grid_q) - 1;
}

}  // namespace

rm_status rm_mesh2d_workspace_size(const rm_attn_desc* desc, int grid_q, int grid_k,
                                   int backward, size_t* bytes) {
  rm_attn_desc d2;
  RM_TRY(mesh2d_desc(desc, grid_q, grid_k, &d2));
  if (!bytes) return fail(RM_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = mesh2d_ws(&d2, grid_k, backward).total;
  return RM_OK;
}

rm_status rm_mesh2d_attn_fwd(const rm_attn_desc* desc, int grid_q, int grid_k, rm_tensor q,
                             rm_tensor k, rm_tensor v, rm_tensor o, float* lse, void* ws,
                             size_t ws_bytes, void* stream) {
  rm_attn_desc d2;
  RM_TRY(mesh2d_desc(desc, grid_q, grid_k, &d2));
  if (d2.B == 0 || d2.N == 0) return RM_OK;
  RM_TRY(check_qkv(&d2, d2.N, q, k, v));
  const int es = esize_of(d2.dtype);
  RM_TRY(check_tensor("o", o, es, (int64_t)d2.B * d2.N, d2.Hq, d2.d));
  if (!lse || ((uintptr_t)lse & 3)) return fail(RM_ERR_INVALID_ARG, "lse NULL/misaligned");
  const MeshWs w = mesh2d_ws(&d2, grid_k, 0);
  if (!ws || ws_bytes < w.total || ((uintptr_t)ws & 255))
    return fail(RM_ERR_WORKSPACE, "workspace needs %zu bytes, 256-byte aligned", w.total);
  cudaStream_t st = (cudaStream_t)stream;
  const int64_t Lq = d2.N / grid_q, Lk = d2.N / grid_k;
  const size_t rows_q = (size_t)d2.B * d2.N * d2.Hq;
  float* o_slots = (float*)((char*)ws + w.o_parts);
  float* lse_slots = (float*)((char*)ws + w.lse_parts);
  for (int i = 0; i < grid_q; ++i) {
    // tile (i, j): partial O into rows of chunk i of slot j, its LSE likewise
    int parts = 0;
    for (int j = 0; j < grid_k && mesh2d_tile_live(&d2, grid_q, grid_k, i, j); ++j, ++parts) {
      rm_tensor o_j = dense_bnhd(o_slots + (size_t)j * rows_q * d2.d, d2.N, d2.Hq, d2.d);
      RM_TRY(block_fwd(&d2, i, j, offset_rows(q, i * Lq, es), offset_rows(k, j * Lk, es),
                       offset_rows(v, j * Lk, es), offset_rows(o_j, i * Lq, 4), 1,
                       lse_slots + (size_t)j * rows_q + i * Lq, d2.N, st, grid_k));
    }
    // the live tiles of a row are a prefix j < parts (parts >= 1: key 0 sees every query)
    MergeArgs m;
    memset(&m, 0, sizeof(m));
    m.B = d2.B;
    m.H = d2.Hq;
    m.d = d2.d;
    m.Nq = Lq;
    m.n_parts = parts;
    m.lse_ld = d2.N;
    for (int j = 0; j < parts; ++j) {
      m.o_ptr[j] = o_slots + (size_t)j * rows_q * d2.d + (size_t)i * Lq * d2.Hq * d2.d;
      m.o_sb[j] = d2.N * d2.Hq * d2.d;
      m.o_sn[j] = (int64_t)d2.Hq * d2.d;
      m.o_sh[j] = d2.d;
      m.lse_ptr[j] = lse_slots + (size_t)j * rows_q + i * Lq;
    }
    const rm_tensor o_i = offset_rows(o, i * Lq, es);
    m.out = o_i.ptr;
    m.out_sb = o.stride_b;
    m.out_sn = o.stride_n;
    m.out_sh = o.stride_h;
    m.lse_out = lse + i * Lq;
    RM_CUDA(launch_lse_merge(m, d2.dtype == RM_BF16, st), "Mesh2D merge launch");
  }
  return RM_OK;
}

rm_status rm_mesh2d_attn_bwd(const rm_attn_desc* desc, int grid_q, int grid_k, rm_tensor q,
                             rm_tensor k, rm_tensor v, rm_tensor o, const float* lse,
                             rm_tensor dout, rm_tensor dq, rm_tensor dk, rm_tensor dv, void* ws,
                             size_t ws_bytes, void* stream) {
  rm_attn_desc d2;
  RM_TRY(mesh2d_desc(desc, grid_q, grid_k, &d2));
  if (d2.B == 0 || d2.N == 0) return RM_OK;
  RM_TRY(check_qkv(&d2, d2.N, q, k, v));
  const int es = esize_of(d2.dtype);
  const int64_t rows = (int64_t)d2.B * d2.N;
  RM_TRY(check_tensor("o", o, es, rows, d2.Hq, d2.d));
  RM_TRY(check_tensor("dout", dout, es, rows, d2.Hq, d2.d));
  RM_TRY(check_tensor("dq", dq, es, rows, d2.Hq, d2.d));
  RM_TRY(check_tensor("dk", dk, es, rows, d2.Hkv, d2.d));
  RM_TRY(check_tensor("dv", dv, es, rows, d2.Hkv, d2.d));
  if (!lse) return fail(RM_ERR_INVALID_ARG, "lse NULL");
  const MeshWs w = mesh2d_ws(&d2, grid_k, 1);
  if (!ws || ws_bytes < w.total || ((uintptr_t)ws & 255))
    return fail(RM_ERR_WORKSPACE, "workspace needs %zu bytes, 256-byte aligned", w.total);
  cudaStream_t st = (cudaStream_t)stream;
  char* base = (char*)ws;
  float* delta = (float*)(base + w.delta);
  const rm_tensor dq_acc = dense_bnhd(base + w.dq, d2.N, d2.Hq, d2.d);
  const rm_tensor dk_acc = dense_bnhd(base + w.dk, d2.N, d2.Hkv, d2.d);
  const rm_tensor dv_acc = dense_bnhd(base + w.dv, d2.N, d2.Hkv, d2.d);
  const size_t kv_bytes = (size_t)rows * d2.Hkv * d2.d * 4;
  // delta from the final O (and the dQ accumulator zeroed in the same pass)
  RM_CUDA(launch_bwd_preprocess(d2.dtype == RM_BF16, d2.B, d2.N, d2.Hq, d2.d, o, dout, delta,
                                (float*)dq_acc.ptr, st),
          "bwd preprocess launch");
  RM_CUDA(cudaMemsetAsync(dk_acc.ptr, 0, kv_bytes, st), "dK accumulator clear");
  RM_CUDA(cudaMemsetAsync(dv_acc.ptr, 0, kv_bytes, st), "dV accumulator clear");
  const int64_t Lq = d2.N / grid_q, Lk = d2.N / grid_k;
  for (int i = 0; i < grid_q; ++i) {
    for (int j = 0; j < grid_k && mesh2d_tile_live(&d2, grid_q, grid_k, i, j); ++j) {
      AttnArgs a = attn_args(&d2, d2.N);
      a.Pk = grid_k;
      a.q = offset_rows(q, i * Lq, es);
      a.dout = offset_rows(dout, i * Lq, es);
      a.k = offset_rows(k, j * Lk, es);
      a.v = offset_rows(v, j * Lk, es);
      a.lse_in = lse + i * Lq;
      a.delta = delta + i * Lq;
      a.dq = offset_rows(dq_acc, i * Lq, 4);
      a.dk = offset_rows(dk_acc, j * Lk, 4);
      a.dv = offset_rows(dv_acc, j * Lk, 4);
      a.accumulate = 1;
      if (d2.dtype == RM_F32 || bf16_simt_bwd(&d2)) {
        RM_CUDA(launch_simt_bwd(a, i, j, d2.dtype == RM_BF16, st), "simt Mesh2D tile bwd launch");
      } else {
        RM_TRY(tc_bwd(a, i, j, st));
      }
    }
  }
  const int out_bf16 = d2.dtype == RM_BF16;
  RM_CUDA(launch_convert_f32(out_bf16, d2.B, d2.N, d2.Hq, d2.d, dq_acc, dq, st), "dQ convert");
  RM_CUDA(launch_convert_f32(out_bf16, d2.B, d2.N, d2.Hkv, d2.d, dk_acc, dk, st), "dK convert");
  RM_CUDA(launch_convert_f32(out_bf16, d2.B, d2.N, d2.Hkv, d2.d, dv_acc, dv, st), "dV convert");
  return RM_OK;
}

}  // extern "C"
