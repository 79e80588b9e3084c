// Internal launchers shared between the translation units of librm_attn.so.
// None of this is exported; the C ABI lives in rm_attn.cu.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/rm_attn.h"

namespace rm {

int num_sms();  // SM count of the current device (cached per device)

// Opt-in launch timing (rm_profile_enable): brackets a launch with events.
namespace prof {
int begin(const char* name, cudaStream_t s);
void end(int idx, cudaStream_t s);
}  // namespace prof
struct ProfScope {
  int idx;
  cudaStream_t s;
  ProfScope(const char* name, cudaStream_t st) : idx(prof::begin(name, st)), s(st) {}
  ~ProfScope() { prof::end(idx, s); }
};
void set_last_error(const char* msg);  // reason returned by rm_last_error()

cudaError_t launch_layout_permute(int esize, int B, int64_t N, int H, int d, int layout, int P,
                                  int inverse, const void* in, void* out, cudaStream_t stream);

cudaError_t launch_seq_head_repack(int esize, int P, int64_t n_local, int H, int d,
                                   int head_to_seq, const void* in, void* out,
                                   cudaStream_t stream);

// LSE merge of up to kMaxMergeParts partials.
constexpr int kMaxMergeParts = 16;
struct MergeArgs {
  int B, H, d;
  int64_t Nq;
  int n_parts;
  const float* o_ptr[kMaxMergeParts];
  int64_t o_sb[kMaxMergeParts], o_sn[kMaxMergeParts], o_sh[kMaxMergeParts];
  const float* lse_ptr[kMaxMergeParts];  // [B, H, *] rows of lse_ld floats
  int64_t lse_ld;                        // stride between (b, h) LSE rows (parts and output)
  void* out;
  int64_t out_sb, out_sn, out_sh;
  float* lse_out;
};
cudaError_t launch_lse_merge(const MergeArgs& a, int out_bf16, cudaStream_t stream);

// delta[b,h,t] = sum_c o*dout; optionally zero-fills an fp32 [B,N,H,d] buffer
// (the dQ accumulator, dense) in the same pass.
cudaError_t launch_bwd_preprocess(int in_bf16, int B, int64_t N, int H, int d, rm_tensor o,
                                  rm_tensor dout, float* delta, float* zero_fill,
                                  cudaStream_t stream);

// fp32 strided [B,N,H,d] -> out dtype strided [B,N,H,d] (RNE for bf16).
cudaError_t launch_convert_f32(int out_bf16, int B, int64_t N, int H, int d, rm_tensor in,
                               rm_tensor out, cudaStream_t stream);

// Arguments of the attention kernels (SIMT fp32 and tensor-core bf16).
struct AttnArgs {
  int B, Hq, Hkv, d;
  int64_t N;
  int P, layout, causal;
  int Pk;                // block calls: KV chunks of a rectangular grid (0: P)
  float scale;
  rm_tensor q, k, v;     // bases of the q / kv operands (see launchers)
  rm_tensor o;           // fwd output
  int o_f32;             // fwd: o in fp32 (else desc dtype)
  float* lse;            // fwd output; element (b, h, row) at (b*Hq + h)*lse_ld + row
  int64_t lse_ld;        // stride between (b, h) rows of lse / lse_in / delta
  rm_tensor dout;        // bwd
  const float* lse_in;   // bwd: final LSE
  const float* delta;    // bwd
  rm_tensor dq, dk, dv;  // bwd fp32 accumulators
  int accumulate;        // bwd: 1 = dq/dk/dv +=, 0 = written (=)
  int global_order;      // ring: operands (and lse / delta) in global token order
  const int* cu_seqlens; // packing boundaries (device) or null
  int num_segments;
  const int* seq_lens;   // right-padding lengths (device) or null
  int seg_div;           // batch entries per seq_lens entry (>= 1; USP head groups)
  unsigned int* status;
};
__host__ __device__ inline int kv_shards(const AttnArgs& a) { return a.Pk > 0 ? a.Pk : a.P; }

// Forward.  q_rank < 0: all ranks (ring, rank-major operands, fused merge);
// else one (q_rank, kv_rank) pair with shard-local operands.
cudaError_t launch_simt_fwd(const AttnArgs& a, int q_rank, int kv_rank, cudaStream_t stream);
// Backward, same rank convention; dq / dk / dv are fp32 (+= when
// a.accumulate); operands fp32, or bf16 (in_bf16) widened as they are read.
cudaError_t launch_simt_bwd(const AttnArgs& a, int q_rank, int kv_rank, int in_bf16,
                            cudaStream_t stream);

// Short sequences (L <= 16, d <= 64): one warp per (sequence, head), any dtype.
bool small_seq_supported(int64_t L, int d);
cudaError_t launch_small_seq_fwd(const AttnArgs& a, int q_rank, int kv_rank, int bf16,
                                 cudaStream_t stream);

cudaError_t launch_debug_expire_wait(uint32_t spin_limit, unsigned int* status,
                                     cudaStream_t stream);
cudaError_t launch_debug_exp2_poly(const float* x, float* y, int64_t n, cudaStream_t stream);

}  // namespace rm
