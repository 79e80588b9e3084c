// Ring backward that allocates nothing.
//
// The ring backward needs scratch device memory: the row term
// delta = rowsum(dO * O), one fp32 value per (batch, query head, token).
// Most callers pass a workspace they allocated; some cannot: for example a runtime that reserved all device memory for its own
// pool at start-up and hands out no raw allocations, or code that must not
// call cudaMalloc because it would synchronise the device.  For them this
// file keeps one fixed scratch array in device memory and forwards to the
// ordinary ring backward with it as the workspace.
#include <stdio.h>

#include "common.cuh"
#include "internal.h"

namespace rm {
namespace {

constexpr size_t kScratchBytes = 64ull << 20;  // 64 MiB on every device that uses it

// Never referenced by device code; host code must not pass its name to a
// kernel: the name is a host-side stand-in, the device address comes from
// cudaGetSymbolAddress below.
__device__ __align__(256) unsigned char g_scratch[kScratchBytes];

// Device address of the scratch in the current context, looked up on every
// call.  A __device__ array's address belongs to the context that loaded the
// module, not to the device ordinal: after cudaDeviceReset, or with another
// driver-API context current, an address cached from an earlier call would
// point into memory that is no longer (or never was) this context's.  Once
// the module is loaded the lookup is a table search.
rm_status scratch_address(void** out) {
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
  if (e != cudaSuccess || !p) {
    char buf[256];
    snprintf(buf, sizeof(buf), "rm_ring_attn_bwd_noalloc: cudaGetSymbolAddress failed: %s",
             cudaGetErrorString(e));
    set_last_error(buf);
    return RM_ERR_CUDA;
  }
  *out = p;
  return RM_OK;
}

}  // namespace
}  // namespace rm

extern "C" rm_status rm_ring_attn_bwd_noalloc(const rm_attn_desc* desc, rm_tensor q,
                                              rm_tensor k, rm_tensor v, rm_tensor o,
                                              const float* lse, rm_tensor dout, rm_tensor dq,
                                              rm_tensor dk, rm_tensor dv, void* stream) {
  size_t need = 0;
  rm_status s = rm_ring_workspace_size(desc, 1, &need);
  if (s != RM_OK) return s;
  if (need > rm::kScratchBytes) {
    char buf[256];
    snprintf(buf, sizeof(buf),
             "rm_ring_attn_bwd_noalloc: this problem needs %zu bytes of scratch; the built-in "
             "scratch holds %zu bytes (use rm_ring_attn_bwd with a workspace)",
             need, rm::kScratchBytes);
    rm::set_last_error(buf);
    return RM_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  s = rm::scratch_address(&scratch);
  if (s != RM_OK) return s;
  // the ring backward writes delta into the scratch before reading it, so the
  // previous call's contents are harmless
  return rm_ring_attn_bwd(desc, q, k, v, o, lse, dout, dq, dk, dv, scratch, rm::kScratchBytes,
                          stream);
}
