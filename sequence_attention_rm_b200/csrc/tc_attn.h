// Tensor-core (tcgen05 / TMEM / TMA) bf16 attention, sm_100a.
#pragma once

#include "internal.h"

namespace rm {

bool tc_supported_head_dim(int d);

// Forward.  q_rank < 0: the fused ring over all P ranks (operands rank-major,
// running softmax state carried across KV shards); else one (q_rank, kv_rank)
// shard pair with shard-local operands.  o is bf16 unless a.o_f32.
rm_status tc_fwd(const AttnArgs& a, int q_rank, int kv_rank, cudaStream_t stream);

// Backward (head dim 128): a key-stationary dK/dV kernel and a
// query-stationary dQ kernel.  Same rank convention.  With a.accumulate,
// dq / dk / dv are fp32 accumulators (+=); otherwise bf16 outputs written once
// (ring mode: every CTA owns complete sums).
rm_status tc_bwd(const AttnArgs& a, int q_rank, int kv_rank, cudaStream_t stream);

}  // namespace rm
