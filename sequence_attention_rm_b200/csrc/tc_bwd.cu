// Backward attention on the sm_100a tensor cores (placeholder until the
// tcgen05 backward kernel lands).
#include "tc_attn.h"

namespace rm {

rm_status tc_bwd(const AttnArgs& a, int q_rank, int kv_rank, cudaStream_t stream) {
  (void)a; (void)q_rank; (void)kv_rank; (void)stream;
  return RM_ERR_UNSUPPORTED;
}

}  // namespace rm
