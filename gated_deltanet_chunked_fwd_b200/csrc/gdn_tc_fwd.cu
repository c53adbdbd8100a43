// gdn_tc_fwd.cu -- tensor-core (tcgen05 / TMEM / TMA) fused forward (sm_100a).
#include "gdn_internal.cuh"

namespace gdn {
bool tc_fwd_supported(const Problem&) { return false; }
size_t tc_fwd_workspace(const Problem&) { return 0; }
int tc_fwd_launches(const Problem&) { return 0; }
gdn_status launch_fwd_tc(const FwdPlan&, char*, cudaStream_t) { return GDN_ERR_UNSUPPORTED; }
}  // namespace gdn
