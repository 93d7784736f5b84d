// tcgen05 tensor-core path of the drafter block attention (placeholder: not enabled).
#include "ls_attend_tc.h"

namespace ls {

bool tc_supported(const Dev&) { return false; }
int tc_prepare(const Dev&, TcPlan*) { return LS_ERR_UNSUPPORTED; }
cudaError_t launch_attend_tc(const Dev&, const TcPlan&, int, int, const void*, const void*,
                             const void*, int64_t, float, void*, int, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace ls
