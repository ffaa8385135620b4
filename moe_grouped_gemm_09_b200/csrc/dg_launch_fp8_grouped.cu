// MoE M-grouped FP8 forms (contiguous and masked): kernel instantiations and launch.
#include "dg_launch.cuh"

namespace dg {

dg_status launch_fp8_grouped(bool* attr_set, const LaunchPlan& plan, cudaStream_t stream) {
  if (plan.form == kFormContiguous) return launch_form<kFormContiguous>(attr_set, plan, stream);
  if (plan.form == kFormMasked) return launch_form<kFormMasked>(attr_set, plan, stream);
  return DG_ERR_UNSUPPORTED;
}

}  // namespace dg
