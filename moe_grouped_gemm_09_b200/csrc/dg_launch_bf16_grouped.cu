// MoE M-grouped forms on BF16 operands (contiguous and masked): kernel
// instantiations and launch.
#include "dg_launch.cuh"

namespace dg {

dg_status launch_bf16_grouped(bool* attr_set, const LaunchPlan& plan, cudaStream_t stream) {
  if (plan.form == kFormBf16Contiguous)
    return launch_form<kFormBf16Contiguous>(attr_set, plan, stream);
  if (plan.form == kFormBf16Masked) return launch_form<kFormBf16Masked>(attr_set, plan, stream);
  return DG_ERR_UNSUPPORTED;
}

}  // namespace dg
