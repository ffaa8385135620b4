// Dense FP8 forms with M-major A and/or N-major B (NN, TN, TT), with FP32
// output (D = A B^T + C), and the K-grouped form (weight gradient, TN, FP32
// output per group): kernel instantiations and launch.
#include "dg_launch.cuh"

namespace dg {

dg_status launch_fp8_layouts(bool* attr_set, const LaunchPlan& plan, cudaStream_t stream) {
  switch (plan.form) {
    case kFormNN: return launch_form<kFormNN>(attr_set, plan, stream);
    case kFormTN: return launch_form<kFormTN>(attr_set, plan, stream);
    case kFormTT: return launch_form<kFormTT>(attr_set, plan, stream);
    case kFormF32: return launch_form<kFormF32>(attr_set, plan, stream);
    case kFormKGrouped: return launch_form<kFormKGrouped>(attr_set, plan, stream);
    default: return DG_ERR_UNSUPPORTED;
  }
}

}  // namespace dg
