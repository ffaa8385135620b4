// Dense form on BF16 operands: kernel instantiations and launch.
#include "dg_launch.cuh"

namespace dg {

dg_status launch_bf16_dense(bool* attr_set, const LaunchPlan& plan, cudaStream_t stream) {
  return launch_form<kFormBf16Dense>(attr_set, plan, stream);
}

}  // namespace dg
