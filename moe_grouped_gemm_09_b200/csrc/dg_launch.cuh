// Kernel instantiation and launch of one form over every variant it is built
// for.  Included only by the per-form translation units (dg_launch_*.cu), so
// that each one instantiates its own kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <type_traits>
#include <utility>

#include "dg_internal.h"

namespace dg {

// Kernel mode of a variant: 0 general, 1 decode, 2 small decode.
constexpr int mode_of(const Variant& v) { return v.small ? 2 : v.decode ? 1 : 0; }

template <int V, bool SCALED = true, bool F32EPI = kVariants[V].f32>
using ShapeOf = KernelShape<kVariants[V].block_n, kVariants[V].stages, kVariants[V].num_acc,
                            kVariants[V].kps, kVariants[V].a_rows, mode_of(kVariants[V]), SCALED,
                            F32EPI>;

// Kernels exist only for the (form, variant) pairs that are used: the decode
// variants and the general ones with several K blocks per stage serve the
// dense forms, the M-/N-major forms take the general variants with
// 128-column B boxes, and the FP32-output forms their own variants.
template <int FORM, int V>
constexpr bool kBuilt =
    kVariants[V].f32
        ? is_f32_form(FORM) && mn_capable(kVariants[V])
        : FORM == kFormDense || FORM == kFormBf16Dense ||
              ((FORM == kFormContiguous || FORM == kFormMasked || FORM == kFormBf16Contiguous ||
                FORM == kFormBf16Masked) &&
               !kVariants[V].decode && kVariants[V].kps == 1) ||
              (FORM >= kFormNN && FORM <= kFormTT && mn_capable(kVariants[V]));

template <int FORM, int V>
auto kernel_of() {
  constexpr Variant var = kVariants[V];
  return fp8_gemm_kernel<kind_of_form(FORM), var.block_n, var.stages, var.num_acc, var.kps,
                         var.a_rows, mode_of(var), layout_of_form(FORM), is_f32_form(FORM),
                         is_bf16_form(FORM)>;
}

template <int FORM, int V>
dg_status set_smem_attr(bool* attr_set) {
  if constexpr (!kBuilt<FORM, V>) {
    return DG_ERR_UNSUPPORTED;
  } else {
    if (!attr_set[V]) {
      if (cudaFuncSetAttribute(kernel_of<FORM, V>(), cudaFuncAttributeMaxDynamicSharedMemorySize,
                               ShapeOf<V, !is_bf16_form(FORM), is_f32_form(FORM)>::kSmemBytes) !=
          cudaSuccess)
        return DG_ERR_CUDA;
      attr_set[V] = true;
    }
    return DG_OK;
  }
}

template <int FORM, int V>
dg_status launch_variant(bool* attr_set, const LaunchPlan& pl, cudaStream_t stream) {
  if constexpr (!kBuilt<FORM, V>) {
    return DG_ERR_UNSUPPORTED;
  } else {
    dg_status s = set_smem_attr<FORM, V>(attr_set);
    if (s != DG_OK) return s;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.grid, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = ShapeOf<V, !is_bf16_form(FORM), is_f32_form(FORM)>::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    int n_attr = 1;
    if (pl.args.split_k > 1) {  // the CTAs of one output tile form a cluster
      attr[1].id = cudaLaunchAttributeClusterDimension;
      attr[1].val.clusterDim.x = pl.args.split_k;
      attr[1].val.clusterDim.y = 1;
      attr[1].val.clusterDim.z = 1;
      n_attr = 2;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n_attr;
    return cudaLaunchKernelEx(&cfg, kernel_of<FORM, V>(), pl.ta, pl.tb, pl.td, pl.args) ==
                   cudaSuccess
               ? DG_OK
               : DG_ERR_CUDA;
  }
}

template <int FORM, int... V>
dg_status launch_dispatch(bool* attr_set, const LaunchPlan& pl, cudaStream_t stream,
                          std::integer_sequence<int, V...>) {
  dg_status s = DG_ERR_UNSUPPORTED;
  ((pl.variant == V ? (s = launch_variant<FORM, V>(attr_set, pl, stream), 0) : 0), ...);
  return s;
}

template <int FORM>
dg_status launch_form(bool* attr_set, const LaunchPlan& pl, cudaStream_t stream) {
  return launch_dispatch<FORM>(attr_set, pl, stream,
                               std::make_integer_sequence<int, kNumVariants>{});
}

}  // namespace dg
