// Host-side internals shared by the library's translation units: the launch
// forms, the plan of one GEMM call (kernel variant, grid, kernel arguments and
// tensor maps) and the per-form launch functions, each compiled in a
// translation unit of its own so that the kernel instantiations build in
// parallel.  Nothing here is part of the C ABI (include/dg.h).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/dg.h"
#include "dg_config.h"
#include "sm100_fp8_gemm.cuh"

namespace dg {

// Launch forms: the three GEMM forms, then the dense form with M-major A
// and/or N-major B, then the dense form with FP32 output (D = A B^T + C),
// then the three GEMM forms on BF16 operands, then the K-grouped form (the
// weight gradient: M-major A, N-major B, FP32 output per group); the forms
// differ in their kernel instantiation.
enum Form : int { kFormDense = 0, kFormContiguous = 1, kFormMasked = 2, kFormNN = 3, kFormTN = 4,
                  kFormTT = 5, kFormF32 = 6, kFormBf16Dense = 7, kFormBf16Contiguous = 8,
                  kFormBf16Masked = 9, kFormKGrouped = 10 };
constexpr int kNumForms = 11;
static_assert(kFormKGrouped + 1 == kNumForms, "one shared-memory attribute row per form");

constexpr bool is_bf16_form(int f) { return f >= kFormBf16Dense && f <= kFormBf16Masked; }
constexpr int kind_of_form(int f) {
  return f < 3 ? f : is_bf16_form(f) ? f - kFormBf16Dense : f == kFormKGrouped ? kKGrouped : kDense;
}
constexpr int layout_of_form(int f) {
  return f == kFormNN ? kLayoutNN
         : (f == kFormTN || f == kFormKGrouped) ? kLayoutTN
         : f == kFormTT ? kLayoutTT
                        : kLayoutNT;
}
// Forms whose kernel writes the FP32 accumulator (plus an optional addend).
constexpr bool is_f32_form(int f) { return f == kFormF32 || f == kFormKGrouped; }
// Variants that serve M-/N-major operands and the FP32 output form: general
// ones with 128-column B boxes.
constexpr bool mn_capable(const Variant& v) {
  return !v.decode && !v.small && v.kps == 1 && v.a_rows == 128 && v.block_n % 128 == 0;
}

// Everything one launch needs, decided on the host before any device work.
struct LaunchPlan {
  int form;
  int variant;  // index into kVariants
  int grid;     // CTAs
  GemmArgs args;
  CUtensorMap ta, tb, td;
};

// Inputs of one GEMM call as the C ABI receives them.
struct GemmCall {
  int form;
  const void* a;
  const float* sfa;
  const void* b;
  const float* sfb;
  void* d;
  const float* c;        // FP32 output form: addend (may be null or d)
  const int* m_indices;  // contiguous form
  const int* masked_m;   // masked form
  int rows, N, K, G, expected_m;
  const int* ks = nullptr;  // K-grouped form: rows of K per group (device)
};

// Device facts the plan depends on (none of them needs device memory).
struct DeviceFacts {
  int num_sms;                  // SMs the library may use
  const ClusterLimits* limits;  // co-resident split-K clusters (null: not known)
};

// Host-side argument checks of a call (no device work): DG_OK and *empty
// set when there is nothing to compute.
dg_status check_gemm_call(const GemmCall& call, bool* empty);

// The launches of one call, in stream order: one, or for a dense problem
// whose last wave of tiles would leave most SMs idle, a first launch over the
// whole waves and one or two tail launches (plan_tail).
struct LaunchPlans {
  int n = 0;
  LaunchPlan plan[3];
};

// Checks the call's arguments, picks the kernel variant and grid, fills the
// kernel arguments and encodes the tensor maps.  DG_OK with plans->n == 0
// means there is nothing to launch (an empty problem).  `error_word` is the
// device word the kernels report into.
dg_status plan_gemm(const GemmCall& call, const DeviceFacts& facts, int* error_word,
                    LaunchPlans* plans);

// Launches the scale-contract check of a call's sfa and sfb (FP8 forms) on
// `stream`, reporting into `error_word`.
dg_status launch_scale_check(const GemmCall& call, int* error_word, cudaStream_t stream);

// Library-wide settings that every entry point applies.
unsigned long long wait_timeout_ns();
int prefetch_enabled();
int check_scales_enabled();
int weight_preload_enabled();

// Per-form launches (one translation unit each).  `attr_set` is the caller's
// per-device row of flags: whether the form's kernel of each variant has had
// its dynamic shared-memory limit raised on this device.
dg_status launch_fp8_dense(bool* attr_set, const LaunchPlan& plan, cudaStream_t stream);
dg_status launch_fp8_grouped(bool* attr_set, const LaunchPlan& plan, cudaStream_t stream);
dg_status launch_fp8_layouts(bool* attr_set, const LaunchPlan& plan, cudaStream_t stream);
dg_status launch_bf16_dense(bool* attr_set, const LaunchPlan& plan, cudaStream_t stream);
dg_status launch_bf16_grouped(bool* attr_set, const LaunchPlan& plan, cudaStream_t stream);

// How many split-K clusters of each size the device co-schedules for every
// decode variant of the dense form (uses the dense form's attribute row).
dg_status query_decode_cluster_limits(bool* dense_attr_set, ClusterLimits* out);

// Shared-memory bytes and TMEM columns of each variant (E4M3 operands).
int variant_smem_bytes(int variant);
int variant_tmem_cols(int variant);

}  // namespace dg
