// dg_fp8_gemm_nt_noalloc: the dense GEMM for callers that cannot allocate
// device memory.  Its scratch -- the device error word the kernel's bounded
// waits and data checks report into -- lives in one file-scope __device__
// array of fixed size instead of memory the library would otherwise
// cudaMalloc on first use.  (Split-K reduces through distributed shared
// memory and needs no global scratch.)  The planning (argument checks,
// picker, tensor maps) and the launch are the regular dense entry point's;
// only the device set-up differs: it allocates nothing.  The declarations and
// the contract are in include/dg.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/dg.h"
#include "dg_internal.h"

namespace dg {
namespace {

// Layout of the static scratch: [error word | pad to 256 bytes]
constexpr size_t kNaScratchBytes = 256;

// Every GPU that loads the library holds this array until the process exits.
// In host code `g_noalloc_scratch` is only a host-side stand-in for the
// symbol; the device address comes from cudaGetSymbolAddress below, and the
// host reads and clears the word through the symbol API
// (cudaMemcpyFromSymbol / cudaMemcpyToSymbol), which allocates nothing.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNaScratchBytes];

constexpr int kNaMaxDevices = 64;

struct NaDevice {
  bool ready = false;
  int num_sms = 0;
  int* error_word = nullptr;          // device address of g_noalloc_scratch
  bool attr_set[kNumVariants] = {};   // dense form: shared-memory limit raised
  ClusterLimits limits = {};          // co-resident split-K clusters
};

std::mutex g_na_mutex;
NaDevice g_na_dev[kNaMaxDevices];

// Once per device, with that device current: check the architecture, find the
// device address of the static scratch and the co-resident cluster limits.
// Nothing here allocates device memory.
dg_status na_setup(NaDevice** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DG_ERR_CUDA;
  if (dev < 0 || dev >= kNaMaxDevices) return DG_ERR_UNSUPPORTED;
  NaDevice& st = g_na_dev[dev];
  if (!st.ready) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return DG_ERR_CUDA;
    if (major != 10 || minor != 0) return DG_ERR_ARCH;
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr)
      return DG_ERR_CUDA;
    st.error_word = static_cast<int*>(ptr);
    st.num_sms = sms;
    dg_status s = query_decode_cluster_limits(st.attr_set, &st.limits);
    if (s != DG_OK) return s;
    st.ready = true;
  }
  *out = &st;
  return DG_OK;
}

}  // namespace
}  // namespace dg

using namespace dg;

extern "C" dg_status dg_fp8_gemm_nt_noalloc(const void* a, const float* sfa, const void* b,
                                            const float* sfb, void* d, int M, int N, int K,
                                            dg_stream_t stream) {
  const GemmCall call{kFormDense, a, sfa, b, sfb, d, nullptr, nullptr, nullptr, M, N, K, 1, 0};
  bool empty = false;
  dg_status s = check_gemm_call(call, &empty);  // before any device work
  if (s != DG_OK || empty) return s;
  std::lock_guard<std::mutex> lock(g_na_mutex);
  NaDevice* st = nullptr;
  s = na_setup(&st);
  if (s != DG_OK) return s;
  LaunchPlans plans;
  s = plan_gemm(call, DeviceFacts{st->num_sms, &st->limits}, st->error_word, &plans);
  if (s != DG_OK || plans.n == 0) return s;
  const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (check_scales_enabled()) {
    s = launch_scale_check(call, st->error_word, cs);
    if (s != DG_OK) return s;
  }
  for (int i = 0; i < plans.n && s == DG_OK; ++i) s = launch_fp8_dense(st->attr_set, plans.plan[i], cs);
  return s;
}

extern "C" dg_status dg_fp8_gemm_nt_noalloc_get_last_device_error(int* code) {
  if (!code) return DG_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_na_mutex);
  NaDevice* st = nullptr;
  dg_status s = na_setup(&st);
  if (s != DG_OK) return s;
  if (cudaDeviceSynchronize() != cudaSuccess) return DG_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_noalloc_scratch, sizeof(int), 0, cudaMemcpyDeviceToHost) !=
      cudaSuccess)
    return DG_ERR_CUDA;
  *code = v;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_noalloc_scratch, &zero, sizeof(int), 0, cudaMemcpyHostToDevice) !=
        cudaSuccess)
      return DG_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return DG_ERR_CUDA;
  }
  return DG_OK;
}
