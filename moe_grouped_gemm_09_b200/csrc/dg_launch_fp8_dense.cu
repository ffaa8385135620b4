// Dense FP8 form: kernel instantiations, launch, and the device's co-resident
// split-K cluster limits of the decode variants.
#include <array>

#include "dg_launch.cuh"

namespace dg {

dg_status launch_fp8_dense(bool* attr_set, const LaunchPlan& plan, cudaStream_t stream) {
  return launch_form<kFormDense>(attr_set, plan, stream);
}

namespace {

template <int V>
dg_status query_cluster_limits(bool* attr_set, ClusterLimits* out) {
  if constexpr (kVariants[V].decode) {
    dg_status s = set_smem_attr<kFormDense, V>(attr_set);
    if (s != DG_OK) return s;
    for (int c = 1; c <= kMaxSplitK; ++c) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(c, 1, 1);
      cfg.blockDim = dim3(kThreads, 1, 1);
      cfg.dynamicSmemBytes = ShapeOf<V>::kSmemBytes;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = c;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kernel_of<kFormDense, V>(), &cfg) != cudaSuccess) {
        cudaGetLastError();  // clear; treat as "not known"
        n = 0;
      }
      out->max_clusters[V][c] = n;
    }
  }
  return DG_OK;
}

template <int... V>
dg_status query_all(bool* attr_set, ClusterLimits* out, std::integer_sequence<int, V...>) {
  dg_status s = DG_OK;
  ((s = (s == DG_OK ? query_cluster_limits<V>(attr_set, out) : s)), ...);
  return s;
}

template <int what, int... V>
constexpr std::array<int, sizeof...(V)> variant_table(std::integer_sequence<int, V...>) {
  return {(what == 0 ? ShapeOf<V>::kSmemBytes : ShapeOf<V>::kTmemCols)...};
}

}  // namespace

dg_status query_decode_cluster_limits(bool* dense_attr_set, ClusterLimits* out) {
  return query_all(dense_attr_set, out, std::make_integer_sequence<int, kNumVariants>{});
}

int variant_smem_bytes(int v) {
  constexpr auto t = variant_table<0>(std::make_integer_sequence<int, kNumVariants>{});
  return t[v];
}

int variant_tmem_cols(int v) {
  constexpr auto t = variant_table<1>(std::make_integer_sequence<int, kNumVariants>{});
  return t[v];
}

}  // namespace dg
