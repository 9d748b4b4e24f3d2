// Table-mode launch for one (PA, PB) plane pair; each gemm_table_p*.cu includes
// this and instantiates one pair, so the kernels compile in parallel.
#pragma once

#include <mutex>

#include "host_common.h"

namespace mao {

template <int PA, int PB, int A_MN, int B_MN>
mao_status launch_table_majors(const GemmTableParams& p, cudaStream_t stream, int kernel_id, double flops) {
  using Cfg = GemmCfg<OP_SPLIT3, A_MN, B_MN, PA, PB>;
  static std::mutex mu;
  static bool attr_set[64] = {};
  DeviceInfo* d = nullptr;
  MAO_TRY(device_info(&d));
  int dev = 0;
  MAO_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return MAO_ERR_UNSUPPORTED;
  auto kern = gemm_tc_table_kernel<A_MN, B_MN, PA, PB>;
  {
    std::lock_guard<std::mutex> lk(mu);
    if (!attr_set[dev]) {
      MAO_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES));
      attr_set[dev] = true;
    }
  }
  if (p.total_tiles <= 0) return MAO_OK;
  const int grid = p.total_tiles < d->sm_count ? p.total_tiles : d->sm_count;
  // tensor-core products per multiply-add: pairs (i, j), i < PA, j < PB, i + j <= max(PA, PB) - 1
  constexpr int kProducts = (PA == 3 && PB == 3) ? 6 : (PA == 1 && PB == 1) ? 1 : 3;
  LaunchScope ls(stream, kernel_id, flops, 0.0, flops * kProducts);
  kern<<<grid, Cfg::TABLE_THREADS, Cfg::SMEM_BYTES, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? MAO_OK : MAO_ERR_CUDA;
}

// CTA-pair kernel (clusters of two): grid = two CTAs per pair, at most one pair per two SMs.
template <int PA, int PB, int A_MN, int B_MN>
mao_status launch_pair_majors(const GemmTableParams& p, cudaStream_t stream, int kernel_id, double flops) {
  using Cfg = GemmPairCfg<A_MN, B_MN, PA, PB>;
  static std::mutex mu;
  static bool attr_set[64] = {};
  DeviceInfo* d = nullptr;
  MAO_TRY(device_info(&d));
  int dev = 0;
  MAO_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return MAO_ERR_UNSUPPORTED;
  auto kern = gemm_tc_pair_kernel<A_MN, B_MN, PA, PB>;
  {
    std::lock_guard<std::mutex> lk(mu);
    if (!attr_set[dev]) {
      MAO_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES));
      attr_set[dev] = true;
    }
  }
  if (p.total_tiles <= 0) return MAO_OK;
  const int max_pairs = d->sm_count / 2;
  const int pairs = p.total_tiles < max_pairs ? p.total_tiles : max_pairs;
  constexpr int kProducts = (PA == 3 && PB == 3) ? 6 : (PA == 1 && PB == 1) ? 1 : 3;
  LaunchScope ls(stream, kernel_id, flops, 0.0, flops * kProducts);
  kern<<<2 * pairs, Cfg::THREADS, Cfg::SMEM_BYTES, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? MAO_OK : MAO_ERR_CUDA;
}

template <int PA, int PB>
mao_status launch_table_planes(const GemmTableParams& p, int a_mn, int b_mn, cudaStream_t stream, int kernel_id,
                               double flops, bool pair) {
  if (pair) {
    if (!a_mn && !b_mn) return launch_pair_majors<PA, PB, 0, 0>(p, stream, kernel_id, flops);
    if (!a_mn && b_mn) return launch_pair_majors<PA, PB, 0, 1>(p, stream, kernel_id, flops);
    if (a_mn && !b_mn) return launch_pair_majors<PA, PB, 1, 0>(p, stream, kernel_id, flops);
    return launch_pair_majors<PA, PB, 1, 1>(p, stream, kernel_id, flops);
  }
  if (!a_mn && !b_mn) return launch_table_majors<PA, PB, 0, 0>(p, stream, kernel_id, flops);
  if (!a_mn && b_mn) return launch_table_majors<PA, PB, 0, 1>(p, stream, kernel_id, flops);
  if (a_mn && !b_mn) return launch_table_majors<PA, PB, 1, 0>(p, stream, kernel_id, flops);
  return launch_table_majors<PA, PB, 1, 1>(p, stream, kernel_id, flops);
}

}  // namespace mao
