// Instantiation unit of the TMA/TMEM expert-FFN kernel for one stage and
// one weight format (MOE_ST, MOE_RF, MOE_RF_CODE set by the including file).
#include "ffn_umma.cuh"

namespace moe {

#define MOE_UM_CAT3(a, b, c) a##b##_##c
#define MOE_UM_NAME(pre, st, f) MOE_UM_CAT3(pre, st, f)

namespace {
cudaLaunchConfig_t um_config(int pairs, cudaStream_t s, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(kUmThreads);
  cfg.dynamicSmemBytes = UmCfg<MOE_ST, MOE_RF_CODE>::smem;
  cfg.stream = s;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}
}  // namespace

bool MOE_UM_NAME(launch_um_s, MOE_ST, MOE_RF)(const UmParams& p, int pairs, cudaStream_t s) {
  cudaLaunchAttribute attr[1];
  const cudaLaunchConfig_t cfg = um_config(pairs, s, attr);
  return cudaLaunchKernelEx(&cfg, ffn_umma_kernel<MOE_ST, MOE_RF_CODE>, p) == cudaSuccess;
}

int MOE_UM_NAME(attrs_um_s, MOE_ST, MOE_RF)() {
  cudaFuncSetAttribute(ffn_umma_kernel<MOE_ST, MOE_RF_CODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)UmCfg<MOE_ST, MOE_RF_CODE>::smem);
  cudaLaunchAttribute attr[1];
  const cudaLaunchConfig_t cfg = um_config(1, nullptr, attr);
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, ffn_umma_kernel<MOE_ST, MOE_RF_CODE>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  return n;
}

}  // namespace moe
