// Instantiation unit of the TMA/TMEM expert-FFN kernel for one stage and
// one weight format (MOE_ST, MOE_RF, MOE_RF_CODE set by the including file).
#include "ffn_umma.cuh"

namespace moe {

#define MOE_UM_CAT3(a, b, c) a##b##_##c
#define MOE_UM_NAME(pre, st, f) MOE_UM_CAT3(pre, st, f)

bool MOE_UM_NAME(launch_um_s, MOE_ST, MOE_RF)(const UmParams& p, int grid, cudaStream_t s) {
  ffn_umma_kernel<MOE_ST, MOE_RF_CODE><<<grid, kUmThreads, UmCfg<MOE_ST, MOE_RF_CODE>::smem, s>>>(p);
  return true;
}

void MOE_UM_NAME(attrs_um_s, MOE_ST, MOE_RF)() {
  cudaFuncSetAttribute(ffn_umma_kernel<MOE_ST, MOE_RF_CODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)UmCfg<MOE_ST, MOE_RF_CODE>::smem);
}

}  // namespace moe
