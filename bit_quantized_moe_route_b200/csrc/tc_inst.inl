// Instantiation unit of the tensor-core expert-FFN kernel for one stage and
// one weight format (MOE_ST, MOE_RF, MOE_RF_CODE set by the including file).
#include "ffn_tc.cuh"

namespace moe {

#define MOE_TC_CAT3(a, b, c) a##b##_##c
#define MOE_TC_NAME(pre, st, f) MOE_TC_CAT3(pre, st, f)

bool MOE_TC_NAME(launch_tc_s, MOE_ST, MOE_RF)(const TcParams& p, int grid, cudaStream_t s) {
  ffn_tc_kernel<MOE_ST, MOE_RF_CODE><<<grid, kTcThreads, TcCfg<MOE_ST, MOE_RF_CODE>::smem, s>>>(p);
  return true;
}

void MOE_TC_NAME(attrs_tc_s, MOE_ST, MOE_RF)() {
  cudaFuncSetAttribute(ffn_tc_kernel<MOE_ST, MOE_RF_CODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)TcCfg<MOE_ST, MOE_RF_CODE>::smem);
}

}  // namespace moe
