// Instantiation unit of the streaming expert-FFN kernels for one stage and
// one routed format (MOE_ST, MOE_RF set by the including file).
#include "ffn_stream.cuh"

namespace moe {

#define MOE_CAT3(a, b, c) a##b##_##c
#define MOE_NAME(pre, st, f) MOE_CAT3(pre, st, f)

bool MOE_NAME(launch_stream_s, MOE_ST, MOE_RF)(int ntmax, int cpl, int grid, cudaStream_t s,
                                                const StreamParams& q) {
  // programmatic stream serialization: the kernel waits (griddepcontrol)
  // for its predecessor's results where it needs them
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kStreamThreads);
  cfg.dynamicSmemBytes = kStreamSmem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
#define MOE_CASE(NT, CP)                                                                          \
  if (ntmax == NT && cpl == CP) {                                                                 \
    cudaLaunchKernelEx(&cfg, ffn_stream_kernel<MOE_ST, NT, CP, MOE_RF_CODE>, q); /* errors: caller checks */ \
    return true;                                                                                  \
  }
  MOE_CASE(1, 4)
  MOE_CASE(1, 2)
  MOE_CASE(1, 1)
  MOE_CASE(2, 2)
  MOE_CASE(2, 1)
  MOE_CASE(4, 1)
#undef MOE_CASE
  return false;
}

void MOE_NAME(attrs_stream_s, MOE_ST, MOE_RF)() {
#define MOE_ATTR(NT, CP)                                                                            \
  cudaFuncSetAttribute(ffn_stream_kernel<MOE_ST, NT, CP, MOE_RF_CODE>,                             \
                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kStreamSmem);
  MOE_ATTR(1, 4)
  MOE_ATTR(1, 2)
  MOE_ATTR(1, 1)
  MOE_ATTR(2, 2)
  MOE_ATTR(2, 1)
  MOE_ATTR(4, 1)
#undef MOE_ATTR
}

}  // namespace moe
