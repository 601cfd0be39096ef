// Streaming expert-FFN kernels: stage 1, routed format A8.
#define MOE_ST 1
#define MOE_RF A8
#define MOE_RF_CODE F_A8
#include "stream_inst.inl"
