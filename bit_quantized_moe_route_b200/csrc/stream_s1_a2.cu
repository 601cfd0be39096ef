// Streaming expert-FFN kernels: stage 1, routed format A2.
#define MOE_ST 1
#define MOE_RF A2
#define MOE_RF_CODE F_A2
#include "stream_inst.inl"
