// Streaming expert-FFN kernels: stage 2, routed format A2.
#define MOE_ST 2
#define MOE_RF A2
#define MOE_RF_CODE F_A2
#include "stream_inst.inl"
