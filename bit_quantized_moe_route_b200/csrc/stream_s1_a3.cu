// Streaming expert-FFN kernels: stage 1, routed format A3.
#define MOE_ST 1
#define MOE_RF A3
#define MOE_RF_CODE F_A3
#include "stream_inst.inl"
