// Streaming expert-FFN kernels: stage 2, routed format A8.
#define MOE_ST 2
#define MOE_RF A8
#define MOE_RF_CODE F_A8
#include "stream_inst.inl"
