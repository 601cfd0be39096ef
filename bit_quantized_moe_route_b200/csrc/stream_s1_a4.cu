// Streaming expert-FFN kernels: stage 1, routed format A4.
#define MOE_ST 1
#define MOE_RF A4
#define MOE_RF_CODE F_A4
#include "stream_inst.inl"
