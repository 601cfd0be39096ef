// Streaming expert-FFN kernels: stage 2, routed format MX4.
#define MOE_ST 2
#define MOE_RF MX4
#define MOE_RF_CODE F_MX4
#include "stream_inst.inl"
