// Streaming expert-FFN kernels: stage 1, routed format MX4.
#define MOE_ST 1
#define MOE_RF MX4
#define MOE_RF_CODE F_MX4
#include "stream_inst.inl"
