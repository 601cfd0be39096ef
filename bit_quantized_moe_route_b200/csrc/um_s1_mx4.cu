// TMA/TMEM expert-FFN kernel: stage 1, weight format MX4.
#define MOE_ST 1
#define MOE_RF MX4
#define MOE_RF_CODE F_MX4
#include "um_inst.inl"
