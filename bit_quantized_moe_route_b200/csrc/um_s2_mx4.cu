// TMA/TMEM expert-FFN kernel: stage 2, weight format MX4.
#define MOE_ST 2
#define MOE_RF MX4
#define MOE_RF_CODE F_MX4
#include "um_inst.inl"
