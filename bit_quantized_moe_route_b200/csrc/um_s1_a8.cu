// TMA/TMEM expert-FFN kernel: stage 1, weight format A8.
#define MOE_ST 1
#define MOE_RF A8
#define MOE_RF_CODE F_A8
#include "um_inst.inl"
