// TMA/TMEM expert-FFN kernel: stage 2, weight format A8.
#define MOE_ST 2
#define MOE_RF A8
#define MOE_RF_CODE F_A8
#include "um_inst.inl"
