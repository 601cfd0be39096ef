// TMA/TMEM expert-FFN kernel: stage 1, weight format A2.
#define MOE_ST 1
#define MOE_RF A2
#define MOE_RF_CODE F_A2
#include "um_inst.inl"
