// TMA/TMEM expert-FFN kernel: stage 2, weight format A2.
#define MOE_ST 2
#define MOE_RF A2
#define MOE_RF_CODE F_A2
#include "um_inst.inl"
