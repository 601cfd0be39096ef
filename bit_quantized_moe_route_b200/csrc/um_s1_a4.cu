// TMA/TMEM expert-FFN kernel: stage 1, weight format A4.
#define MOE_ST 1
#define MOE_RF A4
#define MOE_RF_CODE F_A4
#include "um_inst.inl"
