// TMA/TMEM expert-FFN kernel: stage 2, weight format A3.
#define MOE_ST 2
#define MOE_RF A3
#define MOE_RF_CODE F_A3
#include "um_inst.inl"
