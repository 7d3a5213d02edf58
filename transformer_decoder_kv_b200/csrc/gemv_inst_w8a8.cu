// Projection kernels with int8 weights and int8 activations (Qwen2 W8A8 layers, int8 dot op).
#define DEC_GEMV_DEFINE
#include "gemv_launch.cuh"

namespace dec {
DEC_GEMV_INSTANTIATE(int8_t, true, PRO_RMS, EPI_QKV, MAP_ROPE)
DEC_GEMV_INSTANTIATE(int8_t, true, PRO_NONE, EPI_RESID, MAP_ADJ)
DEC_GEMV_INSTANTIATE(int8_t, true, PRO_RMS, EPI_SWIGLU, MAP_DUAL)
DEC_GEMV_INSTANTIATE(int8_t, true, PRO_RAW_I8, EPI_I32, MAP_ADJ)
}  // namespace dec
