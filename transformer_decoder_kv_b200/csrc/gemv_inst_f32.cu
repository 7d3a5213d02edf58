// Projection kernels with f32 weights and f32 activations (Whisper f32 layers, LM heads).
#define DEC_GEMV_DEFINE
#include "gemv_launch.cuh"

namespace dec {
DEC_GEMV_INSTANTIATE(float, false, PRO_LN, EPI_QKV, MAP_ADJ)
DEC_GEMV_INSTANTIATE(float, false, PRO_NONE, EPI_RESID, MAP_ADJ)
DEC_GEMV_INSTANTIATE(float, false, PRO_LN, EPI_STORE, MAP_ADJ)
DEC_GEMV_INSTANTIATE(float, false, PRO_LN, EPI_GELU, MAP_ADJ)
}  // namespace dec
