// Projection kernels with int8 per-row weights and f32 activations (Whisper W8A32 layers).
#define DEC_GEMV_DEFINE
#include "gemv_launch.cuh"

namespace dec {
DEC_GEMV_INSTANTIATE(int8_t, false, PRO_LN, EPI_QKV, MAP_ADJ)
DEC_GEMV_INSTANTIATE(int8_t, false, PRO_NONE, EPI_RESID, MAP_ADJ)
DEC_GEMV_INSTANTIATE(int8_t, false, PRO_LN, EPI_STORE, MAP_ADJ)
DEC_GEMV_INSTANTIATE(int8_t, false, PRO_LN, EPI_GELU, MAP_ADJ)
}  // namespace dec
