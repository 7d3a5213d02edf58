// Final norm + tied LM head + greedy argmax (f32 embedding table).
#define DEC_GEMV_DEFINE
#include "gemv_launch.cuh"

namespace dec {
DEC_GEMV_INSTANTIATE(float, false, PRO_LN, EPI_HEAD, MAP_ADJ)
DEC_GEMV_INSTANTIATE(float, false, PRO_RMS, EPI_HEAD, MAP_ADJ)
}  // namespace dec
