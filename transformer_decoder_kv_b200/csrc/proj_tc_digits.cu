// Whisper projections (W8A32 and f32 weights) on tcgen05 int8 tensor cores: activation rows
// as three int8 digit planes, weights as one (int8) or three (f32) digit planes.
#define DEC_PROJ_TC_DEFINE
#include <algorithm>

#include "proj_tc.cuh"

namespace dec {
DEC_PROJ_TC_INSTANTIATE(EPI_QKV, MAP_ADJ, 3, 1)
DEC_PROJ_TC_INSTANTIATE(EPI_RESID, MAP_ADJ, 3, 1)
DEC_PROJ_TC_INSTANTIATE(EPI_STORE, MAP_ADJ, 3, 1)
DEC_PROJ_TC_INSTANTIATE(EPI_GELU, MAP_ADJ, 3, 1)
DEC_PROJ_TC_INSTANTIATE(EPI_QKV, MAP_ADJ, 3, 3)
DEC_PROJ_TC_INSTANTIATE(EPI_RESID, MAP_ADJ, 3, 3)
DEC_PROJ_TC_INSTANTIATE(EPI_STORE, MAP_ADJ, 3, 3)
DEC_PROJ_TC_INSTANTIATE(EPI_GELU, MAP_ADJ, 3, 3)
}  // namespace dec
