// Whisper W8A32 projections on tcgen05 int8 tensor cores: the activation rows as three int8
// digit planes, stacked along N, times the int8 weights.
#define DEC_PROJ_TC_DEFINE
#include <algorithm>

#include "proj_tc.cuh"

namespace dec {
DEC_PROJ_TC_INSTANTIATE(EPI_QKV, MAP_ADJ, 3, 1)
DEC_PROJ_TC_INSTANTIATE(EPI_RESID, MAP_ADJ, 3, 1)
DEC_PROJ_TC_INSTANTIATE(EPI_STORE, MAP_ADJ, 3, 1)
DEC_PROJ_TC_INSTANTIATE(EPI_GELU, MAP_ADJ, 3, 1)
}  // namespace dec
