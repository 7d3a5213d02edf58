// W8A8 projections on tcgen05 int8 tensor cores and the weight-row permutation used by
// their RoPE and SwiGLU row maps.
#define DEC_PROJ_TC_DEFINE
#define DEC_PROJ_TC_PERMUTE_DEFINE
#include <algorithm>

#include "proj_tc.cuh"

namespace dec {
DEC_PROJ_TC_INSTANTIATE(EPI_QKV, MAP_ROPE, 1, 1)
DEC_PROJ_TC_INSTANTIATE(EPI_RESID, MAP_ADJ, 1, 1)
DEC_PROJ_TC_INSTANTIATE(EPI_SWIGLU, MAP_DUAL, 1, 1)
DEC_PROJ_TC_INSTANTIATE(EPI_I32, MAP_ADJ, 1, 1)
}  // namespace dec
