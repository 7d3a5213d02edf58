// Tensor-core projections for W8A8 layers (int8 weights, int8 activation rows), the
// int8 row quantiser and the weight-row permutation used by the RoPE and SwiGLU row maps.
#define DEC_I8MMA_DEFINE
#include "proj_i8mma.cuh"

namespace dec {
DEC_I8MMA_INSTANTIATE(EPI_QKV, MAP_ROPE)
DEC_I8MMA_INSTANTIATE(EPI_RESID, MAP_ADJ)
DEC_I8MMA_INSTANTIATE(EPI_SWIGLU, MAP_DUAL)
DEC_ROWPREP_I8_INSTANTIATE(PRO_RMS)
DEC_ROWPREP_I8_INSTANTIATE(PRO_NONE)
}  // namespace dec
