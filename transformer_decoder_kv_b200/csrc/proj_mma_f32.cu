// Tensor-core projections with f32 weights (Whisper f32 layers, LM heads) and the
// row-normalisation prologue kernel they share with the W8A32 projections.
#define DEC_MMA_DEFINE
#include "proj_mma.cuh"

namespace dec {
DEC_MMA_INSTANTIATE(float, EPI_QKV)
DEC_MMA_INSTANTIATE(float, EPI_RESID)
DEC_MMA_INSTANTIATE(float, EPI_STORE)
DEC_MMA_INSTANTIATE(float, EPI_GELU)
DEC_MMA_INSTANTIATE(float, EPI_HEAD)
DEC_ROWPREP_INSTANTIATE(PRO_LN)
DEC_ROWPREP_INSTANTIATE(PRO_RMS)
}  // namespace dec
