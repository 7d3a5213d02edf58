// Tensor-core projections with int8 per-row weights and f32 activations (Whisper W8A32 layers).
#define DEC_MMA_DEFINE
#include "proj_mma.cuh"

namespace dec {
DEC_MMA_INSTANTIATE(int8_t, EPI_QKV)
DEC_MMA_INSTANTIATE(int8_t, EPI_RESID)
DEC_MMA_INSTANTIATE(int8_t, EPI_STORE)
DEC_MMA_INSTANTIATE(int8_t, EPI_GELU)
}  // namespace dec
