// Per-row int8 activation quantiser of the W8A8 tensor-core projections.
#define DEC_ROWPREP_I8_DEFINE
#include "rowprep_i8.cuh"

namespace dec {
DEC_ROWPREP_I8_INSTANTIATE(PRO_RMS)
DEC_ROWPREP_I8_INSTANTIATE(PRO_NONE)
}  // namespace dec
