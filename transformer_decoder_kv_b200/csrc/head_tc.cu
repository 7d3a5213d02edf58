// Tied LM head on tcgen05 int8 tensor cores (three-digit split of the f32 operands) and
// the per-row digit kernel it shares with the load-time embedding split.
#define DEC_HEAD_TC_DEFINE
#include <algorithm>

#include "head_tc.cuh"

namespace dec {
template cudaError_t rowprep_digits_launch<PRO_NONE>(const float*, int, const float*, const float*, float, int, int,
                                                     long long, int8_t*, float*, int*, bool, cudaStream_t);
template cudaError_t rowprep_digits_launch<PRO_LN>(const float*, int, const float*, const float*, float, int, int,
                                                   long long, int8_t*, float*, int*, bool, cudaStream_t);
template cudaError_t rowprep_digits_launch<PRO_RMS>(const float*, int, const float*, const float*, float, int, int,
                                                    long long, int8_t*, float*, int*, bool, cudaStream_t);
}  // namespace dec
