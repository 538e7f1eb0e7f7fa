#include "dsa_internal.h"
namespace dsa {
bool index_scores_tc_supported(const dsa_dims&) { return false; }
cudaError_t launch_index_scores_tc(const dsa_dims&, const void*, const void*, const float*, float,
                                   const int32_t*, const int32_t*, const int32_t*, float*,
                                   cudaStream_t) { return cudaErrorNotSupported; }
}
