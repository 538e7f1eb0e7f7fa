#include "dsa_internal.h"
namespace dsa {
bool attend_tc_supported(const dsa_dims&, int64_t, const void*, const void*, int64_t, int) { return false; }
cudaError_t launch_attend_tc(const dsa_dims&, const void*, const void*, int64_t, const int32_t*, int,
                             float, void*, float*, cudaStream_t) { return cudaErrorNotSupported; }
}
