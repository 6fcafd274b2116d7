// placeholder, replaced by the tcgen05 GEMM
#include "launch.h"
namespace cca {
bool gemm_tc_supported(long long, int, int) { return false; }
cudaError_t launch_gemm_tc(const GemmTcArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace cca
