// Instantiations of the tensor-core chunk kernels for d_k = 16 (all d_v).
#include "gla_tc.cuh"

namespace gtr {
cudaError_t launch_tc_dk16(const TcArgs &a, int mode, cudaStream_t st) { return launch_tc_dk<16>(a, mode, st); }
}  // namespace gtr
