// Host entry of the tcgen05 fused kernel (d_k = d_v = 64, chunk 64).
#include "gla_umma.cuh"

namespace gtr {
cudaError_t launch_fused_umma(const TcArgs &a, cudaStream_t st) { return launch_umma(a, st); }
}  // namespace gtr
