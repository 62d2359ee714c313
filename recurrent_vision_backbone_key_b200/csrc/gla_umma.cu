// Host entry of the tcgen05 fused kernel (d_k = d_v = 64 or 128, chunk 64).
#include "gla_umma.cuh"

namespace gtr {
cudaError_t launch_fused_umma(const TcArgs &a, cudaStream_t st) {
    return a.geo.dk == 128 ? launch_umma<128>(a, st) : launch_umma<64>(a, st);
}
}  // namespace gtr
