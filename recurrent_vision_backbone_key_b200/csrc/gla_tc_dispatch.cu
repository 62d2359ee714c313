// Dispatch of the tensor-core chunk kernels on d_k (host code).
#include "gla_tc.cuh"

namespace gtr {

cudaError_t launch_tc_dk16(const TcArgs &a, int mode, cudaStream_t st);
cudaError_t launch_tc_dk32(const TcArgs &a, int mode, cudaStream_t st);
cudaError_t launch_tc_dk64(const TcArgs &a, int mode, cudaStream_t st);
cudaError_t launch_tc_dk128(const TcArgs &a, int mode, cudaStream_t st);

cudaError_t launch_tc(const TcArgs &a, int mode, cudaStream_t st) {
    switch (a.geo.dk) {
    case 16: return launch_tc_dk16(a, mode, st);
    case 32: return launch_tc_dk32(a, mode, st);
    case 64: return launch_tc_dk64(a, mode, st);
    default: return launch_tc_dk128(a, mode, st);
    }
}

}  // namespace gtr
