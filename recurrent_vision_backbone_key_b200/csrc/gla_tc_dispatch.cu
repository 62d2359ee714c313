// Dispatch of the tensor-core chunk kernels on d_k, d_v (host code).
#include "gla_tc.cuh"

namespace gtr {

cudaError_t launch_tc_dk16(const TcArgs &a, int mode, cudaStream_t st);
cudaError_t launch_tc_dk32(const TcArgs &a, int mode, cudaStream_t st);
cudaError_t launch_tc_dk64(const TcArgs &a, int mode, cudaStream_t st);
cudaError_t launch_tc_dk128(const TcArgs &a, int mode, cudaStream_t st);

namespace {
template <int DK>
size_t smem_dk(int dv, int chunk) {
    switch (dv) {
    case 16: return TcLayout<DK, 16>::bytes(chunk);
    case 32: return TcLayout<DK, 32>::bytes(chunk);
    case 64: return TcLayout<DK, 64>::bytes(chunk);
    default: return TcLayout<DK, 128>::bytes(chunk);
    }
}
}  // namespace

size_t tc_smem_bytes(int dk, int dv, int chunk) {
    switch (dk) {
    case 16: return smem_dk<16>(dv, chunk);
    case 32: return smem_dk<32>(dv, chunk);
    case 64: return smem_dk<64>(dv, chunk);
    default: return smem_dk<128>(dv, chunk);
    }
}

cudaError_t launch_tc(const TcArgs &a, int mode, cudaStream_t st) {
    switch (a.geo.dk) {
    case 16: return launch_tc_dk16(a, mode, st);
    case 32: return launch_tc_dk32(a, mode, st);
    case 64: return launch_tc_dk64(a, mode, st);
    default: return launch_tc_dk128(a, mode, st);
    }
}

}  // namespace gtr
