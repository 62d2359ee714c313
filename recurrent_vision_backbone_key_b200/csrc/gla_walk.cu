// gla_walk.cu -- instantiations and launchers of the tcgen05 walk kernel
// (gla_walk.cuh): d_k in {32, 64, 128}, value slices of 64, chunks of 64.
#include "gla_walk.cuh"

namespace gtr {

cudaError_t launch_walk(const WalkArgs &a, int mode, int grid, cudaStream_t st) {
    const int dk = a.geo.dk;
    if (a.gate && (mode != WALK_SEQ || a.vs != 1)) return cudaErrorInvalidValue;
#define GTR_WALK_CASE(DK)                                                                 \
    if (dk == DK) {                                                                       \
        if (mode == WALK_SEQ)                                                             \
            return a.gate ? launch_walk_t<DK, WALK_SEQ, true>(a, grid, st)                \
                          : launch_walk_t<DK, WALK_SEQ, false>(a, grid, st);              \
        if (mode == WALK_SUMMARY) return launch_walk_t<DK, WALK_SUMMARY, false>(a, grid, st); \
        return launch_walk_t<DK, WALK_OUTPUT, false>(a, grid, st);                        \
    }
    GTR_WALK_CASE(32)
    GTR_WALK_CASE(64)
    GTR_WALK_CASE(128)
#undef GTR_WALK_CASE
    return cudaErrorInvalidValue;
}

cudaError_t walk_ctas_per_sm(int dk, int mode, int *ctas) {
    *ctas = 0;
#define GTR_WALK_OCC(DK)                                                           \
    if (dk == DK) {                                                                \
        if (mode == WALK_SEQ) return walk_occupancy<DK, WALK_SEQ, false>(ctas);    \
        if (mode == WALK_SUMMARY) return walk_occupancy<DK, WALK_SUMMARY, false>(ctas); \
        return walk_occupancy<DK, WALK_OUTPUT, false>(ctas);                       \
    }
    GTR_WALK_OCC(32)
    GTR_WALK_OCC(64)
    GTR_WALK_OCC(128)
#undef GTR_WALK_OCC
    return cudaSuccess;
}

}  // namespace gtr
