// gla_walk.cu -- instantiations and launchers of the tcgen05 walk kernel
// (gla_walk.cuh): d_k in {32, 64, 128}, value slices of 64, chunks of 64;
// fp16 in every mode, bf16 for the whole-sequence walk.
#include "gla_walk.cuh"

namespace gtr {

cudaError_t launch_walk(const WalkArgs &a, int mode, int grid, cudaStream_t st, bool bf16) {
    const int dk = a.geo.dk;
    if (a.gate && (mode != WALK_SEQ || a.vs != 1)) return cudaErrorInvalidValue;
    if (bf16 && mode != WALK_SEQ) return cudaErrorInvalidValue;
#define GTR_WALK_CASE(DK)                                                                                  \
    if (dk == DK) {                                                                                        \
        if (mode == WALK_SEQ) {                                                                            \
            if (bf16)                                                                                      \
                return a.gate ? launch_walk_t<DK, WALK_SEQ, true, __nv_bfloat16>(a, grid, st)              \
                              : launch_walk_t<DK, WALK_SEQ, false, __nv_bfloat16>(a, grid, st);            \
            return a.gate ? launch_walk_t<DK, WALK_SEQ, true, __half>(a, grid, st)                         \
                          : launch_walk_t<DK, WALK_SEQ, false, __half>(a, grid, st);                       \
        }                                                                                                  \
        if (mode == WALK_SUMMARY) return launch_walk_t<DK, WALK_SUMMARY, false, __half>(a, grid, st);      \
        return launch_walk_t<DK, WALK_OUTPUT, false, __half>(a, grid, st);                                 \
    }
    GTR_WALK_CASE(32)
    GTR_WALK_CASE(64)
    GTR_WALK_CASE(128)
#undef GTR_WALK_CASE
    return cudaErrorInvalidValue;
}

cudaError_t walk_ctas_per_sm(int dk, int mode, int *ctas) {
    *ctas = 0;
#define GTR_WALK_OCC(DK)                                                                \
    if (dk == DK) {                                                                     \
        if (mode == WALK_SEQ) return walk_occupancy<DK, WALK_SEQ, false, __half>(ctas); \
        if (mode == WALK_SUMMARY) return walk_occupancy<DK, WALK_SUMMARY, false, __half>(ctas); \
        return walk_occupancy<DK, WALK_OUTPUT, false, __half>(ctas);                    \
    }
    GTR_WALK_OCC(32)
    GTR_WALK_OCC(64)
    GTR_WALK_OCC(128)
#undef GTR_WALK_OCC
    return cudaSuccess;
}

}  // namespace gtr
