// gla_check.cuh -- bounds checks for debug builds.
//
// In a library built with -DGTR_BOUNDS_CHECK, every global-memory access whose
// index is computed at run time first checks that index against the extent of
// its buffer.  An index out of range is recorded in a device-side report of
// the translation unit (the first one: site, index, extent; and a count of
// all of them) and the access is skipped, so a wrong index shows up as a
// report, never as a memory fault.  The host sums and clears the reports of
// every translation unit through gtr_gla_debug_bounds_report.  Without the
// macro the checks compile to nothing and the kernels are unchanged.
#pragma once

#include <cuda_runtime.h>

namespace gtr {

struct BoundsReport {
    unsigned long long count;  // accesses skipped
    long long index, limit;    // the first one: its index and the extent it broke
    int site;                  // the first one: a BoundsSite
    int pad;
};

// Access sites, for the report.
enum BoundsSite : int {
    BS_UMMA_ROW = 1, BS_UMMA_QKV, BS_UMMA_G, BS_UMMA_EXACT, BS_UMMA_OUT, BS_UMMA_RING, BS_UMMA_FLAG,
    BS_TC_ROW = 20, BS_TC_LOAD, BS_TC_EXACT, BS_TC_SUMMARY, BS_TC_SENTER, BS_TC_RING, BS_TC_FLAG, BS_TC_OUT,
    BS_SIMT_LOAD = 40, BS_SIMT_SUMMARY, BS_SIMT_SCAN, BS_SIMT_SENTER, BS_SIMT_OUT,
    BS_WALK_ROW = 60, BS_WALK_LOAD, BS_WALK_G, BS_WALK_EXACT, BS_WALK_OUT, BS_WALK_STATE, BS_WALK_SUMMARY, BS_WALK_GATE,
    BS_SSWIGLU_LOAD = 80, BS_SSWIGLU_W, BS_SSWIGLU_OUT,
};

// Host: each checked translation unit registers a reader of its report
// (adds it into *sum, clears it when asked; returns 0, or -1 on a CUDA error).
typedef int (*BoundsReader)(BoundsReport *sum, int clear);
void register_bounds_reader(BoundsReader reader);

}  // namespace gtr

#ifdef GTR_BOUNDS_CHECK
namespace {

__device__ gtr::BoundsReport g_bounds;

__device__ __forceinline__ bool gtr_in_bounds(long long idx, long long limit, int site) {
    if (idx >= 0 && idx < limit) return true;
    if (atomicAdd(&g_bounds.count, 1ull) == 0ull) {
        g_bounds.index = idx;
        g_bounds.limit = limit;
        g_bounds.site = site;
    }
    return false;
}

int read_bounds_report(gtr::BoundsReport *sum, int clear) {
    gtr::BoundsReport r;
    if (cudaMemcpyFromSymbol(&r, g_bounds, sizeof(r)) != cudaSuccess) return -1;
    if (r.count && !sum->count) {
        sum->index = r.index;
        sum->limit = r.limit;
        sum->site = r.site;
    }
    sum->count += r.count;
    if (clear) {
        const gtr::BoundsReport z = {};
        if (cudaMemcpyToSymbol(g_bounds, &z, sizeof(z)) != cudaSuccess) return -1;
    }
    return 0;
}

struct BoundsRegistration {
    BoundsRegistration() { gtr::register_bounds_reader(&read_bounds_report); }
} g_bounds_registration;

}  // namespace
// true when 0 <= idx < limit; otherwise records the access and returns false
#define GTR_INB(idx, limit, site) gtr_in_bounds((long long)(idx), (long long)(limit), (site))
#else
// the arguments are side-effect free; naming them keeps them "used"
#define GTR_INB(idx, limit, site) ((void)(idx), (void)(limit), true)
#endif
