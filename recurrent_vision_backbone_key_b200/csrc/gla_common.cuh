// gla_common.cuh -- pieces shared by the CUDA kernels of the GLA mixer.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "gla_check.cuh"

namespace gtr {

// Programmatic dependent launch.  A grid launched with programmatic stream
// serialization may start before the grid ahead of it in the stream has
// finished: grid_dep_wait() blocks until that grid has completed and its
// memory is visible (immediately for a normal launch), and must come before
// any read of what it wrote; grid_dep_launch() lets the next such grid start.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

// kern<<<grid, block, smem, st>>>(args...), with programmatic stream
// serialization when `pdl` is set (only for kernels that call grid_dep_wait
// before they read the previous grid's results).
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
                          Args &&...args) {
    if (!pdl) {
        kern<<<grid, block, smem, st>>>(std::forward<Args>(args)...);
        return cudaGetLastError();
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Problem geometry shared by every kernel.  Token layout [B][N][heads][d],
// N = H*W tokens in row-major spatial order.
struct Geom {
    int B, heads, H, W;
    int dk, dv;
    int dir;     // 0 L->R, 1 R->L, 2 T->B, 3 B->T
    int chunk;   // tokens per chunk
    int N;       // H*W
    int nc;      // ceil(N / chunk)
};

// G0, the scan-order index map: scan position t -> row-major token index.
// Left->right is row-major order, right->left its reverse, top->bottom is
// column-major order (t = col*H + row) and bottom->top its reverse (ai.info
// summary of GTR, "Methodology in Plain English"; GTR project page, "How GTR
// Works").  Folded into every load and store: no permuted copy exists.
__device__ __forceinline__ int scan_pos(int dir, int t, int H, int W, int N) {
    if (dir == 1) return N - 1 - t;
    if (dir >= 2) {
        int u = (dir == 3) ? (N - 1 - t) : t;
        int col = u / H;
        int row = u - col * H;
        return row * W + col;
    }
    return t;
}

// Element offset of (b, token p, head h) in a [B][N][heads][d] tensor.
__device__ __forceinline__ int64_t tok_offset(const Geom &g, int b, int p, int h, int d) {
    return (((int64_t)b * g.N + p) * g.heads + h) * (int64_t)d;
}

}  // namespace gtr

// Host-side launchers implemented in the .cu files (internal, C++ linkage).
namespace gtr {
cudaError_t launch_summary_v0(const __half *k, const __half *v, const float *g, const Geom &geo,
                              float *dS, float *gamma, cudaStream_t st);
cudaError_t launch_scan_v0(const float *dS, const float *gamma, int nseq, int nc, int dk, int dv,
                           float *S_enter, cudaStream_t st);
cudaError_t launch_output_v0(const __half *q, const __half *k, const __half *v, const float *g,
                             const float *S_enter, const Geom &geo, __half *out, cudaStream_t st);
// The boundary scan in two passes over segments of chunks (more parallel
// work for long chains and few state elements); agg holds scan_agg_bytes.
int scan_segments(int64_t nseq, int nc, int dk, int dv);
size_t scan_agg_bytes(int64_t nseq, int nc, int dk, int dv);
// pdl: launched with programmatic stream serialization (the scan waits for
// the grid ahead of it before it reads dS).
cudaError_t launch_scan_segmented(const float *dS, const float *gamma, int nseq, int nc, int dk, int dv,
                                  float *S_enter, float *agg, cudaStream_t st, bool pdl = false);
// The same with fp16 dS and S_enter (the running state stays fp32).
cudaError_t launch_scan_segmented(const __half *dS, const float *gamma, int nseq, int nc, int dk, int dv,
                                  __half *S_enter, float *agg, cudaStream_t st, bool pdl = false);
void count_launch(int n = 1);
// Spatial SwiGLU gating with the fused 3x3 depthwise convolution (sswiglu.cu).
cudaError_t launch_sswiglu(const __half *a, const __half *v, const float *wc, const float *bias, int B, int H, int W,
                           int C, __half *y, unsigned *status, cudaStream_t st);
// Records the calling thread's failure text (returned by gtr_gla_last_error)
// and returns s; clear_last_error empties it at the start of a call.
int set_last_error(int s, const char *msg);
void clear_last_error();
}  // namespace gtr
