// sswiglu.cu -- Spatial SwiGLU's gating with its fused 3x3 depthwise
// convolution on the patch grid:
//     y[b][p][c] = silu(a[b][p][c]) * (bias[c] + sum_{dy,dx} w[c][dy+1][dx+1] * v[b][p + dy*W + dx][c])
// with zero padding at the grid border (ai.info summary of GTR, "Methodology
// in Plain English": a 3x3 depthwise convolution inserted in the value branch
// of a SwiGLU block, on the 2-D patch grid; GTR project page, "Spatial
// SwiGLU").  a is the gate branch, v the value branch, both [B][H*W][C] fp16
// in row-major spatial order; y likewise.
//
// HBM-bound (6 bytes per element): one CTA of 128 threads takes a tile of 8
// grid rows x 16 grid columns x 64 channels.  The value tile with its one-token
// halo (10 x 18 tokens x 128 bytes) and the gate tile (8 x 16 tokens) are
// staged in shared memory by cp.async, all in flight at once, zero-filled
// outside the grid, so the stencil needs no border tests.  Thread (column c,
// channel octet j) keeps its 9 x 8 filter taps in registers and walks the
// tile's 8 rows down its column with a 3 x 3 window of 16-byte vectors,
// loading one new row of three per step; the output writes are 16-byte
// vectors, 8 threads per 128-byte line.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gla_common.cuh"

namespace gtr {
namespace {

constexpr int kRows = 8, kCols = 16, kCh = 64;  // tile: grid rows, grid columns, channels
constexpr int kHr = kRows + 2, kHc = kCols + 2; // with the halo
constexpr int kThreads = kCols * (kCh / 8);     // one thread per (column, channel octet)

__device__ __forceinline__ void cp16(uint32_t saddr, const void *g, bool full) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(saddr), "l"(g), "r"(full ? 16 : 0));
}

__device__ __forceinline__ void acc_tap(float (&acc)[8], const float (&w)[8], uint4 x) {
    const __half2 *h = reinterpret_cast<const __half2 *>(&x);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(h[e]);
        acc[2 * e] = fmaf(w[2 * e], f.x, acc[2 * e]);
        acc[2 * e + 1] = fmaf(w[2 * e + 1], f.y, acc[2 * e + 1]);
    }
}

__device__ __forceinline__ float silu(float x) { return __fdividef(x, 1.f + __expf(-x)); }

__global__ void __launch_bounds__(kThreads) sswiglu_kernel(const __half *__restrict__ a, const __half *__restrict__ v,
                                                           const float *__restrict__ wc, const float *__restrict__ bias,
                                                           int B, int H, int W, int C, __half *__restrict__ y) {
    __shared__ __align__(16) uint4 tile[kHr * kHc * (kCh / 8)];     // value branch with halo
    __shared__ __align__(16) uint4 gtile[kRows * kCols * (kCh / 8)];  // gate branch
    const int tid = threadIdx.x;
    const int c0 = blockIdx.y * kCh;
    const int tiles_w = (W + kCols - 1) / kCols;
    const int r0 = (blockIdx.x / tiles_w) * kRows, col0 = (blockIdx.x % tiles_w) * kCols;
    const int b = blockIdx.z;
    const int64_t elems = (int64_t)B * H * W * C;

    // ---- the value tile with its halo and the gate tile, zero outside the
    // grid and past C, all copies in flight at once
    const uint32_t sbase = (uint32_t)__cvta_generic_to_shared(tile);
    for (int idx = tid; idx < kHr * kHc * (kCh / 8); idx += kThreads) {
        const int j = idx & 7, cell = idx >> 3;
        const int hr = cell / kHc, hc = cell - hr * kHc;
        const int gr = r0 - 1 + hr, gc = col0 - 1 + hc, ch = c0 + 8 * j;
        const int64_t o = (((int64_t)b * H + gr) * W + gc) * C + ch;
        const bool ok = gr >= 0 && gr < H && gc >= 0 && gc < W && ch < C && GTR_INB(o + 7, elems, BS_SSWIGLU_LOAD);
        cp16(sbase + idx * 16, v + (ok ? o : 0), ok);
    }
    const uint32_t gbase = (uint32_t)__cvta_generic_to_shared(gtile);
    for (int idx = tid; idx < kRows * kCols * (kCh / 8); idx += kThreads) {
        const int j = idx & 7, cell = idx >> 3;
        const int tr = cell / kCols, tcol = cell - tr * kCols;
        const int gr = r0 + tr, gc = col0 + tcol, ch = c0 + 8 * j;
        const int64_t o = (((int64_t)b * H + gr) * W + gc) * C + ch;
        const bool ok = gr < H && gc < W && ch < C && GTR_INB(o + 7, elems, BS_SSWIGLU_LOAD);
        cp16(gbase + idx * 16, a + (ok ? o : 0), ok);
    }
    asm volatile("cp.async.commit_group;\n" ::: "memory");

    // ---- this thread's channel octet: 9 x 8 taps and the bias (while the tiles land)
    const int j = tid & 7, tc = tid >> 3;
    const int ch = c0 + 8 * j;
    const bool ch_ok = ch < C;
    float w[9][8], bs[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const bool ok = ch_ok && GTR_INB((int64_t)(ch + e) * 9 + 8, (int64_t)C * 9, BS_SSWIGLU_W);
#pragma unroll
        for (int tap = 0; tap < 9; ++tap) w[tap][e] = ok ? __ldg(wc + (int64_t)(ch + e) * 9 + tap) : 0.f;
        bs[e] = (ok && bias) ? __ldg(bias + ch + e) : 0.f;
    }
    asm volatile("cp.async.wait_group 0;\n" ::: "memory");
    __syncthreads();

    // ---- walk down column col0 + tc: window rows (i-1, i, i+1) x columns (tc-1, tc, tc+1) of the halo tile
    const int gc = col0 + tc;
    if (gc >= W || !ch_ok) return;
    auto at = [&](int hr, int hc) { return tile[(hr * kHc + hc) * 8 + j]; };
    uint4 win[3][3];
#pragma unroll
    for (int dy = 0; dy < 2; ++dy)
#pragma unroll
        for (int dx = 0; dx < 3; ++dx) win[dy][dx] = at(dy, tc + dx);
#pragma unroll
    for (int i = 0; i < kRows; ++i) {
        const int gr = r0 + i;
        if (gr >= H) break;
#pragma unroll
        for (int dx = 0; dx < 3; ++dx) win[2][dx] = at(i + 2, tc + dx);
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = bs[e];
#pragma unroll
        for (int dy = 0; dy < 3; ++dy)
#pragma unroll
            for (int dx = 0; dx < 3; ++dx) acc_tap(acc, w[3 * dy + dx], win[dy][dx]);
        const int64_t o = (((int64_t)b * H + gr) * W + gc) * C + ch;
        if (GTR_INB(o + 7, elems, BS_SSWIGLU_OUT)) {
            const uint4 av = gtile[(i * kCols + tc) * 8 + j];
            const __half2 *ah = reinterpret_cast<const __half2 *>(&av);
            uint4 out;
            __half2 *oh = reinterpret_cast<__half2 *>(&out);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __half22float2(ah[e]);
                oh[e] = __floats2half2_rn(silu(f.x) * acc[2 * e], silu(f.y) * acc[2 * e + 1]);
            }
            __stcs(reinterpret_cast<uint4 *>(y + o), out);
        }
#pragma unroll
        for (int dx = 0; dx < 3; ++dx) {
            win[0][dx] = win[1][dx];
            win[1][dx] = win[2][dx];
        }
    }
}

}  // namespace

cudaError_t launch_sswiglu(const __half *a, const __half *v, const float *wc, const float *bias, int B, int H, int W,
                           int C, __half *y, cudaStream_t st) {
    const int64_t tiles = (int64_t)((H + kRows - 1) / kRows) * ((W + kCols - 1) / kCols);
    if (tiles >= ((int64_t)1 << 31) || (C + kCh - 1) / kCh > 65535 || B > 65535) return cudaErrorInvalidConfiguration;
    const dim3 grid((unsigned)tiles, (unsigned)((C + kCh - 1) / kCh), (unsigned)B);
    sswiglu_kernel<<<grid, kThreads, 0, st>>>(a, v, wc, bias, B, H, W, C, y);
    count_launch();
    return cudaGetLastError();
}

}  // namespace gtr
