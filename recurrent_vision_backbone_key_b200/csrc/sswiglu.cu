// sswiglu.cu -- Spatial SwiGLU's gating with its fused 3x3 depthwise
// convolution on the patch grid:
//     y[b][p][c] = silu(a[b][p][c]) * (bias[c] + sum_{dy,dx} w[c][dy+1][dx+1] * v[b][p + dy*W + dx][c])
// with zero padding at the grid border (ai.info summary of GTR, "Methodology
// in Plain English": a 3x3 depthwise convolution inserted in the value branch
// of a SwiGLU block, on the 2-D patch grid; GTR project page, "Spatial
// SwiGLU").  a is the gate branch, v the value branch, both [B][H*W][C] fp16
// in row-major spatial order; y likewise.
//
// HBM-bound (6 bytes per element), so the kernel is built to issue few
// instructions per element and to keep many tiles' loads in flight.  A tile
// is 8 grid rows x 16 grid columns x 32 channels.  Its value block with the
// one-token halo (10 x 18 tokens x 64 bytes) and its gate block (8 x 16
// tokens) are two TMA tile loads of 4-D tensor maps [B][H][W][C], issued by
// one thread; the halo's cells outside the grid and channels past C read as
// zero, so the stencil needs no border tests (the channel coordinate, the
// innermost, is a multiple of 32: 64-byte aligned).  One CTA of 64 threads
// per tile, eight resident per SM (114 registers, 20 KB of shared memory).
// Thread (column pair, channel quad j) keeps its 9 x 4 filter taps in
// registers and walks the tile's 8 rows down its two columns with a 3 x 4
// window held in fp32: each step loads one new row of four 8-byte vectors,
// converts it once, and applies the nine taps to each column with packed
// fp32x2 FMAs (two channels per instruction, fp32 accumulation).  Two
// columns per thread halve the per-thread set-up (taps, addresses) per
// output and share the window's middle columns.  silu takes one
// special-function operation (sigmoid as 1/2 + tanh(x/2)/2 with the hardware
// tanh approximation, whose error is far inside the output's bar).
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "gla_common.cuh"
#include "gla_tcgen05.cuh"

namespace gtr {
namespace {

constexpr int kRows = 8, kCols = 16, kCh = 32;  // tile: grid rows, grid columns, channels
constexpr int kHr = kRows + 2, kHc = kCols + 2; // with the halo
constexpr int kQuads = kCh / 4;                 // 8-byte channel quads per token
constexpr int kThreads = kCols / 2 * kQuads;    // one thread per (column pair, channel quad)

constexpr uint32_t kTileBytes = kHr * kHc * kCh * 2, kGateBytes = kRows * kCols * kCh * 2;

// One 4-D TMA tile load (coordinates innermost first) completing on mbar.
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap *map, int x, int y, int z, int w,
                                            uint32_t mbar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], "
        "[%6];\n" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(mbar)
        : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t mbar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(mbar), "r"(bytes) : "memory");
}

// d = a * b + c on two fp32 lanes at once.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;\n"
        : "=l"(d)
        : "l"(*reinterpret_cast<unsigned long long *>(&a)), "l"(*reinterpret_cast<unsigned long long *>(&b)),
          "l"(*reinterpret_cast<unsigned long long *>(&c)));
    return *reinterpret_cast<float2 *>(&d);
}

// Four fp16 channels (one 8-byte vector) as two fp32 pairs.
struct Quad {
    float2 lo, hi;
};
__device__ __forceinline__ Quad to_quad(uint2 x) {
    Quad q;
    q.lo = __half22float2(*reinterpret_cast<const __half2 *>(&x.x));
    q.hi = __half22float2(*reinterpret_cast<const __half2 *>(&x.y));
    return q;
}

// silu(x) = x * sigmoid(x), sigmoid(x) = 1/2 + tanh(x/2)/2 with the
// hardware tanh approximation (one special-function operation).
__device__ __forceinline__ float silu(float x) {
    float t;
    asm("tanh.approx.f32 %0, %1;\n" : "=f"(t) : "f"(0.5f * x));
    return x * fmaf(0.5f, t, 0.5f);
}

__global__ void __launch_bounds__(kThreads)
    sswiglu_kernel(const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_a,
                   const float *__restrict__ wc, const float *__restrict__ bias, int B, int H, int W, int C,
                   __half *__restrict__ y, unsigned *status) {
    __shared__ __align__(128) uint2 tile[kHr * kHc * kQuads];     // value branch with halo
    __shared__ __align__(128) uint2 gtile[kRows * kCols * kQuads];  // gate branch
    __shared__ __align__(8) uint64_t bar;
    const int tid = threadIdx.x;
    const int c0 = blockIdx.y * kCh;
    const int tiles_w = (W + kCols - 1) / kCols;
    const int r0 = (blockIdx.x / tiles_w) * kRows, col0 = (blockIdx.x % tiles_w) * kCols;
    const int b = blockIdx.z;
    const int64_t elems = (int64_t)B * H * W * C;

    // ---- the value block with its halo and the gate block, one TMA load each
    const uint32_t mbar = (uint32_t)__cvta_generic_to_shared(&bar);
    if (tid == 0) {
        mbar_init(mbar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
        mbar_expect_tx(mbar, kTileBytes + kGateBytes);
        tma_load_4d((uint32_t)__cvta_generic_to_shared(tile), &map_v, c0, col0 - 1, r0 - 1, b, mbar);
        tma_load_4d((uint32_t)__cvta_generic_to_shared(gtile), &map_a, c0, col0, r0, b, mbar);
    }
    __syncthreads();  // the barrier is initialised before anyone waits on it

    // ---- this thread's channel quad: 9 x 4 taps and the bias (while the tiles land)
    const int j = tid % kQuads, tc = 2 * (tid / kQuads);  // first of the thread's two columns
    const int ch = c0 + 4 * j;
    const bool ch_ok = ch < C;  // C is a multiple of 8, so the whole quad
    float2 w[9][2], bs[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float t0[9], t1[9];
        const int e = ch + 2 * h;
        const bool ok = ch_ok && GTR_INB((int64_t)(e + 1) * 9 + 8, (int64_t)C * 9, BS_SSWIGLU_W);
#pragma unroll
        for (int tap = 0; tap < 9; ++tap) {
            t0[tap] = ok ? __ldg(wc + (int64_t)e * 9 + tap) : 0.f;
            t1[tap] = ok ? __ldg(wc + (int64_t)(e + 1) * 9 + tap) : 0.f;
        }
#pragma unroll
        for (int tap = 0; tap < 9; ++tap) w[tap][h] = make_float2(t0[tap], t1[tap]);
        bs[h] = (ok && bias) ? make_float2(__ldg(bias + e), __ldg(bias + e + 1)) : make_float2(0.f, 0.f);
    }
    // ---- the tiles have landed (a wait that gives up records a timeout,
    // waits once more so that no copy is left writing into this CTA's shared
    // memory, and skips the tile)
    if (!mbar_wait(mbar, 0)) {
        if (tid == 0) atomicOr(status, 6u);  // GTR_ERR_TIMEOUT
        mbar_wait(mbar, 0);
        return;
    }

    // ---- walk down columns col0 + tc and col0 + tc + 1: window rows
    // (i-1, i, i+1) x columns (tc-1 .. tc+2) of the halo block, in fp32
    const int gc = col0 + tc;
    if (gc >= W || !ch_ok) return;
    const bool two = gc + 1 < W;
    auto at = [&](int hr, int hc) { return to_quad(tile[(hr * kHc + hc) * kQuads + j]); };
    Quad win[3][4];
#pragma unroll
    for (int dy = 0; dy < 2; ++dy)
#pragma unroll
        for (int dx = 0; dx < 4; ++dx) win[dy][dx] = at(dy, tc + dx);
#pragma unroll
    for (int i = 0; i < kRows; ++i) {
        const int gr = r0 + i;
        if (gr >= H) break;
#pragma unroll
        for (int dx = 0; dx < 4; ++dx) win[2][dx] = at(i + 2, tc + dx);
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            float2 lo = bs[0], hi = bs[1];
#pragma unroll
            for (int dy = 0; dy < 3; ++dy)
#pragma unroll
                for (int dx = 0; dx < 3; ++dx) {
                    lo = ffma2(w[3 * dy + dx][0], win[dy][dx + cc].lo, lo);
                    hi = ffma2(w[3 * dy + dx][1], win[dy][dx + cc].hi, hi);
                }
            const int64_t o = (((int64_t)b * H + gr) * W + gc + cc) * C + ch;
            if ((cc == 0 || two) && GTR_INB(o + 3, elems, BS_SSWIGLU_OUT)) {
                const Quad g = to_quad(gtile[(i * kCols + tc + cc) * kQuads + j]);
                uint2 out;
                *reinterpret_cast<__half2 *>(&out.x) = __floats2half2_rn(silu(g.lo.x) * lo.x, silu(g.lo.y) * lo.y);
                *reinterpret_cast<__half2 *>(&out.y) = __floats2half2_rn(silu(g.hi.x) * hi.x, silu(g.hi.y) * hi.y);
                __stcs(reinterpret_cast<uint2 *>(y + o), out);
            }
        }
#pragma unroll
        for (int dx = 0; dx < 4; ++dx) {
            win[0][dx] = win[1][dx];
            win[1][dx] = win[2][dx];
        }
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled through the driver entry point the runtime hands out
// (no link-time dependency on the driver library); nullptr if unavailable.
EncodeTiledFn encode_tiled() {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
        else
            cudaGetLastError();
    });
    return fn;
}

// Tensor map of a [B][H][W][C] fp16 tensor with a (box_c, box_w, box_h, 1)
// box; cells outside the tensor read as zero.
cudaError_t make_map(CUtensorMap *m, const __half *p, int B, int H, int W, int C, int box_c, int box_w, int box_h) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return cudaErrorNotSupported;
    const cuuint64_t dims[4] = {(cuuint64_t)C, (cuuint64_t)W, (cuuint64_t)H, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)C * 2, (cuuint64_t)W * C * 2, (cuuint64_t)H * W * C * 2};
    const cuuint32_t box[4] = {(cuuint32_t)box_c, (cuuint32_t)box_w, (cuuint32_t)box_h, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, const_cast<__half *>(p), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_sswiglu(const __half *a, const __half *v, const float *wc, const float *bias, int B, int H, int W,
                           int C, __half *y, unsigned *status, cudaStream_t st) {
    const int64_t tiles = (int64_t)((H + kRows - 1) / kRows) * ((W + kCols - 1) / kCols);
    if (tiles >= ((int64_t)1 << 31) || (C + kCh - 1) / kCh > 65535 || B > 65535) return cudaErrorInvalidConfiguration;
    CUtensorMap mv, ma;
    cudaError_t e = make_map(&mv, v, B, H, W, C, kCh, kHc, kHr);
    if (e == cudaSuccess) e = make_map(&ma, a, B, H, W, C, kCh, kCols, kRows);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)tiles, (unsigned)((C + kCh - 1) / kCh), (unsigned)B);
    sswiglu_kernel<<<grid, kThreads, 0, st>>>(mv, ma, wc, bias, B, H, W, C, y, status);
    count_launch();
    return cudaGetLastError();
}

}  // namespace gtr
