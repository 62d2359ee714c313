// gla_phases_simt.cu -- the three-phase chunkwise schedule on CUDA cores.
//
// GTR project page, "A Kernel That Makes Recurrence Fast": per-chunk
// summaries in parallel over the chunk x head grid, a light coalesced scan
// of the boundary states, then an output kernel fusing the within-chunk
// score-value product with the boundary-state readout.  This file is the
// plain-FP32 CUDA-core version of those three phases: every decay factor is
// exp() of a difference of in-chunk prefix sums, so it is safe for any gate
// values.  It is the straightforward schedule the tensor-core kernels are
// checked and timed against.
#include <algorithm>

#include "gla_common.cuh"

namespace gtr {

namespace {

constexpr int kThreads = 256;

// Loads one chunk of a [B][N][heads][d] fp16 tensor into fp32 shared memory
// rows of stride `ld`, visiting tokens in scan order; rows past N are zero.
__device__ void load_rows_h(const __half *src, const Geom &g, int b, int h, int t0, int len,
                            int d, float *dst, int ld) {
    for (int idx = threadIdx.x; idx < g.chunk * d; idx += blockDim.x) {
        int t = idx / d, i = idx - t * d;
        float x = 0.f;
        if (t < len) {
            int p = scan_pos(g.dir, t0 + t, g.H, g.W, g.N);
            const int64_t o = tok_offset(g, b, p, h, d) + i;
            if (GTR_INB(o, (int64_t)g.B * g.N * g.heads * d, BS_SIMT_LOAD)) x = __half2float(src[o]);
        }
        dst[t * ld + i] = x;
    }
}

__device__ void load_rows_f(const float *src, const Geom &g, int b, int h, int t0, int len, int d,
                            float *dst, int ld) {
    for (int idx = threadIdx.x; idx < g.chunk * d; idx += blockDim.x) {
        int t = idx / d, i = idx - t * d;
        float x = 0.f;
        if (t < len) {
            int p = scan_pos(g.dir, t0 + t, g.H, g.W, g.N);
            const int64_t o = tok_offset(g, b, p, h, d) + i;
            if (GTR_INB(o, (int64_t)g.B * g.N * g.heads * d, BS_SIMT_LOAD)) x = src[o];
        }
        dst[t * ld + i] = x;
    }
}

// In-place inclusive prefix sum over the chunk's tokens, one thread per key
// dimension.
__device__ void prefix_rows(float *bs, int ld, int len, int dk) {
    for (int i = threadIdx.x; i < dk; i += blockDim.x) {
        float acc = 0.f;
        for (int t = 0; t < len; ++t) {
            acc += bs[t * ld + i];
            bs[t * ld + i] = acc;
        }
    }
}

// Phase 1: gamma_c = exp(b_last), dS_c = sum_s exp(b_last - b_s) k_s^T v_s.
__global__ void __launch_bounds__(kThreads) summary_simt_kernel(
    const __half *__restrict__ k, const __half *__restrict__ v, const float *__restrict__ gl,
    Geom g, float *__restrict__ dS, float *__restrict__ gamma) {
    extern __shared__ float sm[];
    const int c = (int)(blockIdx.x % (unsigned)g.nc);
    const int seq_i = (int)(blockIdx.x / (unsigned)g.nc);
    const int h = seq_i % g.heads, b = seq_i / g.heads;
    const int C = g.chunk, dk = g.dk, dv = g.dv, ldk = dk + 1;
    float *kw = sm;               // [C][dk+1]
    float *bs = kw + C * ldk;     // [C][dk+1]
    float *vv = bs + C * ldk;     // [C][dv]
    const int t0 = c * C;
    const int len = min(C, g.N - t0);
    load_rows_h(k, g, b, h, t0, len, dk, kw, ldk);
    load_rows_f(gl, g, b, h, t0, len, dk, bs, ldk);
    load_rows_h(v, g, b, h, t0, len, dv, vv, dv);
    __syncthreads();
    prefix_rows(bs, ldk, len, dk);
    __syncthreads();
    const int64_t seq = (int64_t)b * g.heads + h;
    if (!GTR_INB(seq * g.nc + c, (int64_t)g.B * g.heads * g.nc, BS_SIMT_SUMMARY)) return;
    for (int idx = threadIdx.x; idx < len * dk; idx += blockDim.x) {
        int t = idx / dk, i = idx - t * dk;
        kw[t * ldk + i] *= expf(bs[(len - 1) * ldk + i] - bs[t * ldk + i]);
    }
    for (int i = threadIdx.x; i < dk; i += blockDim.x)
        gamma[(seq * g.nc + c) * dk + i] = expf(bs[(len - 1) * ldk + i]);
    __syncthreads();
    float *out = dS + (seq * g.nc + c) * (int64_t)dk * dv;
    for (int e = threadIdx.x; e < dk * dv; e += blockDim.x) {
        int i = e / dv, j = e - i * dv;
        float acc = 0.f;
        for (int t = 0; t < len; ++t) acc = fmaf(kw[t * ldk + i], vv[t * dv + j], acc);
        out[e] = acc;
    }
}

// Phase 2: one thread per state element, serial over chunks; consecutive
// threads own consecutive elements, so every step is one coalesced sweep.
// The loads do not depend on the running state, so they are issued kAhead
// chunks ahead of their use and only the fma chain is serial.  In place is
// allowed: element e of chunk c is read (kAhead steps early) before step c
// writes it, and no step writes an element a later prefetch reads.
constexpr int kAhead = 8;
__global__ void __launch_bounds__(kThreads) scan_simt_kernel(
    const float *dS, const float *__restrict__ gamma, int nseq, int nc, int dk, int dv, float *S_enter) {
    const int per_seq = (dk * dv + blockDim.x - 1) / blockDim.x;
    const int64_t seq = blockIdx.x / per_seq;
    const int e = (blockIdx.x % per_seq) * blockDim.x + threadIdx.x;
    if (e >= dk * dv) return;
    if (!GTR_INB(seq, nseq, BS_SIMT_SCAN)) return;
    const int i = e / dv;
    const int64_t stride = (int64_t)dk * dv;
    const float *src = dS + seq * nc * stride + e;
    const float *gm = gamma + seq * nc * dk + i;
    float *dst = S_enter + seq * nc * stride + e;
    float xs[kAhead], as[kAhead];
#pragma unroll
    for (int u = 0; u < kAhead; ++u) {
        xs[u] = u < nc ? src[u * stride] : 0.f;
        as[u] = u < nc ? gm[(int64_t)u * dk] : 0.f;
    }
    float S = 0.f;
    for (int c0 = 0; c0 < nc; c0 += kAhead) {
#pragma unroll
        for (int u = 0; u < kAhead; ++u) {
            const int c = c0 + u;
            if (c < nc) {
                const float x = xs[u], a = as[u];
                if (c + kAhead < nc) {  // chunk c + kAhead, read before anything writes it
                    xs[u] = src[(c + kAhead) * stride];
                    as[u] = gm[(int64_t)(c + kAhead) * dk];
                }
                dst[c * stride] = S;
                S = fmaf(a, S, x);
            }
        }
    }
}

// The same scan in two passes over segments of each sequence's chunks, with
// four state elements (one float4, one key row) per thread: more independent
// work for problems with few state elements and long chains.
//   pass 1 (APPLY = false): the aggregate of segment s, the state leaving it
//     from zero and the product of its gates, D_s and Gam_s;
//   pass 2 (APPLY = true): the state entering segment s from the aggregates
//     of segments 0..s-1, then the segment's chunks again, writing S_enter.
// Pass 1 only reads dS; pass 2 reads each element before it writes it, so
// S_enter may be dS.  Aggregates: [seq][nseg - 1][d_k*d_v (D) + d_k (Gam)].
// dS and S_enter are fp32 or fp16 (T); the running state and the aggregates
// are fp32.
__device__ __forceinline__ float4 load4(const float *p, int64_t i4) { return reinterpret_cast<const float4 *>(p)[i4]; }
__device__ __forceinline__ float4 load4(const __half *p, int64_t i4) {
    const uint2 u = reinterpret_cast<const uint2 *>(p)[i4];
    const float2 a = __half22float2(*reinterpret_cast<const __half2 *>(&u.x));
    const float2 b = __half22float2(*reinterpret_cast<const __half2 *>(&u.y));
    return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ void store4(float *p, int64_t i4, float4 x) { reinterpret_cast<float4 *>(p)[i4] = x; }
__device__ __forceinline__ void store4(__half *p, int64_t i4, float4 x) {
    uint2 u;
    *reinterpret_cast<__half2 *>(&u.x) = __floats2half2_rn(x.x, x.y);
    *reinterpret_cast<__half2 *>(&u.y) = __floats2half2_rn(x.z, x.w);
    reinterpret_cast<uint2 *>(p)[i4] = u;
}
template <bool APPLY, typename T>
__global__ void __launch_bounds__(kThreads) scan_seg_kernel(const T *dS, const float *__restrict__ gamma,
                                                            int nseq, int nc, int dk, int dv, int L, int nseg,
                                                            float *agg, T *S_enter) {
    // launched programmatically after the summary (or pass 1): let the next
    // grid start, then wait for the one ahead before reading its results
    grid_dep_launch();
    grid_dep_wait();
    const int n4 = dk * dv / 4;
    const int per = (n4 + blockDim.x - 1) / blockDim.x;
    const int segs = APPLY ? nseg : nseg - 1;
    const int64_t ss = blockIdx.x / per;
    const int e4 = (int)(blockIdx.x % per) * blockDim.x + threadIdx.x;
    if (e4 >= n4) return;
    const int64_t seq = ss / segs;
    const int seg = (int)(ss - seq * segs);
    if (!GTR_INB(seq, nseq, BS_SIMT_SCAN)) return;
    const int i = (4 * e4) / dv;  // the key row of the four elements
    const int64_t aggstride = (int64_t)dk * dv + dk;
    const int c0 = seg * L, c1 = min(nc, c0 + L);
    float4 S = make_float4(0.f, 0.f, 0.f, 0.f);
    if (APPLY) {
        const float *ab = agg + seq * (nseg - 1) * aggstride;
        for (int s = 0; s < seg; ++s) {
            const float4 D = reinterpret_cast<const float4 *>(ab + s * aggstride)[e4];
            const float G = ab[s * aggstride + (int64_t)dk * dv + i];
            S = make_float4(fmaf(G, S.x, D.x), fmaf(G, S.y, D.y), fmaf(G, S.z, D.z), fmaf(G, S.w, D.w));
        }
    }
    const int64_t base4 = seq * nc * (int64_t)n4 + e4;  // element quad e4 of the sequence's chunk 0
    const float *gm = gamma + seq * nc * dk + i;
    float4 xs[kAhead];
    float as[kAhead];
#pragma unroll
    for (int u = 0; u < kAhead; ++u) {
        xs[u] = c0 + u < c1 ? load4(dS, base4 + (int64_t)(c0 + u) * n4) : make_float4(0.f, 0.f, 0.f, 0.f);
        as[u] = c0 + u < c1 ? gm[(int64_t)(c0 + u) * dk] : 0.f;
    }
    float G = 1.f;
    for (int b = c0; b < c1; b += kAhead) {
#pragma unroll
        for (int u = 0; u < kAhead; ++u) {
            const int c = b + u;
            if (c < c1) {
                const float4 x = xs[u];
                const float a = as[u];
                if (c + kAhead < c1) {  // chunk c + kAhead, read before anything writes it
                    xs[u] = load4(dS, base4 + (int64_t)(c + kAhead) * n4);
                    as[u] = gm[(int64_t)(c + kAhead) * dk];
                }
                if (APPLY) store4(S_enter, base4 + (int64_t)c * n4, S);
                S = make_float4(fmaf(a, S.x, x.x), fmaf(a, S.y, x.y), fmaf(a, S.z, x.z), fmaf(a, S.w, x.w));
                if (!APPLY) G *= a;
            }
        }
    }
    if (!APPLY) {
        float *ab = agg + (seq * (nseg - 1) + seg) * aggstride;
        reinterpret_cast<float4 *>(ab)[e4] = S;
        if ((4 * e4) % dv == 0) ab[(int64_t)dk * dv + i] = G;
    }
}

// Phase 3: intra-chunk scores A[t][s] = sum_i q~_t[i] k_s[i] exp(b_t[i]-b_s[i])
// for s <= t, then o_t = (q~_t * exp(b_t)) S_enter + sum_s A[t][s] v_s.
__global__ void __launch_bounds__(kThreads) output_simt_kernel(
    const __half *__restrict__ q, const __half *__restrict__ k, const __half *__restrict__ v,
    const float *__restrict__ gl, const float *__restrict__ S_enter, Geom g,
    __half *__restrict__ out) {
    extern __shared__ float sm[];
    const int c = (int)(blockIdx.x % (unsigned)g.nc);
    const int seq_i = (int)(blockIdx.x / (unsigned)g.nc);
    const int h = seq_i % g.heads, b = seq_i / g.heads;
    const int C = g.chunk, dk = g.dk, dv = g.dv, ldk = dk + 1;
    float *qs = sm;               // [C][dk+1]
    float *ks = qs + C * ldk;     // [C][dk+1]
    float *bs = ks + C * ldk;     // [C][dk+1]
    float *vv = bs + C * ldk;     // [C][dv]
    float *A = vv + C * dv;       // [C][C]
    float *S = A + C * C;         // [dk][dv]
    const int t0 = c * C;
    const int len = min(C, g.N - t0);
    const float scale = rsqrtf((float)dk);
    load_rows_h(q, g, b, h, t0, len, dk, qs, ldk);
    load_rows_h(k, g, b, h, t0, len, dk, ks, ldk);
    load_rows_f(gl, g, b, h, t0, len, dk, bs, ldk);
    load_rows_h(v, g, b, h, t0, len, dv, vv, dv);
    const int64_t seq = (int64_t)b * g.heads + h;
    const bool s_ok = GTR_INB(seq * g.nc + c, (int64_t)g.B * g.heads * g.nc, BS_SIMT_SENTER);
    const float *Sg = S_enter + (s_ok ? seq * g.nc + c : 0) * (int64_t)dk * dv;
    for (int e = threadIdx.x; e < dk * dv; e += blockDim.x) S[e] = s_ok ? Sg[e] : 0.f;
    __syncthreads();
    prefix_rows(bs, ldk, len, dk);
    for (int idx = threadIdx.x; idx < C * dk; idx += blockDim.x) {
        int t = idx / dk, i = idx - t * dk;
        qs[t * ldk + i] *= scale;
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < C * C; idx += blockDim.x) {
        int t = idx / C, s = idx - t * C;
        float a = 0.f;
        if (s <= t && t < len) {
            for (int i = 0; i < dk; ++i)
                a = fmaf(qs[t * ldk + i] * ks[s * ldk + i], expf(bs[t * ldk + i] - bs[s * ldk + i]), a);
        }
        A[idx] = a;
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < C * dk; idx += blockDim.x) {
        int t = idx / dk, i = idx - t * dk;
        qs[t * ldk + i] *= expf(bs[t * ldk + i]);
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < len * dv; idx += blockDim.x) {
        int t = idx / dv, j = idx - t * dv;
        float acc = 0.f;
        for (int i = 0; i < dk; ++i) acc = fmaf(qs[t * ldk + i], S[i * dv + j], acc);
        for (int s = 0; s <= t; ++s) acc = fmaf(A[t * C + s], vv[s * dv + j], acc);
        int p = scan_pos(g.dir, t0 + t, g.H, g.W, g.N);
        const int64_t o = tok_offset(g, b, p, h, dv) + j;
        if (GTR_INB(o, (int64_t)g.B * g.N * g.heads * dv, BS_SIMT_OUT)) out[o] = __float2half_rn(acc);
    }
}

size_t summary_smem(const Geom &g) { return sizeof(float) * (size_t)g.chunk * (2 * (g.dk + 1) + g.dv); }
size_t output_smem(const Geom &g) {
    return sizeof(float) * ((size_t)g.chunk * (3 * (g.dk + 1) + g.dv + g.chunk) + (size_t)g.dk * g.dv);
}

}  // namespace

cudaError_t launch_summary_v0(const __half *k, const __half *v, const float *g, const Geom &geo,
                              float *dS, float *gamma, cudaStream_t st) {
    size_t smem = summary_smem(geo);
    cudaError_t e = cudaFuncSetAttribute(summary_simt_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((int64_t)geo.nc * geo.B * geo.heads));
    summary_simt_kernel<<<grid, kThreads, smem, st>>>(k, v, g, geo, dS, gamma);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_scan_v0(const float *dS, const float *gamma, int nseq, int nc, int dk, int dv,
                           float *S_enter, cudaStream_t st) {
    dim3 grid((unsigned)((int64_t)((dk * dv + kThreads - 1) / kThreads) * nseq));
    scan_simt_kernel<<<grid, kThreads, 0, st>>>(dS, gamma, nseq, nc, dk, dv, S_enter);
    count_launch();
    return cudaGetLastError();
}

int scan_segments(int64_t nseq, int nc, int dk, int dv) {
    // as many segments as keep every thread (four elements each) resident at
    // once on a B200 (about 105k threads at this kernel's register count),
    // each segment at least 8 chunks long; chains under 32 chunks are not
    // worth the second launch
    const int64_t threads = nseq * (int64_t)dk * dv / 4;
    if (nc < 32) return 1;
    int64_t nseg = threads > 0 ? 105000 / threads : 1;
    nseg = std::min<int64_t>(nseg, std::max(1, nc / 8));
    return (int)std::max<int64_t>(1, nseg);
}

size_t scan_agg_bytes(int64_t nseq, int nc, int dk, int dv) {
    return (size_t)nseq * (scan_segments(nseq, nc, dk, dv) - 1) * ((size_t)dk * dv + dk) * sizeof(float);
}

template <typename T>
cudaError_t launch_scan_segmented_t(const T *dS, const float *gamma, int nseq, int nc, int dk, int dv, T *S_enter,
                                    float *agg, cudaStream_t st, bool pdl) {
    const int nseg = scan_segments(nseq, nc, dk, dv);
    const int L = (nc + nseg - 1) / nseg;
    const int64_t per = ((int64_t)dk * dv / 4 + kThreads - 1) / kThreads;
    if (nseg > 1) {
        cudaError_t e = launch_kernel(scan_seg_kernel<false, T>, dim3((unsigned)(nseq * (int64_t)(nseg - 1) * per)),
                                      dim3(kThreads), 0, st, pdl, dS, gamma, nseq, nc, dk, dv, L, nseg, agg, S_enter);
        count_launch();
        if (e != cudaSuccess) return e;
    }
    cudaError_t e = launch_kernel(scan_seg_kernel<true, T>, dim3((unsigned)(nseq * (int64_t)nseg * per)), dim3(kThreads),
                                  0, st, pdl, dS, gamma, nseq, nc, dk, dv, L, nseg, agg, S_enter);
    count_launch();
    return e;
}

cudaError_t launch_scan_segmented(const float *dS, const float *gamma, int nseq, int nc, int dk, int dv,
                                  float *S_enter, float *agg, cudaStream_t st, bool pdl) {
    return launch_scan_segmented_t(dS, gamma, nseq, nc, dk, dv, S_enter, agg, st, pdl);
}
cudaError_t launch_scan_segmented(const __half *dS, const float *gamma, int nseq, int nc, int dk, int dv,
                                  __half *S_enter, float *agg, cudaStream_t st, bool pdl) {
    return launch_scan_segmented_t(dS, gamma, nseq, nc, dk, dv, S_enter, agg, st, pdl);
}

cudaError_t launch_output_v0(const __half *q, const __half *k, const __half *v, const float *g,
                             const float *S_enter, const Geom &geo, __half *out, cudaStream_t st) {
    size_t smem = output_smem(geo);
    cudaError_t e = cudaFuncSetAttribute(output_simt_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((int64_t)geo.nc * geo.B * geo.heads));
    output_simt_kernel<<<grid, kThreads, smem, st>>>(q, k, v, g, S_enter, geo, out);
    count_launch();
    return cudaGetLastError();
}

}  // namespace gtr
