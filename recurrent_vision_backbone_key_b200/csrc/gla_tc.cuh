// gla_tc.cuh -- tensor-core chunk kernels of the key-gated GLA mixer.
//
// One kernel template, three modes:
//   SUMMARY : per (sequence, chunk) tile, the decay-weighted chunk summary
//             dS_c (d_k x d_v) and the chunk decay gamma_c (d_k) -- phase 1
//             of the chunkwise operator on the GTR project page ("A Kernel
//             That Makes Recurrence Fast": summaries in parallel over the
//             chunk x head grid);
//   OUTPUT  : per tile, the chunk output from the state entering the chunk
//             (phase 3: the within-chunk score-value product fused with the
//             boundary-state readout);
//   FUSED   : summary, boundary state and output of a tile in one kernel.
//             Tiles are handed out in chunk-major order by an atomic ticket;
//             the state entering chunk c is passed from the tile of chunk c-1
//             of the same sequence through a two-slot ring in L2 with a
//             release/acquire flag (the boundary scan, done as a chain
//             between tiles; the wait is bounded).
//
// Numerics (fp16 tensor-core operands, fp32 accumulation):
//   Inside a chunk the tokens are split into sub-chunks of 16.  With beta_t
//   the inclusive prefix sum of g inside the sub-chunk (per key dimension),
//     qs_t = q~_t exp(beta_t)               (<= |q~_t|)
//     ke_s = k_s exp(beta_end - beta_s)     (<= |k_s|)
//     qe_t = q~_t exp(b_t)                  (b: prefix sum from the chunk start)
//   a local state L runs over the sub-chunks of the chunk from zero,
//     L_{u+1} = diag(exp(beta_end,u)) L_u + ke_u^T V_u,
//   so every factor that meets an fp16 operand is at most one; only the
//   16 x 16 diagonal blocks need exp(beta_t - beta_s) directly.  Those use a
//   reference point in the middle of the sub-chunk (factors within e^{+-R},
//   fp16 tensor-core product) when R <= kDiagRange, and exact per-pair
//   exponentials in fp32 otherwise.  Then
//     o_t = qs_t L_u + sum_{s<=t in u} A_ts v_s + qe_t S_enter,
//     S_leave = diag(exp(b_last)) S_enter + L_last.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "gla_common.cuh"

namespace gtr {

enum TcMode : int { TC_SUMMARY = 0, TC_OUTPUT = 1, TC_FUSED = 2 };

// Largest within-sub-chunk decay (natural-log units, either side of the
// reference point) for which the diagonal block uses fp16 factors.
constexpr float kDiagRange = 6.0f;

struct TcArgs {
    const __half *q, *k, *v;
    const float *g;
    Geom geo;
    float *dS;             // SUMMARY: [nseq][nc][dk][dv]
    float *gamma;          // SUMMARY: [nseq][nc][dk]
    const float *S_enter;  // OUTPUT:  [nseq][nc][dk][dv]
    __half *out;           // OUTPUT / FUSED
    int *ctrl;             // FUSED: [0] ticket, [1] exit count, then nseq flags
    float *ring;           // FUSED: [nseq][2][dk*dv] fragment-ordered states
    unsigned *status;      // FUSED: device status word (GTR_ERR_TIMEOUT on a give-up)
    long long spin_limit;  // FUSED: polls before a wait gives up
    int hold_seq, hold_chunk;  // FUSED test hook: this tile never publishes (-1: off)
};

// ---------------------------------------------------------------- PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, bool full) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(smem)), "l"(gmem),
                 "r"(full ? 16 : 0));
}
__device__ __forceinline__ void cp_async_commit_wait() {
    asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;\n" ::: "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}

// D += A(16x16, row) * B(16x8, col), fp16 in, fp32 accumulate.
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

// 2^x with the MUFU approximation (flushes tiny results to zero).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
    return y;
}
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ int ld_acquire(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];\n" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release(int *p, int v) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;\n" ::"l"(p), "r"(v) : "memory");
}

// ------------------------------------------------------------ smem layout

template <int DK, int DV>
struct TcLayout {
    static constexpr int LDK = DK + 8;  // fp16 row stride (halves): 16-byte rows, conflict-free ldmatrix
    static constexpr int LDV = DV + 8;
    static constexpr int LDA = 24;      // 16x16 diagonal block rows (halves)
    static constexpr int NW = DV / 16;  // warps: one 16-wide value slice each
    static constexpr int NT = NW * 32;
    // byte offsets for a chunk of C tokens
    __host__ __device__ static size_t q(int) { return 0; }
    __host__ __device__ static size_t k(int C) { return q(C) + (size_t)C * LDK * 2; }
    __host__ __device__ static size_t v(int C) { return k(C) + (size_t)C * LDK * 2; }
    __host__ __device__ static size_t g(int C) { return v(C) + (size_t)C * LDV * 2; }
    __host__ __device__ static size_t qd(int C) { return g(C) + (size_t)C * DK * 4; }
    __host__ __device__ static size_t kd(int C) { return qd(C) + (size_t)C * LDK * 2; }
    __host__ __device__ static size_t a(int C) { return kd(C) + (size_t)C * LDK * 2; }
    __host__ __device__ static size_t bend(int C) { return a(C) + (size_t)(C / 16) * 16 * LDA * 2; }
    __host__ __device__ static size_t gu(int C) { return bend(C) + (size_t)(C / 16) * DK * 4; }
    __host__ __device__ static size_t eb(int C) { return gu(C) + (size_t)(C / 16) * DK * 4; }
    __host__ __device__ static size_t gc(int C) { return eb(C) + (size_t)(C / 16) * DK * 4; }
    __host__ __device__ static size_t flags(int C) { return gc(C) + (size_t)DK * 4; }
    // output staging: the qd/kd region when it is large enough, else its own
    __host__ __device__ static bool out_alias(int C) { return (size_t)C * LDV <= (size_t)2 * C * LDK; }
    __host__ __device__ static size_t out(int C) { return out_alias(C) ? qd(C) : flags(C) + 64; }
    __host__ __device__ static size_t bytes(int C) {
        size_t end = flags(C) + 64;
        if (!out_alias(C)) end += (size_t)C * LDV * 2;
        return end;
    }
};

// The last fused tile to finish resets the ticket, the exit count and the
// flags, so the next launch starts from zero without a memset.  Called by
// every thread of a CTA (uniform branch).
__device__ __forceinline__ void fused_finish(const TcArgs &args, int nseq, int *sFlags, int nt) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        sFlags[9] = (atomicAdd(&args.ctrl[1], 1) == (int)gridDim.x - 1);
    }
    __syncthreads();
    if (sFlags[9]) {
        __threadfence();
        for (int i = threadIdx.x; i < nseq; i += nt) args.ctrl[2 + i] = 0;
        if (threadIdx.x == 0) {
            args.ctrl[0] = 0;
            args.ctrl[1] = 0;
        }
    }
}

// --------------------------------------------------------------- the kernel

template <int DK, int DV, int MODE>
__global__ void __launch_bounds__(TcLayout<DK, DV>::NT)
gla_tc_kernel(const TcArgs args) {
    using Lay = TcLayout<DK, DV>;
    constexpr int LDK = Lay::LDK, LDV = Lay::LDV, LDA = Lay::LDA, NT = Lay::NT;
    constexpr int KT = DK / 8;  // 8-wide key tiles of the state
    extern __shared__ __align__(128) unsigned char smem[];
    const Geom &geo = args.geo;
    const int C = geo.chunk;
    const int nsub = C / 16;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    __half *sQ = reinterpret_cast<__half *>(smem + Lay::q(C));
    __half *sK = reinterpret_cast<__half *>(smem + Lay::k(C));
    __half *sV = reinterpret_cast<__half *>(smem + Lay::v(C));
    float *sG = reinterpret_cast<float *>(smem + Lay::g(C));
    __half *sQD = reinterpret_cast<__half *>(smem + Lay::qd(C));
    __half *sKD = reinterpret_cast<__half *>(smem + Lay::kd(C));
    __half *sA = reinterpret_cast<__half *>(smem + Lay::a(C));
    float *sBend = reinterpret_cast<float *>(smem + Lay::bend(C));
    float *sGu = reinterpret_cast<float *>(smem + Lay::gu(C));
    float *sEb = reinterpret_cast<float *>(smem + Lay::eb(C));
    float *sGc = reinterpret_cast<float *>(smem + Lay::gc(C));
    int *sFlags = reinterpret_cast<int *>(smem + Lay::flags(C));  // [0..3] diag range bits, [4..7] overflow, [8] tile
    __half *sOut = reinterpret_cast<__half *>(smem + Lay::out(C));

    // ------------------------------------------------ which tile
    const int nseq = geo.B * geo.heads;
    if (tid < 16 && tid != 8) sFlags[tid] = 0;
    int tile;
    if (MODE == TC_FUSED) {
        if (tid == 0) sFlags[8] = atomicAdd(&args.ctrl[0], 1);
        __syncthreads();
        tile = sFlags[8];
    } else {
        tile = blockIdx.x;
        __syncthreads();
    }
    // A ticket past the grid can only come from control words left behind by
    // an aborted launch: record it and only take part in the reset below.
    if (MODE == TC_FUSED && tile >= geo.nc * nseq) {
        if (tid == 0) atomicOr(args.status, 6u);
        fused_finish(args, nseq, sFlags, NT);
        return;
    }
    // FUSED: chunk-major tickets; other modes: sequence-major blocks
    int c, seq;
    if (MODE == TC_FUSED) {
        c = tile / nseq;
        seq = tile - c * nseq;
    } else {
        seq = tile / geo.nc;
        c = tile - seq * geo.nc;
    }
    const int b = seq / geo.heads, h = seq - b * geo.heads;
    const int t0 = c * C;
    const int len = min(C, geo.N - t0);
    const float qscale = rsqrtf((float)DK);

    // ------------------------------------------------ A: stage the chunk
    {
        constexpr int QCH = DK / 8, VCH = DV / 8, GCH = DK / 4;  // 16-byte pieces per row
        for (int idx = tid; idx < C * (2 * QCH + VCH + GCH); idx += NT) {
            int t, j, which;
            if (idx < C * QCH) { which = 0; t = idx / QCH; j = idx - t * QCH; }
            else if (idx < 2 * C * QCH) { which = 1; int r = idx - C * QCH; t = r / QCH; j = r - t * QCH; }
            else if (idx < C * (2 * QCH + VCH)) { which = 2; int r = idx - 2 * C * QCH; t = r / VCH; j = r - t * VCH; }
            else { which = 3; int r = idx - C * (2 * QCH + VCH); t = r / GCH; j = r - t * GCH; }
            const bool in = t < len;
            const int p = in ? scan_pos(geo.dir, t0 + t, geo.H, geo.W, geo.N) : 0;
            if (MODE == TC_SUMMARY && which == 0) continue;  // q unused
            switch (which) {
            case 0: cp_async16(sQ + t * LDK + j * 8, args.q + tok_offset(geo, b, p, h, DK) + j * 8, in); break;
            case 1: cp_async16(sK + t * LDK + j * 8, args.k + tok_offset(geo, b, p, h, DK) + j * 8, in); break;
            case 2: cp_async16(sV + t * LDV + j * 8, args.v + tok_offset(geo, b, p, h, DV) + j * 8, in); break;
            default: cp_async16(sG + t * DK + j * 4, args.g + tok_offset(geo, b, p, h, DK) + j * 4, in); break;
            }
        }
        cp_async_commit_wait();
        __syncthreads();
    }

    // ------------------------------------------------ B: in-sub-chunk prefix sums (log2 units)
    for (int task = tid; task < DK * nsub; task += NT) {
        const int d = task % DK, u = task / DK;
        float acc = 0.f, b7 = 0.f, b0 = 0.f;
        for (int t = 0; t < 16; ++t) {
            float *p = sG + (16 * u + t) * DK + d;
            acc += *p * kLog2e;
            *p = acc;
            if (t == 0) b0 = acc;
            if (t == 7) b7 = acc;
        }
        sBend[u * DK + d] = acc;
        float r = fmaxf(fmaxf(b0 - b7, b7 - acc), 0.f);  // decay either side of the reference
        atomicMax(&sFlags[u], __float_as_int(r));
    }
    __syncthreads();
    for (int task = tid; task < DK * nsub; task += NT) {
        const int d = task % DK, u = task / DK;
        float base = 0.f, tot = 0.f;
        for (int w = 0; w < nsub; ++w) {
            float be = sBend[w * DK + d];
            if (w < u) base += be;
            tot += be;
        }
        sGu[u * DK + d] = ex2(sBend[u * DK + d]);
        sEb[u * DK + d] = ex2(base);
        if (u == 0) sGc[d] = ex2(tot);
    }
    __syncthreads();

    // ------------------------------------------------ C1: diagonal-block factors
    // qd_t = q~_t 2^(beta_t - beta_7), kd_s = k_s 2^(beta_7 - beta_s) for the
    // sub-chunks whose decay range allows fp16 factors; an fp16 overflow
    // sends that sub-chunk to the exact path as well.
    if (MODE != TC_SUMMARY) {
        for (int task = tid; task < DK * nsub; task += NT) {
            const int d = task % DK, u = task / DK;
            if (!(__int_as_float(sFlags[u]) <= kDiagRange * kLog2e)) continue;
            const float b7 = sG[(16 * u + 7) * DK + d];
            bool ovf = false;
            for (int t = 0; t < 16; ++t) {
                const int row = 16 * u + t;
                const float bt = sG[row * DK + d];
                const __half hq = __float2half_rn(__half2float(sQ[row * LDK + d]) * qscale * ex2(bt - b7));
                const __half hk = __float2half_rn(__half2float(sK[row * LDK + d]) * ex2(b7 - bt));
                ovf |= __hisinf(hq) | __hisinf(hk);
                sQD[row * LDK + d] = hq;
                sKD[row * LDK + d] = hk;
            }
            if (ovf) sFlags[4 + u] = 1;
        }
        __syncthreads();

        // ------------------------------------------------ D: diagonal 16x16 blocks
        for (int u = warp; u < nsub; u += Lay::NW) {
            const bool fast = __int_as_float(sFlags[u]) <= kDiagRange * kLog2e && sFlags[4 + u] == 0;
            __half *Au = sA + u * 16 * LDA;
            if (fast) {
                float acc[2][4] = {};
#pragma unroll
                for (int kk = 0; kk < DK / 16; ++kk) {
                    uint32_t af[4], bf[4];
                    const int r = lane & 7, m = lane >> 3;
                    ldsm_x4(af, sQD + (16 * u + r + 8 * (m & 1)) * LDK + 16 * kk + 8 * (m >> 1));
                    ldsm_x4(bf, sKD + (16 * u + r + 8 * (m >> 1)) * LDK + 16 * kk + 8 * (m & 1));
                    mma16816(acc[0], af, bf[0], bf[1]);
                    mma16816(acc[1], af, bf[2], bf[3]);
                }
                const int tr = lane >> 2, tc = 2 * (lane & 3);
#pragma unroll
                for (int j = 0; j < 2; ++j) {
#pragma unroll
                    for (int hlf = 0; hlf < 2; ++hlf) {
                        const int t = tr + 8 * hlf;
                        const int s0 = 8 * j + tc;
                        const float x0 = (s0 <= t) ? acc[j][2 * hlf] : 0.f;
                        const float x1 = (s0 + 1 <= t) ? acc[j][2 * hlf + 1] : 0.f;
                        *reinterpret_cast<uint32_t *>(Au + t * LDA + s0) = pack_h2(x0, x1);
                    }
                }
            } else {
                // exact: A_ts = sum_d q~_td k_sd 2^(beta_td - beta_sd) from the raw
                // operands; lane -> one query t and eight keys s
                const int t = lane >> 1, sb = 8 * (lane & 1);
                float acc[8] = {};
                for (int d = 0; d < DK; ++d) {
                    const float qv = __half2float(sQ[(16 * u + t) * LDK + d]) * qscale;
                    const float bt = sG[(16 * u + t) * DK + d];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int s = sb + j;
                        if (s <= t) {
                            const float kv = __half2float(sK[(16 * u + s) * LDK + d]);
                            acc[j] = fmaf(qv * kv, ex2(bt - sG[(16 * u + s) * DK + d]), acc[j]);
                        }
                    }
                }
#pragma unroll
                for (int j = 0; j < 8; j += 2)
                    *reinterpret_cast<uint32_t *>(Au + t * LDA + sb + j) = pack_h2(acc[j], acc[j + 1]);
            }
        }
        __syncthreads();
    }

    // ------------------------------------------------ C2: qs, ke in place
    for (int task = tid; task < DK * nsub; task += NT) {
        const int d = task % DK, u = task / DK;
        const float bend = sBend[u * DK + d];
        for (int t = 0; t < 16; ++t) {
            const int row = 16 * u + t;
            const float bt = sG[row * DK + d];
            if (MODE != TC_SUMMARY) {
                const float qv = __half2float(sQ[row * LDK + d]) * qscale;
                sQ[row * LDK + d] = __float2half_rn(qv * ex2(bt));
            }
            const float kv = __half2float(sK[row * LDK + d]);
            sK[row * LDK + d] = __float2half_rn(kv * ex2(bend - bt));
        }
    }
    __syncthreads();
    // qe_t = qs_t 2^(base_u) into the sQD region (the diagonal blocks are done with it)
    if (MODE != TC_SUMMARY) {
        for (int task = tid; task < DK * nsub; task += NT) {
            const int d = task % DK, u = task / DK;
            const float e = sEb[u * DK + d];
            for (int t = 0; t < 16; ++t) {
                const int row = 16 * u + t;
                sQD[row * LDK + d] = __float2half_rn(__half2float(sQ[row * LDK + d]) * e);
            }
        }
        // made visible to every warp by the barrier at the top of phase H
    }

    // ------------------------------------------------ F: local state over sub-chunks
    // Warp w owns value columns [16w, 16w+16).  L^T (16 x DK) lives in the
    // accumulator layout: Lt[n][0..3] covers key columns 8n..8n+7.
    const int v0 = 16 * warp;
    float Lt[KT][4];
#pragma unroll
    for (int n = 0; n < KT; ++n) Lt[n][0] = Lt[n][1] = Lt[n][2] = Lt[n][3] = 0.f;
    float o[4][2][4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int j = 0; j < 2; ++j) o[u][j][0] = o[u][j][1] = o[u][j][2] = o[u][j][3] = 0.f;

    const int r8 = lane & 7, m4 = lane >> 3;
    const int kc = 2 * (lane & 3);  // key column pair inside an 8-wide tile
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        if (u >= nsub) break;
        if (MODE != TC_SUMMARY) {
            // readout of the local state: o_u = qs_u L_u
            if (u > 0) {
#pragma unroll
                for (int kk = 0; kk < DK / 16; ++kk) {
                    uint32_t af[4];
                    ldsm_x4(af, sQ + (16 * u + r8 + 8 * (m4 & 1)) * LDK + 16 * kk + 8 * (m4 >> 1));
                    const uint32_t b00 = pack_h2(Lt[2 * kk][0], Lt[2 * kk][1]);
                    const uint32_t b01 = pack_h2(Lt[2 * kk + 1][0], Lt[2 * kk + 1][1]);
                    const uint32_t b10 = pack_h2(Lt[2 * kk][2], Lt[2 * kk][3]);
                    const uint32_t b11 = pack_h2(Lt[2 * kk + 1][2], Lt[2 * kk + 1][3]);
                    mma16816(o[u][0], af, b00, b01);
                    mma16816(o[u][1], af, b10, b11);
                }
            }
            // diagonal block: o_u += A_uu V_u
            {
                uint32_t af[4], bf[4];
                ldsm_x4(af, sA + u * 16 * LDA + (r8 + 8 * (m4 & 1)) * LDA + 8 * (m4 >> 1));
                ldsm_x4_t(bf, sV + (16 * u + r8 + 8 * (m4 & 1)) * LDV + v0 + 8 * (m4 >> 1));
                mma16816(o[u][0], af, bf[0], bf[1]);
                mma16816(o[u][1], af, bf[2], bf[3]);
            }
        }
        // update: L = diag(gamma_u) L + V_u^T ke_u
        {
            const float *gu = sGu + u * DK;
#pragma unroll
            for (int n = 0; n < KT; ++n) {
                const float g0 = gu[8 * n + kc], g1 = gu[8 * n + kc + 1];
                Lt[n][0] *= g0; Lt[n][1] *= g1; Lt[n][2] *= g0; Lt[n][3] *= g1;
            }
            uint32_t af[4];
            // A = V^T (rows: value columns of this warp, cols: 16 tokens)
            ldsm_x4_t(af, sV + (16 * u + r8 + 8 * (m4 >> 1)) * LDV + v0 + 8 * (m4 & 1));
#pragma unroll
            for (int np = 0; np < KT / 2; ++np) {
                uint32_t bf[4];
                ldsm_x4_t(bf, sK + (16 * u + r8 + 8 * (m4 & 1)) * LDK + 16 * np + 8 * (m4 >> 1));
                mma16816(Lt[2 * np], af, bf[0], bf[1]);
                mma16816(Lt[2 * np + 1], af, bf[2], bf[3]);
            }
        }
    }

    const int64_t sdx = ((int64_t)seq * geo.nc + c);
    if (MODE == TC_SUMMARY) {
        // dS_c[dk][dv] = L^T transposed; gamma_c
        float *dst = args.dS + sdx * DK * DV;
        const int vr = v0 + (lane >> 2);
#pragma unroll
        for (int n = 0; n < KT; ++n) {
            const int kcol = 8 * n + kc;
            dst[(kcol)*DV + vr] = Lt[n][0];
            dst[(kcol + 1) * DV + vr] = Lt[n][1];
            dst[(kcol)*DV + vr + 8] = Lt[n][2];
            dst[(kcol + 1) * DV + vr + 8] = Lt[n][3];
        }
        for (int d = tid; d < DK; d += NT) args.gamma[sdx * DK + d] = sGc[d];
        return;
    }

    // ------------------------------------------------ G: the state entering the chunk
    float Se[KT][4];
    bool have_state = c > 0;
    if (MODE == TC_OUTPUT) {
        const float *src = args.S_enter + sdx * DK * DV;
        const int vr = v0 + (lane >> 2);
#pragma unroll
        for (int n = 0; n < KT; ++n) {
            const int kcol = 8 * n + kc;
            Se[n][0] = src[kcol * DV + vr];
            Se[n][1] = src[(kcol + 1) * DV + vr];
            Se[n][2] = src[kcol * DV + vr + 8];
            Se[n][3] = src[(kcol + 1) * DV + vr + 8];
        }
        have_state = true;
    } else {  // FUSED
        int *flags = args.ctrl + 2;
        if (c > 0) {
            if (tid == 0) {
                long long spins = 0;
                while (ld_acquire(&flags[seq]) < c) {
                    if (++spins > args.spin_limit) {
                        atomicOr(args.status, 6u);  // GTR_ERR_TIMEOUT
                        break;
                    }
                    __nanosleep(spins < 64 ? 32 : 256);
                }
            }
            __syncthreads();
            const float4 *src = reinterpret_cast<const float4 *>(
                args.ring + ((int64_t)seq * 2 + ((c - 1) & 1)) * (DK * DV));
#pragma unroll
            for (int n = 0; n < KT; ++n) {
                float4 x = __ldcg(src + ((warp * KT + n) * 32 + lane));
                Se[n][0] = x.x; Se[n][1] = x.y; Se[n][2] = x.z; Se[n][3] = x.w;
            }
        } else {
#pragma unroll
            for (int n = 0; n < KT; ++n) Se[n][0] = Se[n][1] = Se[n][2] = Se[n][3] = 0.f;
        }
        // publish S_leave = diag(gamma_c) S_enter + L for the next chunk
        const bool hold = (seq == args.hold_seq && c == args.hold_chunk);
        if (c + 1 < geo.nc && !hold) {
            float4 *dst = reinterpret_cast<float4 *>(
                args.ring + ((int64_t)seq * 2 + (c & 1)) * (DK * DV));
#pragma unroll
            for (int n = 0; n < KT; ++n) {
                const float g0 = sGc[8 * n + kc], g1 = sGc[8 * n + kc + 1];
                float4 x;
                x.x = fmaf(g0, Se[n][0], Lt[n][0]);
                x.y = fmaf(g1, Se[n][1], Lt[n][1]);
                x.z = fmaf(g0, Se[n][2], Lt[n][2]);
                x.w = fmaf(g1, Se[n][3], Lt[n][3]);
                __stcg(dst + ((warp * KT + n) * 32 + lane), x);
            }
            __threadfence();
            __syncthreads();
            if (tid == 0) st_release(&flags[seq], c + 1);
        }
    }

    // ------------------------------------------------ H: readout of the entering state
    __syncthreads();  // qe visible to every warp
    if (have_state) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (u >= nsub) break;
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk) {
                uint32_t af[4];
                ldsm_x4(af, sQD + (16 * u + r8 + 8 * (m4 & 1)) * LDK + 16 * kk + 8 * (m4 >> 1));
                const uint32_t b00 = pack_h2(Se[2 * kk][0], Se[2 * kk][1]);
                const uint32_t b01 = pack_h2(Se[2 * kk + 1][0], Se[2 * kk + 1][1]);
                const uint32_t b10 = pack_h2(Se[2 * kk][2], Se[2 * kk][3]);
                const uint32_t b11 = pack_h2(Se[2 * kk + 1][2], Se[2 * kk + 1][3]);
                mma16816(o[u][0], af, b00, b01);
                mma16816(o[u][1], af, b10, b11);
            }
        }
    }

    // ------------------------------------------------ I: store the outputs
    __syncthreads();  // every warp is done reading sQD (the staging may alias it)
    {
        const int tr = lane >> 2;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (u >= nsub) break;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int col = v0 + 8 * j + kc;
                *reinterpret_cast<uint32_t *>(sOut + (16 * u + tr) * LDV + col) = pack_h2(o[u][j][0], o[u][j][1]);
                *reinterpret_cast<uint32_t *>(sOut + (16 * u + tr + 8) * LDV + col) = pack_h2(o[u][j][2], o[u][j][3]);
            }
        }
    }
    __syncthreads();
    {
        constexpr int VCH = DV / 8;
        for (int idx = tid; idx < len * VCH; idx += NT) {
            const int t = idx / VCH, j = idx - t * VCH;
            const int p = scan_pos(geo.dir, t0 + t, geo.H, geo.W, geo.N);
            *reinterpret_cast<int4 *>(args.out + tok_offset(geo, b, p, h, DV) + j * 8) =
                *reinterpret_cast<const int4 *>(sOut + t * LDV + j * 8);
        }
    }

    if (MODE == TC_FUSED) fused_finish(args, nseq, sFlags, NT);
}

// Launch helper used by the per-d_k translation units.
template <int DK, int DV, int MODE>
cudaError_t launch_tc_mode(const TcArgs &a, cudaStream_t st) {
    using Lay = TcLayout<DK, DV>;
    const size_t smem = Lay::bytes(a.geo.chunk);
    cudaError_t e = cudaFuncSetAttribute(gla_tc_kernel<DK, DV, MODE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((int64_t)a.geo.nc * a.geo.B * a.geo.heads);
    gla_tc_kernel<DK, DV, MODE><<<grid, Lay::NT, smem, st>>>(a);
    count_launch();
    return cudaGetLastError();
}

template <int DK, int DV>
cudaError_t launch_tc_dv(const TcArgs &a, int mode, cudaStream_t st) {
    switch (mode) {
    case TC_SUMMARY: return launch_tc_mode<DK, DV, TC_SUMMARY>(a, st);
    case TC_OUTPUT: return launch_tc_mode<DK, DV, TC_OUTPUT>(a, st);
    default: return launch_tc_mode<DK, DV, TC_FUSED>(a, st);
    }
}

template <int DK>
cudaError_t launch_tc_dk(const TcArgs &a, int mode, cudaStream_t st) {
    switch (a.geo.dv) {
    case 16: return launch_tc_dv<DK, 16>(a, mode, st);
    case 32: return launch_tc_dv<DK, 32>(a, mode, st);
    case 64: return launch_tc_dv<DK, 64>(a, mode, st);
    default: return launch_tc_dv<DK, 128>(a, mode, st);
    }
}

size_t tc_smem_bytes(int dk, int dv, int chunk);
cudaError_t launch_tc(const TcArgs &a, int mode, cudaStream_t st);

}  // namespace gtr
