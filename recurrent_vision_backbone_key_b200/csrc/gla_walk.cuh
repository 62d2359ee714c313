// gla_walk.cuh -- the GLA forward walked chunk by chunk on the tcgen05 tensor
// cores, one CTA per (sequence, 64-wide value slice), chunks of 64 tokens.
//
// The recurrence S_t = diag(exp g_t) S_{t-1} + k_t^T v_t splits by value
// column: a slice of 64 value columns of S evolves on its own (ai.info summary
// of GTR, "Methodology in Plain English": key-only gating, value-side decay
// fixed at one).  So a CTA owns a value slice of one sequence and keeps that
// slice of the state in registers while it walks the sequence's chunks in
// scan order; no state ever leaves the CTA and no CTA waits for another.
// Per chunk, with a_t = exp(g_t), E_t = a_0..a_t, Suf_t = a_{t+1}..a_63 and
// gamma = E_63 (the chunk's total decay, per key dimension):
//     ke_s = k_s Suf_s                  qh_t = q~_t E_t / gamma
//     A    = qh ke^T                    (A_ts = sum_d q~_td k_sd exp(b_td - b_sd))
//     dS^T = V^T ke                     (the chunk summary of this value slice)
//     O    = tril(A) V + qh (gamma . S_enter)
//     S_leave = diag(gamma) S_enter + dS
// -- the chunk summary, the step of the boundary scan and the output product
// fused with the boundary readout of the GTR project page ("A Kernel That
// Makes Recurrence Fast"), here run back to back inside one CTA.  Chunks
// whose decay exceeds kChunkRange nats in some key dimension (or with
// |q~| > 16) keep the safe operand qe_t = q~_t E_t and compute the score
// matrix exactly on CUDA cores.
//
// Modes (one kernel template):
//   WALK_SEQ     : item = (sequence, value slice), all chunks, state from zero
//                  or from a given S_0, optional final state S_N;
//   WALK_SUMMARY : item = (sequence, chunk, value slice): dS_c and gamma_c only
//                  (phase 1 of the three-phase schedule);
//   WALK_OUTPUT  : item = (sequence, chunk, value slice): the chunk's outputs
//                  from a given entering state (phase 3).
// A CTA takes items blockIdx.x, blockIdx.x + gridDim.x, ... and walks their
// chunks as one stream: the q, k, v rows (and g for d_k = 128) of the next
// chunk but one are loaded by cp.async into a second stage while the current
// chunk is computed; g (d_k <= 64) is prefetched into registers one chunk
// ahead.
//
// Shared-memory tiles use the 128-byte swizzled canonical layout (16-byte
// chunk j of a 128-byte row r at chunk j ^ (r mod 8)); a row of d_k = 128
// halves is split into two 64-column halves, each a 64 x 128-byte tile.
// d_k = 32 uses 128-byte rows of which the MMAs read the first 64 bytes.
// Accumulators (M = 64) take TMEM lanes 0-15 (A, then O) and 16-31 (dS^T) of
// each 32-lane group; warp w reads rows 16w..16w+15 in the m16n8 fragment
// layout and owns value rows 16w..16w+15 of the state slice.
#pragma once

#include <cuda_bf16.h>

#include "gla_tc.cuh"
#include "gla_tcgen05.cuh"

namespace gtr {

// Element type of q, k, v, the gate and the output (fp16 or bf16): the
// tensor-core operands (q, k, v, the masked scores P and the scaled state S')
// are in this type, accumulation and the state stay fp32.
template <typename T>
struct IoType;
template <>
struct IoType<__half> {
    using T2 = __half2;
    static constexpr int kBf16 = 0;
    static __device__ __forceinline__ T2 from_f2(float x, float y) { return __floats2half2_rn(x, y); }
    static __device__ __forceinline__ float2 to_f2(T2 x) { return __half22float2(x); }
    static __device__ __forceinline__ float to_f(__half x) { return __half2float(x); }
    static __device__ __forceinline__ __half zero() { return __float2half(0.f); }
};
template <>
struct IoType<__nv_bfloat16> {
    using T2 = __nv_bfloat162;
    static constexpr int kBf16 = 1;
    static __device__ __forceinline__ T2 from_f2(float x, float y) { return __floats2bfloat162_rn(x, y); }
    static __device__ __forceinline__ float2 to_f2(T2 x) { return __bfloat1622float2(x); }
    static __device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
    static __device__ __forceinline__ __nv_bfloat16 zero() { return __float2bfloat16(0.f); }
};
template <typename T>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    typename IoType<T>::T2 h = IoType<T>::from_f2(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

enum WalkMode : int { WALK_SEQ = 0, WALK_SUMMARY = 1, WALK_OUTPUT = 2 };

// silu(x) = x * sigmoid(x), sigmoid(x) = 1/2 + tanh(x/2)/2 with the hardware
// tanh approximation: one special-function operation.
__device__ __forceinline__ float silu_tanh(float x) {
    float t;
    asm("tanh.approx.f32 %0, %1;\n" : "=f"(t) : "f"(0.5f * x));
    return x * fmaf(0.5f, t, 0.5f);
}

// Largest total decay over a chunk (nats) for the whole-chunk tensor-core form.
constexpr float kWalkChunkRange = 8.0f;

struct WalkArgs {
    const void *q, *k, *v; // fp16 or bf16 (the kernel's element type)
    const float *g;
    Geom geo;
    void *out;             // SEQ, OUTPUT
    const float *S0;       // SEQ: initial state [nseq][dk][dv] fp32, or null for zero
    float *SN;             // SEQ: final state [nseq][dk][dv] fp32, or null
    float *dS;             // SUMMARY: [nseq][nc][dk][dv]
    float *gamma;          // SUMMARY: [nseq][nc][dk]
    const float *S_enter;  // OUTPUT: [nseq][nc][dk][dv]
    unsigned *status;      // GTR_ERR_TIMEOUT if a wait for tensor-core work gave up
    int vs;                // 64-wide value slices per sequence (d_v / 64)
    int items;             // SEQ: nseq * vs; SUMMARY, OUTPUT: nseq * nc * vs
    // gated output (d_v = 64): out = o / sqrt(mean(o^2) + eps) * w * silu(gate)
    const void *gate;      // [B][N][heads][d_v] gate pre-activation (element type)
    const float *norm_w;   // [d_v] RMS-norm weight
    float norm_eps;
    bool pdl;              // host side: launched with programmatic stream serialization
};

template <int DK>
struct WalkLayout {
    static constexpr bool kGsmem = DK > 64;             // g staged in shared memory (else registers)
    static constexpr int KW = DK < 64 ? 64 : DK;        // q/k tile columns in shared memory
    static constexpr uint32_t TQK = 64u * KW * 2u;      // one q or k tile
    static constexpr uint32_t SQ = 0, SK = TQK, SV = 2 * TQK, SG = 2 * TQK + 8192;
    static constexpr uint32_t STAGE = SG + (kGsmem ? 64u * DK * 4u : 0u);
    static constexpr uint32_t P = 2 * STAGE;            // masked scores, then output staging, exact-path scratch
    static constexpr uint32_t SP = P + 8192;            // (scale . S_enter)^T: 64 value rows x DK, K-major
    static constexpr uint32_t TOT = SP + TQK;           // sub-chunk decay totals [4][DK] fp32
    static constexpr uint32_t GAM = TOT + 4u * DK * 4u; // gamma [DK] fp32
    static constexpr uint32_t ROW = GAM + DK * 4u;      // token-head rows [2 stages][64] int64
    static constexpr uint32_t MISC = ROW + 2u * 64u * 8u;  // tmem base, two mbarriers
    static constexpr uint32_t BYTES = MISC + 64;
    static constexpr uint32_t ALLOC = BYTES + 1024;     // slack for aligning the base to 1024
    static constexpr uint32_t TMEM_COLS = 128u;  // A | O (lanes 0-15), dS^T (lanes 16-31)
    static constexpr int MIN_CTAS = kGsmem ? 1 : 3;
};

// Byte offset of element (row, col) of a 64-row fp16 tile whose rows are
// split in 64-column halves of 128 bytes, 128-byte swizzle.
__device__ __forceinline__ uint32_t swz(int row, int col) {
    return (uint32_t)((col >> 6) * 8192) + sw128(row, col & 63);
}

// GATED (WALK_SEQ, d_v = 64): the output store applies the output gate on
// the RMS-normalised output (ai.info summary, "Methodology in Plain English"):
// out = o / sqrt(mean over the head's d_v values of o^2 + eps) * w * silu(gate).
template <int DK, int MODE, bool GATED, typename T>
__global__ void __launch_bounds__(128, WalkLayout<DK>::MIN_CTAS) gla_walk_kernel(const WalkArgs args) {
    using IO = IoType<T>;
    using T2 = typename IO::T2;
    const T *gq_ = static_cast<const T *>(args.q), *gk_ = static_cast<const T *>(args.k);
    const T *gv_ = static_cast<const T *>(args.v);
    T *gout_ = static_cast<T *>(args.out);
    using L = WalkLayout<DK>;
    constexpr int KT = DK / 8;           // 8-wide key tiles of the state fragment
    constexpr int PPL = DK > 64 ? 2 : 1; // key-dimension pairs per lane in the prep
    constexpr int DV_CTA = 64;
    constexpr bool kOut = MODE != WALK_SUMMARY;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base_addr = (raw_addr + 1023u) & ~1023u;
    unsigned char *base = smem_raw + (base_addr - raw_addr);
    const Geom &geo = args.geo;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tr = lane >> 2, kc = 2 * (lane & 3);
    float *sTot = reinterpret_cast<float *>(base + L::TOT);
    float *sGam = reinterpret_cast<float *>(base + L::GAM);
    int64_t *sRow = reinterpret_cast<int64_t *>(base + L::ROW);  // [stage][64]
    int *misc = reinterpret_cast<int *>(base + L::MISC);
    const uint32_t mbar1 = base_addr + L::MISC + 8, mbar2 = base_addr + L::MISC + 16;
    const int nseq = geo.B * geo.heads;
    const int64_t rows = (int64_t)geo.B * geo.N * geo.heads;  // token-head rows of every tensor
    const int DV = geo.dv;
    const float qscale = rsqrtf((float)DK);
    // the prep's lane map: lane -> key-dimension pair (2 dpair, 2 dpair + 1)
    // of each 64-column half, over TPL of the warp's 16 tokens from tb; at
    // d_k = 32 (16 pairs) the two half-warps take 8 tokens each, so that
    // every lane works
    constexpr bool kSplit = DK == 32;
    constexpr int TPL = kSplit ? 8 : 16;
    const int dpair = kSplit ? (lane & 15) : lane;
    const int tb = kSplit ? 8 * (lane >> 4) : 0;
    const bool lane_on = DK >= 64 || kSplit || lane < 16;  // lanes with key dimensions in the prep

    // ---- the CTA's stream of chunk steps: (item, chunk)
    auto first_chunk = [&](int it) { return MODE == WALK_SEQ ? 0 : (it / args.vs) % geo.nc; };
    auto last_chunk = [&](int it) { return MODE == WALK_SEQ ? geo.nc - 1 : (it / args.vs) % geo.nc; };
    auto seq_of = [&](int it) { return MODE == WALK_SEQ ? it / args.vs : (it / args.vs) / geo.nc; };
    auto next_step = [&](int &it, int &c) {
        if (c < last_chunk(it)) {
            ++c;
        } else {
            it += gridDim.x;
            c = it < args.items ? first_chunk(it) : 0;
        }
    };

    // ---- loads of one step into a stage, each warp its own 16 rows: lanes
    // 0-15 compute the rows of tokens 16w..16w+15, then lane l copies half
    // of the 16-byte pieces of row 16w + l/2 of every tensor
    auto issue_loads = [&](int it, int c, int stage) {
        int64_t *rowt = sRow + stage * 64;
        const uint32_t sb = base_addr + (uint32_t)stage * L::STAGE;
        if (it < args.items) {
            const int seq = seq_of(it), sl = it % args.vs;
            const int b = seq / geo.heads, h = seq - b * geo.heads;
            const int t0 = c * 64, len = min(64, geo.N - t0);
            int64_t r_own = -1;
            if (lane < 16) {
                const int t = 16 * warp + lane;
                if (t < len)
                    r_own = ((int64_t)b * geo.N + scan_pos(geo.dir, t0 + t, geo.H, geo.W, geo.N)) * geo.heads + h;
                if (r_own >= 0 && !GTR_INB(r_own, rows, BS_WALK_ROW)) r_own = -1;
                rowt[t] = r_own;
            }
            // consecutive lanes copy consecutive 16-byte pieces of a row (whole
            // 128-byte lines per 8 lanes); the row index comes from the lane
            // that computed it
            constexpr int QCH = DK / 8;         // pieces of a q or k row
            constexpr int QRPI = 32 / QCH;      // rows per instruction
            const int jq = lane % QCH, rq = lane / QCH;
#pragma unroll
            for (int i = 0; i < 16 / QRPI; ++i) {
                const int tl = rq + QRPI * i, t = 16 * warp + tl;
                const int64_t r = __shfl_sync(0xffffffffu, r_own, tl);
                const bool ok = r >= 0 && GTR_INB(r * DK + jq * 8 + 7, rows * DK, BS_WALK_LOAD);
                const int64_t o = ok ? r * DK + jq * 8 : 0;
                const uint32_t so = (uint32_t)(jq >> 3) * 8192u + (uint32_t)t * 128u +
                                    ((((uint32_t)jq & 7u) ^ (uint32_t)(t & 7)) << 4);
                if (kOut) cp_async16_s(sb + L::SQ + so, gq_ + o, ok);
                cp_async16_s(sb + L::SK + so, gk_ + o, ok);
            }
            const int jv = lane & 7, rv = lane >> 3;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int tl = rv + 4 * i, t = 16 * warp + tl;
                const int64_t r = __shfl_sync(0xffffffffu, r_own, tl);
                const int64_t o = r * DV + sl * DV_CTA + jv * 8;
                const bool ok = r >= 0 && GTR_INB(o + 7, rows * DV, BS_WALK_LOAD);
                cp_async16_s(sb + L::SV + (uint32_t)t * 128u + ((((uint32_t)jv) ^ (uint32_t)(t & 7)) << 4),
                             gv_ + (ok ? o : 0), ok);
            }
            if constexpr (L::kGsmem) {
                constexpr int GCH = DK / 4;     // pieces of a g row (fp32)
                constexpr int GRPI = 32 / GCH;  // rows per instruction (1 for d_k = 128)
                const int jg = lane % GCH, rg = lane / GCH;
#pragma unroll
                for (int i = 0; i < 16 / GRPI; ++i) {
                    const int tl = rg + GRPI * i, t = 16 * warp + tl;
                    const int64_t r = __shfl_sync(0xffffffffu, r_own, tl);
                    const bool ok = r >= 0 && GTR_INB(r * DK + jg * 4 + 3, rows * DK, BS_WALK_LOAD);
                    cp_async16_s(sb + L::SG + (uint32_t)t * (DK * 4) + jg * 16, args.g + (ok ? r * DK + jg * 4 : 0), ok);
                }
            }
        }
        cp_async_commit();  // one group per step, empty past the end
    };

    // g of one step into registers (d_k <= 64): key pair (2 dpair, 2 dpair + 1)
    // of this lane's TPL tokens; padding rows get g = 0 (a = 1)
    auto load_g = [&](int stage, float2 (&gv)[TPL]) {
        const int64_t *rowt = sRow + stage * 64 + 16 * warp + tb;
#pragma unroll
        for (int t = 0; t < TPL; t += 2) {
            const longlong2 rr = *reinterpret_cast<const longlong2 *>(rowt + t);
            const int64_t r2[2] = {rr.x, rr.y};
#pragma unroll
            for (int u = 0; u < 2; ++u)
                gv[t + u] = (lane_on && r2[u] >= 0 && GTR_INB(r2[u] * DK + 2 * dpair + 1, rows * DK, BS_WALK_G))
                                ? __ldcs(reinterpret_cast<const float2 *>(args.g + r2[u] * DK + 2 * dpair))
                                : make_float2(0.f, 0.f);
        }
    };

    // state slice, fragment layout: Se[n][i] = S[dk = 8n + kc + (i & 1)][v = 16*warp + tr + 8*(i >> 1)]
    // of value slice sl; arr[off + dk*DV + sl*64 + v] (extent elements), or zero
    float Se[KT][4];
    auto load_state = [&](const float *arr, int64_t off, int64_t extent, int sl) {
#pragma unroll
        for (int n = 0; n < KT; ++n)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int dk = 8 * n + kc + (i & 1), v = 16 * warp + tr + 8 * (i >> 1);
                const int64_t e = off + (int64_t)dk * DV + sl * DV_CTA + v;
                Se[n][i] = (arr && GTR_INB(e, extent, BS_WALK_STATE)) ? __ldcg(arr + e) : 0.f;
            }
    };
    const int64_t state_elems = (int64_t)nseq * DK * DV;             // S_0, S_N
    const int64_t chunk_state_elems = state_elems * geo.nc;          // dS, S_enter
    auto load_item_state = [&](int item, int cc) {
        const int sq = seq_of(item), sl = item % args.vs;
        if (MODE == WALK_SEQ) load_state(args.S0, (int64_t)sq * DK * DV, state_elems, sl);
        if (MODE == WALK_OUTPUT) load_state(args.S_enter, ((int64_t)sq * geo.nc + cc) * DK * DV, chunk_state_elems, sl);
    };

    // ---- set-up: tensor memory, mbarriers, the first two steps in flight
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(base_addr + L::MISC),
                     "n"(L::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
    }
    if (tid == 0) {
        mbar_init(mbar1, kOut ? 3 : 1);  // pass 1 completes from threads 0, 32 and 64
        mbar_init(mbar2, 1);
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = (uint32_t)misc[0];
    constexpr uint32_t kDsLanes = 16u << 16;  // dS^T: lanes 16-31 of each 32-lane group
    constexpr uint32_t kOCol = 64;            // O: columns 64-127 of lanes 0-15
    // matrix descriptors of stage 0 (a stage's tiles sit L::STAGE bytes
    // further; a descriptor's start-address field counts 16-byte units, so
    // an offset inside shared memory is added as offset >> 4)
    const uint64_t dQk = umma_desc_sw128(base_addr + L::SQ, 16, 1024);    // qh, K-major
    const uint64_t dKk = umma_desc_sw128(base_addr + L::SK, 16, 1024);    // ke, K-major
    const uint64_t dKm = umma_desc_sw128(base_addr + L::SK, 8192, 1024);  // ke, MN-major
    const uint64_t dVm = umma_desc_sw128(base_addr + L::SV, 8192, 1024);  // v, MN-major
    const uint64_t dP = umma_desc_sw128(base_addr + L::P, 16, 1024);
    const uint64_t dSP = umma_desc_sw128(base_addr + L::SP, 16, 1024);
    uint32_t ph1 = 0, ph2 = 0;
    bool mma_ok = true;

    // launched programmatically, the set-up above overlaps the grid ahead of
    // it; the whole-sequence walk and phase 1 wait for that grid before any
    // access to global memory (phase 3 before it reads S_enter, below), and
    // only then let the grid after this one start (phase 3 reads q, k, v, g
    // before its wait, so nothing ahead of a call may still run when it
    // starts)
    if (MODE != WALK_OUTPUT) grid_dep_wait();
    grid_dep_launch();
    int it = blockIdx.x, c = it < args.items ? first_chunk(it) : 0;
    int it1 = it, c1 = c;
    next_step(it1, c1);
    issue_loads(it, c, 0);
    issue_loads(it1, c1, 1);
    float2 gnext[TPL];
    if constexpr (!L::kGsmem) {
        if (it < args.items) load_g(0, gnext);
    }
    (void)gnext;
    // phase 3 reads S_enter, written by the scan: with a programmatic launch
    // the loads above are in flight while the scan finishes
    if (MODE == WALK_OUTPUT) grid_dep_wait();
    if (it < args.items) load_item_state(it, c);

    for (int step = 0; it < args.items; ++step) {
        const int s = step & 1;
        const uint32_t sb = (uint32_t)s * L::STAGE;
        const int seq = seq_of(it), sl = it % args.vs;
        const int t0 = c * 64, len = min(64, geo.N - t0);
        const int64_t *rowt = sRow + s * 64;
        // the step after this one (its loads are in flight in the other stage)
        int itn = it, cn = c;
        next_step(itn, cn);

        // ---- a_t = exp(g_t) of this warp's 16 tokens; per-warp decay totals
        float2 av[PPL][TPL];
        if constexpr (!L::kGsmem) {
#pragma unroll
            for (int t = 0; t < TPL; ++t) av[0][t] = gnext[t];
            if (itn < args.items) load_g(s ^ 1, gnext);  // next step's g, consumed one step later
        }
        cp_async_wait_group<1>();  // this step's stage (the next one may still be in flight)
        __syncwarp();              // the warp's own rows (its own copies) visible to the warp
        if constexpr (L::kGsmem) {
            const float *sg = reinterpret_cast<const float *>(base + sb + L::SG);
#pragma unroll
            for (int p = 0; p < PPL; ++p)
#pragma unroll
                for (int t = 0; t < TPL; ++t)
                    av[p][t] = *reinterpret_cast<const float2 *>(sg + (16 * warp + tb + t) * DK + 64 * p + 2 * dpair);
        }
        float2 oth[PPL];  // kSplit: the other half-warp's decay total over its 8 tokens
#pragma unroll
        for (int p = 0; p < PPL; ++p) {
            float2 tot = make_float2(1.f, 1.f);
#pragma unroll
            for (int t = 0; t < TPL; ++t) {
                av[p][t] = make_float2(ex2(av[p][t].x * kLog2e), ex2(av[p][t].y * kLog2e));
                tot.x *= av[p][t].x;
                tot.y *= av[p][t].y;
            }
            if constexpr (kSplit) {
                oth[p] = make_float2(__shfl_xor_sync(0xffffffffu, tot.x, 16), __shfl_xor_sync(0xffffffffu, tot.y, 16));
                tot.x *= oth[p].x;
                tot.y *= oth[p].y;
            }
            if (lane_on && (!kSplit || lane < 16))
                *reinterpret_cast<float2 *>(sTot + warp * DK + 64 * p + 2 * dpair) = tot;
        }
        // ---- this lane's column pairs of the warp's 16 rows of q and k, read
        // once (all loads before any store), and the |q~| test
        uint32_t ro[PPL][TPL];
        T2 qv[PPL][TPL], kv[PPL][TPL];
        float qm = 0.f;
#pragma unroll
        for (int p = 0; p < PPL; ++p) {
            if (!lane_on) break;
            const int dc = (2 * dpair) & 63;
            const uint32_t cb = (uint32_t)p * 8192u + (uint32_t)(dc & 7) * 2u;
#pragma unroll
            for (int t = 0; t < TPL; ++t) {
                const int row = 16 * warp + tb + t;
                ro[p][t] = cb + (uint32_t)row * 128u + (((uint32_t)(dc >> 3) ^ (uint32_t)(row & 7)) << 4);
            }
#pragma unroll
            for (int t = 0; t < TPL; ++t) kv[p][t] = *reinterpret_cast<const T2 *>(base + sb + L::SK + ro[p][t]);
            if (kOut) {
#pragma unroll
                for (int t = 0; t < TPL; ++t) {
                    qv[p][t] = *reinterpret_cast<const T2 *>(base + sb + L::SQ + ro[p][t]);
                    const float2 qf = IO::to_f2(qv[p][t]);
                    qm = fmaxf(qm, fmaxf(fabsf(qf.x), fabsf(qf.y)));
                }
            }
        }
        // (A) every warp's totals visible; any |q~| > 16 in the chunk
        const bool qbig = __syncthreads_or(kOut && qm * qscale > 16.f) != 0;

        // ---- prep: ke = k Suf (always <= |k|), qh = q~ E / gamma (whole-chunk
        // form) or qe = q~ E (exact form), written over the raw tiles
        float2 Eb[PPL], Sb[PPL], gam[PPL];
#pragma unroll
        for (int p = 0; p < PPL; ++p) {
            Eb[p] = Sb[p] = gam[p] = make_float2(1.f, 1.f);
            const int d0 = 64 * p + 2 * dpair;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float2 tw = lane_on ? *reinterpret_cast<const float2 *>(sTot + w * DK + d0) : make_float2(1.f, 1.f);
                if (w < warp) { Eb[p].x *= tw.x; Eb[p].y *= tw.y; }
                if (w > warp) { Sb[p].x *= tw.x; Sb[p].y *= tw.y; }
                gam[p].x *= tw.x;
                gam[p].y *= tw.y;
            }
            if constexpr (kSplit) {  // the other half-warp's tokens come before (lanes 16-31) or after
                if (lane >= 16) { Eb[p].x *= oth[p].x; Eb[p].y *= oth[p].y; }
                else { Sb[p].x *= oth[p].x; Sb[p].y *= oth[p].y; }
            }
        }
        // every warp covers every key dimension with the same products, so
        // the vote below is the same in every warp
        const float lo = 3.3546263e-4f;  // e^-kWalkChunkRange
        bool in_range = true;
#pragma unroll
        for (int p = 0; p < PPL; ++p)
            in_range = in_range && gam[p].x >= lo && gam[p].y >= lo && gam[p].x <= 1.f / lo && gam[p].y <= 1.f / lo;
        const bool gam_ok = __all_sync(0xffffffffu, in_range);
        // the whole-chunk form needs the gate range and |q~| <= 16 (qh then fits fp16)
        const bool exact = kOut && (!gam_ok || qbig);
#pragma unroll
        for (int p = 0; p < PPL; ++p) {
            if (!lane_on) break;
            const int d0 = 64 * p + 2 * dpair;
            if (kOut) {
                float2 E = exact ? make_float2(Eb[p].x * qscale, Eb[p].y * qscale)
                                 : make_float2(Eb[p].x * (qscale / gam[p].x), Eb[p].y * (qscale / gam[p].y));
#pragma unroll
                for (int t = 0; t < TPL; ++t) {
                    E.x *= av[p][t].x;
                    E.y *= av[p][t].y;
                    *reinterpret_cast<T2 *>(base + sb + L::SQ + ro[p][t]) = __hmul2(qv[p][t], IO::from_f2(E.x, E.y));
                }
            }
            float2 S = Sb[p];  // decay after token t to the chunk end
#pragma unroll
            for (int t = TPL - 1; t >= 0; --t) {
                *reinterpret_cast<T2 *>(base + sb + L::SK + ro[p][t]) = __hmul2(kv[p][t], IO::from_f2(S.x, S.y));
                S.x *= av[p][t].x;
                S.y *= av[p][t].y;
            }
            if (warp == 0 && (!kSplit || lane < 16)) *reinterpret_cast<float2 *>(sGam + d0) = gam[p];
        }

        const bool have_state = MODE == WALK_OUTPUT || (MODE == WALK_SEQ && (c > 0 || args.S0 != nullptr));
        if (kOut && have_state) {
            // ---- S'^T = (sc . S_enter)^T, K-major B operand of the readout
            // (rows: this slice's value columns); sc = gamma (whole-chunk form)
            // or 1 (exact form), gamma of key dim dk taken from the lane of this
            // warp that computed it; pass 2 of the previous step has read it
            const int v0 = 16 * warp + tr;
            const uint32_t rb0 = (uint32_t)v0 * 128u + (uint32_t)kc * 2u, rb1 = rb0 + 8u * 128u;
            const uint32_t x0 = (uint32_t)(v0 & 7), x1 = (uint32_t)((v0 + 8) & 7);
#pragma unroll
            for (int n = 0; n < KT; ++n) {
                const int src = 4 * (n & 7) + (lane & 3);
                const int p = n >> 3;
                float gx = 1.f, gy = 1.f;
#pragma unroll
                for (int pp = 0; pp < PPL; ++pp) {
                    const float ax = __shfl_sync(0xffffffffu, gam[pp].x, src);
                    const float ay = __shfl_sync(0xffffffffu, gam[pp].y, src);
                    if (pp == p) { gx = ax; gy = ay; }
                }
                if (exact) gx = gy = 1.f;
                const uint32_t hb = (uint32_t)p * 8192u, ch = (uint32_t)(n & 7);
                *reinterpret_cast<uint32_t *>(base + L::SP + hb + rb0 + ((ch ^ x0) << 4)) =
                    pack2<T>(gx * Se[n][0], gy * Se[n][1]);
                *reinterpret_cast<uint32_t *>(base + L::SP + hb + rb1 + ((ch ^ x1) << 4)) =
                    pack2<T>(gx * Se[n][2], gy * Se[n][3]);
            }
        }
        fence_async_shared();
        tc_fence_before();
        __syncthreads();  // (B) operands, S' and gamma written

        // ---- pass 1, issued from three threads at once (each issuing thread
        // pays its own per-instruction cost, so three queues of four MMAs
        // finish issuing sooner than one of twelve): A = qh ke^T (lanes 0-15,
        // columns 0-63) from thread 0, dS^T = V^T ke (lanes 16-31) from
        // thread 64 (thread 0 in phase 1, which has no A), the readout
        // O = qh S' (lanes 0-15, columns 64-127) from thread 32; the three
        // write disjoint accumulators
        if (tid == 0) {
            tc_fence_after();
            const uint64_t so = (uint64_t)(sb >> 4);
            if (kOut && !exact) {
                constexpr uint32_t id = umma_idesc(0, 0, 64, 64, IO::kBf16);
#pragma unroll
                for (int ks = 0; ks < DK / 16; ++ks) {
                    const uint64_t ko = so + (uint64_t)(((ks >> 2) * 8192 + (ks & 3) * 32) >> 4);
                    umma_f16(tmem, dQk + ko, dKk + ko, id, ks > 0);
                }
            }
            if (!kOut) {
                constexpr uint32_t id2 = umma_idesc(1, 1, 64, DK, IO::kBf16);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_f16(tmem + kDsLanes, dVm + so + 128 * ks, dKm + so + 128 * ks, id2, ks > 0);
            }
            if (kOut && exact)
                mbar_arrive(mbar1);
            else
                umma_commit(mbar1);
        }
        if (kOut && tid == 64) {
            tc_fence_after();
            const uint64_t so = (uint64_t)(sb >> 4);
            constexpr uint32_t id2 = umma_idesc(1, 1, 64, DK, IO::kBf16);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) umma_f16(tmem + kDsLanes, dVm + so + 128 * ks, dKm + so + 128 * ks, id2, ks > 0);
            umma_commit(mbar1);
        }
        if (kOut && tid == 32) {
            if (have_state) {
                tc_fence_after();
                const uint64_t so = (uint64_t)(sb >> 4);
                constexpr uint32_t id_qs = umma_idesc(0, 0, 64, 64, IO::kBf16);
#pragma unroll
                for (int ks = 0; ks < DK / 16; ++ks) {
                    const uint64_t ko = (uint64_t)(((ks >> 2) * 8192 + (ks & 3) * 32) >> 4);
                    umma_f16(tmem + kOCol, dQk + so + ko, dSP + ko, id_qs, ks > 0);
                }
                umma_commit(mbar1);
            } else {
                mbar_arrive(mbar1);
            }
        }

        // ---- exact form: the score matrix on CUDA cores from the raw operands
        if (kOut && exact) {
            // thread -> query row t = tid / 2, keys s in [32*(tid&1), +32); the
            // log2-domain in-chunk prefix of g, 16 key dims at a time, staged
            // in the score region
            const int t = tid >> 1, sbk = 32 * (tid & 1);
            float pe[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) pe[j] = 0.f;
            T *xq = reinterpret_cast<T *>(base + L::P);         // [64][16]
            T *xk = reinterpret_cast<T *>(base + L::P + 2048);  // [64][16]
            float *xb = reinterpret_cast<float *>(base + L::P + 4096);    // [64][16]
            for (int hd = 0; hd < DK / 16; ++hd) {
                __syncthreads();
                for (int idx = tid; idx < 64 * 16; idx += 128) {
                    const int tt = idx >> 4, d = idx & 15;
                    const int64_t r = rowt[tt];
                    const int64_t o = (r < 0 ? 0 : r) * DK + 16 * hd + d;
                    const bool ok = r >= 0 && GTR_INB(o, rows * DK, BS_WALK_EXACT);
                    xq[idx] = ok ? gq_[o] : IO::zero();
                    xk[idx] = ok ? gk_[o] : IO::zero();
                    xb[idx] = ok ? args.g[o] * kLog2e : 0.f;
                }
                __syncthreads();
                if (tid < 16) {
                    float acc = 0.f;
                    for (int tt = 0; tt < 64; ++tt) {
                        acc += xb[tt * 16 + tid];
                        xb[tt * 16 + tid] = acc;
                    }
                }
                __syncthreads();
                for (int d = 0; d < 16; ++d) {
                    const float qq = IO::to_f(xq[t * 16 + d]) * qscale;
                    const float bt = xb[t * 16 + d];
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int sk = sbk + j;
                        if (sk <= t) pe[j] = fmaf(qq * IO::to_f(xk[sk * 16 + d]), ex2(bt - xb[sk * 16 + d]), pe[j]);
                    }
                }
            }
            __syncthreads();  // the staging in the score region is consumed
#pragma unroll
            for (int j = 0; j < 32; j += 2)
                *reinterpret_cast<uint32_t *>(base + L::P + sw128(t, sbk + j)) = pack2<T>(pe[j], pe[j + 1]);
        }

        if (!mbar_wait(mbar1, ph1)) mma_ok = false;
        ph1 ^= 1u;
        tc_fence_after();
        if constexpr (GATED) {
            // the gate rows of this warp's tokens into the S' tile (pass 1 has
            // read it; the readout is in TMEM), swizzled like the output rows,
            // in flight while the scores and pass 2 are done
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t = 16 * warp + 4 * i + (lane >> 3), j = lane & 7;
                const int64_t r = rowt[t];
                const int64_t o_off = r * DV + j * 8;
                const bool ok = t < len && r >= 0 && GTR_INB(o_off + 7, rows * DV, BS_WALK_GATE);
                cp_async16_s(base_addr + L::SP + t * 128 + (((j ^ (t & 7)) & 7) << 4),
                             static_cast<const T *>(args.gate) + (ok ? o_off : 0), ok);
            }
            cp_async_commit();
        }

        // ---- the chunk summary of this value slice: the state update, or
        // (phase 1) dS_c and gamma_c written out
        {
            const bool last = c == last_chunk(it);
#pragma unroll
            for (int q4 = 0; q4 < (DK + 31) / 32; ++q4) {
                float dS[16];
                if constexpr (DK >= 32) {
                    tmem_ld_16x32(tmem + kDsLanes + ((uint32_t)(32 * warp) << 16) + 32 * q4, dS);
                    tc_wait_ld();
                }
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const int n = 4 * q4 + m;
                    if (n >= KT) break;
                    const int dk = 8 * n + kc;
                    if (MODE == WALK_SUMMARY) {
                        const int64_t o = ((int64_t)seq * geo.nc + c) * DK * DV + sl * DV_CTA + 16 * warp + tr;
                        const int64_t e[4] = {o + (int64_t)dk * DV, o + (int64_t)(dk + 1) * DV,
                                              o + (int64_t)dk * DV + 8, o + (int64_t)(dk + 1) * DV + 8};
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            if (GTR_INB(e[i], chunk_state_elems, BS_WALK_SUMMARY)) args.dS[e[i]] = dS[4 * m + i];
                    } else if (MODE == WALK_SEQ) {
                        const float2 gg = *reinterpret_cast<const float2 *>(sGam + dk);
                        Se[n][0] = fmaf(gg.x, Se[n][0], dS[4 * m + 0]);
                        Se[n][1] = fmaf(gg.y, Se[n][1], dS[4 * m + 1]);
                        Se[n][2] = fmaf(gg.x, Se[n][2], dS[4 * m + 2]);
                        Se[n][3] = fmaf(gg.y, Se[n][3], dS[4 * m + 3]);
                    }
                }
            }
            if (MODE == WALK_SUMMARY && sl == 0)
                for (int d = tid; d < DK; d += 128) {
                    const int64_t e = ((int64_t)seq * geo.nc + c) * DK + d;
                    if (GTR_INB(e, (int64_t)nseq * geo.nc * DK, BS_WALK_SUMMARY)) args.gamma[e] = sGam[d];
                }
            if (MODE == WALK_SEQ && last && args.SN) {
#pragma unroll
                for (int n = 0; n < KT; ++n)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int dk = 8 * n + kc + (i & 1), v = 16 * warp + tr + 8 * (i >> 1);
                        const int64_t e = (int64_t)seq * DK * DV + (int64_t)dk * DV + sl * DV_CTA + v;
                        if (GTR_INB(e, state_elems, BS_WALK_STATE)) args.SN[e] = Se[n][i];
                    }
            }
        }

        if (kOut) {
            // ---- the masked scores P (fp16, swizzled), this warp's 16 query rows
            if (!exact) {
                float a[32];
                tmem_ld_16x64(tmem + ((uint32_t)(32 * warp) << 16), a);
                tc_wait_ld();
#pragma unroll
                for (int n = 0; n < 8; ++n) {
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        const int t = 16 * warp + tr + 8 * hf, sk = 8 * n + kc;
                        const float x0 = sk <= t ? a[4 * n + 2 * hf] : 0.f;
                        const float x1 = sk + 1 <= t ? a[4 * n + 2 * hf + 1] : 0.f;
                        *reinterpret_cast<uint32_t *>(base + L::P + sw128(t, sk)) = pack2<T>(x0, x1);
                    }
                }
            }
            fence_async_shared();
            tc_fence_before();
            __syncthreads();  // (C) P and S' written; A and dS^T read by every warp

            // ---- pass 2: O += P V (O holds qh S' from pass 1 when there is state)
            if (tid == 0) {
                tc_fence_after();
                const uint64_t so = (uint64_t)(sb >> 4);
                constexpr uint32_t id_pv = umma_idesc(0, 1, 64, 64, IO::kBf16);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_f16(tmem + kOCol, dP + 2 * ks, dVm + so + 128 * ks, id_pv, (ks > 0 || have_state) ? 1u : 0u);
                umma_commit(mbar2);
            }
            if (!mbar_wait(mbar2, ph2)) mma_ok = false;
            ph2 ^= 1u;
            tc_fence_after();

            // ---- store O: each warp stages its own 16 rows (swizzled, in the
            // score region) and writes them as 16-byte row pieces
            {
                float o[32];
                tmem_ld_16x64(tmem + kOCol + ((uint32_t)(32 * warp) << 16), o);
                tc_wait_ld();
                unsigned char *st = base + L::P;
                if constexpr (GATED) {
                    // the gate rows (copied into the S' tile after pass 1) have landed
                    cp_async_wait_group<0>();
                    __syncwarp();
                    // 1 / rms of rows tr and tr + 8 (fp32, over the 64 values
                    // that lanes 4tr..4tr+3 hold)
                    float ss0 = 0.f, ss1 = 0.f;
#pragma unroll
                    for (int n = 0; n < 8; ++n) {
                        ss0 = fmaf(o[4 * n], o[4 * n], fmaf(o[4 * n + 1], o[4 * n + 1], ss0));
                        ss1 = fmaf(o[4 * n + 2], o[4 * n + 2], fmaf(o[4 * n + 3], o[4 * n + 3], ss1));
                    }
                    ss0 += __shfl_xor_sync(0xffffffffu, ss0, 1);
                    ss1 += __shfl_xor_sync(0xffffffffu, ss1, 1);
                    ss0 += __shfl_xor_sync(0xffffffffu, ss0, 2);
                    ss1 += __shfl_xor_sync(0xffffffffu, ss1, 2);
                    const float inv0 = rsqrtf(ss0 * (1.f / 64.f) + args.norm_eps);
                    const float inv1 = rsqrtf(ss1 * (1.f / 64.f) + args.norm_eps);
#pragma unroll
                    for (int n = 0; n < 8; ++n) {
                        const int t = 16 * warp + tr, col = 8 * n + kc;
                        const float2 w = __ldg(reinterpret_cast<const float2 *>(args.norm_w + col));
                        const float2 r0 = IO::to_f2(*reinterpret_cast<const T2 *>(base + L::SP + sw128(t, col)));
                        const float2 r1 = IO::to_f2(*reinterpret_cast<const T2 *>(base + L::SP + sw128(t + 8, col)));
                        o[4 * n + 0] *= inv0 * w.x * silu_tanh(r0.x);
                        o[4 * n + 1] *= inv0 * w.y * silu_tanh(r0.y);
                        o[4 * n + 2] *= inv1 * w.x * silu_tanh(r1.x);
                        o[4 * n + 3] *= inv1 * w.y * silu_tanh(r1.y);
                    }
                }
#pragma unroll
                for (int n = 0; n < 8; ++n) {
                    const int t = 16 * warp + tr, col = 8 * n + kc;
                    *reinterpret_cast<uint32_t *>(st + sw128(t, col)) = pack2<T>(o[4 * n], o[4 * n + 1]);
                    *reinterpret_cast<uint32_t *>(st + sw128(t + 8, col)) = pack2<T>(o[4 * n + 2], o[4 * n + 3]);
                }
                __syncwarp();
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int t = 16 * warp + 4 * i + (lane >> 3), j = lane & 7;
                    const int64_t r = rowt[t];
                    const int64_t o_off = r * DV + sl * DV_CTA + j * 8;
                    if (t < len && r >= 0 && GTR_INB(o_off + 7, rows * DV, BS_WALK_OUT))
                        *reinterpret_cast<int4 *>(gout_ + o_off) =
                            *reinterpret_cast<const int4 *>(st + t * 128 + (((j ^ (t & 7)) & 7) << 4));
                }
            }
        } else {
            // phase 1: the next step's pass 1 overwrites dS^T only after every
            // warp has read it (barrier A of the next step)
            tc_fence_before();
        }

        // ---- this stage is free (both passes complete): the step after the
        // next one is loaded into it; the next item's entering state
        {
            int it2 = itn, c2 = cn;
            if (itn < args.items) next_step(it2, c2);
            else it2 = args.items;
            issue_loads(it2, c2, s);
        }
        if (itn < args.items && itn != it) load_item_state(itn, cn);
        it = itn;
        c = cn;
    }

    if (!mma_ok && tid == 0) atomicOr(args.status, 6u);  // GTR_ERR_TIMEOUT
    cp_async_wait_all();
    // ---- release tensor memory
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "n"(L::TMEM_COLS)
                     : "memory");
    }
}

// Resident CTAs per SM of one instantiation (cached per device by the caller).
template <int DK, int MODE, bool GATED, typename T>
cudaError_t walk_occupancy(int *ctas) {
    using L = WalkLayout<DK>;
    cudaError_t e = cudaFuncSetAttribute(gla_walk_kernel<DK, MODE, GATED, T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::ALLOC);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(gla_walk_kernel<DK, MODE, GATED, T>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(ctas, gla_walk_kernel<DK, MODE, GATED, T>, 128, L::ALLOC);
}

template <int DK, int MODE, bool GATED, typename T>
cudaError_t launch_walk_t(const WalkArgs &a, int grid, cudaStream_t st) {
    using L = WalkLayout<DK>;
    cudaError_t e = cudaFuncSetAttribute(gla_walk_kernel<DK, MODE, GATED, T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::ALLOC);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(gla_walk_kernel<DK, MODE, GATED, T>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    e = launch_kernel(gla_walk_kernel<DK, MODE, GATED, T>, dim3(grid), dim3(128), L::ALLOC, st,
                      a.pdl, a);
    count_launch();
    return e;
}

// Launchers (gla_walk.cu): grid CTAs; `grid` <= a.items.  a.gate != null
// selects the gated output (WALK_SEQ with d_v = 64 only); bf16 selects bf16
// q, k, v, gate and output (WALK_SEQ only).
cudaError_t launch_walk(const WalkArgs &a, int mode, int grid, cudaStream_t st, bool bf16 = false);
// Resident CTAs per SM for (d_k, mode), or 0 for an unsupported d_k.
cudaError_t walk_ctas_per_sm(int dk, int mode, int *ctas);

}  // namespace gtr
