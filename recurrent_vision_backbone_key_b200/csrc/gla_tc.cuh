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
//             A tile is one chunk, or two consecutive chunks of a sequence
//             (d_v <= 64).  Tiles are handed out in chunk-major order by an
//             atomic ticket; the state entering a tile is passed from the
//             tile before it in the same sequence through a ring slot in L2
//             with a release/acquire flag, and from the first chunk of a
//             tile to the second through shared memory (the boundary scan,
//             done as a chain between tiles; the wait is bounded).
//
// Numerics (fp16 tensor-core operands, fp32 accumulation):
//   The chunk's tokens form sub-chunks of 16.  Per key dimension, with
//   a_t = exp(g_t), P_t = a_0..a_t (decay since the sub-chunk start) and
//   Suf_t = a_{t+1}..a_15 (decay to the sub-chunk end):
//     qs_t = q~_t P_t      ke_s = k_s Suf_s      (both <= the raw operand)
//   A local state runs over the sub-chunks of the chunk from zero,
//     L_{u+1} = diag(P_15,u) L_u + ke_u^T V_u,
//   so every factor that meets an fp16 operand is at most one.  Only the
//   16 x 16 diagonal blocks need exp(b_t - b_s) directly: when the decay
//   over the sub-chunk is at most kDiagRange nats they use the reference
//   token 7 (qd = qs / P_7, kd = ke / Suf_7, factors within e^{+-kDiagRange},
//   fp16 tensor-core product); when it is at most kMidRange nats, the same
//   reference with fp32 factors taken from the raw operands and a tf32
//   tensor-core product (factors within e^{+-kMidRange}, inside fp32 and
//   tf32 range); otherwise exact per-pair exponentials in fp32.
//   Then, with E_u the decay from the chunk start to sub-chunk u,
//     o_t = qs_t L_u + sum_{s<=t in u} A_ts v_s + (qs_t E_u) S_enter,
//     S_leave = diag(gamma_c) S_enter + L_last.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "gla_common.cuh"

namespace gtr {

enum TcMode : int { TC_SUMMARY = 0, TC_OUTPUT = 1, TC_FUSED = 2, TC_FUSED_PAIR = 3 };

// Largest decay over a 16-token sub-chunk (nats, either sign) for which the
// diagonal block uses fp16 factors around the reference token.
constexpr float kDiagRange = 5.0f;
// Largest |q~| or |k| for that path (keeps e^{kDiagRange} * value in fp16).
constexpr float kDiagMaxAbs = 64.0f;
// Largest ratio (nats) between two in-sub-chunk decay prefixes for the tf32
// form of the diagonal block, and the largest |q~| or |k| it takes (keeps
// e^{kMidRange} * value inside fp32).
constexpr float kMidRange = 80.0f;
constexpr float kMidMaxAbs = 1024.0f;
// Diagonal-block forms of a sub-chunk (its flag word).
enum DiagForm : int { DIAG_FP16 = 0, DIAG_TF32 = 1, DIAG_EXACT = 2 };

struct TcArgs {
    const __half *q, *k, *v;
    const float *g;
    Geom geo;
    float *dS;             // SUMMARY: [nseq][nc][dk][dv]
    float *gamma;          // SUMMARY: [nseq][nc][dk]
    const float *S_enter;  // OUTPUT:  [nseq][nc][dk][dv]
    __half *dS_h;          // SUMMARY: dS in fp16 instead (when set)
    const __half *S_enter_h;  // OUTPUT: S_enter in fp16 instead (when set)
    __half *out;           // OUTPUT / FUSED
    int *ctrl;             // FUSED: [0] ticket, [1] unused, then 4 flags per sequence; zeroed before each launch
    float *ring;           // FUSED: [nseq][2][dk*dv] fragment-ordered states
    unsigned *status;      // FUSED: device status word (GTR_ERR_TIMEOUT on a give-up)
    long long spin_limit;  // FUSED: polls before a wait gives up
    int hold_seq, hold_chunk;  // FUSED test hook: this tile never publishes (-1: off)
    bool pdl;              // host side: SUMMARY / OUTPUT launched with programmatic stream serialization
};

// ---------------------------------------------------------------- PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, bool full) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(smem)), "l"(gmem),
                 "r"(full ? 16 : 0));
}
// The same with a shared-state-space address.
__device__ __forceinline__ void cp_async16_s(uint32_t saddr, const void *gmem, bool full) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(saddr), "l"(gmem), "r"(full ? 16 : 0));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }
// Wait until at most N of this thread's cp.async groups are still pending.
template <int N>
__device__ __forceinline__ void cp_async_wait_group() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

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

// D += A(16x8, row) * B(8x8, col), tf32 in, fp32 accumulate.
__device__ __forceinline__ void mma1688_tf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// fp32 -> tf32 (round to nearest, ties away), as a 32-bit operand.
__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t y;
    asm("cvt.rna.tf32.f32 %0, %1;\n" : "=r"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ float2 unpack_h2(uint32_t x) {
    return __half22float2(*reinterpret_cast<__half2 *>(&x));
}
// Packed fp16 pair times a packed fp16 pair.
__device__ __forceinline__ uint32_t hmul2u(uint32_t x, uint32_t s) {
    __half2 r = __hmul2(*reinterpret_cast<__half2 *>(&x), *reinterpret_cast<__half2 *>(&s));
    return *reinterpret_cast<uint32_t *>(&r);
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

// One block of shared memory per chunk of the tile (NCH chunks per tile).
// GDIRECT: g is read from global memory straight into registers by the
// prep, not staged, and the tf32 diagonal factors are built one sub-chunk
// at a time; the output phase at d_k = 64 takes this to fit five CTAs per
// SM instead of four (43.6 KB against 52.8 KB at C = 64).
template <int DK, int DV, int NCH, bool MID, bool GDIRECT = false>
struct TcLayout {
    static constexpr int LDK = DK + 8;  // fp16 row stride (halves): 16-byte rows, conflict-free ldmatrix
    static constexpr int LDV = DV + 8;
    static constexpr int LDA = 24;      // 16x16 diagonal block rows (halves)
    static constexpr int NW = DV / 16;  // warps per chunk: one 16-wide value slice each
    static constexpr int NT = NW * 32 * NCH;
    // byte offsets inside a chunk block, for a chunk of C tokens (nsub = C/16 sub-chunks)
    __host__ __device__ static size_t q(int) { return 0; }                                 // qs fp16 [C][LDK]
    __host__ __device__ static size_t k(int C) { return q(C) + (size_t)C * LDK * 2; }      // ke fp16 [C][LDK]
    __host__ __device__ static size_t v(int C) { return k(C) + (size_t)C * LDK * 2; }      // v  fp16 [C][LDV]
    __host__ __device__ static size_t a(int C) { return v(C) + (size_t)C * LDV * 2; }      // A  fp16 [nsub][16][LDA]
    __host__ __device__ static size_t gu(int C) { return a(C) + (size_t)(C / 16) * 16 * LDA * 2; }  // P_15 per (u,d)
    __host__ __device__ static size_t rp(int C) { return gu(C) + (size_t)(C / 16) * DK * 4; }  // 1/P_7 (fp16)
    __host__ __device__ static size_t rs(int C) { return rp(C) + (size_t)(C / 16) * DK * 2; }  // 1/Suf_7 (fp16)
    __host__ __device__ static size_t eb(int C) { return rs(C) + (size_t)(C / 16) * DK * 2; }  // E_u (fp16)
    __host__ __device__ static size_t gc(int C) { return eb(C) + (size_t)(C / 16) * DK * 2; }  // gamma_c
    __host__ __device__ static size_t row(int C) { return gc(C) + (size_t)DK * 4; }            // token-head row index
    __host__ __device__ static size_t flags(int C) { return row(C) + (size_t)C * 8; }          // exact-path sub-chunks
    // scratch, used in turn for the staged g rows (fp32 [C][DK], unless
    // GDIRECT), the tf32 diagonal factors, the exact
    // diagonal path's raw operands, the state handed from the first chunk of
    // a tile to the second, and the output staging
    __host__ __device__ static size_t scratch(int C) { return flags(C) + 64; }
    __host__ __device__ static size_t scratch_bytes(int C) {
        size_t o = (size_t)C * LDV * 2, e = (size_t)16 * DK * 8, gs = GDIRECT ? 0 : (size_t)C * DK * 4;
        size_t hs = NCH > 1 ? (size_t)DK * DV * 4 : 0;
        size_t md = (size_t)(C >= 32 ? kMidGroup : 1) * 32 * DK * 4;  // tf32 diagonal factors
        size_t m = o > e ? o : e;
        m = m > gs ? m : gs;
        m = m > md ? m : md;
        return m > hs ? m : hs;
    }
    // MID (the fused schedule) with d_k = d_v = 128 (one CTA per SM, shared
    // memory to spare): the prepared qs, ke go to a second pair of buffers
    // (fp16 [2][C][LDK]) so that the raw q, k stay in the first, and the
    // tf32 diagonal factors of every sub-chunk fit at once (fp32
    // [nsub][2][16][DK]).  The output phase of the three-phase schedule keeps
    // the smaller layout, which fits two CTAs per SM.
    static constexpr bool kMidSmem = MID && DK >= 128 && DV >= 128;
    static constexpr bool kGDirect = GDIRECT;
    // tf32 sub-chunks whose factors are built together
    static constexpr int kMidGroup = kMidSmem ? 4 : (GDIRECT ? 1 : 2);
    __host__ __device__ static size_t prep(int C) { return scratch(C) + scratch_bytes(C); }
    __host__ __device__ static size_t fac(int C) { return prep(C) + (kMidSmem ? (size_t)2 * C * LDK * 2 : 0); }
    __host__ __device__ static size_t block(int C) {
        return (fac(C) + (kMidSmem ? (size_t)C * DK * 8 : 0) + 127) & ~(size_t)127;
    }
    __host__ __device__ static size_t misc(int C) { return NCH * block(C); }  // tile index
    __host__ __device__ static size_t bytes(int C) { return misc(C) + 64; }
};
template <int DK, int DV, int MODE, int NCH>
using TcLayoutOf = TcLayout<DK, DV, NCH, MODE == TC_FUSED, MODE == TC_OUTPUT && DK == 64>;

// --------------------------------------------------------------- the kernel
//
// NCH chunks per tile (2 for the fused schedule with d_v <= 64, else 1):
// warps [NW*ch, NW*ch + NW) work on chunk ch of the tile.  The state enters
// the tile's first chunk from the ring and is handed to the second chunk
// through shared memory, so only every NCH-th chunk boundary goes through L2.

template <int DK, int DV, int MODE, int NCH>
__global__ void __launch_bounds__(TcLayoutOf<DK, DV, MODE, NCH>::NT)
gla_tc_kernel(const TcArgs args) {
    using Lay = TcLayoutOf<DK, DV, MODE, NCH>;
    // the output phase lets the grid launched after it start at once (that
    // grid waits for this one before it reads what this one writes); the
    // summary does so only after its own wait, below
    constexpr int LDK = Lay::LDK, LDV = Lay::LDV, LDA = Lay::LDA, NT = Lay::NT, NW = Lay::NW;
    constexpr int KT = DK / 8;  // 8-wide key tiles of the state
    static_assert(NCH == 1 || MODE == TC_FUSED, "multi-chunk tiles are for the fused schedule");
    extern __shared__ __align__(128) unsigned char smem[];
    const Geom &geo = args.geo;
    const int C = geo.chunk;
    const int nsub = C / 16;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int ch = warp / NW, wl = warp - ch * NW;  // chunk of this warp, value slice within it
    const size_t BLK = Lay::block(C);
    int *sTile = reinterpret_cast<int *>(smem + Lay::misc(C));

    // per-chunk views
    auto blk = [&](int i) { return smem + (size_t)i * BLK; };
    auto Q_ = [&](int i) { return reinterpret_cast<__half *>(blk(i) + Lay::q(C)); };
    auto K_ = [&](int i) { return reinterpret_cast<__half *>(blk(i) + Lay::k(C)); };
    auto V_ = [&](int i) { return reinterpret_cast<__half *>(blk(i) + Lay::v(C)); };
    auto A_ = [&](int i) { return reinterpret_cast<__half *>(blk(i) + Lay::a(C)); };
    auto Gu_ = [&](int i) { return reinterpret_cast<float *>(blk(i) + Lay::gu(C)); };
    auto Rp_ = [&](int i) { return reinterpret_cast<__half *>(blk(i) + Lay::rp(C)); };
    auto Rs_ = [&](int i) { return reinterpret_cast<__half *>(blk(i) + Lay::rs(C)); };
    auto Eb_ = [&](int i) { return reinterpret_cast<__half *>(blk(i) + Lay::eb(C)); };
    auto Gc_ = [&](int i) { return reinterpret_cast<float *>(blk(i) + Lay::gc(C)); };
    auto Row_ = [&](int i) { return reinterpret_cast<int64_t *>(blk(i) + Lay::row(C)); };  // (b*N + p)*heads + h, or -1
    auto Fl_ = [&](int i) { return reinterpret_cast<int *>(blk(i) + Lay::flags(C)); };
    auto Scr_ = [&](int i) { return blk(i) + Lay::scratch(C); };
    auto Fac_ = [&](int i) { return reinterpret_cast<float *>(blk(i) + Lay::fac(C)); };  // kMidSmem: tf32 factors
    // the prepared operands qs, ke: over the raw q, k, or (kMidSmem) beside them
    auto QP_ = [&](int i) {
        return Lay::kMidSmem ? reinterpret_cast<__half *>(blk(i) + Lay::prep(C)) : Q_(i);
    };
    auto KP_ = [&](int i) {
        return Lay::kMidSmem ? reinterpret_cast<__half *>(blk(i) + Lay::prep(C)) + C * LDK : K_(i);
    };

    // ------------------------------------------------ which tile
    const int nseq = geo.B * geo.heads;
    const int64_t rows = (int64_t)geo.B * geo.N * geo.heads;  // token-head rows of every tensor
    if (tid < 4 * NCH) Fl_(tid >> 2)[tid & 3] = 0;
    int tile;
    if (MODE == TC_FUSED) {
        if (tid == 0) sTile[0] = atomicAdd(&args.ctrl[0], 1);
        __syncthreads();
        tile = sTile[0];
        // The control words are zeroed before every launch, so a ticket past
        // the grid cannot happen; guard the indexing anyway.
        if (tile >= ((geo.nc + NCH - 1) / NCH) * nseq) {
            if (tid == 0) atomicOr(args.status, 6u);
            return;
        }
    } else {
        tile = blockIdx.x;
    }
    int c0, seq;
    if (MODE == TC_FUSED) {  // chunk-major: chunk group g of every sequence before group g+1
        const int grp = tile / nseq;
        seq = tile - grp * nseq;
        c0 = grp * NCH;
    } else {
        seq = tile / geo.nc;
        c0 = tile - seq * geo.nc;
    }
    const int b = seq / geo.heads, h = seq - b * geo.heads;
    const float qscale = rsqrtf((float)DK);
    auto chunk_len = [&](int i) {
        const int cc = c0 + i;
        return cc < geo.nc ? min(C, geo.N - cc * C) : 0;
    };

    // ------------------------------------------------ S0: the scan-order row tables
    // Row t of chunk i is token-head row (b*N + p)*heads + h of every
    // [B][N][heads][d] tensor; -1 past the end of the sequence.
    // chunk of a flat index over NCH equal parts of size `part` (no division)
    auto part_of = [](int idx, int part) { return (NCH > 1 && idx >= part) ? 1 : 0; };
    for (int idx = tid; idx < NCH * C; idx += NT) {
        const int i = part_of(idx, C), t = idx - i * C;
        const int cc = c0 + i;
        int64_t r = (t < chunk_len(i))
                        ? ((int64_t)b * geo.N + scan_pos(geo.dir, cc * C + t, geo.H, geo.W, geo.N)) * geo.heads + h
                        : (int64_t)-1;
        if (r >= 0 && !GTR_INB(r, rows, BS_TC_ROW)) r = -1;
        Row_(i)[t] = r;
    }
    __syncthreads();

    // a summary launched programmatically waits here for the grid ahead of
    // it before any access to global memory (that grid may still produce k,
    // v, g, or read the buffers this one writes)
    if (MODE == TC_SUMMARY) grid_dep_wait();
    // A grid launched after this one may start now.  The output phase (two
    // launches on) reads q, k, v, g before it waits for its predecessor, so
    // the first kernel of a call must not let the others start before
    // everything ahead of the call is complete.
    if (MODE != TC_FUSED) grid_dep_launch();

    // ------------------------------------------------ S1: stage q, k, v, g; prepare qs / ke
    // Every row of the tile is requested at once (cp.async, 16 bytes per
    // request, rows past the sequence end zero-filled), so the whole tile is
    // in flight together; q and k land in the operand buffers and are turned
    // into qs / ke in place (d_k = d_v = 128: into the second pair of
    // buffers, the raw tiles kept for the tf32 diagonal form), g lands in the
    // scratch region (GDIRECT: g is read by the prep itself).
    {
        constexpr int QCH = DK / 8, VCH = DV / 8, GCH = DK / 4;
        for (int idx = tid; idx < NCH * C * VCH; idx += NT) {
            const int i = part_of(idx, C * VCH), rem = idx - i * (C * VCH);
            const int t = rem / VCH, j = rem - t * VCH;
            const int64_t r = Row_(i)[t];
            const bool ok = r >= 0 && GTR_INB(r * DV + j * 8 + 7, rows * DV, BS_TC_LOAD);
            cp_async16(V_(i) + t * LDV + j * 8, args.v + (ok ? r * DV + j * 8 : 0), ok);
        }
        for (int idx = tid; idx < NCH * C * QCH; idx += NT) {
            const int i = part_of(idx, C * QCH), rem = idx - i * (C * QCH);
            const int t = rem / QCH, j = rem - t * QCH;
            const int64_t r = Row_(i)[t];
            const bool ok = r >= 0 && GTR_INB(r * DK + j * 8 + 7, rows * DK, BS_TC_LOAD);
            const int64_t o = ok ? r * DK + j * 8 : 0;
            if (MODE != TC_SUMMARY) cp_async16(Q_(i) + t * LDK + j * 8, args.q + o, ok);
            cp_async16(K_(i) + t * LDK + j * 8, args.k + o, ok);
        }
        for (int idx = tid; idx < (Lay::kGDirect ? 0 : NCH * C * GCH); idx += NT) {
            const int i = part_of(idx, C * GCH), rem = idx - i * (C * GCH);
            const int t = rem / GCH, j = rem - t * GCH;
            const int64_t r = Row_(i)[t];
            const bool ok = r >= 0 && GTR_INB(r * DK + j * 4 + 3, rows * DK, BS_TC_LOAD);
            cp_async16(reinterpret_cast<float *>(Scr_(i)) + t * DK + j * 4, args.g + (ok ? r * DK + j * 4 : 0), ok);
        }
        cp_async_commit();
        cp_async_wait_all();
        __syncthreads();
    }
    for (int task = tid; task < NCH * (DK / 2) * nsub; task += NT) {
        const int i = part_of(task, (DK / 2) * nsub), rem = task - i * ((DK / 2) * nsub);
        const int dp = rem % (DK / 2), u = rem / (DK / 2);
        const int d0 = 2 * dp;
        const __half *sQ = Q_(i), *sK = K_(i);  // raw
        __half *dQ = QP_(i), *dK = KP_(i);       // prepared
        const float *sG = reinterpret_cast<const float *>(Scr_(i));
        __half2 qv[16], kv[16];
        float2 av[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) {
            const int row = 16 * u + t;
            if (MODE != TC_SUMMARY) qv[t] = *reinterpret_cast<const __half2 *>(sQ + row * LDK + d0);
            kv[t] = *reinterpret_cast<const __half2 *>(sK + row * LDK + d0);
            if constexpr (Lay::kGDirect) {
                const int64_t r = Row_(i)[row];
                av[t] = (r >= 0 && GTR_INB(r * DK + d0 + 1, rows * DK, BS_TC_LOAD))
                            ? __ldg(reinterpret_cast<const float2 *>(args.g + r * DK + d0))
                            : make_float2(0.f, 0.f);
            } else {
                av[t] = *reinterpret_cast<const float2 *>(sG + row * DK + d0);
            }
        }
        // forward: a_t = exp(g_t), P_t = prod a_0..a_t, qs_t = q~_t P_t
        float2 P = make_float2(1.f, 1.f), P7 = P;
        float2 Pmn = P, Pmx = P;  // extremes of the prefixes (P_{-1} = 1 included)
        __half2 qmax = __float2half2_rn(0.f), kmax = qmax;
#pragma unroll
        for (int t = 0; t < 16; ++t) {
            av[t].x = ex2(av[t].x * kLog2e);
            av[t].y = ex2(av[t].y * kLog2e);
            P.x *= av[t].x;
            P.y *= av[t].y;
            if (t == 7) P7 = P;
            Pmn = make_float2(fminf(Pmn.x, P.x), fminf(Pmn.y, P.y));
            Pmx = make_float2(fmaxf(Pmx.x, P.x), fmaxf(Pmx.y, P.y));
            if (MODE != TC_SUMMARY) {
                qmax = __hmax2(qmax, __habs2(qv[t]));
                *reinterpret_cast<__half2 *>(dQ + (16 * u + t) * LDK + d0) =
                    __hmul2(qv[t], __floats2half2_rn(P.x * qscale, P.y * qscale));
            }
        }
        // backward: Suf_t = prod a_{t+1}..a_15, ke_t = k_t Suf_t
        float2 S = make_float2(1.f, 1.f), S7 = S;
#pragma unroll
        for (int t = 15; t >= 0; --t) {
            if (t == 7) S7 = S;
            kmax = __hmax2(kmax, __habs2(kv[t]));
            *reinterpret_cast<__half2 *>(dK + (16 * u + t) * LDK + d0) = __hmul2(kv[t], __floats2half2_rn(S.x, S.y));
            S.x *= av[t].x;
            S.y *= av[t].y;
        }
        *reinterpret_cast<float2 *>(Gu_(i) + u * DK + d0) = P;
        if (MODE != TC_SUMMARY) {
            const float lo = 6.737947e-3f /* e^-5 */, hi = 148.41316f /* e^5 */;
            const float2 qm = __half22float2(qmax), km = __half22float2(kmax);
            const bool fast = P.x >= lo && P.y >= lo && P.x <= hi && P.y <= hi &&
                              fmaxf(qm.x, qm.y) * qscale <= kDiagMaxAbs && fmaxf(km.x, km.y) <= kDiagMaxAbs;
            // the tf32 form: every ratio of two prefixes (so every factor
            // around token 7) within e^{+-kMidRange}
            const float mlo = 1.8048513e-35f;  // e^-kMidRange
            const bool mid = Pmn.x >= Pmx.x * mlo && Pmn.y >= Pmx.y * mlo && Pmx.x <= 3.0e35f &&
                             Pmx.y <= 3.0e35f && fmaxf(qm.x, qm.y) * qscale <= kMidMaxAbs &&
                             fmaxf(km.x, km.y) <= kMidMaxAbs;
            if (!fast) atomicMax(&Fl_(i)[u], mid ? DIAG_TF32 : DIAG_EXACT);
            *reinterpret_cast<__half2 *>(Rp_(i) + u * DK + d0) =
                __floats2half2_rn(P7.x > 0.f ? 1.f / P7.x : 0.f, P7.y > 0.f ? 1.f / P7.y : 0.f);
            *reinterpret_cast<__half2 *>(Rs_(i) + u * DK + d0) =
                __floats2half2_rn(S7.x > 0.f ? 1.f / S7.x : 0.f, S7.y > 0.f ? 1.f / S7.y : 0.f);
        }
    }
    __syncthreads();

    // ------------------------------------------------ S2: decay to each sub-chunk, chunk decay
    for (int task = tid; task < NCH * DK; task += NT) {
        const int i = part_of(task, DK), d = task - i * DK;
        float e = 1.f;
        for (int u = 0; u < nsub; ++u) {
            Eb_(i)[u * DK + d] = __float2half_rn(e);
            e *= Gu_(i)[u * DK + d];
        }
        Gc_(i)[d] = e;
    }

    const int r8 = lane & 7, m4 = lane >> 3;
    const int kc = 2 * (lane & 3);  // key column pair inside an 8-wide tile

    // ------------------------------------------------ S3: diagonal 16x16 blocks
    if (MODE != TC_SUMMARY) {
        for (int pr = warp; pr < NCH * nsub; pr += NCH * NW) {
            const int i = part_of(pr, nsub), u = pr - i * nsub;
            if (Fl_(i)[u]) continue;
            const __half *sQ = QP_(i), *sK = KP_(i), *sRp = Rp_(i), *sRs = Rs_(i);
            float acc[2][4] = {};
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk) {
                uint32_t af[4], bf[4];
                ldsm_x4(af, sQ + (16 * u + r8 + 8 * (m4 & 1)) * LDK + 16 * kk + 8 * (m4 >> 1));
                ldsm_x4(bf, sK + (16 * u + r8 + 8 * (m4 >> 1)) * LDK + 16 * kk + 8 * (m4 & 1));
                const uint32_t p0 = *reinterpret_cast<const uint32_t *>(sRp + u * DK + 16 * kk + kc);
                const uint32_t p1 = *reinterpret_cast<const uint32_t *>(sRp + u * DK + 16 * kk + 8 + kc);
                const uint32_t s0 = *reinterpret_cast<const uint32_t *>(sRs + u * DK + 16 * kk + kc);
                const uint32_t s1 = *reinterpret_cast<const uint32_t *>(sRs + u * DK + 16 * kk + 8 + kc);
                af[0] = hmul2u(af[0], p0); af[1] = hmul2u(af[1], p0);
                af[2] = hmul2u(af[2], p1); af[3] = hmul2u(af[3], p1);
                bf[0] = hmul2u(bf[0], s0); bf[2] = hmul2u(bf[2], s0);
                bf[1] = hmul2u(bf[1], s1); bf[3] = hmul2u(bf[3], s1);
                mma16816(acc[0], af, bf[0], bf[1]);
                mma16816(acc[1], af, bf[2], bf[3]);
            }
            __half *Au = A_(i) + u * 16 * LDA;
            const int tr = lane >> 2;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
#pragma unroll
                for (int hlf = 0; hlf < 2; ++hlf) {
                    const int t = tr + 8 * hlf;
                    const int s0i = 8 * j + kc;
                    const float x0 = (s0i <= t) ? acc[j][2 * hlf] : 0.f;
                    const float x1 = (s0i + 1 <= t) ? acc[j][2 * hlf + 1] : 0.f;
                    *reinterpret_cast<uint32_t *>(Au + t * LDA + s0i) = pack_h2(x0, x1);
                }
            }
        }
        // tf32 form (DIAG_TF32), by the whole CTA, with beta the in-sub-chunk
        // prefix sum of g*log2(e):
        //   qf_t = q~_t 2^(beta_t - beta_7),  kf_s = k_s 2^(beta_7 - beta_s),
        //   A = qf kf^T  (m16n8k8 tf32, fp32 accumulate).
        // The factors (fp32 [sub-chunk][qf, kf][16][DK], columns XOR-swizzled
        // by the row so that the fragment loads are free of bank conflicts)
        // meet only inside fp32 range; pairs s > t, whose product may
        // overflow, are dropped by the mask.
        for (int i = 0; i < NCH; ++i) {
            const int *fl = Fl_(i);
            uint32_t mids = 0;  // the tf32 sub-chunks, 4 bits each, in order
            int nm = 0;
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (u < nsub && fl[u] == DIAG_TF32) mids |= (uint32_t)u << (4 * nm++);
            // with kMidSmem every tf32 sub-chunk at once, from the raw q, k
            // and the staged g still in shared memory; else kMidGroup (two,
            // or one with GDIRECT) at a time in the scratch region, from the
            // raw operands in global memory
            constexpr int kGroup = Lay::kMidGroup;
            float *xf = Lay::kMidSmem ? Fac_(i) : reinterpret_cast<float *>(Scr_(i));
            const int64_t *sRow = Row_(i);
            __half *sA = A_(i);
            auto xsw = [](int row) { return (4 * row) & 28 & (DK - 1); };
            for (int m0 = 0; m0 < nm; m0 += kGroup) {
                const int gcnt = min(kGroup, nm - m0);
                if constexpr (Lay::kMidSmem) {
                    const __half *rq = Q_(i), *rk = K_(i);  // raw q, k (kept beside qs, ke)
                    const float *sG = reinterpret_cast<const float *>(Scr_(i));
                    for (int task = tid; task < gcnt * DK; task += NT) {
                        const int sl = task / DK, d = task - sl * DK;
                        const int u = (mids >> (4 * (m0 + sl))) & 15;
                        float bv[16];
#pragma unroll
                        for (int t = 0; t < 16; ++t) bv[t] = sG[(16 * u + t) * DK + d] * kLog2e;
#pragma unroll
                        for (int t = 1; t < 16; ++t) bv[t] += bv[t - 1];
                        float *xq = xf + sl * (32 * DK), *xk = xq + 16 * DK;
#pragma unroll 4
                        for (int t = 0; t < 16; ++t) {
                            const int row = 16 * u + t, cs = d ^ xsw(t);
                            xq[t * DK + cs] = __half2float(rq[row * LDK + d]) * qscale * ex2(bv[t] - bv[7]);
                            xk[t * DK + cs] = __half2float(rk[row * LDK + d]) * ex2(bv[7] - bv[t]);
                        }
                    }
                } else {
                    for (int task = tid; task < gcnt * DK; task += NT) {
                        const int sl = task / DK, d = task - sl * DK;
                        const int u = (mids >> (4 * (m0 + sl))) & 15;
                        const int64_t *rw = sRow + 16 * u;
                        auto off = [&](int t) {
                            const int64_t r = rw[t];
                            const int64_t o = (r < 0 ? 0 : r) * DK + d;
                            return (r >= 0 && GTR_INB(o, rows * DK, BS_TC_EXACT)) ? o : (int64_t)-1;
                        };
                        // beta: the 16 g loads in flight together, then the prefix
                        float bv[16];
#pragma unroll
                        for (int t = 0; t < 16; ++t) {
                            const int64_t o = off(t);
                            bv[t] = o >= 0 ? args.g[o] * kLog2e : 0.f;
                        }
#pragma unroll
                        for (int t = 1; t < 16; ++t) bv[t] += bv[t - 1];
                        float *xq = xf + sl * (32 * DK), *xk = xq + 16 * DK;
#pragma unroll 4
                        for (int t = 0; t < 16; ++t) {
                            const int64_t o = off(t);
                            const float qv = o >= 0 ? __half2float(args.q[o]) : 0.f;
                            const float kv = o >= 0 ? __half2float(args.k[o]) : 0.f;
                            const int cs = d ^ xsw(t);
                            xq[t * DK + cs] = qv * qscale * ex2(bv[t] - bv[7]);
                            xk[t * DK + cs] = kv * ex2(bv[7] - bv[t]);
                        }
                    }
                }
                __syncthreads();
                // job j (one warp each): sub-chunk m0 + (j >> 1), key columns 8 (j & 1) .. + 7
                for (int job = warp; job < 2 * gcnt; job += NCH * NW) {
                    const int sl = job >> 1, n0 = 8 * (job & 1);
                    const float *xq = xf + sl * (32 * DK), *xk = xq + 16 * DK;
                    const int g8 = lane >> 2, t4 = lane & 3;
                    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
                    for (int k0 = 0; k0 < DK; k0 += 8) {
                        uint32_t af[4];
                        af[0] = to_tf32(xq[g8 * DK + ((k0 + t4) ^ xsw(g8))]);
                        af[1] = to_tf32(xq[(g8 + 8) * DK + ((k0 + t4) ^ xsw(g8 + 8))]);
                        af[2] = to_tf32(xq[g8 * DK + ((k0 + t4 + 4) ^ xsw(g8))]);
                        af[3] = to_tf32(xq[(g8 + 8) * DK + ((k0 + t4 + 4) ^ xsw(g8 + 8))]);
                        const uint32_t b0 = to_tf32(xk[(n0 + g8) * DK + ((k0 + t4) ^ xsw(n0 + g8))]);
                        const uint32_t b1 = to_tf32(xk[(n0 + g8) * DK + ((k0 + t4 + 4) ^ xsw(n0 + g8))]);
                        mma1688_tf32(acc, af, b0, b1);
                    }
                    __half *Au = sA + ((mids >> (4 * (m0 + sl))) & 15) * 16 * LDA;
#pragma unroll
                    for (int hlf = 0; hlf < 2; ++hlf) {
                        const int t = g8 + 8 * hlf, s0i = n0 + 2 * t4;
                        const float x0 = (s0i <= t) ? acc[2 * hlf] : 0.f;
                        const float x1 = (s0i + 1 <= t) ? acc[2 * hlf + 1] : 0.f;
                        *reinterpret_cast<uint32_t *>(Au + t * LDA + s0i) = pack_h2(x0, x1);
                    }
                }
                __syncthreads();
            }
        }
        // Exact path (DIAG_EXACT), one sub-chunk at a time by the whole CTA:
        // A_ts = sum_d q~_td k_sd 2^(beta_td - beta_sd) with beta the in-sub-chunk
        // prefix sum of g*log2(e), from the raw operands.
        for (int i = 0; i < NCH; ++i) {
            int *fl = Fl_(i);
            if (!((fl[0] | fl[1] | fl[2] | fl[3]) & DIAG_EXACT)) continue;
            __half *xq = reinterpret_cast<__half *>(Scr_(i));
            __half *xk = xq + 16 * DK;
            float *xb = reinterpret_cast<float *>(xk + 16 * DK);
            const int64_t *sRow = Row_(i);
            __half *sA = A_(i);
            for (int u = 0; u < nsub; ++u) {
                if (fl[u] != DIAG_EXACT) continue;
                for (int idx = tid; idx < 16 * DK; idx += NT) {
                    const int t = idx / DK, d = idx - t * DK;
                    const int64_t r = sRow[16 * u + t];
                    const int64_t o = (r < 0 ? 0 : r) * DK + d;
                    const bool ok = r >= 0 && GTR_INB(o, rows * DK, BS_TC_EXACT);
                    xq[idx] = ok ? args.q[o] : __float2half(0.f);
                    xk[idx] = ok ? args.k[o] : __float2half(0.f);
                    xb[idx] = ok ? args.g[o] * kLog2e : 0.f;
                }
                __syncthreads();
                for (int d = tid; d < DK; d += NT) {
                    float acc = 0.f;
                    for (int t = 0; t < 16; ++t) {
                        acc += xb[t * DK + d];
                        xb[t * DK + d] = acc;
                    }
                }
                __syncthreads();
                for (int pr = tid; pr < 256; pr += NT) {
                    const int t = pr >> 4, s = pr & 15;
                    float acc = 0.f;
                    if (s <= t) {
                        for (int d = 0; d < DK; ++d)
                            acc = fmaf(__half2float(xq[t * DK + d]) * __half2float(xk[s * DK + d]),
                                       ex2(xb[t * DK + d] - xb[s * DK + d]), acc);
                        acc *= qscale;
                    }
                    sA[u * 16 * LDA + t * LDA + s] = __float2half_rn(acc);
                }
                __syncthreads();
            }
        }
    }
    __syncthreads();

    // ------------------------------------------------ S4: local state over sub-chunks
    // Warp (ch, wl) owns value columns [16wl, 16wl+16) of chunk ch.  L^T
    // (16 x DK) lives in the accumulator layout: Lt[n][0..3] covers key
    // columns 8n..8n+7.
    const __half *sQ = QP_(ch), *sK = KP_(ch), *sV = V_(ch), *sA = A_(ch), *sEb = Eb_(ch);
    const float *sGu = Gu_(ch), *sGc = Gc_(ch);
    const int v0 = 16 * wl;
    const int c = c0 + ch;
    float Lt[KT][4];
#pragma unroll
    for (int n = 0; n < KT; ++n) Lt[n][0] = Lt[n][1] = Lt[n][2] = Lt[n][3] = 0.f;
    float o[4][2][4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int j = 0; j < 2; ++j) o[u][j][0] = o[u][j][1] = o[u][j][2] = o[u][j][3] = 0.f;

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
                    mma16816(o[u][0], af, pack_h2(Lt[2 * kk][0], Lt[2 * kk][1]),
                             pack_h2(Lt[2 * kk + 1][0], Lt[2 * kk + 1][1]));
                    mma16816(o[u][1], af, pack_h2(Lt[2 * kk][2], Lt[2 * kk][3]),
                             pack_h2(Lt[2 * kk + 1][2], Lt[2 * kk + 1][3]));
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
        // update: L = diag(P_15,u) L + V_u^T ke_u
        {
            const float *gu = sGu + u * DK;
#pragma unroll
            for (int n = 0; n < KT; ++n) {
                const float2 gg = *reinterpret_cast<const float2 *>(gu + 8 * n + kc);
                Lt[n][0] *= gg.x; Lt[n][1] *= gg.y; Lt[n][2] *= gg.x; Lt[n][3] *= gg.y;
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
        if (!GTR_INB(sdx, (int64_t)nseq * geo.nc, BS_TC_SUMMARY)) return;
        const int vr = v0 + (lane >> 2);
        if (args.dS_h) {
            __half *dst = args.dS_h + sdx * DK * DV;
#pragma unroll
            for (int n = 0; n < KT; ++n) {
                const int kcol = 8 * n + kc;
                dst[(kcol)*DV + vr] = __float2half_rn(Lt[n][0]);
                dst[(kcol + 1) * DV + vr] = __float2half_rn(Lt[n][1]);
                dst[(kcol)*DV + vr + 8] = __float2half_rn(Lt[n][2]);
                dst[(kcol + 1) * DV + vr + 8] = __float2half_rn(Lt[n][3]);
            }
        } else {
            float *dst = args.dS + sdx * DK * DV;
#pragma unroll
            for (int n = 0; n < KT; ++n) {
                const int kcol = 8 * n + kc;
                dst[(kcol)*DV + vr] = Lt[n][0];
                dst[(kcol + 1) * DV + vr] = Lt[n][1];
                dst[(kcol)*DV + vr + 8] = Lt[n][2];
                dst[(kcol + 1) * DV + vr + 8] = Lt[n][3];
            }
        }
        for (int d = tid; d < DK; d += NT) args.gamma[sdx * DK + d] = sGc[d];
        return;
    }

    // ------------------------------------------------ S5: the state entering each chunk
    float Se[KT][4];
    bool have_state = c > 0;
    if (MODE == TC_OUTPUT) {
        // everything above reads only q, k, v, g: with a programmatic launch
        // it runs while the scan that writes S_enter finishes
        grid_dep_wait();
        const int64_t so = (GTR_INB(sdx, (int64_t)nseq * geo.nc, BS_TC_SENTER) ? sdx : 0) * DK * DV;
        const int vr = v0 + (lane >> 2);
        if (args.S_enter_h) {  // fp16 states: the readout's B fragments are fp16 anyway
            const __half *src = args.S_enter_h + so;
#pragma unroll
            for (int n = 0; n < KT; ++n) {
                const int kcol = 8 * n + kc;
                Se[n][0] = __half2float(src[kcol * DV + vr]);
                Se[n][1] = __half2float(src[(kcol + 1) * DV + vr]);
                Se[n][2] = __half2float(src[kcol * DV + vr + 8]);
                Se[n][3] = __half2float(src[(kcol + 1) * DV + vr + 8]);
            }
        } else {
            const float *src = args.S_enter + so;
#pragma unroll
            for (int n = 0; n < KT; ++n) {
                const int kcol = 8 * n + kc;
                Se[n][0] = src[kcol * DV + vr];
                Se[n][1] = src[(kcol + 1) * DV + vr];
                Se[n][2] = src[kcol * DV + vr + 8];
                Se[n][3] = src[(kcol + 1) * DV + vr + 8];
            }
        }
        have_state = true;
    } else {  // FUSED
        int *flags = args.ctrl + 2;
        // ring slot of the state entering the tile and of the one it leaves
        // (two alternating slots with one chunk per tile; a single slot with
        // two, since the tile reads it before it writes it)
        const int slot_in = NCH == 1 ? ((c0 - 1) & 1) : 0;
        const int slot_out = NCH == 1 ? (c0 & 1) : 0;
        // seq < nseq indexes the flags and both ring slots
        const bool seq_ok = GTR_INB(seq, nseq, BS_TC_FLAG) && GTR_INB((int64_t)seq * 2 + 1, (int64_t)nseq * 2, BS_TC_RING);
        if (c0 > 0) {
            if (tid == 0 && seq_ok) {
                long long spins = 0;
                while (ld_acquire(&flags[seq]) < c0) {
                    if (++spins > args.spin_limit) {
                        atomicOr(args.status, 6u);  // GTR_ERR_TIMEOUT
                        break;
                    }
                    __nanosleep(spins < 64 ? 32 : 256);
                }
            }
            __syncthreads();
            if (ch == 0 && seq_ok) {
                const float4 *src = reinterpret_cast<const float4 *>(
                    args.ring + ((int64_t)seq * 2 + slot_in) * (DK * DV));
#pragma unroll
                for (int n = 0; n < KT; ++n) {
                    float4 x = __ldcg(src + ((wl * KT + n) * 32 + lane));
                    Se[n][0] = x.x; Se[n][1] = x.y; Se[n][2] = x.z; Se[n][3] = x.w;
                }
            }
        } else if (ch == 0) {
#pragma unroll
            for (int n = 0; n < KT; ++n) Se[n][0] = Se[n][1] = Se[n][2] = Se[n][3] = 0.f;
        }
        if (NCH > 1) {
            // chunk c0 hands diag(gamma) S_enter + L to chunk c0+1 through shared memory
            float4 *hand = reinterpret_cast<float4 *>(Scr_(1));
            if (ch == 0) {
#pragma unroll
                for (int n = 0; n < KT; ++n) {
                    const float2 gg = *reinterpret_cast<const float2 *>(sGc + 8 * n + kc);
                    hand[(wl * KT + n) * 32 + lane] =
                        make_float4(fmaf(gg.x, Se[n][0], Lt[n][0]), fmaf(gg.y, Se[n][1], Lt[n][1]),
                                    fmaf(gg.x, Se[n][2], Lt[n][2]), fmaf(gg.y, Se[n][3], Lt[n][3]));
                }
            }
            __syncthreads();
            if (ch == NCH - 1) {
#pragma unroll
                for (int n = 0; n < KT; ++n) {
                    const float4 x = hand[(wl * KT + n) * 32 + lane];
                    Se[n][0] = x.x; Se[n][1] = x.y; Se[n][2] = x.z; Se[n][3] = x.w;
                }
                have_state = true;
            }
            __syncthreads();  // the hand-over region is reused for output staging below
        }
        // the tile's last chunk publishes diag(gamma_c) S_enter + L for the next tile
        const bool hold = (seq == args.hold_seq && args.hold_chunk >= c0 && args.hold_chunk < c0 + NCH);
        if (c0 + NCH < geo.nc && !hold && seq_ok) {
            if (ch == NCH - 1) {
                float4 *dst = reinterpret_cast<float4 *>(args.ring + ((int64_t)seq * 2 + slot_out) * (DK * DV));
#pragma unroll
                for (int n = 0; n < KT; ++n) {
                    const float2 gg = *reinterpret_cast<const float2 *>(sGc + 8 * n + kc);
                    float4 x;
                    x.x = fmaf(gg.x, Se[n][0], Lt[n][0]);
                    x.y = fmaf(gg.y, Se[n][1], Lt[n][1]);
                    x.z = fmaf(gg.x, Se[n][2], Lt[n][2]);
                    x.w = fmaf(gg.y, Se[n][3], Lt[n][3]);
                    __stcg(dst + ((wl * KT + n) * 32 + lane), x);
                }
            }
            __syncthreads();
            if (tid == 0) st_release(&flags[seq], c0 + NCH);
        }
    }

    // ------------------------------------------------ S6: readout of the entering state
    // qe_t = qs_t E_u is formed in registers from the qs fragments.
    if (have_state) {
        uint32_t Sb[KT][2];  // the entering state as fp16 B fragments
#pragma unroll
        for (int n = 0; n < KT; ++n) {
            Sb[n][0] = pack_h2(Se[n][0], Se[n][1]);
            Sb[n][1] = pack_h2(Se[n][2], Se[n][3]);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (u >= nsub) break;
#pragma unroll
            for (int kk = 0; kk < DK / 16; ++kk) {
                uint32_t af[4];
                ldsm_x4(af, sQ + (16 * u + r8 + 8 * (m4 & 1)) * LDK + 16 * kk + 8 * (m4 >> 1));
                const uint32_t e0 = *reinterpret_cast<const uint32_t *>(sEb + u * DK + 16 * kk + kc);
                const uint32_t e1 = *reinterpret_cast<const uint32_t *>(sEb + u * DK + 16 * kk + 8 + kc);
                af[0] = hmul2u(af[0], e0); af[1] = hmul2u(af[1], e0);
                af[2] = hmul2u(af[2], e1); af[3] = hmul2u(af[3], e1);
                mma16816(o[u][0], af, Sb[2 * kk][0], Sb[2 * kk + 1][0]);
                mma16816(o[u][1], af, Sb[2 * kk][1], Sb[2 * kk + 1][1]);
            }
        }
    }

    // ------------------------------------------------ S7: store the outputs
    {
        __half *sOut = reinterpret_cast<__half *>(Scr_(ch));
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
        __syncthreads();
        constexpr int VCH = DV / 8;
        for (int i = 0; i < NCH; ++i) {
            const int len = chunk_len(i);
            const __half *so = reinterpret_cast<const __half *>(Scr_(i));
            const int64_t *sRow = Row_(i);
            for (int idx = tid; idx < len * VCH; idx += NT) {
                const int t = idx / VCH, j = idx - t * VCH;
                if (sRow[t] >= 0 && GTR_INB(sRow[t] * DV + j * 8 + 7, rows * DV, BS_TC_OUT))
                    *reinterpret_cast<int4 *>(args.out + sRow[t] * DV + j * 8) =
                        *reinterpret_cast<const int4 *>(so + t * LDV + j * 8);
            }
        }
    }
}

// Launch helper used by the per-d_k translation units.
template <int DK, int DV, int MODE, int NCH>
cudaError_t launch_tc_mode(const TcArgs &a, cudaStream_t st) {
    using Lay = TcLayoutOf<DK, DV, MODE, NCH>;
    const size_t smem = Lay::bytes(a.geo.chunk);
    cudaError_t e = cudaFuncSetAttribute(gla_tc_kernel<DK, DV, MODE, NCH>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t groups = (a.geo.nc + NCH - 1) / NCH;
    const unsigned grid = (unsigned)(groups * a.geo.B * a.geo.heads);
    e = launch_kernel(gla_tc_kernel<DK, DV, MODE, NCH>, dim3(grid), dim3(Lay::NT), smem, st,
                      MODE != TC_FUSED && a.pdl, a);
    count_launch();
    return e;
}

// mode TC_FUSED_PAIR: the fused schedule with two chunks per tile (d_v <= 64).
template <int DK, int DV>
cudaError_t launch_tc_dv(const TcArgs &a, int mode, cudaStream_t st) {
    switch (mode) {
    case TC_SUMMARY: return launch_tc_mode<DK, DV, TC_SUMMARY, 1>(a, st);
    case TC_OUTPUT: return launch_tc_mode<DK, DV, TC_OUTPUT, 1>(a, st);
    case TC_FUSED_PAIR:
        if constexpr (DV <= 64) return launch_tc_mode<DK, DV, TC_FUSED, 2>(a, st);
        return launch_tc_mode<DK, DV, TC_FUSED, 1>(a, st);
    default: return launch_tc_mode<DK, DV, TC_FUSED, 1>(a, st);
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

cudaError_t launch_tc(const TcArgs &a, int mode, cudaStream_t st);
// tcgen05 fused kernel (d_k = d_v = 64, chunk 64), gla_umma.cu.
cudaError_t launch_fused_umma(const TcArgs &a, cudaStream_t st);

}  // namespace gtr
