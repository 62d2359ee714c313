// gla_umma.cuh -- fused GLA forward on the 5th-generation tensor cores
// (tcgen05 MMAs from shared-memory descriptors into tensor memory) for
// d_k = d_v in {64, 128} and chunks of 64 tokens.
//
// Same schedule as the fused mode of gla_tc.cuh (one (sequence, chunk, 64
// value columns) tile per CTA, chunk-major tickets, boundary state chained
// through an L2 ring with release/acquire flags, bounded waits), with the
// chunk's dense products done as whole-chunk M = 64 MMAs:
//   with a_t = exp(g_t), E_t = a_0..a_t (decay since the chunk start),
//   Suf_t = a_{t+1}..a_63 (decay to the chunk end), gamma_c = E_63:
//     ke_s  = k_s Suf_s                       (<= |k|)
//     qh_t  = q~_t E_t / gamma_c = q~_t / Suf_t
//     A     = qh ke^T            -> A_ts = sum_d q~_td k_sd exp(b_td - b_sd)
//     dS^T  = V^T ke             (the chunk summary; value rows)
//     O     = tril(A) V + qh (gamma_c . S_enter)
//     S_leave = diag(gamma_c) S_enter + dS
//   GTR project page, "A Kernel That Makes Recurrence Fast": the summary
//   (dS), the boundary scan (the chain), and the output product fused with
//   the boundary readout.
// qh grows like exp(chunk decay); the whole-chunk form is used when the decay
// over the chunk is at most kChunkRange nats in every key dimension.  Other
// chunks keep the other MMAs with the safe operands qe_t = q~_t E_t (<= |q~|)
// and compute the score matrix exactly on CUDA cores.
//
// Operands live in shared memory as 64 x 64 fp16 row-major tiles with 128-byte
// rows in the 128-byte swizzled canonical layout (16-byte chunk j of row r
// stored at chunk j ^ (r mod 8)), read as K-major or MN-major by the MMA
// descriptors; a 64 x 128 operand (q, k, S'^T at d_k = 128) is two such tiles,
// key dims 0..63 then 64..127.  Accumulators: with M = 64, row m of an
// accumulator sits in TMEM lane (m mod 16) + 32 (m / 16) + base, base 0 or 16,
// so two of them share columns: A (base 0, 64 columns) and dS^T (base 16, d_k
// columns) in one MMA pass, then O over A.  Warp w reads rows 16w..16w+15 of
// either with the 16x256b load, in the m16n8 accumulator-fragment layout.
// At d_k = 128 the two value halves of a chunk are two CTAs with adjacent
// tickets: each preps the same q, k, g rows (the second read comes from L2)
// and carries its own 128 x 64 slice of the state.
#pragma once

#include "gla_tc.cuh"
#include "gla_tcgen05.cuh"

namespace gtr {

// Largest total decay over a chunk (nats) for the whole-chunk tensor-core form.
constexpr float kChunkRange = 8.0f;

// ---------------------------------------------------------------- layout
template <int DK>
struct UmmaLayout {
    static constexpr uint32_t KTILE = DK * 128;  // a 64-row operand over all key dims (DK/64 tiles)
    // all offsets relative to a 1024-byte aligned base; every tile is swizzled
    static constexpr uint32_t QH = 0;            // raw q, then the qh (or qe) tile in place
    static constexpr uint32_t KE = KTILE;        // raw k, then the ke tile in place; then S'^T
    static constexpr uint32_t SP = KE;           // (scaled entering state)^T, rows = value columns,
                                                 // written once the summary MMA has read ke
    static constexpr uint32_t V = 2 * KTILE;     // v tile, 64 value columns (also read as MN-major)
    static constexpr uint32_t P = V + 8192;      // exact path's staging, then the masked scores,
                                                 // then the output staging
    static constexpr uint32_t VEC = P + 8192;    // gamma_c[DK], unused[DK], sub-chunk totals [4][DK] (fp32)
    static constexpr uint32_t ROW = VEC + 6 * DK * 4;  // int64 [64]
    static constexpr uint32_t MISC = ROW + 64 * 8;     // tile, tmem base, mbarrier (8-aligned)
    static constexpr uint32_t BYTES = MISC + 64;
    static constexpr uint32_t ALLOC = BYTES + 1024;    // slack for aligning the base
    static constexpr uint32_t TMEM_COLS = DK;          // dS^T is the widest accumulator
    static constexpr int CTAS_PER_SM = DK == 64 ? 6 : 4;
    // swizzled operand tiles on 1024-byte boundaries; the resident CTAs fit
    // the SM's 228 KB of shared memory (1 KB reserved per CTA) and its 512
    // TMEM columns
    static_assert(QH % 1024 == 0 && KE % 1024 == 0 && V % 1024 == 0 && P % 1024 == 0, "tile alignment");
    static_assert(CTAS_PER_SM * (ALLOC + 1024) <= 228 * 1024, "shared memory per SM");
    static_assert(CTAS_PER_SM * TMEM_COLS <= 512, "tensor memory per SM");
};

// ---------------------------------------------------------------- the kernel
// Chain of boundary states: warp w owns value rows 16w..16w+15 of the CTA's
// slice of S^T (its TMEM lanes), and that slice of S_leave depends only on
// the same slice of S_enter and of dS.  So each warp waits for, reads and
// publishes its own slice, with one flag per (sequence, value half, warp): no
// CTA barrier on the chain.
template <int DK>
__global__ void __launch_bounds__(128, UmmaLayout<DK>::CTAS_PER_SM) gla_umma_kernel(const TcArgs args) {
    using L = UmmaLayout<DK>;
    // DVC value columns per CTA, NVH CTAs per (sequence, chunk); d_v = d_k
    constexpr int DVC = 64, NVH = DK / 64, DV = DK, C = 64, KT = DK / 8, NKA = DK / 64;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    // 1024-byte aligned base (the swizzled operand tiles need it)
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base_addr = (raw_addr + 1023u) & ~1023u;
    unsigned char *base = smem_raw + (base_addr - raw_addr);
    const Geom &geo = args.geo;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tr = lane >> 2, kc = 2 * (lane & 3);
    float *vGc = reinterpret_cast<float *>(base + L::VEC);
    float *vTot = vGc + 2 * DK;  // [4][DK]
    int64_t *sRow = reinterpret_cast<int64_t *>(base + L::ROW);
    int *misc = reinterpret_cast<int *>(base + L::MISC);  // [0] tile [2] tmem base; mbar at +16
    const uint32_t mbar = base_addr + L::MISC + 16;
    const int nseq = geo.B * geo.heads;
    const int nslot = nseq * NVH;  // chains: one per (sequence, value half)
    const int64_t rows = (int64_t)geo.B * geo.N * geo.heads;  // token-head rows of every tensor

    // ---- tensor memory first (before the ticket: a CTA waiting for TMEM holds no ticket)
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(base_addr + L::MISC + 8),
                     "r"(L::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
    }
    // the ticket comes from warp 1, so its round trip overlaps the allocation
    if (tid == 32) misc[0] = atomicAdd(&args.ctrl[0], 1);
    if (tid == 0) {
        mbar_init(mbar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = (uint32_t)misc[2];
    const int tile = misc[0];
    bool ok_tile = tile < geo.nc * nslot;
    if (!ok_tile && tid == 0) atomicOr(args.status, 6u);

    // chunk-major tickets; the value halves of a (sequence, chunk) adjacent
    const int c = ok_tile ? tile / nslot : 0;
    const int slot = ok_tile ? tile - c * nslot : 0;
    const int seq = slot / NVH, vh = slot - seq * NVH;
    const int b = seq / geo.heads, h = seq - b * geo.heads;
    const int t0 = c * C;
    const int len = ok_tile ? min(C, geo.N - t0) : 0;
    const float qscale = rsqrtf((float)DK);

    if (ok_tile) {
        // ---- row table: each warp its own 16 rows (tokens 16w..16w+15),
        // which are the only rows it loads, preps and stores (the exact
        // path, which reads all rows, starts with a CTA barrier)
        if (lane < 16) {
            const int t = 16 * warp + lane;
            int64_t r = (t < len) ? ((int64_t)b * geo.N + scan_pos(geo.dir, t0 + t, geo.H, geo.W, geo.N)) * geo.heads + h
                                  : (int64_t)-1;
            if (r >= 0 && !GTR_INB(r, rows, BS_UMMA_ROW)) r = -1;
            sRow[t] = r;
        }
        __syncwarp();

        // ---- q, k, v rows into swizzled tiles (one cp.async batch per warp);
        // 16-byte piece j of a q / k row goes to key tile j / 8, pieces
        // 0..7 of the CTA's 64 value columns to the v tile
        constexpr int QP = DK / 8;  // 16-byte pieces of a q or k row
        for (int idx = lane; idx < 16 * QP; idx += 32) {
            const int t = 16 * warp + idx / QP, j = idx % QP;
            const int64_t r = sRow[t];
            const bool ok = r >= 0 && GTR_INB(r * DK + j * 8 + 7, rows * DK, BS_UMMA_QKV);
            const int64_t o = ok ? r * DK + j * 8 : 0;
            const uint32_t sw = ((((j & 7) ^ (t & 7)) & 7) << 4);
            const uint32_t so = (j >> 3) * 8192 + t * 128 + sw;
            cp_async16(base + L::QH + so, args.q + o, ok);
            cp_async16(base + L::KE + so, args.k + o, ok);
            if (j < 8) {
                const bool okv = r >= 0 && GTR_INB(r * DV + vh * DVC + j * 8 + 7, rows * DV, BS_UMMA_QKV);
                cp_async16(base + L::V + t * 128 + sw, args.v + (okv ? r * DV + vh * DVC + j * 8 : 0), okv);
            }
        }
        cp_async_commit();

        // ---- g straight into registers: warp u takes sub-chunk u (tokens
        // 16u..16u+15), lane dp the key dims 64p + (2dp, 2dp+1) of each
        // 64-dim part p; one 256-byte row piece per warp load.  a_t = exp(g_t);
        // padding rows get g = 0 (a = 1).
        const int u = warp;
        float2 av[NKA][16];
#pragma unroll
        for (int p = 0; p < NKA; ++p) {
            const int d0 = 64 * p + 2 * lane;
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                const int64_t r = sRow[16 * u + t];
                av[p][t] = (r >= 0 && GTR_INB(r * DK + d0 + 1, rows * DK, BS_UMMA_G))
                               ? __ldcs(reinterpret_cast<const float2 *>(args.g + r * DK + d0))
                               : make_float2(0.f, 0.f);
            }
        }
#pragma unroll
        for (int p = 0; p < NKA; ++p) {
            float2 tot = make_float2(1.f, 1.f);
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                av[p][t] = make_float2(ex2(av[p][t].x * kLog2e), ex2(av[p][t].y * kLog2e));
                tot.x *= av[p][t].x;
                tot.y *= av[p][t].y;
            }
            *reinterpret_cast<float2 *>(vTot + u * DK + 64 * p + 2 * lane) = tot;
        }
        cp_async_wait_all();
        __syncthreads();  // sub-chunk totals and the q, k, v tiles visible

        float2 Ebase[NKA], Sbase[NKA], gam[NKA];
        bool in_range = true;
        const float lo = 3.3546263e-4f;  // e^-kChunkRange
#pragma unroll
        for (int p = 0; p < NKA; ++p) {
            const int d0 = 64 * p + 2 * lane;
            Ebase[p] = Sbase[p] = gam[p] = make_float2(1.f, 1.f);
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float2 tw = *reinterpret_cast<const float2 *>(vTot + w * DK + d0);
                if (w < u) { Ebase[p].x *= tw.x; Ebase[p].y *= tw.y; }
                if (w > u) { Sbase[p].x *= tw.x; Sbase[p].y *= tw.y; }
                gam[p].x *= tw.x;
                gam[p].y *= tw.y;
            }
            in_range = in_range && gam[p].x >= lo && gam[p].y >= lo && gam[p].x <= 1.f / lo && gam[p].y <= 1.f / lo;
        }
        // Every warp covers all key dims with the same products, so the vote
        // is the same in every warp.
        const bool gam_ok = __all_sync(0xffffffffu, in_range);
        // qh = q~ E_t / gamma_c (whole-chunk form) or qe = q~ E_t, in place
        __half2 qmax = __float2half2_rn(0.f);
#pragma unroll
        for (int p = 0; p < NKA; ++p) {
            const int d0 = 2 * lane;  // inside key tile p
            // E_t / gamma_c * qscale (or E_t * qscale), carried as one product
            float2 E = gam_ok ? make_float2(Ebase[p].x * (qscale / gam[p].x), Ebase[p].y * (qscale / gam[p].y))
                              : make_float2(Ebase[p].x * qscale, Ebase[p].y * qscale);
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                __half2 *pq = reinterpret_cast<__half2 *>(base + L::QH + p * 8192 + sw128(16 * u + t, d0));
                const __half2 qv = *pq;
                qmax = __hmax2(qmax, __habs2(qv));
                E.x *= av[p][t].x;
                E.y *= av[p][t].y;
                *pq = __hmul2(qv, __floats2half2_rn(E.x, E.y));
            }
            float2 S = Sbase[p];  // decay after token t to the chunk end
#pragma unroll
            for (int t = 15; t >= 0; --t) {
                __half2 *pk = reinterpret_cast<__half2 *>(base + L::KE + p * 8192 + sw128(16 * u + t, d0));
                *pk = __hmul2(*pk, __floats2half2_rn(S.x, S.y));
                S.x *= av[p][t].x;
                S.y *= av[p][t].y;
            }
        }
        const float2 qm = __half22float2(qmax);
        if (warp == 0) {
#pragma unroll
            for (int p = 0; p < NKA; ++p) *reinterpret_cast<float2 *>(vGc + 64 * p + 2 * lane) = gam[p];
        }
        fence_async_shared();
        tc_fence_before();
        // the whole-chunk form needs the gate range and |q~| <= 16 (qh then fits fp16)
        const bool exact = __syncthreads_or(!gam_ok || fmaxf(qm.x, qm.y) * qscale > 16.f) != 0;

        // Two MMA passes through the same TMEM columns.  Pass 1: A = qh ke^T
        // (whole-chunk form only; columns 0-63) in TMEM lanes 0-15 of each
        // 32-lane group and dS^T = V^T ke (columns 0..DK-1, one N = 64 MMA
        // chain per key tile) in lanes 16-31 (an M = 64 accumulator uses half
        // of each group).  Pass 2: O = P V + qh S' over A.  `phase` is the
        // parity of the next mbarrier completion.
        uint32_t phase = 0;
        const uint32_t aQH = base_addr + L::QH, aKE = base_addr + L::KE, aV = base_addr + L::V;
        constexpr uint32_t kDsLanes = 16u << 16;
        if (tid == 0) {
            tc_fence_after();
            if (!exact) {
                const uint32_t id = umma_idesc_f16(0, 0);
#pragma unroll
                for (int ks = 0; ks < DK / 16; ++ks) {
                    const uint32_t ko = (ks >> 2) * 8192 + 32 * (ks & 3);  // key tile, 16-dim step
                    umma_f16(tmem, umma_desc_sw128(aQH + ko, 16, 1024), umma_desc_sw128(aKE + ko, 16, 1024), id,
                             ks > 0);
                }
            }
            const uint32_t id2 = umma_idesc_f16(1, 1);
#pragma unroll
            for (int na = 0; na < NKA; ++na)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_f16(tmem + kDsLanes + 64 * na, umma_desc_sw128(aV + 2048 * ks, 8192, 1024),
                             umma_desc_sw128(aKE + na * 8192 + 2048 * ks, 8192, 1024), id2, ks > 0);
            umma_commit(mbar);
        }

        // ---- exact form: the score matrix on CUDA cores from the raw operands
        float pe[32];
        if (exact) {
            if (gam_ok) {
                // qh was written with 1 / gamma_c: rewrite qe = q~ E_t from the raw rows
#pragma unroll
                for (int p = 0; p < NKA; ++p) {
                    const int d0 = 64 * p + 2 * lane;
                    float2 E = Ebase[p];
#pragma unroll
                    for (int t = 0; t < 16; ++t) {
                        const int64_t r = sRow[16 * u + t];
                        const bool ok = r >= 0 && GTR_INB(r * DK + d0 + 1, rows * DK, BS_UMMA_EXACT);
                        const float2 gv = ok ? *reinterpret_cast<const float2 *>(args.g + r * DK + d0)
                                             : make_float2(0.f, 0.f);
                        const __half2 qv = ok ? *reinterpret_cast<const __half2 *>(args.q + r * DK + d0)
                                              : __float2half2_rn(0.f);
                        E.x *= ex2(gv.x * kLog2e);
                        E.y *= ex2(gv.y * kLog2e);
                        *reinterpret_cast<__half2 *>(base + L::QH + p * 8192 + sw128(16 * u + t, 2 * lane)) =
                            __hmul2(qv, __floats2half2_rn(E.x * qscale, E.y * qscale));
                    }
                }
                fence_async_shared();
            }
            // thread -> query row t = tid / 2, keys s in [32*(tid&1), +32)
            const int t = tid >> 1, sb = 32 * (tid & 1);
#pragma unroll
            for (int j = 0; j < 32; ++j) pe[j] = 0.f;
            // log2-domain in-chunk prefix of g, DK/16 parts of 16 dims,
            // staged in the (not yet used) score region
            __half *xq = reinterpret_cast<__half *>(base + L::P);          // [64][16]
            __half *xk = reinterpret_cast<__half *>(base + L::P + 2048);   // [64][16]
            float *xb = reinterpret_cast<float *>(base + L::P + 4096);     // [64][16]
            for (int hd = 0; hd < DK / 16; ++hd) {
                __syncthreads();
                for (int idx = tid; idx < 64 * 16; idx += 128) {
                    const int tt = idx >> 4, d = idx & 15;
                    const int64_t r = sRow[tt];
                    const int64_t o = (r < 0 ? 0 : r) * DK + 16 * hd + d;
                    const bool ok = r >= 0 && GTR_INB(o, rows * DK, BS_UMMA_EXACT);
                    xq[idx] = ok ? args.q[o] : __float2half(0.f);
                    xk[idx] = ok ? args.k[o] : __float2half(0.f);
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
                    const float qq = __half2float(xq[t * 16 + d]) * qscale;
                    const float bt = xb[t * 16 + d];
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int s = sb + j;
                        if (s <= t)
                            pe[j] = fmaf(qq * __half2float(xk[s * 16 + d]), ex2(bt - xb[s * 16 + d]), pe[j]);
                    }
                }
            }
            __syncthreads();  // the exact path's staging (in the score region) is consumed
            const int t2 = tid >> 1, sb2 = 32 * (tid & 1);
#pragma unroll
            for (int j = 0; j < 32; j += 2)
                *reinterpret_cast<uint32_t *>(base + L::P + sw128(t2, sb2 + j)) = pack_h2(pe[j], pe[j + 1]);
        }

        // ---- this warp's slice of the state entering the chunk (bounded
        // wait on the predecessor's flag for the same slice), while pass 1 runs
        // ring slot (chain, chunk parity): the chain's DK x 64 slice of the
        // state, warp-major float4 fragments
        constexpr int64_t kSlot = (int64_t)DK * DVC;
        const int64_t ring_n = (int64_t)nslot * 2 * kSlot;
        float Se[KT][4];
        int *flag = args.ctrl + 2 + (int64_t)slot * 4 + warp;
        if (c > 0) {
            const float4 *ring_in = reinterpret_cast<const float4 *>(args.ring + ((int64_t)slot * 2 + ((c - 1) & 1)) * kSlot);
            if (lane == 0 && GTR_INB(2 + (int64_t)slot * 4 + warp, 2 + (int64_t)nslot * 4, BS_UMMA_FLAG)) {
                long long spins = 0;
                while (ld_acquire(flag) < c) {
                    if (++spins > args.spin_limit) {
                        atomicOr(args.status, 6u);  // GTR_ERR_TIMEOUT
                        break;
                    }
                    __nanosleep(spins < 64 ? 32 : 256);
                }
            }
            __syncwarp();
#pragma unroll
            for (int n = 0; n < KT; ++n) {
                const int64_t e = ((int64_t)slot * 2 + ((c - 1) & 1)) * kSlot + ((warp * KT + n) * 32 + lane) * 4;
                const float4 x = GTR_INB(e + 3, ring_n, BS_UMMA_RING)
                                     ? __ldcg(ring_in + ((warp * KT + n) * 32 + lane))
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
                Se[n][0] = x.x; Se[n][1] = x.y; Se[n][2] = x.z; Se[n][3] = x.w;
            }
        } else {
#pragma unroll
            for (int n = 0; n < KT; ++n) Se[n][0] = Se[n][1] = Se[n][2] = Se[n][3] = 0.f;
        }

        if (!mbar_wait(mbar, phase) && tid == 0) atomicOr(args.status, 6u);
        phase ^= 1u;
        tc_fence_after();
        // ---- publish this warp's slice of S_leave = diag(gamma_c) S_enter + dS,
        // half the columns at a time, as soon as pass 1 is done: the chain of
        // boundary states waits on this release
        {
            const bool hold = (seq == args.hold_seq && c == args.hold_chunk);
            const bool publish = c + 1 < geo.nc && !hold;
            float4 *dst = reinterpret_cast<float4 *>(args.ring + ((int64_t)slot * 2 + (c & 1)) * kSlot);
#pragma unroll
            for (int hf = 0; hf < DK / 32; ++hf) {
                float dS[16];
                tmem_ld_16x32(tmem + kDsLanes + ((uint32_t)(32 * warp) << 16) + 32 * hf, dS);
                tc_wait_ld();
                if (publish) {
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const int n = 4 * hf + m;
                        const float2 gg = *reinterpret_cast<const float2 *>(vGc + 8 * n + kc);
                        float4 x;
                        x.x = fmaf(gg.x, Se[n][0], dS[4 * m + 0]);
                        x.y = fmaf(gg.y, Se[n][1], dS[4 * m + 1]);
                        x.z = fmaf(gg.x, Se[n][2], dS[4 * m + 2]);
                        x.w = fmaf(gg.y, Se[n][3], dS[4 * m + 3]);
                        const int64_t e = ((int64_t)slot * 2 + (c & 1)) * kSlot + ((warp * KT + n) * 32 + lane) * 4;
                        if (GTR_INB(e + 3, ring_n, BS_UMMA_RING))
                            __stcg(dst + ((warp * KT + n) * 32 + lane), x);
                    }
                }
            }
            if (publish) {
                __syncwarp();
                if (lane == 0 && GTR_INB(2 + (int64_t)slot * 4 + warp, 2 + (int64_t)nslot * 4, BS_UMMA_FLAG))
                    st_release(flag, c + 1);
            }
        }
        // ---- the masked scores P (fp16, swizzled), this warp's 16 query rows
        if (!exact) {
            float a[32];
            tmem_ld_16x64(tmem + ((uint32_t)(32 * warp) << 16), a);
            tc_wait_ld();
#pragma unroll
            for (int n = 0; n < 8; ++n) {
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const int t = 16 * warp + tr + 8 * hf, s = 8 * n + kc;
                    const float x0 = s <= t ? a[4 * n + 2 * hf] : 0.f;
                    const float x1 = s + 1 <= t ? a[4 * n + 2 * hf + 1] : 0.f;
                    *reinterpret_cast<uint32_t *>(base + L::P + sw128(t, s)) = pack_h2(x0, x1);
                }
            }
        }
        // S'^T = (sc . S_enter)^T as the K-major B operand (rows: value
        // columns), over ke (pass 1 is complete); sc = gamma_c (written before
        // the barrier that decided `exact`) or 1 in the exact form
#pragma unroll
        for (int n = 0; n < KT; ++n) {
            const float2 sc = exact ? make_float2(1.f, 1.f) : *reinterpret_cast<const float2 *>(vGc + 8 * n + kc);
            const int dv0 = 16 * warp + tr, dk = 8 * (n & 7) + kc;  // key tile n / 8
            unsigned char *sp = base + L::SP + (n >> 3) * 8192;
            *reinterpret_cast<uint32_t *>(sp + sw128(dv0, dk)) = pack_h2(sc.x * Se[n][0], sc.y * Se[n][1]);
            *reinterpret_cast<uint32_t *>(sp + sw128(dv0 + 8, dk)) = pack_h2(sc.x * Se[n][2], sc.y * Se[n][3]);
        }
        fence_async_shared();
        tc_fence_before();
        __syncthreads();  // P and S' written; A and dS^T read by every warp

        // ---- pass 2: O = P V + qh S' over A
        if (tid == 0) {
            tc_fence_after();
            const uint32_t aP = base_addr + L::P, aSP = base_addr + L::SP;
            const uint32_t id_pv = umma_idesc_f16(0, 1), id_qs = umma_idesc_f16(0, 0);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                umma_f16(tmem, umma_desc_sw128(aP + 32 * ks, 16, 1024), umma_desc_sw128(aV + 2048 * ks, 8192, 1024),
                         id_pv, ks > 0);
            if (c > 0) {
#pragma unroll
                for (int ks = 0; ks < DK / 16; ++ks) {
                    const uint32_t ko = (ks >> 2) * 8192 + 32 * (ks & 3);
                    umma_f16(tmem, umma_desc_sw128(aQH + ko, 16, 1024), umma_desc_sw128(aSP + ko, 16, 1024), id_qs, 1);
                }
            }
            umma_commit(mbar);
        }
        if (!mbar_wait(mbar, phase) && tid == 0) atomicOr(args.status, 6u);
        phase ^= 1u;
        tc_fence_after();

        // ---- store O: each warp stages its own 16 rows (swizzled, in the
        // finished score region) and writes them as 16-byte row pieces
        {
            float o[32];
            tmem_ld_16x64(tmem + ((uint32_t)(32 * warp) << 16), o);
            tc_wait_ld();
            unsigned char *st = base + L::P;
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                const int t = 16 * warp + tr, col = 8 * n + kc;
                *reinterpret_cast<uint32_t *>(st + sw128(t, col)) = pack_h2(o[4 * n], o[4 * n + 1]);
                *reinterpret_cast<uint32_t *>(st + sw128(t + 8, col)) = pack_h2(o[4 * n + 2], o[4 * n + 3]);
            }
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t = 16 * warp + 4 * i + (lane >> 3), j = lane & 7;
                if (t < len && sRow[t] >= 0 && GTR_INB(sRow[t] * DV + vh * DVC + j * 8 + 7, rows * DV, BS_UMMA_OUT))
                    *reinterpret_cast<int4 *>(args.out + sRow[t] * DV + vh * DVC + j * 8) =
                        *reinterpret_cast<const int4 *>(st + t * 128 + (((j ^ (t & 7)) & 7) << 4));
            }
        }
    }

    // ---- release tensor memory
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"(L::TMEM_COLS) : "memory");
    }
}

template <int DK>
cudaError_t launch_umma(const TcArgs &a, cudaStream_t st) {
    const size_t smem = UmmaLayout<DK>::ALLOC;
    cudaError_t e = cudaFuncSetAttribute(gla_umma_kernel<DK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // six CTAs of ~36 KB (d_k = 64) or four of ~53 KB (d_k = 128) per SM:
    // ask for the largest shared-memory carveout
    e = cudaFuncSetAttribute(gla_umma_kernel<DK>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((int64_t)a.geo.nc * a.geo.B * a.geo.heads * (DK / 64));
    gla_umma_kernel<DK><<<grid, 128, smem, st>>>(a);
    count_launch();
    return cudaGetLastError();
}

}  // namespace gtr
