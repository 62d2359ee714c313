// gla_umma.cuh -- fused GLA forward on the 5th-generation tensor cores
// (tcgen05 MMAs from shared-memory descriptors into tensor memory) for
// d_k = d_v = 64 and chunks of 64 tokens.
//
// Same schedule as the fused mode of gla_tc.cuh (one (sequence, chunk) tile
// per CTA, chunk-major tickets, boundary state chained through an L2 ring with
// release/acquire flags, bounded waits), with the chunk's dense products done
// as whole-chunk 64x64x64 MMAs:
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
// descriptors.  Accumulators: with M = 64, row m of an accumulator sits in TMEM
// lane (m mod 16) + 32 (m / 16) + base, base 0 or 16, so two of them share 64
// columns: A (base 0) and dS^T (base 16) in one MMA pass, then O over A.
// Warp w reads rows 16w..16w+15 of either with the 16x256b load, in the m16n8
// accumulator-fragment layout.
#pragma once

#include "gla_tc.cuh"
#include "gla_tcgen05.cuh"

namespace gtr {

// Largest total decay over a chunk (nats) for the whole-chunk tensor-core form.
constexpr float kChunkRange = 8.0f;

// ---------------------------------------------------------------- layout
struct UmmaLayout {
    // all offsets relative to a 1024-byte aligned base; every tile is swizzled
    static constexpr uint32_t QH = 0;          // raw q, then the qh (or qe) tile in place
    static constexpr uint32_t KE = 8192;       // raw k, then the ke tile in place; then S'^T
    static constexpr uint32_t SP = KE;         // (scaled entering state)^T, rows = value columns,
                                               // written once the summary MMA has read ke
    static constexpr uint32_t V = 16384;       // v tile (also read as MN-major)
    static constexpr uint32_t P = 24576;       // exact path's staging, then the masked scores,
                                               // then the output staging
    static constexpr uint32_t VEC = 32768;     // gamma_c[64], unused[64], sub-chunk totals [4][64] (fp32)
    static constexpr uint32_t ROW = VEC + 6 * 64 * 4;  // int64 [64]
    static constexpr uint32_t MISC = ROW + 64 * 8;     // tile, tmem base, mbarrier (8-aligned)
    static constexpr uint32_t BYTES = MISC + 64;
    static constexpr uint32_t ALLOC = BYTES + 1024;    // slack for aligning the base
};

// ---------------------------------------------------------------- the kernel
// Chain of boundary states: warp w owns value rows 16w..16w+15 of S^T (its
// TMEM lanes), and that slice of S_leave depends only on the same slice of
// S_enter and of dS.  So each warp waits for, reads and publishes its own
// slice, with one flag per (sequence, warp): no CTA barrier on the chain.
__global__ void __launch_bounds__(128, 6) gla_umma_kernel(const TcArgs args) {
    using L = UmmaLayout;
    constexpr int DK = 64, DV = 64, C = 64, KT = 8;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    // 1024-byte aligned base (the swizzled operand tiles need it)
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base_addr = (raw_addr + 1023u) & ~1023u;
    unsigned char *base = smem_raw + (base_addr - raw_addr);
    const Geom &geo = args.geo;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tr = lane >> 2, kc = 2 * (lane & 3);
    float *vGc = reinterpret_cast<float *>(base + L::VEC);
    float *vTot = vGc + 128;  // [4][64]
    int64_t *sRow = reinterpret_cast<int64_t *>(base + L::ROW);
    int *misc = reinterpret_cast<int *>(base + L::MISC);  // [0] tile [2] tmem base; mbar at +16
    const uint32_t mbar = base_addr + L::MISC + 16;
    const int nseq = geo.B * geo.heads;
    const int64_t rows = (int64_t)geo.B * geo.N * geo.heads;  // token-head rows of every tensor

    // ---- tensor memory first (before the ticket: a CTA waiting for TMEM holds no ticket)
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 64;\n" ::"r"(base_addr + L::MISC + 8)
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
    bool ok_tile = tile < geo.nc * nseq;
    if (!ok_tile && tid == 0) atomicOr(args.status, 6u);

    const int c = ok_tile ? tile / nseq : 0;
    const int seq = ok_tile ? tile - c * nseq : 0;
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

        // ---- q, k, v rows into swizzled tiles (one cp.async batch per warp)
        for (int idx = lane; idx < 16 * 8; idx += 32) {
            const int t = 16 * warp + (idx >> 3), j = idx & 7;
            const int64_t r = sRow[t];
            const bool ok = r >= 0 && GTR_INB(r * 64 + j * 8 + 7, rows * 64, BS_UMMA_QKV);
            const int64_t o = ok ? r * 64 + j * 8 : 0;
            const uint32_t so = t * 128 + (((j ^ (t & 7)) & 7) << 4);
            cp_async16(base + L::QH + so, args.q + o, ok);
            cp_async16(base + L::KE + so, args.k + o, ok);
            cp_async16(base + L::V + so, args.v + o, ok);
        }
        cp_async_commit();

        // ---- g straight into registers: warp u takes sub-chunk u (tokens
        // 16u..16u+15), lane dp the key dims (2dp, 2dp+1); one 256-byte row
        // per warp load.  a_t = exp(g_t); padding rows get g = 0 (a = 1).
        const int u = warp, d0 = 2 * lane;
        float2 av[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) {
            const int64_t r = sRow[16 * u + t];
            av[t] = (r >= 0 && GTR_INB(r * 64 + d0 + 1, rows * 64, BS_UMMA_G))
                        ? __ldcs(reinterpret_cast<const float2 *>(args.g + r * 64 + d0))
                        : make_float2(0.f, 0.f);
        }
        float2 tot = make_float2(1.f, 1.f);
#pragma unroll
        for (int t = 0; t < 16; ++t) {
            av[t] = make_float2(ex2(av[t].x * kLog2e), ex2(av[t].y * kLog2e));
            tot.x *= av[t].x;
            tot.y *= av[t].y;
        }
        *reinterpret_cast<float2 *>(vTot + u * 64 + d0) = tot;
        cp_async_wait_all();
        __syncthreads();  // sub-chunk totals and the q, k, v tiles visible

        float2 Ebase = make_float2(1.f, 1.f), Sbase = make_float2(1.f, 1.f), gam = make_float2(1.f, 1.f);
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            const float2 tw = *reinterpret_cast<const float2 *>(vTot + w * 64 + d0);
            if (w < u) { Ebase.x *= tw.x; Ebase.y *= tw.y; }
            if (w > u) { Sbase.x *= tw.x; Sbase.y *= tw.y; }
            gam.x *= tw.x;
            gam.y *= tw.y;
        }
        // Every warp covers all 64 key dims with the same products, so the
        // vote is the same in every warp.
        const float lo = 3.3546263e-4f;  // e^-kChunkRange
        const bool gam_ok = __all_sync(0xffffffffu, gam.x >= lo && gam.y >= lo && gam.x <= 1.f / lo &&
                                                        gam.y <= 1.f / lo);
        // qh = q~ E_t / gamma_c (whole-chunk form) or qe = q~ E_t, in place
        __half2 qmax = __float2half2_rn(0.f);
        {
            // E_t / gamma_c * qscale (or E_t * qscale), carried as one product
            float2 E = gam_ok ? make_float2(Ebase.x * (qscale / gam.x), Ebase.y * (qscale / gam.y))
                              : make_float2(Ebase.x * qscale, Ebase.y * qscale);
#pragma unroll
            for (int t = 0; t < 16; ++t) {
                __half2 *p = reinterpret_cast<__half2 *>(base + L::QH + sw128(16 * u + t, d0));
                const __half2 qv = *p;
                qmax = __hmax2(qmax, __habs2(qv));
                E.x *= av[t].x;
                E.y *= av[t].y;
                *p = __hmul2(qv, __floats2half2_rn(E.x, E.y));
            }
            float2 S = Sbase;  // decay after token t to the chunk end
#pragma unroll
            for (int t = 15; t >= 0; --t) {
                __half2 *p = reinterpret_cast<__half2 *>(base + L::KE + sw128(16 * u + t, d0));
                *p = __hmul2(*p, __floats2half2_rn(S.x, S.y));
                S.x *= av[t].x;
                S.y *= av[t].y;
            }
        }
        const float2 qm = __half22float2(qmax);
        if (warp == 0) *reinterpret_cast<float2 *>(vGc + d0) = gam;
        fence_async_shared();
        tc_fence_before();
        // the whole-chunk form needs the gate range and |q~| <= 16 (qh then fits fp16)
        const bool exact = __syncthreads_or(!gam_ok || fmaxf(qm.x, qm.y) * qscale > 16.f) != 0;

        // Two MMA passes through the same 64 TMEM columns.  Pass 1: A = qh ke^T
        // (whole-chunk form only) in TMEM lanes 0-15 of each 32-lane group and
        // dS^T = V^T ke in lanes 16-31 (an M = 64 accumulator uses half of each
        // group).  Pass 2: O = P V + qh S' over A.  `phase` is the parity of the
        // next mbarrier completion.
        uint32_t phase = 0;
        const uint32_t aQH = base_addr + L::QH, aKE = base_addr + L::KE, aV = base_addr + L::V;
        constexpr uint32_t kDsLanes = 16u << 16;
        if (tid == 0) {
            tc_fence_after();
            if (!exact) {
                const uint32_t id = umma_idesc_f16(0, 0);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_f16(tmem, umma_desc_sw128(aQH + 32 * ks, 16, 1024), umma_desc_sw128(aKE + 32 * ks, 16, 1024),
                             id, ks > 0);
            }
            const uint32_t id2 = umma_idesc_f16(1, 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                umma_f16(tmem + kDsLanes, umma_desc_sw128(aV + 2048 * ks, 8192, 1024),
                         umma_desc_sw128(aKE + 2048 * ks, 8192, 1024), id2, ks > 0);
            umma_commit(mbar);
        }

        // ---- exact form: the score matrix on CUDA cores from the raw operands
        float pe[32];
        if (exact) {
            if (gam_ok) {
                // qh was written with 1 / gamma_c: rewrite qe = q~ E_t from the raw rows
                float2 E = Ebase;
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    const int64_t r = sRow[16 * u + t];
                    const bool ok = r >= 0 && GTR_INB(r * 64 + d0 + 1, rows * 64, BS_UMMA_EXACT);
                    const float2 gv = ok ? *reinterpret_cast<const float2 *>(args.g + r * 64 + d0)
                                         : make_float2(0.f, 0.f);
                    const __half2 qv = ok ? *reinterpret_cast<const __half2 *>(args.q + r * 64 + d0)
                                          : __float2half2_rn(0.f);
                    E.x *= ex2(gv.x * kLog2e);
                    E.y *= ex2(gv.y * kLog2e);
                    *reinterpret_cast<__half2 *>(base + L::QH + sw128(16 * u + t, d0)) =
                        __hmul2(qv, __floats2half2_rn(E.x * qscale, E.y * qscale));
                }
                fence_async_shared();
            }
            // thread -> query row t = tid / 2, keys s in [32*(tid&1), +32)
            const int t = tid >> 1, sb = 32 * (tid & 1);
#pragma unroll
            for (int j = 0; j < 32; ++j) pe[j] = 0.f;
            // log2-domain in-chunk prefix of g, four quarters of 16 dims,
            // staged in the (not yet used) score region
            __half *xq = reinterpret_cast<__half *>(base + L::P);          // [64][16]
            __half *xk = reinterpret_cast<__half *>(base + L::P + 2048);   // [64][16]
            float *xb = reinterpret_cast<float *>(base + L::P + 4096);     // [64][16]
            for (int hd = 0; hd < 4; ++hd) {
                __syncthreads();
                for (int idx = tid; idx < 64 * 16; idx += 128) {
                    const int tt = idx >> 4, d = idx & 15;
                    const int64_t r = sRow[tt];
                    const int64_t o = (r < 0 ? 0 : r) * 64 + 16 * hd + d;
                    const bool ok = r >= 0 && GTR_INB(o, rows * 64, BS_UMMA_EXACT);
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
        float Se[KT][4];
        int *flag = args.ctrl + 2 + (int64_t)seq * 4 + warp;
        if (c > 0) {
            const float4 *ring_in =
                reinterpret_cast<const float4 *>(args.ring + ((int64_t)seq * 2 + ((c - 1) & 1)) * (DK * DV));
            if (lane == 0 && GTR_INB(2 + (int64_t)seq * 4 + warp, 2 + (int64_t)nseq * 4, BS_UMMA_FLAG)) {
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
                const int64_t e = ((int64_t)seq * 2 + ((c - 1) & 1)) * (DK * DV) + ((warp * KT + n) * 32 + lane) * 4;
                const float4 x = GTR_INB(e + 3, (int64_t)nseq * 2 * DK * DV, BS_UMMA_RING)
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
            float4 *dst = reinterpret_cast<float4 *>(args.ring + ((int64_t)seq * 2 + (c & 1)) * (DK * DV));
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
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
                        const int64_t e = ((int64_t)seq * 2 + (c & 1)) * (DK * DV) + ((warp * KT + n) * 32 + lane) * 4;
                        if (GTR_INB(e + 3, (int64_t)nseq * 2 * DK * DV, BS_UMMA_RING))
                            __stcg(dst + ((warp * KT + n) * 32 + lane), x);
                    }
                }
            }
            if (publish) {
                __syncwarp();
                if (lane == 0 && GTR_INB(2 + (int64_t)seq * 4 + warp, 2 + (int64_t)nseq * 4, BS_UMMA_FLAG))
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
            const int dv0 = 16 * warp + tr, dk = 8 * n + kc;
            *reinterpret_cast<uint32_t *>(base + L::SP + sw128(dv0, dk)) = pack_h2(sc.x * Se[n][0], sc.y * Se[n][1]);
            *reinterpret_cast<uint32_t *>(base + L::SP + sw128(dv0 + 8, dk)) = pack_h2(sc.x * Se[n][2], sc.y * Se[n][3]);
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
                for (int ks = 0; ks < 4; ++ks)
                    umma_f16(tmem, umma_desc_sw128(aQH + 32 * ks, 16, 1024),
                             umma_desc_sw128(aSP + 32 * ks, 16, 1024), id_qs, 1);
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
                if (t < len && sRow[t] >= 0 && GTR_INB(sRow[t] * DV + j * 8 + 7, rows * DV, BS_UMMA_OUT))
                    *reinterpret_cast<int4 *>(args.out + sRow[t] * DV + j * 8) =
                        *reinterpret_cast<const int4 *>(st + t * 128 + (((j ^ (t & 7)) & 7) << 4));
            }
        }
    }

    // ---- release tensor memory
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 64;\n" ::"r"(tmem) : "memory");
    }
}

inline cudaError_t launch_umma(const TcArgs &a, cudaStream_t st) {
    const size_t smem = UmmaLayout::ALLOC;
    cudaError_t e = cudaFuncSetAttribute(gla_umma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // six CTAs of ~36 KB per SM: ask for the largest shared-memory carveout
    e = cudaFuncSetAttribute(gla_umma_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((int64_t)a.geo.nc * a.geo.B * a.geo.heads);
    gla_umma_kernel<<<grid, 128, smem, st>>>(a);
    count_launch();
    return cudaGetLastError();
}

}  // namespace gtr
