// gtr_gla_api.cu -- the C ABI (include/gtr_gla.h): argument checks, the
// internal workspace, and dispatch to the kernels.  Host code only.
#include "gtr_gla.h"

#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>
#include <vector>

#include "gla_common.cuh"
#include "gla_tc.cuh"
#include "gla_walk.cuh"

namespace gtr {

static std::atomic<uint64_t> g_launches{0};
void count_launch(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

// Readers of the per-translation-unit bounds reports (checked builds only
// register any); function-local statics, so registration at load time does
// not depend on the order in which translation units initialise.
std::mutex &bounds_readers_mu() {
    static std::mutex mu;
    return mu;
}
std::vector<BoundsReader> &bounds_readers() {
    static std::vector<BoundsReader> readers;
    return readers;
}
void register_bounds_reader(BoundsReader reader) {
    std::lock_guard<std::mutex> lk(bounds_readers_mu());
    bounds_readers().push_back(reader);
}

namespace {

thread_local char t_err[256] = "";

gtr_status_t fail(gtr_status_t s, const char *fmt, const char *detail = "") {
    std::snprintf(t_err, sizeof t_err, fmt, detail);
    return s;
}

void t_err_clear() { t_err[0] = '\0'; }

gtr_status_t cuda_fail(cudaError_t e, const char *what) {
    std::snprintf(t_err, sizeof t_err, "%s: %s", what, cudaGetErrorString(e));
    return GTR_ERR_CUDA;
}

bool supported_d(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }
bool supported_chunk(int c) { return c == 16 || c == 32 || c == 64; }
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Range {
    uintptr_t lo, hi;
};
Range span(const void *p, size_t bytes) {
    uintptr_t a = reinterpret_cast<uintptr_t>(p);
    return {a, a + bytes};
}
bool overlap(Range a, Range b) { return a.lo < b.hi && b.lo < a.hi && a.hi > a.lo && b.hi > b.lo; }

// Shape checks common to every token-layout entry point.  Sets `geo`.
// Returns GTR_OK, or an error; `empty` is set when there is no work.
gtr_status_t check_shape(int B, int heads, int grid_h, int grid_w, int d_k, int d_v,
                         int direction, int chunk, Geom &geo, bool &empty) {
    if (B < 0 || heads < 0 || grid_h < 0 || grid_w < 0)
        return fail(GTR_ERR_INVALID_ARG, "negative size%s");
    if (direction < 0 || direction > 3) return fail(GTR_ERR_INVALID_ARG, "bad direction%s");
    if (!supported_d(d_k) || !supported_d(d_v))
        return fail(GTR_ERR_UNSUPPORTED_SHAPE, "d_k and d_v must be 16, 32, 64 or 128%s");
    if (!supported_chunk(chunk))
        return fail(GTR_ERR_UNSUPPORTED_SHAPE, "chunk must be 16, 32 or 64%s");
    int64_t N = (int64_t)grid_h * grid_w;
    if (N > (int64_t)1 << 30) return fail(GTR_ERR_UNSUPPORTED_SHAPE, "more than 2^30 tokens%s");
    empty = (B == 0 || heads == 0 || N == 0);
    int64_t nc = (N + chunk - 1) / chunk;
    if (!empty && nc * B * heads >= ((int64_t)1 << 31))
        return fail(GTR_ERR_UNSUPPORTED_SHAPE, "more than 2^31 chunk tiles%s");
    geo.B = B; geo.heads = heads; geo.H = grid_h; geo.W = grid_w;
    geo.dk = d_k; geo.dv = d_v; geo.dir = direction; geo.chunk = chunk;
    geo.N = (int)N; geo.nc = (int)nc;
    return GTR_OK;
}

size_t tok_bytes(const Geom &g, int d, size_t elem) {
    return (size_t)g.B * g.N * g.heads * d * elem;
}

// Internal workspaces: one grow-only, zero-initialised device buffer per
// (device, stream, kind).  Kinds keep the schedules apart: the fused
// kernel's control words must never be overwritten by another schedule.
enum WsKind {
    WS_THREE_PHASE = 0, WS_FUSED = 1, WS_STAGING = 2, WS_STATUS = 3, WS_SCAN = 4
};
struct Workspace {
    void *ptr = nullptr;
    size_t bytes = 0;
};
struct WsKey {
    int dev;
    cudaStream_t st;
    int kind;
    bool operator<(const WsKey &o) const {
        if (dev != o.dev) return dev < o.dev;
        if (st != o.st) return st < o.st;
        return kind < o.kind;
    }
};
std::mutex g_ws_mu;
std::map<WsKey, Workspace> g_ws;

gtr_status_t get_workspace(size_t bytes, cudaStream_t st, void **out, int kind = WS_THREE_PHASE) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    std::lock_guard<std::mutex> lk(g_ws_mu);
    Workspace &w = g_ws[WsKey{dev, st, kind}];
    if (w.bytes < bytes) {
        // Growing is stream-ordered on `st` (the only stream that uses this
        // workspace): the old buffer is freed after the work already queued
        // on it, the new one is allocated and zeroed in stream order.  An
        // allocation cannot be recorded into a stream capture.
        cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
        if ((e = cudaStreamIsCapturing(st, &cap)) != cudaSuccess) return cuda_fail(e, "cudaStreamIsCapturing");
        if (cap != cudaStreamCaptureStatusNone)
            return fail(GTR_ERR_INVALID_ARG,
                        "the internal workspace must grow, which cannot happen inside a stream capture; "
                        "make a first call of this size on this stream before capturing%s");
        if (w.ptr) {
            e = cudaFreeAsync(w.ptr, st);
            w.ptr = nullptr;
            w.bytes = 0;
            if (e != cudaSuccess) return cuda_fail(e, "cudaFreeAsync");
        }
        size_t want = (bytes + 0xFFFFF) & ~(size_t)0xFFFFF;  // round up to 1 MiB
        e = cudaMallocAsync(&w.ptr, want, st);
        if (e != cudaSuccess) {
            w.ptr = nullptr;
            cudaGetLastError();
            return fail(GTR_ERR_OOM, "workspace allocation failed%s");
        }
        e = cudaMemsetAsync(w.ptr, 0, want, st);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
        w.bytes = want;
    }
    *out = w.ptr;
    return GTR_OK;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

size_t three_phase_ws(const Geom &g) {
    size_t nseq = (size_t)g.B * g.heads;
    return align256(nseq * g.nc * g.dk * g.dv * sizeof(float)) +
           align256(nseq * g.nc * g.dk * sizeof(float)) + align256(scan_agg_bytes((int64_t)nseq, g.nc, g.dk, g.dv));
}

// Fused kernels: control words (ticket, unused, four flags per sequence and
// 64 value columns: the mma.sync kernel uses one per sequence, the tcgen05
// kernel one per (value half, warp)) then a two-slot ring of boundary states
// per sequence.
size_t fused_ctrl_bytes(const Geom &g) {
    return align256(((size_t)g.B * g.heads * 4 * ((g.dv + 63) / 64) + 2) * sizeof(int));
}
size_t fused_ws(const Geom &g) {
    return fused_ctrl_bytes(g) + (size_t)g.B * g.heads * 2 * g.dk * g.dv * sizeof(float);
}
// Device status word of (current device, stream), zeroed at creation: the
// kernels a call enqueues on `st` record a bounded wait that gave up here.
gtr_status_t status_word(cudaStream_t st, unsigned **out) {
    void *p = nullptr;
    gtr_status_t s = get_workspace(256, st, &p, WS_STATUS);
    *out = static_cast<unsigned *>(p);
    return s;
}

constexpr int kSchedLast = GTR_SCHED_THREE_PHASE_MMA;  // largest gtr_schedule_t value
constexpr long long kSpinLimit = 1LL << 22;  // bounded wait: about a second of polling
// At most this many (batch, head) sequences: GTR_SCHED_AUTO runs the
// three-phase schedule (the fused chain is the bottleneck then).  Measured at
// 40x40, d = 64: three phases win at 24 sequences, the two-chunk fused
// kernel from 48.
constexpr int64_t kFewSequences = 24;

// Streaming multiprocessors of the current device (cached per device).
cudaError_t sm_count(int *out) {
    static std::mutex mu;
    static std::map<int, int> cache;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lk(mu);
    auto it = cache.find(dev);
    if (it == cache.end()) {
        int n = 0;
        if ((e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        it = cache.emplace(dev, n).first;
    }
    *out = it->second;
    return cudaSuccess;
}

TcArgs make_args(const __half *q, const __half *k, const __half *v, const float *g, const Geom &geo) {
    TcArgs a;
    a.q = q; a.k = k; a.v = v; a.g = g; a.geo = geo;
    a.dS = nullptr; a.gamma = nullptr; a.S_enter = nullptr; a.out = nullptr;
    a.dS_h = nullptr; a.S_enter_h = nullptr;
    a.ctrl = nullptr; a.ring = nullptr; a.status = nullptr;
    a.spin_limit = kSpinLimit; a.hold_seq = -1; a.hold_chunk = -1;
    a.pdl = false;
    return a;
}

// Shapes of the chained tcgen05 kernel (its tile index, chunk-major over
// (sequence, 64 value columns), is a 32-bit int).
bool tcgen05_shape(const Geom &g) {
    return g.dk == g.dv && (g.dk == 64 || g.dk == 128) && g.chunk == 64 &&
           (int64_t)g.B * g.heads * g.nc * (g.dv / 64) < ((int64_t)1 << 31);
}
// Shapes of the tcgen05 walk kernel (and of the tcgen05 three-phase phases).
bool walk_shape(const Geom &g) {
    return g.chunk == 64 && (g.dk == 32 || g.dk == 64 || g.dk == 128) && (g.dv == 64 || g.dv == 128) &&
           (int64_t)g.B * g.heads * g.nc * (g.dv / 64) < ((int64_t)1 << 31);
}

// The kernels a schedule launches for a problem: a host-only decision, so
// it can be asked without a device (gtr_gla_plan).  With chain_only (the
// bounded-wait test hook) AUTO keeps to the fused kernels whose tiles wait
// on one another.
gtr_plan_t plan_for(const Geom &geo, int schedule, int sms, bool chain_only = false) {
    const int64_t nseq = (int64_t)geo.B * geo.heads;
    if (schedule == GTR_SCHED_THREE_PHASE) return GTR_PLAN_THREE_PHASE;
    if (schedule == GTR_SCHED_THREE_PHASE_MMA) return GTR_PLAN_THREE_PHASE_MMA;
    if (schedule == GTR_SCHED_THREE_PHASE_SIMT) return GTR_PLAN_THREE_PHASE_SIMT;
    if (schedule == GTR_SCHED_WALK_TCGEN05 && walk_shape(geo)) return GTR_PLAN_WALK_TCGEN05;
    // With few sequences every per-sequence chain (the fused kernels' hand-
    // over of boundary states, or the walk's chunk loop) is long next to the
    // work; the three-phase schedule has chunk-parallel phases and a
    // pipelined scan, and its state traffic is small then, so AUTO takes it
    // (with the mma.sync phases: measured faster there than the tcgen05 ones,
    // whose one-chunk CTAs wait on their own tensor-core passes).
    if (schedule == GTR_SCHED_AUTO && !chain_only && nseq <= kFewSequences) return GTR_PLAN_THREE_PHASE_MMA;
    // The walk keeps each (sequence, value slice) on one CTA with no chain
    // between CTAs; it is the fastest measured when those items fill between
    // two and three CTAs per SM (one wave at its occupancy of 3 per SM for
    // d_k <= 64): the batched workload.  Fewer items leave SMs idle, more
    // need a second wave.
    const int64_t items = nseq * (geo.dv / 64);
    if (schedule == GTR_SCHED_AUTO && !chain_only && walk_shape(geo) && geo.dk <= 64 && items >= 2 * (int64_t)sms &&
        items <= 3 * (int64_t)sms)
        return GTR_PLAN_WALK_TCGEN05;
    // Few sequences leave the chain of boundary states as the critical path:
    // then two chunks per tile halve its length (d_v <= 64).  Many sequences
    // keep every SM busy anyway: then one chunk per tile gives more resident
    // CTAs.  The chained tcgen05 kernel does one chunk per tile (AUTO takes
    // it at d_k = 64).
    const bool pair = nseq < 2 * (int64_t)sms;
    if (tcgen05_shape(geo) &&
        (schedule == GTR_SCHED_FUSED_TCGEN05 || (schedule == GTR_SCHED_AUTO && !pair && geo.dk == 64)))
        return GTR_PLAN_FUSED_TCGEN05;
    return (pair && geo.dv <= 64) ? GTR_PLAN_FUSED_MMA_PAIR : GTR_PLAN_FUSED_MMA;
}

// Grid of a persistent walk launch over `items` work items: every resident
// CTA slot of the device, at most one per item (cached per device and mode).
cudaError_t walk_grid(int dk, int mode, int64_t items, int *grid) {
    static std::mutex mu;
    static std::map<std::pair<int, int>, int> cache;  // (device, dk*8 + mode) -> slots
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if ((e = sm_count(&sms)) != cudaSuccess) return e;
    int slots = 0;
    {
        std::lock_guard<std::mutex> lk(mu);
        auto key = std::make_pair(dev, dk * 8 + mode);
        auto it = cache.find(key);
        if (it == cache.end()) {
            int per_sm = 0;
            if ((e = walk_ctas_per_sm(dk, mode, &per_sm)) != cudaSuccess) return e;
            it = cache.emplace(key, std::max(1, per_sm) * sms).first;
        }
        slots = it->second;
    }
    *grid = (int)std::min<int64_t>(items, slots);
    return cudaSuccess;
}

WalkArgs make_walk_args(const __half *q, const __half *k, const __half *v, const float *g, const Geom &geo,
                        unsigned *status) {
    WalkArgs a;
    std::memset(&a, 0, sizeof a);
    a.q = q; a.k = k; a.v = v; a.g = g; a.geo = geo; a.status = status;
    a.vs = geo.dv / 64;
    return a;
}

// The whole forward as one walk launch: one CTA per (sequence, value slice).
// S0 / SN: initial and final states [B*heads][d_k][d_v] fp32, or null.
gtr_status_t run_walk(const __half *q, const __half *k, const __half *v, const float *g, const Geom &geo,
                      __half *out, cudaStream_t st, const float *S0 = nullptr, float *SN = nullptr,
                      const __half *gate = nullptr, const float *norm_w = nullptr, float norm_eps = 0.f,
                      bool bf16 = false) {
    unsigned *status = nullptr;
    gtr_status_t s = status_word(st, &status);
    if (s != GTR_OK) return s;
    WalkArgs a = make_walk_args(q, k, v, g, geo, status);
    a.out = out;
    a.S0 = S0;
    a.SN = SN;
    a.gate = gate;
    a.norm_w = norm_w;
    a.norm_eps = norm_eps;
    a.items = geo.B * geo.heads * a.vs;
    // launched programmatically: the kernel waits for the grid ahead of it
    // before it touches global memory, so only its set-up overlaps that grid
    a.pdl = true;
    cudaError_t e = launch_walk(a, WALK_SEQ, a.items, st, bf16);
    return e == cudaSuccess ? GTR_OK : cuda_fail(e, "walk kernel launch");
}

gtr_status_t run_fused(const __half *q, const __half *k, const __half *v, const float *g,
                       const Geom &geo, __half *out, cudaStream_t st, gtr_plan_t plan,
                       int hold_seq = -1, int hold_chunk = -1, long long spin_limit = kSpinLimit) {
    void *ws = nullptr;
    gtr_status_t s = get_workspace(fused_ws(geo), st, &ws, WS_FUSED);
    if (s != GTR_OK) return s;
    unsigned *status = nullptr;
    if ((s = status_word(st, &status)) != GTR_OK) return s;
    TcArgs a = make_args(q, k, v, g, geo);
    a.out = out;
    a.ctrl = static_cast<int *>(ws);
    a.ring = reinterpret_cast<float *>(static_cast<char *>(ws) + fused_ctrl_bytes(geo));
    a.status = status;
    a.spin_limit = spin_limit;
    a.hold_seq = hold_seq;
    a.hold_chunk = hold_chunk;
    // Ticket and flags start from zero for every launch (a memset of the
    // current problem's control words, recorded into a graph with the
    // launch when captured).
    cudaError_t e = cudaMemsetAsync(a.ctrl, 0, fused_ctrl_bytes(geo), st);
    if (e != cudaSuccess) return cuda_fail(e, "control-word reset");
    if (plan == GTR_PLAN_FUSED_TCGEN05)
        e = launch_fused_umma(a, st);
    else
        e = launch_tc(a, plan == GTR_PLAN_FUSED_MMA_PAIR ? TC_FUSED_PAIR : TC_FUSED, st);
    return e == cudaSuccess ? GTR_OK : cuda_fail(e, "fused kernel launch");
}

// Phase 1 and phase 3 on tensor cores: the tcgen05 walk kernel in its
// single-chunk modes for its shapes, the mma.sync kernel otherwise.
// pdl: launched with programmatic stream serialization (the kernel waits for
// the grid ahead of it before it touches global memory).
cudaError_t summary_tc(const __half *k, const __half *v, const float *g, const Geom &geo, float *dS,
                       float *gamma, cudaStream_t st, unsigned *status, bool tcgen05 = true, bool pdl = false,
                       __half *dS_h = nullptr) {
    if (tcgen05 && walk_shape(geo)) {
        WalkArgs a = make_walk_args(nullptr, k, v, g, geo, status);
        a.pdl = pdl;
        a.dS = dS;
        a.gamma = gamma;
        a.items = geo.B * geo.heads * geo.nc * a.vs;
        int grid = 0;
        cudaError_t e = walk_grid(geo.dk, WALK_SUMMARY, a.items, &grid);
        if (e != cudaSuccess) return e;
        return launch_walk(a, WALK_SUMMARY, grid, st);
    }
    TcArgs a = make_args(nullptr, k, v, g, geo);
    a.pdl = pdl;
    a.dS = dS;
    a.dS_h = dS_h;
    a.gamma = gamma;
    return launch_tc(a, TC_SUMMARY, st);
}

// pdl: launched with programmatic stream serialization after the scan.
cudaError_t output_tc(const __half *q, const __half *k, const __half *v, const float *g,
                      const float *S_enter, const Geom &geo, __half *out, cudaStream_t st, unsigned *status,
                      bool tcgen05 = true, bool pdl = false, const __half *S_enter_h = nullptr) {
    if (tcgen05 && walk_shape(geo)) {
        WalkArgs a = make_walk_args(q, k, v, g, geo, status);
        a.pdl = pdl;
        a.S_enter = S_enter;
        a.out = out;
        a.items = geo.B * geo.heads * geo.nc * a.vs;
        int grid = 0;
        cudaError_t e = walk_grid(geo.dk, WALK_OUTPUT, a.items, &grid);
        if (e != cudaSuccess) return e;
        return launch_walk(a, WALK_OUTPUT, grid, st);
    }
    TcArgs a = make_args(q, k, v, g, geo);
    a.pdl = pdl;
    a.S_enter = S_enter;
    a.S_enter_h = S_enter_h;
    a.out = out;
    return launch_tc(a, TC_OUTPUT, st);
}

// Three-phase schedule; `simt` selects the CUDA-core summary/output kernels.
gtr_status_t run_three_phase(const __half *q, const __half *k, const __half *v, const float *g,
                             const Geom &geo, __half *out, cudaStream_t st, gtr_plan_t plan) {
    const bool simt = plan == GTR_PLAN_THREE_PHASE_SIMT, mma = plan == GTR_PLAN_THREE_PHASE_MMA;
    void *ws = nullptr;
    gtr_status_t s = get_workspace(three_phase_ws(geo), st, &ws);
    if (s != GTR_OK) return s;
    unsigned *status = nullptr;
    if ((s = status_word(st, &status)) != GTR_OK) return s;
    size_t nseq = (size_t)geo.B * geo.heads;
    float *dS = static_cast<float *>(ws);
    float *gamma = reinterpret_cast<float *>(static_cast<char *>(ws) +
                                             align256(nseq * geo.nc * geo.dk * geo.dv * sizeof(float)));
    // the mma.sync phases keep dS and S_enter in fp16 (the output phase's
    // readout takes the entering state as fp16 tensor-core operands anyway;
    // the scan's running state stays fp32): half the state traffic
    __half *dSh = mma ? static_cast<__half *>(ws) : nullptr;
    cudaError_t e = simt ? launch_summary_v0(k, v, g, geo, dS, gamma, st)
                         : summary_tc(k, v, g, geo, dS, gamma, st, status, !mma, true, dSh);
    if (e != cudaSuccess) return cuda_fail(e, "chunk summary launch");
    float *agg = reinterpret_cast<float *>(reinterpret_cast<char *>(gamma) +
                                           align256(nseq * geo.nc * geo.dk * sizeof(float)));
    // the tensor-core phases and the scan are launched programmatically: each
    // starts while the grid ahead of it finishes and waits for it where it
    // first needs it (the summary before any access to global memory, the
    // scan before it reads dS, the output phase after its loads and its
    // within-chunk work, before it reads S_enter)
    e = mma ? launch_scan_segmented(dSh, gamma, (int)nseq, geo.nc, geo.dk, geo.dv, dSh, agg, st, true)
            : launch_scan_segmented(dS, gamma, (int)nseq, geo.nc, geo.dk, geo.dv, dS, agg, st, true);
    if (e != cudaSuccess) return cuda_fail(e, "boundary scan launch");
    e = simt ? launch_output_v0(q, k, v, g, dS, geo, out, st)
             : output_tc(q, k, v, g, dS, geo, out, st, status, !mma, true, dSh);
    if (e != cudaSuccess) return cuda_fail(e, "chunk output launch");
    return GTR_OK;
}

gtr_status_t forward_impl(const void *q, const void *k, const void *v, const float *g, int B,
                          int heads, int grid_h, int grid_w, int d_k, int d_v, int direction,
                          int chunk, int schedule, void *out, void *stream) {
    t_err[0] = '\0';
    Geom geo;
    bool empty = false;
    gtr_status_t s = check_shape(B, heads, grid_h, grid_w, d_k, d_v, direction, chunk, geo, empty);
    if (s != GTR_OK) return s;
    if (schedule < GTR_SCHED_AUTO || schedule > kSchedLast)
        return fail(GTR_ERR_INVALID_ARG, "bad schedule%s");
    if (!q || !k || !v || !g || !out) return fail(GTR_ERR_INVALID_ARG, "null pointer%s");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(out))
        return fail(GTR_ERR_MISALIGNED, "device pointers must be 16-byte aligned%s");
    Range ro = span(out, tok_bytes(geo, d_v, 2));
    if (overlap(ro, span(q, tok_bytes(geo, d_k, 2))) || overlap(ro, span(k, tok_bytes(geo, d_k, 2))) ||
        overlap(ro, span(v, tok_bytes(geo, d_v, 2))) || overlap(ro, span(g, tok_bytes(geo, d_k, 4))))
        return fail(GTR_ERR_ALIAS, "out overlaps an input%s");
    if (empty) return GTR_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const __half *hq = static_cast<const __half *>(q), *hk = static_cast<const __half *>(k);
    const __half *hv = static_cast<const __half *>(v);
    __half *ho = static_cast<__half *>(out);
    int sms = 0;
    cudaError_t e = sm_count(&sms);
    if (e != cudaSuccess) return cuda_fail(e, "device query");
    const gtr_plan_t plan = plan_for(geo, schedule, sms);
    if (plan == GTR_PLAN_THREE_PHASE || plan == GTR_PLAN_THREE_PHASE_SIMT || plan == GTR_PLAN_THREE_PHASE_MMA)
        return run_three_phase(hq, hk, hv, g, geo, ho, st, plan);
    if (plan == GTR_PLAN_WALK_TCGEN05) return run_walk(hq, hk, hv, g, geo, ho, st);
    return run_fused(hq, hk, hv, g, geo, ho, st, plan);
}

// Checks shared by the walk-only entry points (state in/out, gated output):
// the forward's checks plus the walk kernel's shapes.
gtr_status_t check_walk_call(const void *q, const void *k, const void *v, const float *g, int B, int heads,
                             int grid_h, int grid_w, int d_k, int d_v, int direction, int chunk, const void *out,
                             Geom &geo, bool &empty) {
    gtr_status_t s = check_shape(B, heads, grid_h, grid_w, d_k, d_v, direction, chunk, geo, empty);
    if (s != GTR_OK) return s;
    if (!walk_shape(geo))
        return fail(GTR_ERR_UNSUPPORTED_SHAPE, "this call needs chunk 64, d_k in {32, 64, 128}, d_v in {64, 128}%s");
    if (!q || !k || !v || !g || !out) return fail(GTR_ERR_INVALID_ARG, "null pointer%s");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(out))
        return fail(GTR_ERR_MISALIGNED, "device pointers must be 16-byte aligned%s");
    Range ro = span(out, tok_bytes(geo, d_v, 2));
    if (overlap(ro, span(q, tok_bytes(geo, d_k, 2))) || overlap(ro, span(k, tok_bytes(geo, d_k, 2))) ||
        overlap(ro, span(v, tok_bytes(geo, d_v, 2))) || overlap(ro, span(g, tok_bytes(geo, d_k, 4))))
        return fail(GTR_ERR_ALIAS, "out overlaps an input%s");
    return GTR_OK;
}

}  // namespace

// The calling thread's failure text, for entry points in other translation
// units (gtr_gla_last_error returns it).
int set_last_error(int s, const char *msg) {
    std::snprintf(t_err, sizeof t_err, "%s", msg);
    return s;
}
void clear_last_error() { t_err[0] = '\0'; }

}  // namespace gtr

using namespace gtr;

extern "C" {

gtr_status_t gtr_gla_forward(const void *q, const void *k, const void *v, const float *g, int B,
                             int heads, int grid_h, int grid_w, int d_k, int d_v, int direction,
                             int chunk, void *out, void *stream) {
    return forward_impl(q, k, v, g, B, heads, grid_h, grid_w, d_k, d_v, direction, chunk,
                        GTR_SCHED_AUTO, out, stream);
}

gtr_status_t gtr_gla_forward_ex(const void *q, const void *k, const void *v, const float *g,
                                int B, int heads, int grid_h, int grid_w, int d_k, int d_v,
                                int direction, int chunk, int schedule, void *out, void *stream) {
    return forward_impl(q, k, v, g, B, heads, grid_h, grid_w, d_k, d_v, direction, chunk,
                        schedule, out, stream);
}

gtr_status_t gtr_gla_forward_state(const void *q, const void *k, const void *v, const float *g,
                                              const float *S0, int B, int heads, int grid_h, int grid_w,
                                              int d_k, int d_v, int direction, int chunk, void *out, float *SN,
                                              void *stream) {
    t_err_clear();
    Geom geo;
    bool empty = false;
    gtr_status_t s = check_walk_call(q, k, v, g, B, heads, grid_h, grid_w, d_k, d_v, direction, chunk, out,
                                     geo, empty);
    if (s != GTR_OK) return s;
    if ((S0 && !aligned16(S0)) || (SN && !aligned16(SN)))
        return fail(GTR_ERR_MISALIGNED, "S0 and SN must be 16-byte aligned%s");
    const size_t sb = (size_t)B * heads * d_k * d_v * 4;
    if (SN) {
        const Range rn = span(SN, sb);
        if (overlap(rn, span(q, tok_bytes(geo, d_k, 2))) || overlap(rn, span(k, tok_bytes(geo, d_k, 2))) ||
            overlap(rn, span(v, tok_bytes(geo, d_v, 2))) || overlap(rn, span(g, tok_bytes(geo, d_k, 4))) ||
            overlap(rn, span(out, tok_bytes(geo, d_v, 2))))
            return fail(GTR_ERR_ALIAS, "SN overlaps an input or out%s");
        if (S0 && S0 != SN && overlap(rn, span(S0, sb))) return fail(GTR_ERR_ALIAS, "SN partially overlaps S0%s");
    }
    if (S0 && overlap(span(out, tok_bytes(geo, d_v, 2)), span(S0, sb))) return fail(GTR_ERR_ALIAS, "out overlaps S0%s");
    if (empty) {
        // no token: the final state is the initial one (or zero)
        if (!SN || B == 0 || heads == 0) return GTR_OK;
        cudaError_t e = S0 ? (S0 == SN ? cudaSuccess
                                       : cudaMemcpyAsync(SN, S0, sb, cudaMemcpyDeviceToDevice, (cudaStream_t)stream))
                           : cudaMemsetAsync(SN, 0, sb, (cudaStream_t)stream);
        return e == cudaSuccess ? GTR_OK : cuda_fail(e, "empty-problem state copy");
    }
    return run_walk(static_cast<const __half *>(q), static_cast<const __half *>(k), static_cast<const __half *>(v),
                    g, geo, static_cast<__half *>(out), static_cast<cudaStream_t>(stream), S0, SN);
}

gtr_status_t gtr_gla_forward_bf16(const void *q, const void *k, const void *v, const float *g, int B, int heads,
                                  int grid_h, int grid_w, int d_k, int d_v, int direction, int chunk, void *out,
                                  void *stream) {
    t_err_clear();
    Geom geo;
    bool empty = false;
    gtr_status_t s = check_walk_call(q, k, v, g, B, heads, grid_h, grid_w, d_k, d_v, direction, chunk, out,
                                     geo, empty);
    if (s != GTR_OK) return s;
    if (empty) return GTR_OK;
    // the buffers hold bf16 values; the walk kernel reads them through its
    // bf16 instantiation (the pointer types below only carry the addresses)
    return run_walk(static_cast<const __half *>(q), static_cast<const __half *>(k), static_cast<const __half *>(v),
                    g, geo, static_cast<__half *>(out), static_cast<cudaStream_t>(stream), nullptr, nullptr,
                    nullptr, nullptr, 0.f, true);
}

gtr_status_t gtr_gla_forward_gated(const void *q, const void *k, const void *v, const float *g,
                                              const void *gate, const float *norm_weight, float norm_eps, int B,
                                              int heads, int grid_h, int grid_w, int d_k, int d_v, int direction,
                                              int chunk, void *out, void *stream) {
    t_err_clear();
    Geom geo;
    bool empty = false;
    gtr_status_t s = check_walk_call(q, k, v, g, B, heads, grid_h, grid_w, d_k, d_v, direction, chunk, out,
                                     geo, empty);
    if (s != GTR_OK) return s;
    if (d_v != 64) return fail(GTR_ERR_UNSUPPORTED_SHAPE, "the gated output needs d_v = 64%s");
    if (!gate || !norm_weight) return fail(GTR_ERR_INVALID_ARG, "null pointer%s");
    if (!aligned16(gate) || !aligned16(norm_weight))
        return fail(GTR_ERR_MISALIGNED, "gate and norm_weight must be 16-byte aligned%s");
    if (!(norm_eps >= 0.f) || norm_eps > 1e30f) return fail(GTR_ERR_INVALID_ARG, "norm_eps must be finite and >= 0%s");
    const Range ro = span(out, tok_bytes(geo, d_v, 2));
    if (overlap(ro, span(gate, tok_bytes(geo, d_v, 2))) || overlap(ro, span(norm_weight, (size_t)d_v * 4)))
        return fail(GTR_ERR_ALIAS, "out overlaps the gate or the norm weight%s");
    if (empty) return GTR_OK;
    return run_walk(static_cast<const __half *>(q), static_cast<const __half *>(k), static_cast<const __half *>(v),
                    g, geo, static_cast<__half *>(out), static_cast<cudaStream_t>(stream), nullptr, nullptr,
                    static_cast<const __half *>(gate), norm_weight, norm_eps);
}

// Copy/compute pipeline of the host-buffer entry point.  Every batch item is
// one contiguous byte range of every tensor, so the batch is cut into up to
// kHostSlices slices; slice i's upload, forward and download run on three
// streams of their own, and the uploads of later slices overlap the forward
// and the download of earlier ones (PCIe carries both directions at once).
constexpr int kHostSlices = 8;
constexpr size_t kHostSliceMinBytes = 8u << 20;  // smaller problems run as one slice
struct HostPipe {
    cudaStream_t up = nullptr, run = nullptr, down = nullptr;
    cudaEvent_t start = nullptr, up_done[kHostSlices] = {}, run_done[kHostSlices] = {};
};
std::map<WsKey, HostPipe> g_pipes;  // (device, caller's stream); guarded by g_ws_mu

cudaError_t host_pipe(int dev, cudaStream_t st, HostPipe **out) {
    HostPipe &hp = g_pipes[WsKey{dev, st, WS_STAGING}];
    cudaError_t e = cudaSuccess;
    if (!hp.up) {
        if ((e = cudaStreamCreateWithFlags(&hp.up, cudaStreamNonBlocking)) != cudaSuccess ||
            (e = cudaStreamCreateWithFlags(&hp.run, cudaStreamNonBlocking)) != cudaSuccess ||
            (e = cudaStreamCreateWithFlags(&hp.down, cudaStreamNonBlocking)) != cudaSuccess ||
            (e = cudaEventCreateWithFlags(&hp.start, cudaEventDisableTiming)) != cudaSuccess)
            return e;
        for (int i = 0; i < kHostSlices; ++i)
            if ((e = cudaEventCreateWithFlags(&hp.up_done[i], cudaEventDisableTiming)) != cudaSuccess ||
                (e = cudaEventCreateWithFlags(&hp.run_done[i], cudaEventDisableTiming)) != cudaSuccess)
                return e;
    }
    *out = &hp;
    return e;
}

gtr_status_t gtr_gla_forward_host(const void *q, const void *k, const void *v, const float *g,
                                  int B, int heads, int grid_h, int grid_w, int d_k, int d_v,
                                  int direction, int chunk, void *out, void *stream) {
    t_err[0] = '\0';
    Geom geo;
    bool empty = false;
    gtr_status_t s = check_shape(B, heads, grid_h, grid_w, d_k, d_v, direction, chunk, geo, empty);
    if (s != GTR_OK) return s;
    if (!q || !k || !v || !g || !out) return fail(GTR_ERR_INVALID_ARG, "null pointer%s");
    const size_t nq = tok_bytes(geo, d_k, 2), nv = tok_bytes(geo, d_v, 2), ng = tok_bytes(geo, d_k, 4);
    {
        const Range ro = span(out, nv);
        if (overlap(ro, span(q, nq)) || overlap(ro, span(k, nq)) || overlap(ro, span(v, nv)) ||
            overlap(ro, span(g, ng)))
            return fail(GTR_ERR_ALIAS, "out overlaps an input%s");
    }
    if (empty) return GTR_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t bq = align256(nq), bv = align256(nv), bg = align256(ng);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    // Staging for inputs and output lives in the workspace of a private key
    // (the stream's workspace is used by the forward call itself).
    void *stage = nullptr;
    HostPipe *hp = nullptr;
    {
        size_t need = 2 * bq + 2 * bv + bg;
        std::lock_guard<std::mutex> lk(g_ws_mu);
        Workspace &w = g_ws[WsKey{dev, st, WS_STAGING}];
        if (w.bytes < need) {
            if (w.ptr) {
                e = cudaStreamSynchronize(st);
                if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
                cudaFree(w.ptr);
                w.ptr = nullptr;
                w.bytes = 0;
            }
            e = cudaMalloc(&w.ptr, need);
            if (e != cudaSuccess) {
                w.ptr = nullptr;
                cudaGetLastError();
                return fail(GTR_ERR_OOM, "staging allocation failed%s");
            }
            w.bytes = need;
        }
        stage = w.ptr;
        if ((e = host_pipe(dev, st, &hp)) != cudaSuccess) return cuda_fail(e, "pipeline streams");
    }
    char *p = static_cast<char *>(stage);
    char *dq = p, *dk_ = p + bq, *dv_ = p + 2 * bq, *dg = p + 2 * bq + bv, *dout = p + 2 * bq + bv + bg;
    const char *hq = static_cast<const char *>(q), *hk = static_cast<const char *>(k);
    const char *hv = static_cast<const char *>(v), *hg = reinterpret_cast<const char *>(g);
    char *hout = static_cast<char *>(out);
    // slices of whole batch items, none below kHostSliceMinBytes of traffic
    const size_t total = 2 * nq + 2 * nv + ng;
    int S = (int)std::min<size_t>(std::min<size_t>((size_t)B, kHostSlices), std::max<size_t>(1, total / kHostSliceMinBytes));
    // On an error part-way, wait for what was already queued on the internal
    // streams before returning: no copy may still touch the caller's host
    // buffers after this call returns.
    auto drain = [&](gtr_status_t r) {
        cudaStreamSynchronize(hp->up);
        cudaStreamSynchronize(hp->run);
        cudaStreamSynchronize(hp->down);
        return r;
    };
    // the uploads start after the work already queued on the caller's stream
    if ((e = cudaEventRecord(hp->start, st)) != cudaSuccess || (e = cudaStreamWaitEvent(hp->up, hp->start, 0)) != cudaSuccess)
        return drain(cuda_fail(e, "pipeline start"));
    for (int i = 0; i < S; ++i) {
        const int b0 = (int)((int64_t)B * i / S), b1 = (int)((int64_t)B * (i + 1) / S), nb = b1 - b0;
        const size_t per_b = (size_t)geo.N * heads;  // token-heads per batch item
        const size_t oq = (size_t)b0 * per_b * d_k * 2, ov = (size_t)b0 * per_b * d_v * 2, og = (size_t)b0 * per_b * d_k * 4;
        const size_t sq = (size_t)nb * per_b * d_k * 2, sv = (size_t)nb * per_b * d_v * 2, sg = (size_t)nb * per_b * d_k * 4;
        if ((e = cudaMemcpyAsync(dq + oq, hq + oq, sq, cudaMemcpyHostToDevice, hp->up)) != cudaSuccess ||
            (e = cudaMemcpyAsync(dk_ + oq, hk + oq, sq, cudaMemcpyHostToDevice, hp->up)) != cudaSuccess ||
            (e = cudaMemcpyAsync(dv_ + ov, hv + ov, sv, cudaMemcpyHostToDevice, hp->up)) != cudaSuccess ||
            (e = cudaMemcpyAsync(dg + og, hg + og, sg, cudaMemcpyHostToDevice, hp->up)) != cudaSuccess ||
            (e = cudaEventRecord(hp->up_done[i], hp->up)) != cudaSuccess ||
            (e = cudaStreamWaitEvent(hp->run, hp->up_done[i], 0)) != cudaSuccess)
            return drain(cuda_fail(e, "host-to-device copy"));
        s = forward_impl(dq + oq, dk_ + oq, dv_ + ov, reinterpret_cast<const float *>(dg + og), nb, heads, grid_h,
                         grid_w, d_k, d_v, direction, chunk, GTR_SCHED_AUTO, dout + ov, hp->run);
        if (s != GTR_OK) return drain(s);
        if ((e = cudaEventRecord(hp->run_done[i], hp->run)) != cudaSuccess ||
            (e = cudaStreamWaitEvent(hp->down, hp->run_done[i], 0)) != cudaSuccess ||
            (e = cudaMemcpyAsync(hout + ov, dout + ov, sv, cudaMemcpyDeviceToHost, hp->down)) != cudaSuccess)
            return drain(cuda_fail(e, "device-to-host copy"));
    }
    if ((e = cudaStreamSynchronize(hp->down)) != cudaSuccess) return drain(cuda_fail(e, "cudaStreamSynchronize"));
    // the forward ran on the internal compute stream: report its bounded waits here
    return gtr_gla_get_last_device_status(hp->run);
}

gtr_status_t gtr_sswiglu_forward(const void *a, const void *v, const float *w, const float *bias, int B, int grid_h,
                                 int grid_w, int C, void *out, void *stream) {
    t_err_clear();
    if (B < 0 || grid_h < 0 || grid_w < 0 || C < 0) return fail(GTR_ERR_INVALID_ARG, "negative size%s");
    if (C % 8 != 0) return fail(GTR_ERR_UNSUPPORTED_SHAPE, "C must be a multiple of 8%s");
    const int64_t N = (int64_t)grid_h * grid_w;
    if (N > ((int64_t)1 << 30)) return fail(GTR_ERR_UNSUPPORTED_SHAPE, "more than 2^30 tokens%s");
    if (B > 65535 || (C + 31) / 32 > 65535) return fail(GTR_ERR_UNSUPPORTED_SHAPE, "B or C too large%s");
    if (!a || !v || !w || !out) return fail(GTR_ERR_INVALID_ARG, "null pointer%s");
    if (!aligned16(a) || !aligned16(v) || !aligned16(out) || (reinterpret_cast<uintptr_t>(w) & 3u) ||
        (bias && (reinterpret_cast<uintptr_t>(bias) & 3u)))
        return fail(GTR_ERR_MISALIGNED, "a, v, out must be 16-byte aligned, w and bias 4-byte aligned%s");
    const size_t nb = (size_t)B * N * C * 2;
    const Range ro = span(out, nb);
    if (overlap(ro, span(a, nb)) || overlap(ro, span(v, nb)) || overlap(ro, span(w, (size_t)C * 36)) ||
        (bias && overlap(ro, span(bias, (size_t)C * 4))))
        return fail(GTR_ERR_ALIAS, "out overlaps an input%s");
    if (B == 0 || N == 0 || C == 0) return GTR_OK;
    unsigned *status = nullptr;
    gtr_status_t s = status_word(static_cast<cudaStream_t>(stream), &status);
    if (s != GTR_OK) return s;
    cudaError_t e = launch_sswiglu(static_cast<const __half *>(a), static_cast<const __half *>(v), w, bias, B, grid_h,
                                   grid_w, C, static_cast<__half *>(out), status, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? GTR_OK : cuda_fail(e, "S-SwiGLU kernel launch");
}

gtr_status_t gtr_gla_chunk_summary(const void *k, const void *v, const float *g, int B, int heads,
                                   int grid_h, int grid_w, int d_k, int d_v, int direction,
                                   int chunk, float *dS, float *gamma, void *stream) {
    t_err[0] = '\0';
    Geom geo;
    bool empty = false;
    gtr_status_t s = check_shape(B, heads, grid_h, grid_w, d_k, d_v, direction, chunk, geo, empty);
    if (s != GTR_OK) return s;
    if (!k || !v || !g || !dS || !gamma) return fail(GTR_ERR_INVALID_ARG, "null pointer%s");
    if (!aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(dS) || !aligned16(gamma))
        return fail(GTR_ERR_MISALIGNED, "device pointers must be 16-byte aligned%s");
    size_t nseq = (size_t)geo.B * geo.heads;
    Range rs = span(dS, nseq * geo.nc * d_k * d_v * 4), rg = span(gamma, nseq * geo.nc * d_k * 4);
    Range in[3] = {span(k, tok_bytes(geo, d_k, 2)), span(v, tok_bytes(geo, d_v, 2)),
                   span(g, tok_bytes(geo, d_k, 4))};
    for (const Range &r : in)
        if (overlap(rs, r) || overlap(rg, r)) return fail(GTR_ERR_ALIAS, "an output overlaps an input%s");
    if (overlap(rs, rg)) return fail(GTR_ERR_ALIAS, "dS overlaps gamma%s");
    if (empty) return GTR_OK;
    unsigned *status = nullptr;
    if ((s = status_word(static_cast<cudaStream_t>(stream), &status)) != GTR_OK) return s;
    cudaError_t e = summary_tc(static_cast<const __half *>(k), static_cast<const __half *>(v), g, geo,
                               dS, gamma, static_cast<cudaStream_t>(stream), status);
    return e == cudaSuccess ? GTR_OK : cuda_fail(e, "chunk summary launch");
}

gtr_status_t gtr_gla_boundary_scan(const float *dS, const float *gamma, int B, int heads,
                                   int n_chunks, int d_k, int d_v, float *S_enter, void *stream) {
    t_err[0] = '\0';
    if (B < 0 || heads < 0 || n_chunks < 0) return fail(GTR_ERR_INVALID_ARG, "negative size%s");
    if (!supported_d(d_k) || !supported_d(d_v))
        return fail(GTR_ERR_UNSUPPORTED_SHAPE, "d_k and d_v must be 16, 32, 64 or 128%s");
    if (!dS || !gamma || !S_enter) return fail(GTR_ERR_INVALID_ARG, "null pointer%s");
    if (!aligned16(dS) || !aligned16(gamma) || !aligned16(S_enter))
        return fail(GTR_ERR_MISALIGNED, "device pointers must be 16-byte aligned%s");
    int64_t nseq = (int64_t)B * heads;
    if (nseq * (((int64_t)d_k * d_v + 255) / 256) >= ((int64_t)1 << 31))
        return fail(GTR_ERR_UNSUPPORTED_SHAPE, "too many sequences%s");
    size_t sb = (size_t)nseq * n_chunks * d_k * d_v * 4;
    Range rs = span(S_enter, sb);
    if (S_enter != dS && overlap(rs, span(dS, sb))) return fail(GTR_ERR_ALIAS, "S_enter partially overlaps dS%s");
    if (overlap(rs, span(gamma, (size_t)nseq * n_chunks * d_k * 4)))
        return fail(GTR_ERR_ALIAS, "S_enter overlaps gamma%s");
    if (nseq == 0 || n_chunks == 0) return GTR_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    void *agg = nullptr;
    const size_t ab = scan_agg_bytes(nseq, n_chunks, d_k, d_v);
    if (ab > 0) {  // segment aggregates in an internal workspace
        gtr_status_t s = get_workspace(ab, st, &agg, WS_SCAN);
        if (s != GTR_OK) return s;
    }
    cudaError_t e = launch_scan_segmented(dS, gamma, (int)nseq, n_chunks, d_k, d_v, S_enter,
                                          static_cast<float *>(agg), st);
    return e == cudaSuccess ? GTR_OK : cuda_fail(e, "boundary scan launch");
}

gtr_status_t gtr_gla_chunk_output(const void *q, const void *k, const void *v, const float *g,
                                  const float *S_enter, int B, int heads, int grid_h, int grid_w,
                                  int d_k, int d_v, int direction, int chunk, void *out,
                                  void *stream) {
    t_err[0] = '\0';
    Geom geo;
    bool empty = false;
    gtr_status_t s = check_shape(B, heads, grid_h, grid_w, d_k, d_v, direction, chunk, geo, empty);
    if (s != GTR_OK) return s;
    if (!q || !k || !v || !g || !S_enter || !out) return fail(GTR_ERR_INVALID_ARG, "null pointer%s");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(S_enter) ||
        !aligned16(out))
        return fail(GTR_ERR_MISALIGNED, "device pointers must be 16-byte aligned%s");
    size_t nseq = (size_t)geo.B * geo.heads;
    Range ro = span(out, tok_bytes(geo, d_v, 2));
    Range in[5] = {span(q, tok_bytes(geo, d_k, 2)), span(k, tok_bytes(geo, d_k, 2)),
                   span(v, tok_bytes(geo, d_v, 2)), span(g, tok_bytes(geo, d_k, 4)),
                   span(S_enter, nseq * geo.nc * d_k * d_v * 4)};
    for (const Range &r : in)
        if (overlap(ro, r)) return fail(GTR_ERR_ALIAS, "out overlaps an input%s");
    if (empty) return GTR_OK;
    unsigned *status = nullptr;
    if ((s = status_word(static_cast<cudaStream_t>(stream), &status)) != GTR_OK) return s;
    cudaError_t e = output_tc(static_cast<const __half *>(q), static_cast<const __half *>(k),
                              static_cast<const __half *>(v), g, S_enter, geo, static_cast<__half *>(out),
                              static_cast<cudaStream_t>(stream), status);
    return e == cudaSuccess ? GTR_OK : cuda_fail(e, "chunk output launch");
}

size_t gtr_gla_workspace_bytes_ex(int B, int heads, int grid_h, int grid_w, int d_k, int d_v,
                                  int chunk, int schedule) {
    Geom geo;
    bool empty = false;
    if (check_shape(B, heads, grid_h, grid_w, d_k, d_v, 0, chunk, geo, empty) != GTR_OK) return 0;
    if (schedule < GTR_SCHED_AUTO || schedule > kSchedLast || empty) return 0;
    const size_t status = 256;  // the stream's device status word
    if (schedule == GTR_SCHED_THREE_PHASE || schedule == GTR_SCHED_THREE_PHASE_SIMT ||
        schedule == GTR_SCHED_THREE_PHASE_MMA)
        return three_phase_ws(geo) + status;
    if (schedule == GTR_SCHED_AUTO) return std::max(three_phase_ws(geo), fused_ws(geo)) + status;
    if (schedule == GTR_SCHED_WALK_TCGEN05) return (walk_shape(geo) ? 0 : fused_ws(geo)) + status;
    return fused_ws(geo) + status;
}

size_t gtr_gla_workspace_bytes(int B, int heads, int grid_h, int grid_w, int d_k, int d_v, int chunk) {
    return gtr_gla_workspace_bytes_ex(B, heads, grid_h, grid_w, d_k, d_v, chunk, GTR_SCHED_AUTO);
}

gtr_status_t gtr_gla_get_last_device_status(void *stream) {
    t_err[0] = '\0';
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    unsigned *word = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_ws_mu);
        auto it = g_ws.find(WsKey{dev, st, WS_STATUS});
        if (it != g_ws.end()) word = static_cast<unsigned *>(it->second.ptr);
    }
    if (!word) return GTR_OK;  // nothing that reports has run on this stream
    unsigned v = 0;
    if ((e = cudaMemcpyAsync(&v, word, sizeof v, cudaMemcpyDeviceToHost, st)) != cudaSuccess ||
        (e = cudaStreamSynchronize(st)) != cudaSuccess)
        return cuda_fail(e, "status read");
    if (v != 0) {
        if ((e = cudaMemsetAsync(word, 0, sizeof v, st)) != cudaSuccess ||
            (e = cudaStreamSynchronize(st)) != cudaSuccess)
            return cuda_fail(e, "status reset");
        return fail(GTR_ERR_TIMEOUT, "a bounded device wait gave up%s");
    }
    return GTR_OK;
}

gtr_status_t gtr_gla_debug_forward_fused(const void *q, const void *k, const void *v, const float *g,
                                         int B, int heads, int grid_h, int grid_w, int d_k, int d_v,
                                         int direction, int chunk, int schedule, int hold_seq,
                                         int hold_chunk, long long spin_limit, void *out, void *stream) {
    t_err[0] = '\0';
    Geom geo;
    bool empty = false;
    gtr_status_t s = check_shape(B, heads, grid_h, grid_w, d_k, d_v, direction, chunk, geo, empty);
    if (s != GTR_OK) return s;
    if (!q || !k || !v || !g || !out) return fail(GTR_ERR_INVALID_ARG, "null pointer%s");
    if (spin_limit < 1) return fail(GTR_ERR_INVALID_ARG, "spin_limit must be positive%s");
    if (schedule != GTR_SCHED_AUTO && schedule != GTR_SCHED_FUSED && schedule != GTR_SCHED_FUSED_TCGEN05)
        return fail(GTR_ERR_INVALID_ARG, "schedule must be AUTO, FUSED or FUSED_TCGEN05%s");
    if (empty) return GTR_OK;
    int sms = 0;
    cudaError_t e = sm_count(&sms);
    if (e != cudaSuccess) return cuda_fail(e, "device query");
    return run_fused(static_cast<const __half *>(q), static_cast<const __half *>(k),
                     static_cast<const __half *>(v), g, geo, static_cast<__half *>(out),
                     static_cast<cudaStream_t>(stream), plan_for(geo, schedule, sms, true), hold_seq,
                     hold_chunk, spin_limit);
}

gtr_status_t gtr_gla_release_workspace(void) {
    std::lock_guard<std::mutex> lk(g_ws_mu);
    int cur = 0;
    cudaGetDevice(&cur);
    for (auto &kv : g_ws) {
        if (kv.second.ptr) {
            cudaSetDevice(kv.first.dev);
            cudaDeviceSynchronize();
            cudaFree(kv.second.ptr);
        }
    }
    g_ws.clear();
    for (auto &kv : g_pipes) {
        HostPipe &hp = kv.second;
        cudaSetDevice(kv.first.dev);
        if (hp.up) {
            cudaStreamDestroy(hp.up);
            cudaStreamDestroy(hp.run);
            cudaStreamDestroy(hp.down);
            cudaEventDestroy(hp.start);
            for (int i = 0; i < kHostSlices; ++i) {
                cudaEventDestroy(hp.up_done[i]);
                cudaEventDestroy(hp.run_done[i]);
            }
        }
    }
    g_pipes.clear();
    cudaSetDevice(cur);
    return GTR_OK;
}

const char *gtr_gla_status_string(gtr_status_t s) {
    switch (s) {
    case GTR_OK: return "ok";
    case GTR_ERR_INVALID_ARG: return "invalid argument";
    case GTR_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case GTR_ERR_MISALIGNED: return "misaligned pointer";
    case GTR_ERR_ALIAS: return "output aliases an input";
    case GTR_ERR_CUDA: return "CUDA error";
    case GTR_ERR_TIMEOUT: return "device wait timed out";
    case GTR_ERR_OOM: return "out of device memory";
    }
    return "unknown status";
}

const char *gtr_gla_last_error(void) { return t_err; }

uint64_t gtr_gla_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int gtr_gla_version(void) { return 200; }

int gtr_gla_plan(int B, int heads, int grid_h, int grid_w, int d_k, int d_v, int chunk, int schedule,
                 int sm_count) {
    Geom geo;
    bool empty = false;
    if (check_shape(B, heads, grid_h, grid_w, d_k, d_v, 0, chunk, geo, empty) != GTR_OK) return -1;
    if (schedule < GTR_SCHED_AUTO || schedule > kSchedLast || sm_count < 1) return -1;
    return (int)plan_for(geo, schedule, sm_count);
}

int gtr_gla_bounds_checked(void) {
#ifdef GTR_BOUNDS_CHECK
    return 1;
#else
    return 0;
#endif
}

gtr_status_t gtr_gla_debug_bounds_report(unsigned long long *count, int *site, long long *index,
                                         long long *limit, int clear) {
    t_err[0] = '\0';
    if (!count || !site || !index || !limit) return fail(GTR_ERR_INVALID_ARG, "null pointer%s");
    *count = 0;
    *site = 0;
    *index = 0;
    *limit = 0;
    if (!gtr_gla_bounds_checked()) return fail(GTR_ERR_INVALID_ARG, "library built without bounds checks%s");
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
    gtr::BoundsReport sum = {};
    std::lock_guard<std::mutex> lk(gtr::bounds_readers_mu());
    for (gtr::BoundsReader r : gtr::bounds_readers())
        if (r(&sum, clear) != 0) return fail(GTR_ERR_CUDA, "reading a bounds report failed%s");
    *count = sum.count;
    *site = sum.site;
    *index = sum.index;
    *limit = sum.limit;
    return GTR_OK;
}

}  // extern "C"
