// gtr_gla_noalloc.cu -- gtr_gla_forward_noalloc: the three-phase GLA forward
// with its scratch in a fixed, file-scope device array, so that the call
// itself never allocates device memory.
//
// Who needs it: callers that must not call cudaMalloc (or anything that may
// allocate) once they are running -- hosts that hand out every byte of device
// memory through their own allocator or fixed budget and treat a foreign
// allocation as a leak or a failure (engine plugins, serving runtimes), and
// real-time loops that forbid allocation after start-up.  gtr_gla_forward
// grows an internal workspace on demand, which these callers cannot accept.
//
// The scratch holds the per-chunk summaries dS and gamma of the three-phase
// schedule (the boundary scan then overwrites dS with the entering states in
// place).  It runs the CUDA-core versions of the three phases.  Every GPU
// that loads this library reserves the whole array until the process exits.
#include "gtr_gla.h"

#include <cuda.h>  // CUcontext (types only; the driver call is looked up at run time)

#include <mutex>

#include "gla_common.cuh"

namespace {

constexpr size_t kScratchBytes = size_t(16) << 20;  // 16 MiB per device

// File-scope scratch.  In host code `g_noalloc_scratch` names a host-side
// stand-in, not the device array: its device address must be looked up with
// cudaGetSymbolAddress (done once per device below) before a kernel gets it.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
struct ScratchAddr {
    void *ptr = nullptr;
    CUcontext ctx = nullptr;  // the context the address belongs to
};
ScratchAddr g_scratch[kMaxDevices];

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);

// The current CUDA context, through the driver entry point the runtime hands
// out (no link-time dependency on the driver library); nullptr if unknown.
CUcontext current_context() {
    static CtxGetCurrentFn fn = [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess) {
            cudaGetLastError();
            return (CtxGetCurrentFn) nullptr;
        }
        return reinterpret_cast<CtxGetCurrentFn>(f);
    }();
    CUcontext c = nullptr;
    if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
    return c;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

int err(gtr_status_t s, const char *msg) { return gtr::set_last_error(s, msg); }

// Device address of the scratch on the current device.  Looked up on the
// first call per device (with that device current) and cached together with
// the device's context; a new context (after cudaDeviceReset the module is
// loaded again) is looked up again, so a stale address is never used.
gtr_status_t scratch_address(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return (gtr_status_t)err(GTR_ERR_CUDA, "cudaGetDevice failed");
    if (dev < 0 || dev >= kMaxDevices)
        return (gtr_status_t)err(GTR_ERR_INVALID_ARG, "device index above the no-allocation limit of 64 devices");
    // null before the device's context exists: then the address is looked up
    // (which creates the context) and looked up once more on the next call
    const CUcontext ctx = current_context();
    std::lock_guard<std::mutex> lk(g_mu);
    ScratchAddr &a = g_scratch[dev];
    if (!a.ptr || a.ctx != ctx || !ctx) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            a.ptr = nullptr;
            return (gtr_status_t)err(GTR_ERR_CUDA, "cudaGetSymbolAddress of the static scratch failed");
        }
        a.ptr = p;
        a.ctx = ctx;
    }
    *out = a.ptr;
    return GTR_OK;
}

bool supported_d(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool overlap(const void *a, size_t na, const void *b, size_t nb) {
    uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return na && nb && x < y + nb && y < x + na;
}

}  // namespace

extern "C" {

gtr_status_t gtr_gla_forward_noalloc(const void *q, const void *k, const void *v, const float *g,
                                     int B, int heads, int grid_h, int grid_w, int d_k, int d_v,
                                     int direction, int chunk, void *out, void *stream) {
    gtr::clear_last_error();
    auto fail = [](gtr_status_t s, const char *msg) { return (gtr_status_t)err(s, msg); };
    if (B < 0 || heads < 0 || grid_h < 0 || grid_w < 0) return fail(GTR_ERR_INVALID_ARG, "negative size");
    if (direction < 0 || direction > 3) return fail(GTR_ERR_INVALID_ARG, "bad direction");
    if (!supported_d(d_k) || !supported_d(d_v))
        return fail(GTR_ERR_UNSUPPORTED_SHAPE, "d_k and d_v must be 16, 32, 64 or 128");
    if (chunk != 16 && chunk != 32 && chunk != 64)
        return fail(GTR_ERR_UNSUPPORTED_SHAPE, "chunk must be 16, 32 or 64");
    if (!q || !k || !v || !g || !out) return fail(GTR_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(out))
        return fail(GTR_ERR_MISALIGNED, "device pointers must be 16-byte aligned");
    const int64_t N = (int64_t)grid_h * grid_w;
    if (N > ((int64_t)1 << 30)) return fail(GTR_ERR_UNSUPPORTED_SHAPE, "more than 2^30 tokens");
    const size_t ntok = (size_t)B * (size_t)N * (size_t)heads;
    if (overlap(out, ntok * d_v * 2, q, ntok * d_k * 2) || overlap(out, ntok * d_v * 2, k, ntok * d_k * 2) ||
        overlap(out, ntok * d_v * 2, v, ntok * d_v * 2) || overlap(out, ntok * d_v * 2, g, ntok * d_k * 4))
        return fail(GTR_ERR_ALIAS, "out overlaps an input");
    if (ntok == 0) return GTR_OK;
    const int64_t nc = (N + chunk - 1) / chunk;
    const size_t nseq = (size_t)B * heads;
    const size_t ds_bytes = align256(nseq * nc * d_k * d_v * sizeof(float));
    const size_t need = ds_bytes + align256(nseq * nc * d_k * sizeof(float));
    if (need > kScratchBytes)  // B*heads*ceil(N/chunk)*d_k*(d_v+1)*4 bytes must fit
        return fail(GTR_ERR_UNSUPPORTED_SHAPE, "problem larger than the 16 MiB no-allocation scratch");
    void *scratch = nullptr;
    gtr_status_t s = scratch_address(&scratch);
    if (s != GTR_OK) return s;

    gtr::Geom geo;
    geo.B = B; geo.heads = heads; geo.H = grid_h; geo.W = grid_w;
    geo.dk = d_k; geo.dv = d_v; geo.dir = direction; geo.chunk = chunk;
    geo.N = (int)N; geo.nc = (int)nc;
    float *dS = static_cast<float *>(scratch);
    float *gamma = reinterpret_cast<float *>(static_cast<char *>(scratch) + ds_bytes);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // The summary kernel writes every dS and gamma entry the scan and the
    // output kernel read, so nothing in the scratch has to start at zero.
    cudaError_t e = gtr::launch_summary_v0(static_cast<const __half *>(k), static_cast<const __half *>(v),
                                           g, geo, dS, gamma, st);
    if (e == cudaSuccess) e = gtr::launch_scan_v0(dS, gamma, (int)nseq, geo.nc, d_k, d_v, dS, st);
    if (e == cudaSuccess)
        e = gtr::launch_output_v0(static_cast<const __half *>(q), static_cast<const __half *>(k),
                                  static_cast<const __half *>(v), g, dS, geo,
                                  static_cast<__half *>(out), st);
    if (e != cudaSuccess) return fail(GTR_ERR_CUDA, cudaGetErrorString(e));
    return GTR_OK;
}

}  // extern "C"
