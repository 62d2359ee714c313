/*
 * gtr_gla.h -- C ABI of the B200 (sm_100a) key-gated GLA token mixer.
 *
 * Operation (the GTR token mixer; sources by page and section):
 *   For each batch b and head h, over the N = grid_h*grid_w patch tokens
 *   visited in one scan order, with S_0 = 0:
 *       S_t = diag(exp(g_t)) S_{t-1} + k_t^T v_t          (d_k x d_v state)
 *       o_t = (q_t / sqrt(d_k)) S_t
 *   and o_t written back at the token's own spatial position.
 *   - key-only gated linear attention, value-side decay fixed at one; one
 *     directional scan per block, spatial order restored afterwards:
 *     ai.info summary of "GTR: Gated Token Recurrence for Efficient Dense
 *     Prediction", section "Methodology in Plain English";
 *   - scan orders left->right, right->left, top->bottom, bottom->top cycled
 *     across the 12 blocks: GTR project page, section "How GTR Works";
 *   - the inference operator: per-chunk summaries computed in parallel over
 *     the chunk x head grid, a light coalesced scan of the chunk boundary
 *     states, and an output kernel that fuses the intra-chunk score-value
 *     product with the boundary-state readout; zero initial state; fp16:
 *     GTR project page, section "A Kernel That Makes Recurrence Fast", and
 *     the ai.info summary, "Methodology in Plain English".
 *
 * Conventions shared by every entry point:
 *   - Buffers marked (device) are CUDA device pointers of the current device,
 *     buffers marked (host) are host pointers.  The caller owns every buffer.
 *   - fp16 buffers hold IEEE binary16 values (CUDA __half); fp32 buffers
 *     hold IEEE binary32 values.
 *   - Token layout: q, k and g are [B][N][heads][d_k], v and out are
 *     [B][N][heads][d_v], contiguous, N = grid_h*grid_w tokens in row-major
 *     spatial order (row r, column c -> token r*grid_w + c), both in and out.
 *     The scan order is applied inside the kernels' loads and stores; no
 *     permuted copy is ever made.
 *   - Scan orders (gtr_dir_t): L2R visits t -> t; R2L visits t -> N-1-t;
 *     T2B visits column-major, t -> (t mod grid_h)*grid_w + t div grid_h;
 *     B2T visits the reverse of T2B.
 *   - Supported sizes: d_k, d_v in {16, 32, 64, 128}; chunk in {16, 32, 64};
 *     any grid_h, grid_w >= 1 (a ragged last chunk is masked), any B,
 *     heads >= 1.  B == 0 or N == 0 is an empty problem: GTR_OK, nothing
 *     is launched.
 *   - Every device pointer must be 16-byte aligned (GTR_ERR_MISALIGNED).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Device entry points are asynchronous: they enqueue work on
 *     `stream` and return without synchronising.  On any error status
 *     nothing is enqueued, except GTR_ERR_CUDA from a failed launch.
 *   - Errors never cross the ABI as exceptions.  gtr_gla_last_error()
 *     returns a short text for the calling thread's last failure.
 *   - Thread safety: calls on distinct streams may run concurrently.  Calls
 *     that use the library's internal workspace on the same stream are
 *     ordered by that stream.
 *   - log-gates g are expected to be <= 0 (the accuracy bound holds for
 *     g <= 0); other values are accepted and computed, not clamped.
 */
#ifndef GTR_GLA_H
#define GTR_GLA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GTR_DIR_L2R = 0,
    GTR_DIR_R2L = 1,
    GTR_DIR_T2B = 2,
    GTR_DIR_B2T = 3
} gtr_dir_t;

typedef enum {
    GTR_OK = 0,
    GTR_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad enum */
    GTR_ERR_UNSUPPORTED_SHAPE = 2, /* d_k, d_v or chunk outside the supported set */
    GTR_ERR_MISALIGNED = 3,        /* a device pointer not 16-byte aligned */
    GTR_ERR_ALIAS = 4,             /* an output overlaps an input */
    GTR_ERR_CUDA = 5,              /* a CUDA runtime call or launch failed */
    GTR_ERR_TIMEOUT = 6,           /* a bounded device-side wait gave up */
    GTR_ERR_OOM = 7                /* the internal workspace could not grow */
} gtr_status_t;

typedef enum {
    GTR_SCHED_AUTO = 0,             /* library choice (gtr_gla_plan), the fastest measured for the
                                       problem's size: GTR_SCHED_THREE_PHASE_MMA for at most 24
                                       sequences (B*heads); GTR_SCHED_WALK_TCGEN05 for its shapes
                                       with d_k <= 64 and 2 to 3 (sequence, value slice) items per
                                       SM; else GTR_SCHED_FUSED_TCGEN05 for its shape with at least
                                       2 sequences per SM; else GTR_SCHED_FUSED */
    GTR_SCHED_FUSED = 1,            /* one kernel (mma.sync tensor cores): summaries, chained
                                       boundary states, outputs */
    GTR_SCHED_THREE_PHASE = 2,      /* chunk_summary -> boundary_scan -> chunk_output, the phases on
                                       tcgen05 tensor cores for chunk 64, d_k in {32, 64, 128},
                                       d_v in {64, 128} (mma.sync for other shapes) */
    GTR_SCHED_THREE_PHASE_SIMT = 3, /* the same three phases on CUDA cores only (comparison) */
    GTR_SCHED_FUSED_TCGEN05 = 4,    /* fused, one (sequence, chunk, 64 value columns) tile per CTA
                                       with the boundary state chained between CTAs, whole-chunk
                                       products on tcgen05 (d_k = d_v in {64, 128}, chunk 64;
                                       other shapes run GTR_SCHED_FUSED) */
    GTR_SCHED_WALK_TCGEN05 = 5,     /* one CTA per (sequence, 64 value columns) walks the chunks
                                       in scan order with its slice of the state on chip,
                                       whole-chunk products on tcgen05 (chunk 64, d_k in
                                       {32, 64, 128}, d_v in {64, 128}; other shapes run
                                       GTR_SCHED_FUSED) */
    GTR_SCHED_THREE_PHASE_MMA = 6   /* the three phases with mma.sync tensor-core phases, every
                                       shape */
} gtr_schedule_t;

/* The kernels a schedule launches (gtr_gla_plan). */
typedef enum {
    GTR_PLAN_THREE_PHASE = 0,       /* chunk summaries, boundary scan, chunk outputs; tcgen05 phases
                                       for the walk kernel's shapes, else mma.sync */
    GTR_PLAN_THREE_PHASE_SIMT = 1,  /* the same three phases on CUDA cores */
    GTR_PLAN_FUSED_MMA = 2,         /* fused mma.sync kernel, one chunk per tile */
    GTR_PLAN_FUSED_MMA_PAIR = 3,    /* fused mma.sync kernel, two chunks per tile (d_v <= 64) */
    GTR_PLAN_FUSED_TCGEN05 = 4,     /* fused tcgen05 kernel, chained tiles (d_k = d_v in {64, 128},
                                       chunk 64) */
    GTR_PLAN_WALK_TCGEN05 = 5,      /* tcgen05 walk kernel, one CTA per (sequence, value slice) */
    GTR_PLAN_THREE_PHASE_MMA = 6    /* the three phases with mma.sync phases */
} gtr_plan_t;

/* The GLA forward over all B*heads sequences (see the operation above).
 *   q, k (device, fp16) [B][N][heads][d_k]; v (device, fp16) [B][N][heads][d_v];
 *   g (device, fp32) [B][N][heads][d_k] log-gates; out (device, fp16)
 *   [B][N][heads][d_v], written in full (every token, every head);
 *   direction: gtr_dir_t; chunk: tokens per chunk of the chunkwise schedule.
 * out must not overlap q, k, v or g (GTR_ERR_ALIAS).  Uses an internal
 * per-device, per-stream workspace that grows on demand, in stream order on
 * `stream` (cudaFreeAsync / cudaMallocAsync / cudaMemsetAsync; GTR_ERR_OOM if
 * it cannot).  Growing cannot be captured: a call that needs to grow it
 * inside a stream capture returns GTR_ERR_INVALID_ARG, so make the first call
 * of the largest size on that stream outside any capture.  After that, calls
 * on the stream can be captured into a CUDA graph and replayed.
 * Stream order: some schedules (the walk, the three phases) launch their
 * kernels with programmatic stream serialization.  Each such kernel waits for
 * the kernel ahead of it on `stream` to complete before it touches q, k, v,
 * g, out or the workspace, so the call is ordered after earlier work on the
 * stream exactly as a normal launch is.  Each also lets the grid launched
 * after it start early: a kernel the caller launches next with programmatic
 * stream serialization must itself wait for its predecessor
 * (cudaGridDependencySynchronize / griddepcontrol.wait) before it reads out,
 * as that attribute requires anyway; a normal launch waits as usual. */
gtr_status_t gtr_gla_forward(const void *q, const void *k, const void *v, const float *g,
                             int B, int heads, int grid_h, int grid_w, int d_k, int d_v,
                             int direction, int chunk, void *out, void *stream);

/* gtr_gla_forward with an explicit schedule (gtr_schedule_t).  Both
 * schedules compute the same recurrence; results agree to rounding. */
gtr_status_t gtr_gla_forward_ex(const void *q, const void *k, const void *v, const float *g,
                                int B, int heads, int grid_h, int grid_w, int d_k, int d_v,
                                int direction, int chunk, int schedule, void *out, void *stream);

/* The forward from a given initial state, returning the final state: the
 * recurrence above with S_0 = S0 instead of zero, and SN = S_N, the state
 * after the last token of the scan.  This carries the state across calls,
 * e.g. across video frames (ai.info summary, "Future Directions": carrying
 * the state across frames is the natural extension; the pages' own operator
 * fixes S_0 = 0, "Methodology in Plain English").
 *   S0 (device, fp32) [B][heads][d_k][d_v] row-major per (b, h), or NULL for
 *   a zero initial state; SN (device, fp32) [B][heads][d_k][d_v], or NULL
 *   when the final state is not wanted; other arguments as gtr_gla_forward.
 * Runs the walk kernel (GTR_SCHED_WALK_TCGEN05) and supports its shapes only:
 * chunk 64, d_k in {32, 64, 128}, d_v in {64, 128} (else
 * GTR_ERR_UNSUPPORTED_SHAPE).  SN may be the same buffer as S0 (updated in
 * place); any other overlap of SN with S0, an input or out, or of out with
 * S0, is GTR_ERR_ALIAS.  S0 and SN must be 16-byte aligned.  With no token
 * (grid_h*grid_w == 0) SN receives S0 (or zeros).  Needs no workspace. */
gtr_status_t gtr_gla_forward_state(const void *q, const void *k, const void *v, const float *g,
                                   const float *S0, int B, int heads, int grid_h, int grid_w, int d_k,
                                   int d_v, int direction, int chunk, void *out, float *SN, void *stream);

/* gtr_gla_forward with bf16 instead of fp16 for q, k, v and out (g stays
 * fp32): the same recurrence, layouts, checks and error statuses.  The GTR
 * pages specialise their operator to fp16 and leave other precisions open
 * (ai.info summary, "Future Directions": broadening kernel coverage to other
 * precisions); this is that variant.  The tensor-core operands (the
 * decay-scaled q and k, the masked scores and the scaled state) are bf16,
 * accumulation and the state fp32.  Runs the walk kernel: chunk 64, d_k in
 * {32, 64, 128}, d_v in {64, 128} (else GTR_ERR_UNSUPPORTED_SHAPE).  Needs
 * no workspace. */
gtr_status_t gtr_gla_forward_bf16(const void *q, const void *k, const void *v, const float *g, int B,
                                  int heads, int grid_h, int grid_w, int d_k, int d_v, int direction,
                                  int chunk, void *out, void *stream);

/* The forward followed by the output gate on the RMS-normalised output
 * (ai.info summary, "Methodology in Plain English": a separate data-dependent
 * output gate applied to the RMS-normalised output), fused into the output
 * store.  For every token t and head h, with o = o_t of that head (d_v values):
 *     out[e] = o[e] / sqrt(mean_e'(o[e']^2) + norm_eps) * norm_weight[e]
 *              * gate[e] * sigmoid(gate[e])
 * (RMSNorm over the head's d_v values, Zhang and Sennrich; the swish gate of
 * gated linear attention, Yang et al.; both on the GTR reference list).
 *   gate (device, fp16) [B][N][heads][d_v]: the gate's pre-activation;
 *   norm_weight (device, fp32) [d_v]; norm_eps >= 0 and finite;
 *   out (device, fp16) [B][N][heads][d_v] receives the gated values (o
 *   itself is not stored); other arguments as gtr_gla_forward.
 * Runs the walk kernel with d_v = 64 (the pages' deployment shape): chunk
 * 64, d_k in {32, 64, 128}, d_v = 64 (else GTR_ERR_UNSUPPORTED_SHAPE).  out
 * must not overlap any input (GTR_ERR_ALIAS); gate and norm_weight must be
 * 16-byte aligned.  Needs no workspace. */
gtr_status_t gtr_gla_forward_gated(const void *q, const void *k, const void *v, const float *g,
                                   const void *gate, const float *norm_weight, float norm_eps, int B,
                                   int heads, int grid_h, int grid_w, int d_k, int d_v, int direction,
                                   int chunk, void *out, void *stream);

/* End-to-end call on HOST buffers: copies q, k, v, g (host) to the device,
 * runs the forward (GTR_SCHED_AUTO), copies the result into out (host) and
 * returns once out is complete.  Layouts as gtr_gla_forward.  The batch is
 * cut into up to 8 slices of whole batch items (problems under 8 MiB of
 * traffic run as one); each slice's upload, forward and download run on three
 * internal streams of this (device, stream) pair, so uploads overlap the
 * forward and the downloads of earlier slices.  Those streams start after the
 * work queued on `stream` before the call.  Device staging buffers come from
 * the internal workspace.  Page-locked host buffers give the fastest copies
 * and the overlap; pageable ones work too.  out must not overlap q, k, v or g
 * (GTR_ERR_ALIAS).  Returns GTR_ERR_TIMEOUT if a bounded wait inside the
 * forward gave up.  On any error, the internal streams are drained before
 * the call returns: no copy touches the caller's buffers afterwards. */
gtr_status_t gtr_gla_forward_host(const void *q, const void *k, const void *v, const float *g,
                                  int B, int heads, int grid_h, int grid_w, int d_k, int d_v,
                                  int direction, int chunk, void *out, void *stream);

/* gtr_gla_forward without any device allocation.  The GTR pages have no
 * counterpart to this call; it exists for callers that cannot let a library
 * allocate device memory while they run: hosts that own every byte of device
 * memory through their own allocator or a fixed budget (engine plugins,
 * serving runtimes) and real-time loops that forbid allocation after
 * start-up.  Arguments, layouts and error statuses as gtr_gla_forward (its
 * own argument checks, the same codes; the failure text is set as for every
 * other entry point).  It runs the CUDA-core versions of the three phases
 * (chunk summaries, boundary scan, chunk outputs), so its result matches
 * gtr_gla_forward within the forward's tolerance (max |difference| <=
 * 2e-3 * max |output|), not bit for bit.  Its scratch is a 16 MiB array in
 * the library's own device memory, which every GPU that loads the library
 * holds until the process exits.  Problems needing more, i.e.
 * B*heads*ceil(N/chunk)*d_k*(d_v+1)*4 bytes above 16 MiB (after 256-byte
 * rounding of the two parts), are rejected with GTR_ERR_UNSUPPORTED_SHAPE and
 * nothing is launched.  The first call on a device (and the first after the
 * device's context was recreated, e.g. by cudaDeviceReset) looks up that
 * device's scratch address (cudaGetSymbolAddress); make that first call
 * before any stream capture.  All calls on a device share the one scratch
 * array: calls whose kernels may overlap on the GPU (different streams
 * without ordering between them) race and give wrong results; order them on
 * one stream or with events.  The scratch keeps the last call's contents;
 * every entry a call reads is first written by the same call, so nothing
 * needs clearing. */
gtr_status_t gtr_gla_forward_noalloc(const void *q, const void *k, const void *v, const float *g,
                                     int B, int heads, int grid_h, int grid_w, int d_k, int d_v,
                                     int direction, int chunk, void *out, void *stream);

/* Spatial SwiGLU's gating with its 3x3 depthwise convolution, the other
 * half of each GTR block (ai.info summary, "Methodology in Plain English":
 * a 3x3 depthwise convolution inserted in the value branch of a SwiGLU
 * block, on the 2-D patch grid; GTR project page, "Spatial SwiGLU").  For
 * every batch b, token p = row*grid_w + col and channel c:
 *     out[b][p][c] = silu(a[b][p][c])
 *                    * (bias[c] + sum_{dy,dx in -1..1} w[c][dy+1][dx+1] * v[b][p + dy*grid_w + dx][c])
 * with silu(x) = x * sigmoid(x) and zero padding outside the grid.
 *   a (device, fp16) [B][grid_h*grid_w][C]: the gate branch;
 *   v (device, fp16) [B][grid_h*grid_w][C]: the value branch;
 *   w (device, fp32) [C][3][3]: the depthwise filter; bias (device, fp32) [C],
 *   or NULL for none; out (device, fp16) [B][grid_h*grid_w][C].
 * The projections around it (into a and v, and out of the block) are plain
 * GEMMs outside this library.  C must be a multiple of 8
 * (GTR_ERR_UNSUPPORTED_SHAPE); a, v and out 16-byte aligned, w and bias 4-byte
 * aligned (GTR_ERR_MISALIGNED); out must not overlap an input (GTR_ERR_ALIAS).
 * B == 0, an empty grid or C == 0 is an empty problem.  Needs no workspace
 * beyond the stream's device status word: a tile whose loads did not arrive
 * within about a second is skipped and GTR_ERR_TIMEOUT is recorded there
 * (gtr_gla_get_last_device_status). */
gtr_status_t gtr_sswiglu_forward(const void *a, const void *v, const float *w, const float *bias, int B,
                                 int grid_h, int grid_w, int C, void *out, void *stream);

/* Phase 1, chunk summaries (GTR project page, "A Kernel That Makes
 * Recurrence Fast": per-chunk summaries in parallel over the chunk x head
 * grid).  With nc = ceil(N/chunk) and b_s the inclusive prefix sum of g
 * inside chunk c (scan order), for every (b, h, c):
 *   gamma[b][h][c][i]   = exp(b_last[i])
 *   dS[b][h][c][i][j]   = sum_s exp(b_last[i] - b_s[i]) k_s[i] v_s[j]
 * k (device, fp16), v (device, fp16), g (device, fp32) as in gtr_gla_forward;
 * dS (device, fp32) [B][heads][nc][d_k][d_v]; gamma (device, fp32)
 * [B][heads][nc][d_k].  Outputs must not overlap inputs. */
gtr_status_t gtr_gla_chunk_summary(const void *k, const void *v, const float *g,
                                   int B, int heads, int grid_h, int grid_w, int d_k, int d_v,
                                   int direction, int chunk, float *dS, float *gamma,
                                   void *stream);

/* Phase 2, boundary-state scan (same section: only the boundary states are
 * propagated sequentially).  For every (b, h):
 *   S_enter[0] = 0,  S_enter[c+1][i][j] = gamma[c][i] * S_enter[c][i][j] + dS[c][i][j]
 * dS, gamma (device, fp32) as written by gtr_gla_chunk_summary with
 * n_chunks chunks; S_enter (device, fp32) [B][heads][n_chunks][d_k][d_v].
 * S_enter may be the same buffer as dS (in place); any other overlap with
 * the inputs is GTR_ERR_ALIAS.  Long chains with few state elements run in
 * two passes over segments of chunks; their segment aggregates live in an
 * internal per-device, per-stream workspace (GTR_ERR_OOM if it cannot grow;
 * make the first call of the largest size outside any stream capture). */
gtr_status_t gtr_gla_boundary_scan(const float *dS, const float *gamma, int B, int heads,
                                   int n_chunks, int d_k, int d_v, float *S_enter, void *stream);

/* Phase 3, chunk outputs (same section: the output kernel fuses the
 * within-chunk score-value product with the boundary-state readout).  For
 * token t of chunk c:
 *   o_t = sum_i q~_t[i] exp(b_t[i]) S_enter[c][i][:]
 *       + sum_{s <= t in chunk} (sum_i q~_t[i] exp(b_t[i] - b_s[i]) k_s[i]) v_s
 * with q~ = q / sqrt(d_k).  q, k, v, g, out as gtr_gla_forward; S_enter
 * (device, fp32) as written by gtr_gla_boundary_scan. */
gtr_status_t gtr_gla_chunk_output(const void *q, const void *k, const void *v, const float *g,
                                  const float *S_enter, int B, int heads, int grid_h, int grid_w,
                                  int d_k, int d_v, int direction, int chunk, void *out,
                                  void *stream);

/* Bytes of internal device workspace (per device and stream) that a
 * gtr_gla_forward call of this size may use: the larger of what its
 * schedules need, plus the stream's status word (informational; 0 for
 * invalid arguments or an empty problem). */
size_t gtr_gla_workspace_bytes(int B, int heads, int grid_h, int grid_w, int d_k, int d_v,
                               int chunk);

/* The same for gtr_gla_forward_ex(..., schedule, ...) (gtr_schedule_t). */
size_t gtr_gla_workspace_bytes_ex(int B, int heads, int grid_h, int grid_w, int d_k, int d_v,
                                  int chunk, int schedule);

/* Synchronises `stream`, then returns and clears the device-side status
 * word of (current device, stream): GTR_OK, or GTR_ERR_TIMEOUT if a bounded
 * wait inside a kernel enqueued on `stream` gave up since the last query.
 * Each stream has its own word, so a query never sees or clears another
 * stream's report. */
gtr_status_t gtr_gla_get_last_device_status(void *stream);

/* Test hook for the bounded wait of the fused schedules: runs
 * gtr_gla_forward_ex(..., schedule, ...) for schedule GTR_SCHED_AUTO,
 * GTR_SCHED_FUSED or GTR_SCHED_FUSED_TCGEN05 (others: GTR_ERR_INVALID_ARG),
 * except that the tile of sequence hold_seq (= b*heads + h), chunk hold_chunk
 * never publishes its boundary state, and the wait for a predecessor's
 * boundary state gives up after spin_limit polls (> 0, else
 * GTR_ERR_INVALID_ARG).  spin_limit bounds only that wait: a CTA's waits for
 * its own tensor-core work keep a fixed bound of about one second.  The
 * successor tile then times out, records GTR_ERR_TIMEOUT in the stream's
 * device status word (read it with gtr_gla_get_last_device_status) and the
 * kernel still finishes; its output is not meaningful.  hold_seq = -1
 * disables the hold. */
gtr_status_t gtr_gla_debug_forward_fused(const void *q, const void *k, const void *v, const float *g,
                                         int B, int heads, int grid_h, int grid_w, int d_k, int d_v,
                                         int direction, int chunk, int schedule, int hold_seq,
                                         int hold_chunk, long long spin_limit, void *out, void *stream);

/* Frees every internal workspace of every device (synchronises each device
 * that has one).  Later calls allocate again on demand. */
gtr_status_t gtr_gla_release_workspace(void);

/* Static text for a status code. */
const char *gtr_gla_status_string(gtr_status_t status);

/* Text describing the calling thread's most recent failed call ("" if none). */
const char *gtr_gla_last_error(void);

/* Number of kernels this library has launched in this process. */
uint64_t gtr_gla_launch_count(void);

/* ABI version: major*10000 + minor*100 + patch. */
int gtr_gla_version(void);

/* Which kernels gtr_gla_forward_ex(..., schedule, ...) launches for this
 * problem on a device with sm_count streaming multiprocessors: a gtr_plan_t,
 * or -1 for invalid arguments.  Host-only; needs no device.  AUTO takes the
 * three-phase schedule with mma.sync phases for at most 24 sequences
 * (B*heads); the walk kernel for chunk 64, d_k in {32, 64}, d_v in {64, 128}
 * when B*heads*d_v/64 lies in [2*sm_count, 3*sm_count]; the chained tcgen05
 * kernel for d_k = d_v = 64, chunk 64 with at least 2*sm_count sequences;
 * else the mma.sync kernel with two chunks per tile below 2*sm_count
 * sequences when d_v <= 64, one chunk per tile otherwise. */
int gtr_gla_plan(int B, int heads, int grid_h, int grid_w, int d_k, int d_v, int chunk, int schedule,
                 int sm_count);

/* 1 if this library is the bounds-checked debug build, else 0.  The checked
 * build (libgtr_gla_checked.so, compiled with GTR_BOUNDS_CHECK) tests every
 * global-memory index a kernel computes at run time against its buffer's
 * extent before the access; an index out of range is counted, the first one
 * recorded, and the access skipped instead of made.  It is slower, and meant
 * for tests. */
int gtr_gla_bounds_checked(void);

/* Checked build only: waits for the device (cudaDeviceSynchronize), then
 * returns in *count the accesses skipped since the last clear, and for the
 * first of them its site code (*site), index (*index) and the extent it broke
 * (*limit); all zero when none.  clear != 0 resets the report.  The normal
 * build returns GTR_ERR_INVALID_ARG with everything zero. */
gtr_status_t gtr_gla_debug_bounds_report(unsigned long long *count, int *site, long long *index,
                                         long long *limit, int clear);

#ifdef __cplusplus
}
#endif

#endif /* GTR_GLA_H */
