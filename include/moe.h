/*
 * moe.h -- C ABI of the B200 (sm_100a) routed-expert MoE layer library, libmoe.so.
 *
 * The layer is the one the Colibri pages describe for streaming-MoE inference
 * of GLM-5.2 (744B): a DeepSeek-V3-style router picks top-k of E routed
 * experts per token (takumi3488 article, teacher-forcing section; top-8 of 256
 * in the coli info log), every expert is a feed-forward block whose weights are
 * packed int4, int2 or int8 codes with per-row scales, dequantised on use and
 * multiplied against int8 activations with integer dot products (agentlenshq
 * summary, "Integer-Dot Kernels" and "Quantization"), and the routed outputs
 * are combined with the always-resident shared expert (agentlenshq summary,
 * "Memory split").  An expert requested by several tokens of a batch is read
 * once (remio.ai analysis, the paragraph on merging duplicate expert requests).
 *
 * Conventions for every call:
 *  - Tensor pointers are DEVICE pointers owned by the caller.  The library
 *    never allocates, frees or keeps caller memory beyond the stream work it
 *    enqueues.  Pointers must be 16-byte aligned (MOE_EALIGN otherwise).
 *  - All work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) with no implicit synchronisation.  Argument errors are detected
 *    on the host before anything is enqueued and return synchronously.  A
 *    failed launch returns MOE_ECUDA.  Errors found by the kernels themselves
 *    are written to a status word in the workspace; read it with
 *    moe_poll_status after synchronising the stream.
 *  - The library keeps no global handles and is safe to call from several
 *    host threads; calls that share one workspace must not overlap on the GPU.
 *  - moe_last_error() returns a thread-local description of the last failure.
 *
 * Numerics (identical on every entry point):
 *  - activation quantiser: per token s = max|x| / 127 (fp32, IEEE division),
 *    code = clamp(round_half_even(x / s), -127, 127); an all-zero token gets
 *    s = 0 and zero codes; bf16 inputs are widened exactly to fp32 first.
 *  - router: logits = W_r x in fp32 on the UNQUANTISED x; score = sigmoid;
 *    selection on score + bias, descending, ties to the lower expert index;
 *    weights = selected scores / their sum * routed_scale (bias not included).
 *  - codes: two's complement, low bits first (int4 byte = c0 | c1 << 4; int2
 *    byte = c0 | c1 << 2 | c2 << 4 | c3 << 6; int8: one code per byte, the
 *    third width of the agentlenshq summary's "Quantization" item);
 *    int32 accumulation is exact.
 *  - gate/up: g = acc_g * (s_row * s_x), u likewise, h = g / (1 + exp(-g)) * u
 *    (SwiGLU); h is requantised per (token, expert) with the activation rule.
 *  - down: y = acc_d * (s_row * s_h); out = sum_j w_j y_j + y_shared (fp32).
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* same object as cudaStream_t */

typedef enum {
    MOE_OK = 0,
    MOE_EINVAL = -1,   /* bad dimension, null pointer or unsupported combination   */
    MOE_EALIGN = -2,   /* a pointer is not 16-byte aligned                          */
    MOE_ENOSPACE = -3, /* workspace smaller than moe_workspace_bytes(cfg, T)        */
    MOE_ECUDA = -4,    /* a CUDA runtime call or kernel launch failed               */
    MOE_ETIMEOUT = -5, /* a bounded device-side wait ran out (status word only)     */
    MOE_EDEVICE = -6   /* a kernel found an invalid value, e.g. an index out of range */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

/* Shape of one MoE layer.
 *  d: hidden size; f: expert intermediate size; n_experts: routed experts E;
 *  top_k: experts per token k; has_shared: 1 if a shared expert follows the E
 *  routed blobs; wbits: 4, 2 or 8 (codes per byte: 2, 4 or 1);
 *  routed_scale: factor on the renormalised routed weights (2.5 for GLM-5.2).
 *  tc_min_tokens: calls of at least this many tokens run the experts on the
 *  int8 tensor-core (tcgen05) path (moe_layer with MOE_PATH_AUTO,
 *  moe_expert_ffn, moe_expert_down); 0 = library default (3: on B200 at the
 *  GLM-5.2 expert shape the single-launch decode kernel is faster for one and
 *  two tokens, the tensor-core path from three on), < 0 = never.
 *  topp: TOPK/TOPP truncation of the router, opt-in (0 or 1 = off, the
 *  router as above).  With 0 < topp < 1 each token keeps the smallest prefix
 *  of its k selected slots (selection order) whose scores, normalised over
 *  the k, sum to at least topp: slot j is kept iff j == 0 or the float32 sum
 *  of the scores of slots 0..j-1, added in slot order, is below
 *  float32(topp * sum of all k).  A dropped slot selects no expert: its
 *  topk_idx is -1, its weight 0, and no expert is read for it; the kept
 *  weights are the kept scores over their sum, times routed_scale.  (A
 *  reading of the pages' TOPP option: agentlenshq, benchmark table, the
 *  --topp 0.7 rows; takumi3488, the TOPK / TOPP options of the run logs.)
 * Limits (MOE_EINVAL otherwise): 1 <= k <= min(E, 32); E <= 1024;
 * d * wbits / 8 and f * wbits / 8 multiples of 16; d <= 8192; f <= 8192;
 * 0 <= topp <= 1. */
typedef struct {
    int32_t d, f, n_experts, top_k, has_shared, wbits;
    float routed_scale;
    int32_t tc_min_tokens;
    float topp;
} moe_config;

/* One layer's experts in device memory, canonical layout.
 *  w: E + has_shared blobs of 3*d*f*wbits/8 bytes each, expert e at offset
 *     e * blob_bytes, the shared expert last.  A blob is
 *     [gate f x d | up f x d | down d x f], each matrix row-major by output
 *     row, codes packed as above ("adjacent matrices stored together").
 *  s: fp32 [E + has_shared][f + f + d] per-output-row scales, same order
 *     (always every expert's: 10 KB each at the GLM-5.2 shape).
 *  slot_of: NULL, or an HBM expert cache's slot table (moe_cache below):
 *     device int32 [E + has_shared]; then w holds n_slots blobs and expert e's
 *     blob is at w + slot_of[e] * blob_bytes.  Every expert a call selects
 *     must be resident (moe_cache_fetch); an index outside [0, n_slots) is
 *     clamped (and recorded as MOE_EDEVICE by the bounds-checked build).
 *  n_slots: the blobs w holds when slot_of is set. */
typedef struct {
    const uint8_t* w;
    const float* s;
    const int32_t* slot_of;
    int32_t n_slots;
} moe_pool;

/* Bytes of workspace the calls below need for up to max_tokens tokens. */
MOE_API size_t moe_workspace_bytes(const moe_config* cfg, int32_t max_tokens);

/* Zero the whole workspace (its control words and counters).  Call once after
 * allocating a workspace, and again after a call that reported a device error,
 * before its next use; the kernels leave every counter at zero between calls. */
MOE_API moe_status moe_workspace_init(void* ws, size_t ws_bytes, moe_stream_t stream);

/* Activation quantiser alone (step a0), exposed for parity checks.
 * x [T][d] (dtype) -> xq int8 [T][d], sx fp32 [T]. */
MOE_API moe_status moe_quantize(const moe_config* cfg, const void* x, moe_dtype dtype, int32_t T, int8_t* xq,
                        float* sx, moe_stream_t stream);

/* Router alone (step a1): x [T][d] (dtype), w_router fp32 [E][d], bias fp32
 * [E] -> topk_idx int32 [T][k] (slot order = selection score descending),
 * topk_w fp32 [T][k]. */
MOE_API moe_status moe_route(const moe_config* cfg, const void* x, moe_dtype dtype, int32_t T,
                     const float* w_router, const float* bias, int32_t* topk_idx, float* topk_w,
                     void* ws, size_t ws_bytes, moe_stream_t stream);

/* The router of moe_route for callers that cannot provide a workspace.
 * The Colibri pages have no counterpart for this entry point: it exists for
 * callers of this library that cannot allocate device memory on their call
 * path -- a host framework that owns all device memory and forbids allocations
 * after start-up, a serving loop that must not pay cudaMalloc's implicit device
 * synchronisation, a plugin interface with no way to request scratch space.
 * Same arguments and results as moe_route, without ws/ws_bytes.  Its scratch
 * (64 KB) is a fixed array inside libmoe.so that every GPU loading the library
 * keeps until the process exits; the call allocates nothing.
 *  - Limits: T <= 8 tokens, n_experts <= 1024, top_k <= 32; larger requests
 *    return MOE_EINVAL with a message naming the limit.
 *  - Each call looks up that array's device address on the current device
 *    (cudaGetSymbolAddress, with that device current; nothing is kept between
 *    calls, so a device reset by the caller is harmless).  The first call on
 *    a device also loads the library's device code there: make that first
 *    call before any stream capture.
 *  - Every call, on every stream, shares the one array: calls whose work
 *    overlaps on the GPU race and give undefined results.  Each call clears
 *    the control word it needs at its start. */
MOE_API moe_status moe_route_static(const moe_config* cfg, const void* x, moe_dtype dtype, int32_t T,
                                    const float* w_router, const float* bias, int32_t* topk_idx, float* topk_w,
                                    moe_stream_t stream);

/* One expert over T tokens (steps a3 + a4): expert in [0, E) is a routed
 * expert, -1 the shared one.  xq int8 [T][d], sx fp32 [T] -> y fp32 [T][d]
 * (overwritten).  Optional debug outputs (NULL to skip): dbg_acc_gu int32
 * [T][2f] (gate accumulators then up accumulators), dbg_hq int8 [T][f],
 * dbg_sh fp32 [T], dbg_acc_d int32 [T][d]. */
MOE_API moe_status moe_expert_ffn(const moe_config* cfg, const moe_pool* pool, int32_t expert, const int8_t* xq,
                          const float* sx, int32_t T, float* y, int32_t* dbg_acc_gu, int8_t* dbg_hq,
                          float* dbg_sh, int32_t* dbg_acc_d, void* ws, size_t ws_bytes,
                          moe_stream_t stream);

/* Down projection alone from given h codes (step a4, for teacher-forced
 * parity): hq int8 [T][f], sh fp32 [T] -> y fp32 [T][d]; dbg_acc_d optional. */
MOE_API moe_status moe_expert_down(const moe_config* cfg, const moe_pool* pool, int32_t expert, const int8_t* hq,
                           const float* sh, int32_t T, float* y, int32_t* dbg_acc_d, void* ws,
                           size_t ws_bytes, moe_stream_t stream);

/* The whole layer (steps a0-a7): quantise, route, bucket tokens by expert
 * (each selected expert is read once per call), gate/up, requantise, down,
 * weighted combine with the shared expert.
 * x [T][d] (dtype) -> out fp32 [T][d]: overwritten if accumulate == 0, added
 * to if accumulate != 0 (residual stream of stacked layers).  topk_idx_out
 * int32 [T][k] and topk_w_out fp32 [T][k] are optional copies of the routing. */
MOE_API moe_status moe_layer(const moe_config* cfg, const moe_pool* pool, const float* w_router, const float* bias,
                     const void* x, moe_dtype dtype, int32_t T, float* out, int32_t accumulate,
                     int32_t* topk_idx_out, float* topk_w_out, void* ws, size_t ws_bytes,
                     moe_stream_t stream);

/* Options of moe_layer_ex (all optional; zero-initialise).
 *  events: cudaEvent_t handles (or NULL) recorded on `stream` before routing
 *          [0], after routing and bucketing [1], after gate/up [2] and after
 *          down + combine [3]; for timing the phases on the launching stream.
 *          The single-launch decode path records [0] before and [3] after
 *          its one kernel and leaves [1] and [2] untouched (its phases share
 *          the kernel; each extra record after it cost ~2.7 us of GPU time).
 *  path: MOE_PATH_AUTO (0), MOE_PATH_MULTI (1: separate routing, gate/up and
 *        down kernels on dp4a integer dots), MOE_PATH_DECODE (2: one
 *        persistent kernel for T <= 8; MOE_EINVAL if the shape does not fit
 *        it) or MOE_PATH_TC (3: routing, then gate/up and down as int8
 *        grouped GEMMs on the tensor cores, tasks of up to 64 tokens per
 *        expert, then the combine).  AUTO takes TC when T >= tc_min_tokens
 *        (and the shape fits it), else DECODE where it fits, else MULTI.
 *  path_ran: set to the path that ran (MOE_PATH_DECODE, _MULTI or _TC).
 *  n_launches: set to the number of kernels the call launched.
 *  trace: optional DEVICE buffer of (number of SMs) x 32 uint64 that the
 *         single-launch decode path fills with per-CTA global-timer stamps
 *         (ns) at its phase boundaries: [0] start, [1] tokens quantised,
 *         [2] router rows done, [3] shared-expert gate/up done, [4] grid
 *         barrier passed, [5] routing derived, [6] routed gate/up done,
 *         [7] first down staging ready, [8] down done, [11] top-k done,
 *         [18] router logits loaded for the top-k (first warp);
 *         totals: [9] consumer wait for data, [10] producer wait for slots;
 *         producer: [12] rows known before routing issued, [13] routing
 *         received, [14] all rows issued, [15] all copies landed; one-token
 *         row-range down: [7] the CTA's designated tasks requantised, [16]
 *         its first designated task's h row complete (polled), [17] its
 *         codes and scale written, [20] every task's codes staged, [22] the
 *         first down unit done, [21] the last.  Untouched entries are left
 *         as is. */
enum { MOE_PATH_AUTO = 0, MOE_PATH_MULTI = 1, MOE_PATH_DECODE = 2, MOE_PATH_TC = 3 };
typedef struct {
    void* events[4];
    int32_t path;
    int32_t n_launches;
    void* trace;
    int32_t path_ran;
    /* in: bound of the decode kernel's device-side waits in microseconds
     * (0 = 2 s; its waits for ring slots take twice this, so that a stalled
     * hand-off reports before the slot waits behind it); a wait that runs out
     * records MOE_ETIMEOUT with a site code (moe_poll_status) and the kernel
     * finishes without the missing data. */
    int32_t wait_limit_us;
    /* in, for tests of the bounded waits: 1 + t makes the one-token decode
     * with row-range down (the GLM-5.2 expert shapes) leave task t's h values
     * unwritten (task 0 is the shared expert when there is one, then the
     * routed experts in ascending id order), so that every wait on them runs
     * out; ignored on every other path; 0 = off. */
    int32_t test_skip_h;
    /* in: where x and out live.  MOE_IO_X_HOST: x is pinned host memory
     * mapped into the device's address space (cudaHostAlloc, or
     * cudaHostRegister with mapping; with unified addressing the host pointer
     * is the device pointer); the call first copies it into the workspace with
     * a small kernel (one read over the host link, no DMA copy), then runs
     * the layer on the copy.  MOE_IO_OUT_HOST: out is such memory; the
     * kernels write (and in accumulate mode read) it directly.  0 = both in
     * device memory. */
    int32_t io_host;
} moe_layer_opts;
enum { MOE_IO_X_HOST = 1, MOE_IO_OUT_HOST = 2 };

/* moe_layer with options (opts may be NULL, then identical to moe_layer). */
MOE_API moe_status moe_layer_ex(const moe_config* cfg, const moe_pool* pool, const float* w_router,
                                const float* bias, const void* x, moe_dtype dtype, int32_t T, float* out,
                                int32_t accumulate, int32_t* topk_idx_out, float* topk_w_out, void* ws,
                                size_t ws_bytes, moe_stream_t stream, moe_layer_opts* opts);

/* Parameter-free RMSNorm of a residual stream, used between stacked layers:
 * x_in = x / sqrt(mean(x^2) + eps).  x [T][d] (dtype) -> x_in fp32 [T][d].
 * If x_copy is not NULL it receives x widened to fp32 (to start a residual
 * stream from bf16 activations). */
MOE_API moe_status moe_rmsnorm(const void* x, moe_dtype dtype, int32_t T, int32_t d, float eps, float* x_in,
                       float* x_copy, moe_stream_t stream);

/* Device-side status word of a workspace (MOE_OK if no kernel reported an
 * error).  Synchronises `stream` first.  *info (optional) receives a detail
 * word. */
MOE_API moe_status moe_poll_status(const void* ws, int32_t* info, moe_stream_t stream);

/* HBM expert cache with host-memory overflow, one per layer: the layer's
 * full pool stays in pinned host memory, n_slots blobs of it are resident in
 * device memory, and moe_cache_fetch makes the experts a call selects
 * resident before the call runs, evicting the least recently used others
 * (the pages' per-layer LRU of experts with readahead -- agentlenshq,
 * "ロードメカニズム"; remio.ai, the async I/O pool paragraph -- moved one tier
 * up: host RAM behind HBM instead of disk behind RAM).  All memory is the
 * caller's:
 *  host_w: pinned host memory, the layer's E + has_shared blobs (canonical
 *          layout, as moe_pool.w);
 *  slots: device memory, n_slots blobs (16-byte aligned);
 *  slot_of: device int32 [E + has_shared], written by the calls below;
 *  state: host memory of moe_cache_state_bytes(cfg, n_slots) bytes (the LRU
 *         book-keeping);
 *  n_slots: >= the distinct experts of one call (+ the shared expert).
 * Use: moe_cache_init once; per call: route (moe_route), copy the indices to
 * the host, moe_cache_fetch, then moe_layer with the pool {slots, scales,
 * slot_of, n_slots} on the same stream (the layer routes again and finds the
 * same experts).  The shared expert is fetched at init and never evicted. */
typedef struct {
    const uint8_t* host_w;
    uint8_t* slots;
    int32_t* slot_of;
    void* state;
    int32_t n_slots;
} moe_cache;
typedef struct {
    int64_t hits;    /* experts a fetch found resident */
    int64_t misses;  /* experts it copied in */
    int64_t bytes;   /* host -> device bytes it issued */
} moe_cache_stats;
MOE_API size_t moe_cache_state_bytes(const moe_config* cfg, int32_t n_slots);
/* Empties the cache, copies the shared expert in (slot 0) and writes slot_of
 * (-1 for every other expert).  Host errors return synchronously. */
MOE_API moe_status moe_cache_init(const moe_config* cfg, moe_cache* cache, moe_stream_t stream);
/* Makes every expert in idx (host int32 [T][top_k], -1 entries skipped)
 * resident: a hit refreshes the expert's use; a miss takes a free slot or
 * the least recently used slot whose expert this call does not select, and
 * issues one cudaMemcpyAsync of its blob on `stream`; the changed slot_of
 * entries are then written on `stream` by a small kernel whose (expert, slot)
 * pairs travel as kernel arguments, so no host buffer outlives the call.
 * MOE_ENOSPACE if n_slots cannot hold the call's experts.  stats (nullable)
 * receives this call's counts. */
MOE_API moe_status moe_cache_fetch(const moe_config* cfg, moe_cache* cache, const int32_t* idx, int32_t T,
                                   moe_stream_t stream, moe_cache_stats* stats);

MOE_API const char* moe_status_string(moe_status status);
MOE_API const char* moe_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H_ */
