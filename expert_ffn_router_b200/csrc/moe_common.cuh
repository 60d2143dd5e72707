// Shared device/host helpers of libmoe: workspace layout, kernel parameters,
// PTX wrappers, block reductions and the int8 activation staging layout.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "moe.h"

namespace moe {

constexpr int kThreads = 256;  // every kernel of the library runs 256-thread CTAs
constexpr int kWarps = kThreads / 32;
constexpr unsigned kFull = 0xffffffffu;

// ---------------------------------------------------------------------------
// Workspace: a 256-byte header of control words followed by the per-call
// buffers.  The layout is that of the workspace's capacity -- the largest
// token count it can hold for the config (ws_capacity) -- so every call on one
// workspace finds its counters at the same offsets whatever its own T.
// ---------------------------------------------------------------------------
struct WsHeader {
    int32_t status;       // first error code a kernel reported (0 = none)
    int32_t status_info;  // detail word of that error
    uint32_t route_ctr;   // arrival ticket of the router CTAs (self-resetting)
    int32_t n_tasks;      // tasks = (expert, <= CH tokens) pairs of this call
    int32_t n_asg;        // assignments incl. shared-expert ones
    int32_t n_items3;     // gate/up work items
    int32_t n_items4;     // down work items
    uint32_t epoch;       // calls of the persistent decode kernel so far
    uint32_t b1_count;    // its grid barrier: arrivals (self-resetting)
    uint32_t b1_gen;      // its grid barrier: epoch of the last completion
    int32_t tc_rows;      // padded rows of all tensor-core tasks of this call
    int32_t pad[53];
};
static_assert(sizeof(WsHeader) == 256, "header must stay 256 bytes");

// Decode-kernel control words after the header: [0, 1024) and [1024, 2048)
// gate/up rows finished per task of the several-token kernel (the two halves
// alternate by call parity).
constexpr int kReadyFlags = 2048;
constexpr size_t kCtrlBytes = sizeof(WsHeader) + kReadyFlags * 4;  // zeroed by moe_workspace_init

struct Ws {
    WsHeader* hdr;
    uint32_t* ready;   // [kReadyFlags] decode-kernel per-task counters and flags (see kReadyFlags)
    int8_t* xq;        // [T][d]     quantised activations
    float* sx;         // [T]        activation scales
    int32_t* xcs;      // [T]        sum of each token's codes
    float* logits;     // [ksplit][T][E] router logits (partials when split over d)
    int32_t* idx;      // [T][k]     routing
    float* w;          // [T][k]     routing weights
    int32_t* asg;      // [T*S]      assignment ids (token*S + slot) grouped by task
    int4* tasks;       // [max_tasks] (blob, asg start, n tokens, 0)
    uint32_t* task_ctr;// [max_tasks] gate/up item arrivals per task (self-resetting)
    uint32_t* amax;    // [T*S]      max |h| per assignment (float bits)
    uint32_t* amax2;   // [T*S]      second copy: the decode kernel alternates by call parity
    float* h;          // [T*S][f]   SwiGLU output
    int8_t* hq;        // [T*S][f]   requantised h
    float* sh;         // [T*S]      scale of hq
    float* ybuf;       // [T*S][d]   per-assignment down outputs before the combine
    uint32_t* rb_ctr;  // [ceil(d/rb4)] down item arrivals per row block (self-resetting)
    int32_t* hcs;      // [T*S]      sum of the hq codes of each assignment (tensor-core down)
    uint8_t* xb;       // tensor-core operand B of gate/up: per task, activation rows in MMA layout
    uint8_t* hb;       // tensor-core operand B of down: per task, hq rows in MMA layout
    uint8_t* xin;      // [T][d] x as given (<= 4 bytes per value), copied in from host memory
    size_t bytes;
};

constexpr int kRouterKsplitMax = 64;

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct Dims {
    int d, f, E, k, has_shared, wb, T, S;
};

inline int max_tasks(const Dims& m) { return m.T * m.S + m.E + 2; }

// Tensor-core path: tasks hold at most kTcNT tokens (the MMA N), padded to
// tc_npad rows; a K chunk is 64 packed weight bytes (128 int4 / 256 int2 codes).
constexpr int kTcNT = 64;
__host__ __device__ constexpr int tc_npad(int n) { return n <= 8 ? 8 : (n + 15) & ~15; }
__host__ __device__ constexpr int tc_kc(int wb) { return 512 / wb; }
__host__ __device__ constexpr int tc_kpad(int k, int wb) { return (k + tc_kc(wb) - 1) / tc_kc(wb) * tc_kc(wb); }
// Bound on the padded rows of all tasks of a call: every task has >= 1 token
// and pads by < 16 rows; tasks <= experts present + assignments / kTcNT.
__host__ __device__ inline size_t tc_rows_bound(const Dims& m) {
    const size_t A = (size_t)m.T * m.S;
    const size_t t2 = (size_t)(m.E + m.has_shared) + (A + kTcNT - 1) / kTcNT;
    return A + 15 * (A < t2 ? A : t2);
}
// Rows per warp per work item of the gate/up and down kernels (one definition
// for the kernels' template arguments and the host's item counts).
constexpr int rpw3() { return 2; }
constexpr int rpw4(int ncl) { return ncl >= 8 ? 1 : 8 / ncl; }
constexpr int kMinRowBlock4 = 8;  // smallest down row block: 8 warps x rpw4(8)

inline Ws ws_carve(const Dims& m, void* base) {
    Ws w{};
    char* b = static_cast<char*>(base);
    size_t off = 0;
    auto take = [&](size_t bytes) -> void* {
        void* p = b ? b + off : nullptr;
        off = align_up(off + bytes, 256);
        return p;
    };
    const size_t T = (size_t)m.T, A = (size_t)m.T * m.S;
    w.hdr = (WsHeader*)take(sizeof(WsHeader));
    w.ready = (uint32_t*)take(kReadyFlags * 4);
    w.xq = (int8_t*)take(T * m.d);
    w.sx = (float*)take(T * 4);
    w.xcs = (int32_t*)take(T * 4);
    w.logits = (float*)take((size_t)kRouterKsplitMax * T * m.E * 4);
    w.idx = (int32_t*)take(T * m.k * 4);
    w.w = (float*)take(T * m.k * 4);
    w.asg = (int32_t*)take(A * 4);
    w.tasks = (int4*)take((size_t)max_tasks(m) * 16);
    w.task_ctr = (uint32_t*)take((size_t)max_tasks(m) * 4);
    w.amax = (uint32_t*)take(A * 4);
    w.amax2 = (uint32_t*)take(A * 4);
    w.h = (float*)take(A * m.f * 4);
    w.hq = (int8_t*)take(A * m.f);
    w.sh = (float*)take(A * 4);
    w.ybuf = (float*)take(A * m.d * 4);
    w.rb_ctr = (uint32_t*)take((size_t)((m.d + kMinRowBlock4 - 1) / kMinRowBlock4) * 4);
    w.hcs = (int32_t*)take(A * 4);
    w.xb = (uint8_t*)take(tc_rows_bound(m) * tc_kpad(m.d, m.wb));
    w.hb = (uint8_t*)take(tc_rows_bound(m) * tc_kpad(m.f, m.wb));
    w.xin = (uint8_t*)take(T * m.d * 4);
    w.bytes = off;
    return w;
}

// Largest T whose layout fits in `bytes` (0 if none): the layout of a
// workspace is carved for this capacity, with S = top_k + has_shared slots.
inline int ws_capacity(Dims m, size_t bytes) {
    int lo = 0, hi = 1 << 20;
    while (lo < hi) {
        const int mid = lo + (hi - lo + 1) / 2;
        m.T = mid;
        if (ws_carve(m, nullptr).bytes <= bytes) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// ---------------------------------------------------------------------------
// Kernel parameters (passed by value).
// ---------------------------------------------------------------------------
struct Params {
    Dims m;
    float routed_scale;
    const uint8_t* pool;
    const float* scales;
    long long blob_bytes;
    int scale_rows;
    int CH;          // max tokens per task
    int rb3, nrb3;   // gate/up rows per item, items per task
    int rb4, nrb4;   // down rows per item, items per task
    int ksplit;      // router split of d
    int tc;          // tasks are tensor-core tasks (<= kTcNT tokens, padded-row offsets in task.w)
    Ws ws;
    int a_cap;       // assignments the workspace layout holds (capacity T x S)
    unsigned long long* trace;  // optional per-CTA phase stamps of the decode kernel
    unsigned long long wait_ns; // bound of the decode kernel's device-side waits (its slot waits: twice this)
    int skip_h_task;            // testing: the one-token decode leaves this task's h unwritten (-1 = none)
    float topp;                 // TOPK/TOPP truncation of the router (0 or 1 = off)
    const int32_t* slot_of;     // HBM expert cache: expert -> blob slot of `pool` (nullptr: the expert's index)
    int n_slots;                // with slot_of: the blobs `pool` holds
    const float* w_router;
    const float* bias;
    float* out;
    int accumulate;
    int32_t* idx_out;
    float* w_out;
    // single-expert entry points
    int direct_out;        // write y[token][d] instead of the slot buffer + combine
    const int8_t* hq_in;   // teacher-forced down: given codes [T][f]
    const float* sh_in;    // and scales [T]
    // debug outputs
    int32_t* dbg_acc_gu;
    int8_t* dbg_hq;
    float* dbg_sh;
    int32_t* dbg_acc_d;
};

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
// Streaming 16-byte load of read-only weights: no L1 allocation.
__device__ __forceinline__ uint4 ld_stream(const void* p) {
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(p));
    return v;
}
__device__ __forceinline__ float4 ld_stream_f4(const void* p) {
    float4 v;
    asm("ld.global.nc.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
        : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
        : "l"(p));
    return v;
}
// unsigned 8-bit x signed 8-bit 4-way dot product accumulate
__device__ __forceinline__ int dp4a_us(unsigned a, int b, int c) {
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

__device__ __forceinline__ void set_status(WsHeader* h, int code, int info) {
    if (atomicCAS(&h->status, 0, code) == 0) atomicExch(&h->status_info, info);
}

// Indices the kernels read from data -- routed experts, task lists,
// assignment ids, padded-row offsets -- pass through idx_in(): it keeps v in
// [lo, hi) so that no access leaves its buffer, whatever the data.  The
// bounds-checked build of the library (compiled with MOE_BOUNDS,
// libmoe_bounds.so) also records a value outside the range as MOE_EDEVICE
// with the site code in the status word, which the tests read.
__device__ __forceinline__ int idx_in(WsHeader* h, int v, int lo, int hi, int site) {
#ifdef MOE_BOUNDS
    if (v < lo || v >= hi) set_status(h, MOE_EDEVICE, site);
#else
    (void)h;
    (void)site;
#endif
    return min(max(v, lo), hi - 1);
}

// ---------------------------------------------------------------------------
// mbarrier / bulk-copy / ordering wrappers (sm_90+ PTX, used on sm_100a)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("{ .reg .b64 st; mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1; }" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("{ .reg .b64 st; mbarrier.arrive.shared::cta.b64 st, [%0]; }" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// 1-D bulk copy global -> this CTA's shared memory, completion counted in bytes
// on `bar`.  Addresses 16-byte aligned, size a multiple of 16.  No multicast.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}
// The same with an L2 cache policy (e.g. evict-first for bytes read once).
__device__ __forceinline__ void bulk_g2s_hint(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                              uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::
            "r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}
// TOPK/TOPP truncation of one warp's k selected slots (lane j holds slot j).
// With 0 < topp < 1, slot j is kept iff j == 0 or cex -- the float sum of the
// scores of slots 0..j-1, added in slot order -- is below fl(topp * ssum),
// ssum the float sum over all k slots: the smallest prefix whose normalised
// scores reach topp.  Returns the normaliser of the kept weights, cin (the
// inclusive sum) of the last kept slot.  Any other topp keeps every slot and
// returns ssum.  topp is the same for the whole warp.
__device__ __forceinline__ float topp_keep(float topp, int k, float ssum, float cex, float cin, bool& kept) {
    const int lane = threadIdx.x & 31;
    if (!(topp > 0.0f && topp < 1.0f)) {
        kept = lane < k;
        return ssum;
    }
    const float thr = __fmul_rn(topp, ssum);
    kept = lane < k && (lane == 0 || cex < thr);
    const int m = __popc(__ballot_sync(0xffffffffu, kept));
    return __shfl_sync(0xffffffffu, cin, m - 1);
}
// The blob of `pool` that holds expert e: its own index, or its slot in an
// HBM expert cache (every expert a call selects is resident).
__device__ __forceinline__ int blob_slot(const Params& p, int e, int site) {
    return p.slot_of ? idx_in(p.ws.hdr, __ldg(p.slot_of + e), 0, p.n_slots, site) : e;
}
__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void named_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_relaxed_u32(uint32_t* p, uint32_t v) {
    asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void st_relaxed_f32(float* p, float v) {
    asm volatile("st.relaxed.gpu.global.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}
// Morally strong (relaxed, gpu-scope) accesses for values that other CTAs poll
// without a fence: each reader checks every value it uses against the preset
// "not written" pattern, so no ordering between values is needed.
constexpr uint32_t kNotWritten = 0x7fbadbadu;       // a NaN payload that arithmetic never produces
constexpr uint32_t kCodesNotWritten = 0x80808080u;  // -128 bytes: never a code
__device__ __forceinline__ float ld_relaxed_f32(const float* p) {
    float v;
    asm volatile("ld.relaxed.gpu.global.f32 %0, [%1];" : "=f"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ float4 ld_relaxed_f4(const float* p) {
    float4 v;
    asm volatile("ld.relaxed.gpu.global.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p)
                 : "memory");
    return v;
}
__device__ __forceinline__ uint4 ld_relaxed_u4(const void* p) {
    uint4 v;
    asm volatile("ld.relaxed.gpu.global.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p)
                 : "memory");
    return v;
}
__device__ __forceinline__ void st_relaxed_u4(void* p, uint4 v) {
    asm volatile("st.relaxed.gpu.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}
// Nonzero iff some byte of w is 0x80.
__device__ __forceinline__ uint32_t has_byte_80(uint32_t w) {
    const uint32_t v = w ^ 0x80808080u;
    return (v - 0x01010101u) & ~v & 0x80808080u;
}
// Fire-and-forget add (no value returned to the thread).
__device__ __forceinline__ void red_add_u32(uint32_t* p, uint32_t v) {
    asm volatile("red.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// Orders this thread's earlier global writes before its later ones at GPU scope.
__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }
__device__ __forceinline__ int ld_volatile_status(const WsHeader* h) {
    return *reinterpret_cast<const volatile int*>(&h->status);
}

// ---------------------------------------------------------------------------
// Tensor-core (tcgen05) and 2-D TMA wrappers (sm_100a)
// ---------------------------------------------------------------------------
// 2-D tiled TMA load of box {x bytes, y rows} at coordinates (x, y) into this
// CTA's shared memory; completion counted in bytes on `bar`.  No multicast.
__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, int x, int y, uint64_t* bar,
                                            uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
        "l"(tmap), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// TMEM allocation by one full warp; the column base is written to *dst_smem.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// Shared-memory matrix descriptor, no swizzle, K-major core matrices of 8 rows
// x 16 bytes: lbo = byte distance of K-adjacent core matrices, sbo = of
// M/N-adjacent 8-row groups.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}
// D[tmem] (+)= A[tmem] x B[smem]^T, 8-bit x 8-bit -> int32, M = 128, one CTA.
// A: row i in TMEM lane i, K bytes packed four to a 32-bit column.
__device__ __forceinline__ void tc_mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
    asm volatile(
        "{ .reg .pred p; setp.ne.b32 p, %4, 0; tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p; }" ::"r"(
            d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive on `bar` once every tcgen05.mma this thread issued before has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
// 16 consecutive 32-bit TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, int v[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
          "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, int v[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
                 : "r"(taddr)
                 : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// 8 / 16 / 32 consecutive 32-bit TMEM columns of this thread's lane <- registers.
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t v[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(v[0]),
                 "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
                 : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t v[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t v[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
        "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
        "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// Instruction descriptor of tcgen05.mma.kind::i8: D s32, A unsigned 8-bit
// (offset-binary weight codes), B signed 8-bit (activations), both K-major,
// M = 128, N = 8 or a multiple of 16 up to 256.
__host__ __device__ constexpr uint32_t tc_idesc_u8s8(int n) {
    return (2u << 4) | (0u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}
// L2 policy for data read exactly once (the weight stream).
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// Bound of every device-side wait: after this long the waiter records
// MOE_ETIMEOUT in the status word and stops waiting (as do all later waits of
// the call, which see the status word set).
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// Wait for an mbarrier phase with a time bound; false if the wait gave up.
// Unlike the flag waits this does not stop early when another wait has already
// failed: the slots' bulk copies must still be waited for, so that no copy is
// in flight into shared memory when the CTA exits.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, WsHeader* hdr, int site,
                                                  uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > limit_ns) {
            set_status(hdr, MOE_ETIMEOUT, site);
            return false;
        }
    }
    return true;
}
// Wait until *flag == want (acquire), with the same bound.
__device__ __forceinline__ bool flag_wait_bounded(const uint32_t* flag, uint32_t want, WsHeader* hdr, int site,
                                                  uint64_t limit_ns = kWaitLimitNs) {
    if (ld_acquire_u32(flag) == want) return true;
    const uint64_t t0 = global_timer_ns();
    while (ld_acquire_u32(flag) != want) {
        if (ld_volatile_status(hdr) != 0) return false;
        if (global_timer_ns() - t0 > limit_ns) {
            set_status(hdr, MOE_ETIMEOUT, site);
            return false;
        }
        __nanosleep(64);
    }
    return true;
}

// ---------------------------------------------------------------------------
// Reductions for 256-thread CTAs
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    return v;
}
// Block reductions; `red` is a kWarps-element shared scratch the caller owns.
__device__ __forceinline__ float block_max(float v, float* red) {
    v = warp_max(v);
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    float r = red[0];
#pragma unroll
    for (int i = 1; i < kWarps; ++i) r = fmaxf(r, red[i]);
    return r;
}
__device__ __forceinline__ float block_sum(float v, float* red) {
    v = warp_sum(v);
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    float r = red[0];
#pragma unroll
    for (int i = 1; i < kWarps; ++i) r += red[i];
    return r;
}
__device__ __forceinline__ int block_sum_int(int v, int* red) {
    v = __reduce_add_sync(kFull, v);
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    int r = 0;
#pragma unroll
    for (int i = 0; i < kWarps; ++i) r += red[i];
    return r;
}

// In-place exclusive scan of n <= 4 * 256 ints in shared memory by a 256-thread
// CTA; returns the total.  `red` is kWarps ints of shared scratch.
static __device__ int block_exscan(int* a, int n, int* red) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = (n + kThreads - 1) / kThreads;
    const int b = tid * per;
    int local = 0;
    for (int i = 0; i < per; ++i)
        if (b + i < n) local += a[b + i];
    int v = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(kFull, v, o);
        if (lane >= o) v += y;
    }
    __syncthreads();
    if (lane == 31) red[warp] = v;
    __syncthreads();
    int base = 0, total = 0;
#pragma unroll
    for (int i = 0; i < kWarps; ++i) {
        if (i < warp) base += red[i];
        total += red[i];
    }
    int run = base + v - local;
    for (int i = 0; i < per; ++i)
        if (b + i < n) {
            int t = a[b + i];
            a[b + i] = run;
            run += t;
        }
    __syncthreads();
    return total;
}

// ---------------------------------------------------------------------------
// Activation staging layout.  A 16-byte chunk of packed weights holds 32 int4
// codes (or 64 int2, or 16 int8 codes).  The dot kernels split each weight
// word into byte lanes with one mask (offset-binary codes u = c + 8, c + 2 or
// c + 128), so the int8 activations are stored per chunk in the matching byte
// order (int8 weights: the natural order):
//  int4: per 8 columns, word E = (x0,x2,x4,x6) then word O = (x1,x3,x5,x7);
//        sub-array s (s = 0, 1) of a chunk holds columns 16s .. 16s+15.
//  int2: per 16 columns, words P_m = (x_m, x_{m+4}, x_{m+8}, x_{m+12}),
//        m = 0..3; sub-array s (s = 0..3) holds columns 16s .. 16s+15.
// Shared-memory layout of one staged row: [NSUB][nch] uint4, nch = chunks per
// row, NSUB = 8 / wbits, so a warp reading consecutive chunks is conflict-free.
// ---------------------------------------------------------------------------
template <int WB>
__device__ __forceinline__ uint4 permute16(uint4 n) {
    uint4 r;
    if (WB == 8) {  // one code per byte: the natural order
        r = n;
    } else if (WB == 4) {
        r.x = __byte_perm(n.x, n.y, 0x6420);
        r.y = __byte_perm(n.x, n.y, 0x7531);
        r.z = __byte_perm(n.z, n.w, 0x6420);
        r.w = __byte_perm(n.z, n.w, 0x7531);
    } else {
        unsigned a_lo = __byte_perm(n.x, n.y, 0x5140), b_lo = __byte_perm(n.z, n.w, 0x5140);
        unsigned a_hi = __byte_perm(n.x, n.y, 0x7362), b_hi = __byte_perm(n.z, n.w, 0x7362);
        r.x = __byte_perm(a_lo, b_lo, 0x5410);
        r.y = __byte_perm(a_lo, b_lo, 0x7632);
        r.z = __byte_perm(a_hi, b_hi, 0x5410);
        r.w = __byte_perm(a_hi, b_hi, 0x7632);
    }
    return r;
}

// Sum of the 16 signed bytes of a uint4.
__device__ __forceinline__ int sum16(uint4 v) {
    int s = 0;
    s = __dp4a((int)v.x, 0x01010101, s);
    s = __dp4a((int)v.y, 0x01010101, s);
    s = __dp4a((int)v.z, 0x01010101, s);
    s = __dp4a((int)v.w, 0x01010101, s);
    return s;
}

// Stage one int8 row of `ncols` codes (global, 16-byte aligned) into the
// permuted layout at `dst` ([NSUB][nch] uint4); returns this thread's partial
// sum of the codes (the caller reduces it).
template <int WB>
__device__ __forceinline__ int stage_row(const int8_t* src, int ncols, uint4* dst) {
    constexpr int NSUB = 8 / WB;
    const int n16 = ncols / 16;          // 16-byte pieces
    const int nch = n16 / NSUB;          // weight chunks per row
    int s = 0;
    for (int i = threadIdx.x; i < n16; i += kThreads) {
        uint4 v = __ldcg(reinterpret_cast<const uint4*>(src) + i);
        s += sum16(v);
        const int c = i / NSUB, sub = i % NSUB;
        dst[sub * nch + c] = permute16<WB>(v);
    }
    return s;
}

// Dot of one 16-byte weight chunk with one staged activation chunk.
template <int WB>
__device__ __forceinline__ int dot_chunk(const uint4 w, const uint4* xs, int nch, int c, int acc) {
    if (WB == 8) {  // 16 codes, offset-binary bytes c + 128 by flipping each sign bit
        const uint4 x0 = xs[c];
        acc = dp4a_us(w.x ^ 0x80808080u, (int)x0.x, acc);
        acc = dp4a_us(w.y ^ 0x80808080u, (int)x0.y, acc);
        acc = dp4a_us(w.z ^ 0x80808080u, (int)x0.z, acc);
        acc = dp4a_us(w.w ^ 0x80808080u, (int)x0.w, acc);
    } else if (WB == 4) {
        const uint4 x0 = xs[c], x1 = xs[nch + c];
        const unsigned a = w.x ^ 0x88888888u, b = w.y ^ 0x88888888u;
        const unsigned cc = w.z ^ 0x88888888u, dd = w.w ^ 0x88888888u;
        acc = dp4a_us(a & 0x0F0F0F0Fu, (int)x0.x, acc);
        acc = dp4a_us((a >> 4) & 0x0F0F0F0Fu, (int)x0.y, acc);
        acc = dp4a_us(b & 0x0F0F0F0Fu, (int)x0.z, acc);
        acc = dp4a_us((b >> 4) & 0x0F0F0F0Fu, (int)x0.w, acc);
        acc = dp4a_us(cc & 0x0F0F0F0Fu, (int)x1.x, acc);
        acc = dp4a_us((cc >> 4) & 0x0F0F0F0Fu, (int)x1.y, acc);
        acc = dp4a_us(dd & 0x0F0F0F0Fu, (int)x1.z, acc);
        acc = dp4a_us((dd >> 4) & 0x0F0F0F0Fu, (int)x1.w, acc);
    } else {
        const unsigned ws[4] = {w.x ^ 0xAAAAAAAAu, w.y ^ 0xAAAAAAAAu, w.z ^ 0xAAAAAAAAu, w.w ^ 0xAAAAAAAAu};
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            const uint4 xv = xs[s * nch + c];
            acc = dp4a_us(ws[s] & 0x03030303u, (int)xv.x, acc);
            acc = dp4a_us((ws[s] >> 2) & 0x03030303u, (int)xv.y, acc);
            acc = dp4a_us((ws[s] >> 4) & 0x03030303u, (int)xv.z, acc);
            acc = dp4a_us((ws[s] >> 6) & 0x03030303u, (int)xv.w, acc);
        }
    }
    return acc;
}

// Offset of the offset-binary codes: sum c*x = sum u*x - kOff * sum x.
template <int WB>
__device__ __forceinline__ constexpr int code_offset() { return WB == 8 ? 128 : WB == 4 ? 8 : 2; }

// Order-preserving map of a float to an unsigned key (larger float, larger key).
__device__ __forceinline__ unsigned float_key(float v) {
    const unsigned b = __float_as_uint(v);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Quantiser rule of the layer (fp32, IEEE division, round half to even).
__device__ __forceinline__ int quant_code(float v, float s) {
    int q = __float2int_rn(__fdiv_rn(v, s));
    return max(-127, min(127, q));
}

// The same codes without a division per value.  r = quant_recip(s) is the
// correctly rounded 1/s; q = fl(v r) is within 1.5 * 2^-23 * |v / s| <= 2.3e-5
// of the IEEE quotient fl(v / s) for |v / s| <= 128 (two roundings of 2^-24
// each against one), so unless q lies within 1e-3 of a half-integer both round
// to the same integer; those rare values, and any |q| > 128 (or an infinite
// r from a denormal s), take the exact quotient.
__device__ __forceinline__ float quant_recip(float s) { return __fdiv_rn(1.0f, s); }
// The exact quotient out of line: taken for well under 1% of values, it keeps
// the division's instructions out of every unrolled copy of the fast path
// (code that a kernel runs once per call is fetched cold, from HBM, while the
// weight streams saturate it).
static __device__ __noinline__ int quant_code_slow(float v, float s) { return quant_code(v, s); }
__device__ __forceinline__ int quant_code_r(float v, float s, float r) {
    const float q = __fmul_rn(v, r);
    const float aq = fabsf(q);
    if (!(aq <= 128.0f) || fabsf(aq - floorf(aq) - 0.5f) < 1e-3f) return quant_code_slow(v, s);
    return max(-127, min(127, __float2int_rn(q)));
}

template <typename XT>
__device__ __forceinline__ float load_x(const XT* x, size_t i);
template <>
__device__ __forceinline__ float load_x<float>(const float* x, size_t i) { return __ldg(x + i); }
template <>
__device__ __forceinline__ float load_x<__nv_bfloat16>(const __nv_bfloat16* x, size_t i) {
    return __bfloat162float(x[i]);
}

// 4 consecutive activations (i multiple of 4) as float4.
template <typename XT>
__device__ __forceinline__ float4 load_x4(const XT* x, size_t i);
template <>
__device__ __forceinline__ float4 load_x4<float>(const float* x, size_t i) {
    return __ldg(reinterpret_cast<const float4*>(x + i));
}
template <>
__device__ __forceinline__ float4 load_x4<__nv_bfloat16>(const __nv_bfloat16* x, size_t i) {
    uint2 v = __ldg(reinterpret_cast<const uint2*>(x + i));
    float4 r;
    r.x = __uint_as_float(v.x << 16);
    r.y = __uint_as_float(v.x & 0xFFFF0000u);
    r.z = __uint_as_float(v.y << 16);
    r.w = __uint_as_float(v.y & 0xFFFF0000u);
    return r;
}

}  // namespace moe
