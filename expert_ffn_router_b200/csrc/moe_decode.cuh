// The whole MoE layer for decode-sized batches (T <= 8) in one persistent,
// cooperatively launched kernel: one CTA per SM, two groups of 8 consumer
// warps and one producer warp.
//
// The producer streams every weight row the CTA needs -- its router rows, its
// share of the shared expert's gate/up rows, then (once the routing is known)
// its share of the routed gate/up rows and of all down rows -- into a ring of
// shared-memory slots with 1-D bulk copies (cp.async.bulk, completion counted
// on an mbarrier per slot).  The consumers work through the same unit
// sequence, the two consumer groups taking alternate units (4 warps per
// scheduler to hide the dot products' latencies):
//   1. the router bias into shared memory;
//   2. quantise the T tokens (every CTA, into its own shared memory) while
//      the first rows are on their way;
//   3. router units: logits of this CTA's experts (from x as given), turned
//      at once into (selection value, score) pairs -> workspace; arrive at
//      the one grid barrier; meanwhile the other consumer group runs the
//      CTA's first shared-expert gate/up unit (its rows were copied with the
//      router rows);
//   4. after the barrier every CTA reads all pairs and derives the same
//      top-k routing and the same expert task list (no second barrier), so
//      the producer can issue routed rows at once;
//   5. gate/up units: the remaining shared-expert ones, then the routed ones;
//      with several tokens each warp counts the rows it finished per task
//      and, once at the end of the phase, publishes the counts (one release
//      fence, then fire-and-forget adds on per-task counters);
//   6r. single token: no counts and no fences -- the call's h rows, code
//      rows and scales are preset to "not written" before the grid barrier;
//      one CTA per task polls the task's h values until all are written,
//      requantises them into int8 codes in the dot layout (max |h| from the
//      values themselves) and writes codes and scale; every CTA owns a
//      contiguous range of output rows, streams those rows of every task's
//      down matrix (each CTA starting at its own task, so that the CTAs read
//      different matrices at once), stages every task's codes and scale in
//      shared memory in one batch of polled loads, and combines its rows
//      locally;
//   6. otherwise: down units (waiting, bounded, until their task's counter
//      shows every gate/up row) requantise and stage the task's h; at the end
//      each CTA signs its row blocks off and the CTA bringing a row block's
//      last task combines it.
// Each expert selected by several tokens is streamed once: a task is one
// expert with all its tokens.  Every wait is bounded (MOE_ETIMEOUT).
#pragma once

#include <float.h>

#include "moe_common.cuh"

namespace moe {

constexpr int kDecWarps = 8;                         // warps of a consumer group = rows per gate/up unit
constexpr int kDecGroups = 2;
constexpr int kDecConsWarps = kDecWarps * kDecGroups;
constexpr int kDecThreads = (kDecConsWarps + 1) * 32;
constexpr int kDecCons = kDecConsWarps * 32;           // consumer threads
constexpr int kDecGrp = kDecWarps * 32;                // threads of one group
constexpr int kDecMaxSlots = 4;  // ring slots; always even (see decode_plan)
constexpr int kDecMaxT = 8;
constexpr int kDecMaxK = 32;
constexpr int kDecMaxTasks = kDecMaxT * kDecMaxK + 1;
constexpr int kDecBiasCache = 256;  // experts whose bias the kernel keeps in shared memory
constexpr int kDecBar = 1;  // named barrier of all consumer warps; 2 + g: group g
constexpr int kDecNQ = 6;   // down rows per warp per unit of the unrolled shapes (rd = 48)
constexpr int kDecXr = 8;   // router float4 inputs per thread for one token (d <= 8 * 4 * 256)
constexpr int kDecTraceSlots = 32;  // phase stamps per CTA (moe_layer_opts.trace)

struct DecPlan {
    int slot_bytes, nslot;
    int wbytes;        // weight bytes of a slot; the row scales follow at this offset
    int rd;            // down rows per unit (multiple of kDecWarps)
    int rr;            // router rows per unit (1 or 2)
    int nu_gu, nu_dn;  // units per task
    int xs_off, hs_off, ring_off, smem_bytes;
    int hs_grp_bytes;  // h staging bytes of one consumer group (T * f)
    int rowrange;      // single-token down by output-row ranges (see step 6r)
    int dn_rot;        // row-range: CTA c takes the down tasks from task c mod n_tasks on
    int gu_rmaj;       // row-range: routed gate/up units ordered row block first, tasks inner
};
// Row-range down unit (single token): [rows x down row][row scales at wbytes].
constexpr int kDecRRMaxRows = 44;

constexpr int kDecRRMaxTasks = kDecMaxK + 1;  // tasks of a single token (row-range down)
constexpr int kDecRRChunks = 3;     // row-range: 16-byte chunks of the tasks' codes each consumer thread stages
constexpr int kDecSlotCache = 260;  // experts (+ shared) whose cache slot the kernel keeps in shared memory

// Shared control block of the kernel, sized for TM tokens.
template <int TM>
struct DecCtl {
    static constexpr int kTasks = TM * kDecMaxK + 1;  // the shared expert + one task per (token, slot) at most
    uint64_t full[kDecMaxSlots];
    uint64_t empty[kDecMaxSlots];
    uint64_t route_ready;
    uint32_t epoch;
    int n_tasks;
    int hq_task[kDecGroups];
    int n_last;
    float sx[TM];
    int xcs[TM];
    int idx[TM][kDecMaxK];
    float w[TM][kDecMaxK];
    int4 tasks[kTasks];  // (expert, n tokens, blob slot in the pool, -)
    int ttok[kTasks][TM];
    int sorted[TM * kDecMaxK];    // assignment ids by (expert, token, slot)
    int sorted_e[TM * kDecMaxK];  // their experts
    int hcs[kDecGroups][TM];
    float hsh[kDecGroups][TM];
    int last_rb[kDecCons];
    float bias_s[kDecBiasCache];  // the router bias (E <= kDecBiasCache)
    float redf[kDecConsWarps];
    int redi[kDecConsWarps];
    float part[kDecGroups][kDecWarps][2 * TM];
    float rsh[kDecRRMaxTasks];  // one token: the scale of each task's staged codes
    int slot_s[kDecSlotCache];  // HBM expert cache: each expert's blob slot (E + shared <= kDecSlotCache)
};

// --- consumer reductions over all consumer warps (named barrier 1) ---------
__device__ __forceinline__ float cons_max(float v, float* red) {
    v = warp_max(v);
    named_sync(kDecBar, kDecCons);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    named_sync(kDecBar, kDecCons);
    float r = red[0];
#pragma unroll
    for (int i = 1; i < kDecConsWarps; ++i) r = fmaxf(r, red[i]);
    return r;
}
__device__ __forceinline__ int cons_sum_int(int v, int* red) {
    v = __reduce_add_sync(kFull, v);
    named_sync(kDecBar, kDecCons);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    named_sync(kDecBar, kDecCons);
    int r = 0;
#pragma unroll
    for (int i = 0; i < kDecConsWarps; ++i) r += red[i];
    return r;
}
// ... and over one group's 8 warps (named barrier 2 + g); red has kDecConsWarps entries
__device__ __forceinline__ int grp_sum_int(int v, int* red, int g) {
    v = __reduce_add_sync(kFull, v);
    named_sync(2 + g, kDecGrp);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    named_sync(2 + g, kDecGrp);
    int r = 0;
#pragma unroll
    for (int i = 0; i < kDecWarps; ++i) r += red[g * kDecWarps + i];
    return r;
}

// One 16-byte weight chunk against one activation chunk held in registers
// (x[s] = sub-array s of the staged layout), into two accumulators (even and
// odd weight words) to halve the dependent dp4a chain.
template <int WB>
__device__ __forceinline__ void dot_chunk_regs(const uint4 w, const uint4* x, int& a0, int& a1) {
    if (WB == 8) {  // 16 codes, offset-binary by flipping each sign bit
        a0 = dp4a_us(w.x ^ 0x80808080u, (int)x[0].x, a0);
        a1 = dp4a_us(w.y ^ 0x80808080u, (int)x[0].y, a1);
        a0 = dp4a_us(w.z ^ 0x80808080u, (int)x[0].z, a0);
        a1 = dp4a_us(w.w ^ 0x80808080u, (int)x[0].w, a1);
    } else if (WB == 4) {
        const unsigned p = w.x ^ 0x88888888u, q = w.y ^ 0x88888888u;
        const unsigned r = w.z ^ 0x88888888u, t = w.w ^ 0x88888888u;
        a0 = dp4a_us(p & 0x0F0F0F0Fu, (int)x[0].x, a0);
        a1 = dp4a_us((p >> 4) & 0x0F0F0F0Fu, (int)x[0].y, a1);
        a0 = dp4a_us(q & 0x0F0F0F0Fu, (int)x[0].z, a0);
        a1 = dp4a_us((q >> 4) & 0x0F0F0F0Fu, (int)x[0].w, a1);
        a0 = dp4a_us(r & 0x0F0F0F0Fu, (int)x[1].x, a0);
        a1 = dp4a_us((r >> 4) & 0x0F0F0F0Fu, (int)x[1].y, a1);
        a0 = dp4a_us(t & 0x0F0F0F0Fu, (int)x[1].z, a0);
        a1 = dp4a_us((t >> 4) & 0x0F0F0F0Fu, (int)x[1].w, a1);
    } else {
        const unsigned ws[4] = {w.x ^ 0xAAAAAAAAu, w.y ^ 0xAAAAAAAAu, w.z ^ 0xAAAAAAAAu, w.w ^ 0xAAAAAAAAu};
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            a0 = dp4a_us(ws[s] & 0x03030303u, (int)x[s].x, a0);
            a1 = dp4a_us((ws[s] >> 2) & 0x03030303u, (int)x[s].y, a1);
            a0 = dp4a_us((ws[s] >> 4) & 0x03030303u, (int)x[s].z, a0);
            a1 = dp4a_us((ws[s] >> 6) & 0x03030303u, (int)x[s].w, a1);
        }
    }
}

// 16 consecutive activations (i a multiple of 16) as floats.
template <typename XT>
__device__ __forceinline__ void load16(const XT* x, size_t i, float v[16]) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float4 f4 = load_x4(x, i + 4 * q);
        v[4 * q + 0] = f4.x;
        v[4 * q + 1] = f4.y;
        v[4 * q + 2] = f4.z;
        v[4 * q + 3] = f4.w;
    }
}

// Router output of one (token, expert) as the decode kernel keeps it: the
// selection value sigmoid(logit) + bias and the score sigmoid(logit), fp32
// bits, computed by the CTA that owns the expert's router row.
__device__ __forceinline__ uint2 route_pair(float logit, float bias) {
    const float s = __fdiv_rn(1.0f, __fadd_rn(1.0f, expf(-logit)));
    return make_uint2(__float_as_uint(__fadd_rn(s, bias)), __float_as_uint(s));
}

// Top-k of one token by one warp from its row of (selection, score) pairs in
// global memory; lane j (< k) returns slot j's expert and weight (-1 and 0 for
// a slot the TOPP truncation drops).  Same rule as topk_token.
__device__ __forceinline__ void topk_warp(const uint2* prow, int E, int k, float scale, float topp, float* s_sm,
                                          float* sel_sm, int& my_e, float& my_w) {
    const int lane = threadIdx.x & 31;
    for (int e = lane; e < E; e += 32) {
        const uint2 pr = __ldcg(prow + e);
        s_sm[e] = __uint_as_float(pr.y);
        sel_sm[e] = __uint_as_float(pr.x);
    }
    __syncwarp();
    float ssum = 0.0f, my_s = 0.0f, cex = 0.0f, cin = 0.0f;
    my_e = 0;
    for (int j = 0; j < k; ++j) {
        float bv = -FLT_MAX;
        int be = 0x7fffffff;
        for (int e = lane; e < E; e += 32) {
            const float v = sel_sm[e];
            if (v > bv) {
                bv = v;
                be = e;
            }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            const float ov = __shfl_xor_sync(kFull, bv, o);
            const int oe = __shfl_xor_sync(kFull, be, o);
            if (ov > bv || (ov == bv && oe < be)) {
                bv = ov;
                be = oe;
            }
        }
        const float sj = s_sm[be];
        if (lane == j) {
            my_e = be;
            my_s = sj;
            cex = ssum;
        }
        ssum = __fadd_rn(ssum, sj);
        if (lane == j) cin = ssum;
        __syncwarp();
        if (lane == 0) sel_sm[be] = -INFINITY;
        __syncwarp();
    }
    bool kept;
    const float norm = topp_keep(topp, k, ssum, cex, cin, kept);
    my_w = kept ? __fmul_rn(__fdiv_rn(my_s, norm), scale) : 0.0f;
    if (!kept) my_e = -1;
}

// NG / ND: 16-byte weight chunks per lane of a gate/up row / a down row when
// the row is exactly 32 * NG (32 * ND) chunks (fully unrolled, weights loaded
// up front); 0 = any shape (runtime loop).

// Top-k of one token by one warp for E <= 256: lane l holds experts l + 32 i
// in registers; each round takes the largest selection score (lowest index on
// ties) with two warp reductions.  Same rule and arithmetic as topk_warp.
__device__ __forceinline__ void topk_warp_small(const uint2* prow, int E, int k, float scale, float topp, int& my_e,
                                                float& my_w, unsigned long long* tr) {
    const int lane = threadIdx.x & 31;
    float sv[8];
    unsigned key[8];
    uint2 pr[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) pr[i] = lane + 32 * i < E ? __ldcg(prow + lane + 32 * i) : make_uint2(0u, 0u);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        sv[i] = __uint_as_float(pr[i].y);
        key[i] = lane + 32 * i < E ? float_key(__uint_as_float(pr[i].x)) : 0u;  // 0: below every real key
    }
    if (tr && lane == 0 && key[0] != 1u) *tr = global_timer_ns();  // once loaded (the branch reads a value)
    float ssum = 0.0f, my_s = 0.0f, cex = 0.0f, cin = 0.0f;
    my_e = 0;
    for (int j = 0; j < k; ++j) {
        unsigned best = 0u;
        int bi = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (key[i] > best) {  // ascending index within the lane: strict keeps the lower one
                best = key[i];
                bi = i;
            }
        const unsigned mx = __reduce_max_sync(kFull, best);
        const int e_win = __reduce_min_sync(kFull, best == mx ? lane + 32 * bi : 0x7fffffff);
        const int owner = e_win & 31, slot = e_win >> 5;
        float s_mine = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (i == slot) s_mine = sv[i];
        const float sj = __shfl_sync(kFull, s_mine, owner);
        if (lane == owner) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (i == slot) key[i] = 0u;
        }
        if (lane == j) {
            my_e = e_win;
            my_s = sj;
            cex = ssum;
        }
        ssum = __fadd_rn(ssum, sj);
        if (lane == j) cin = ssum;
    }
    bool kept;
    const float norm = topp_keep(topp, k, ssum, cex, cin, kept);
    my_w = kept ? __fmul_rn(__fdiv_rn(my_s, norm), scale) : 0.0f;
    if (!kept) my_e = -1;
}

template <int WB, int TM, int NG, int ND, typename XT>
__global__ void __launch_bounds__(kDecThreads, 1) k_decode(const Params p, const DecPlan pl, const XT* __restrict__ x) {
    constexpr int NSUB = 8 / WB;
    extern __shared__ __align__(128) uint8_t dec_smem[];
    DecCtl<TM>& C = *reinterpret_cast<DecCtl<TM>*>(dec_smem);
    constexpr int kTasks = DecCtl<TM>::kTasks;
    uint4* xs = reinterpret_cast<uint4*>(dec_smem + pl.xs_off);
    uint8_t* hsb = dec_smem + pl.hs_off;
    uint8_t* ring = dec_smem + pl.ring_off;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = gridDim.x, c = blockIdx.x;
    const int d = p.m.d, f = p.m.f, E = p.m.E, k = p.m.k, T = p.m.T, S = p.m.S, HS = p.m.has_shared;
    const int rb_gu = d * WB / 8, rb_dn = f * WB / 8;
    const int nch_gu = rb_gu / 16, nch_dn = rb_dn / 16;
    const int nslot = pl.nslot, slot_bytes = pl.slot_bytes;
    WsHeader* hdr = p.ws.hdr;
    unsigned long long* trace = p.trace ? p.trace + (size_t)blockIdx.x * kDecTraceSlots : nullptr;
#define DEC_TRACE(i)                                   \
    do {                                               \
        if (trace) trace[i] = global_timer_ns();       \
    } while (0)

    if (tid == 0) {
        for (int i = 0; i < nslot; ++i) {
            mbar_init(&C.full[i], 1);
            mbar_init(&C.empty[i], kDecWarps);
        }
        mbar_init(&C.route_ready, 1);
        fence_mbar_init();
        C.epoch = __ldcg(&hdr->epoch);
        for (int g = 0; g < kDecGroups; ++g) C.hq_task[g] = -1;
        if (HS) {  // the shared task (task 0): every token, known before any routing
            C.tasks[0] = make_int4(E, T, E, 0);  // (a cached pool's slot is filled in below)
            for (int t = 0; t < T; ++t) C.ttok[0][t] = t * S + k;
        }
    }
    __syncthreads();  // the only CTA-wide barrier: producer and consumers part here
    const uint32_t epoch = C.epoch;
    // running maxima of |h| alternate between two arrays by call parity; each
    // call zeroes the one the next call uses
    uint32_t* amax_cur = (epoch & 1) ? p.ws.amax2 : p.ws.amax;
    uint32_t* amax_nxt = (epoch & 1) ? p.ws.amax : p.ws.amax2;
    // the same for the per-task counts of finished gate/up rows
    uint32_t* rows_cur = p.ws.ready + (epoch & 1) * 1024;
    uint32_t* rows_nxt = p.ws.ready + ((epoch & 1) ^ 1) * 1024;
    // this CTA's output rows in the row-range down: whole quads of rows, so
    // the row scales are whole 16-byte bulk copies
    const int rr_lo = (int)((long long)c * (d / 4) / G) * 4;
    const int rr_rows = (int)((long long)(c + 1) * (d / 4) / G) * 4 - rr_lo;
    const bool rowrange = TM == 1 && ND > 0 && pl.rowrange;
    // every CTA takes an equal share of every routed expert's rows (experts
    // stream at different speeds, and a CTA's finish time is then the average)
    const bool rmaj = rowrange && pl.gu_rmaj;
    if (tid == 0) DEC_TRACE(0);
    const int n_my_router = c < E ? (E - c + G - 1) / G : 0;  // experts c, c+G, ...
    const int n_router_units = (n_my_router + pl.rr - 1) / pl.rr;
    const int n_sh_units = HS && c < pl.nu_gu ? (pl.nu_gu - c + G - 1) / G : 0;  // shared units c, c+G, ...

    // =====================================================================
    // producer: lane 0 of the last warp
    // =====================================================================
    if (warp == kDecConsWarps) {
        if (lane != 0) return;
        // ring position of the next unit, advanced without divisions
        int ps = 0;          // slot
        uint32_t pr = 0;     // round of that slot (times it has been filled before)
        uint32_t issued = 0; // units issued
        unsigned long long t_empty = 0;  // time blocked on free slots (traced)
        auto take = [&](uint32_t bytes) -> uint8_t* {
            if (pr > 0) {
                const unsigned long long t0 = trace ? global_timer_ns() : 0;
                mbar_wait_bounded(&C.empty[ps], (pr - 1) & 1, hdr, 100 + ps, 2 * p.wait_ns);
                if (trace) t_empty += global_timer_ns() - t0;
            }
            mbar_arrive_expect_tx(&C.full[ps], bytes);
            return ring + (size_t)ps * slot_bytes;
        };
        auto advance = [&]() {
            ++issued;
            if (++ps == nslot) {
                ps = 0;
                ++pr;
            }
        };
        const int n_blobs = p.slot_of ? p.n_slots : E + HS;  // blobs the pool holds
        // the shared expert's blob (its slot in a cached pool, looked up here:
        // the producer issues the shared rows before the routing)
        const int sh_slot = blob_slot(p, E, 610);
        // expert rows are read once per call: evict-first keeps L2 for what
        // the call reads again (h rows, codes, the polled hand-off values);
        // measured on B200 at one token: 55.8 us per call instead of 56.7
        const uint64_t pol_w = l2_policy_evict_first();
        auto issue_gu = [&](int e, int blob, int j) {  // expert e (its scales), in pool blob `blob`
            blob = idx_in(hdr, blob, 0, n_blobs, 611);  // never copy outside the pool, whatever happened
            e = idx_in(hdr, e, 0, E + HS, 609);
            const int r0 = j * kDecWarps, rows = min(kDecWarps, f - r0);  // f % 8 == 0: rows == 8
            const uint32_t bytes = (uint32_t)rows * rb_gu;
            const uint8_t* base = p.pool + (size_t)blob * p.blob_bytes;
            const float* sc = p.scales + (size_t)e * p.scale_rows;
            uint64_t* bar = &C.full[ps];
            uint8_t* dst = take(2 * bytes + 2 * rows * 4);
            bulk_g2s_hint(dst, base + (size_t)r0 * rb_gu, bytes, bar, pol_w);
            bulk_g2s_hint(dst + (size_t)kDecWarps * rb_gu, base + ((size_t)f + r0) * rb_gu, bytes, bar, pol_w);
            bulk_g2s(dst + pl.wbytes, sc + r0, rows * 4, bar);                      // gate row scales
            bulk_g2s(dst + pl.wbytes + kDecWarps * 4, sc + f + r0, rows * 4, bar);  // up row scales
            advance();
        };
        for (int ru = 0; ru < n_router_units; ++ru) {
            const int rows = min(pl.rr, n_my_router - ru * pl.rr);
            uint8_t* dst = take((uint32_t)rows * d * 4);
            for (int i = 0; i < rows; ++i) {
                const int e = c + (ru * pl.rr + i) * G;
                bulk_g2s(dst + (size_t)i * d * 4, p.w_router + (size_t)e * d, (uint32_t)d * 4, &C.full[ps]);
            }
            advance();
        }
        // gate/up rows: the shared expert's units c, c + G, ... first, then,
        // once the routing is known, this CTA's share of the routed units.
        // One call site for both (the routed copies are issued by code that
        // is already in the instruction cache, not by a cold second copy).
        int n_tasks = HS;
#pragma unroll 1
        for (int ph = 0; ph < 2; ++ph) {
            long long n_units = n_sh_units;
            int ti = 0, j = c, jstep = G, jwrap = 0x7fffffff, sh_blob = E;
            if (ph == 1) {
                DEC_TRACE(12);
                mbar_wait_bounded(&C.route_ready, 0, hdr, 110, 2 * p.wait_ns);
                DEC_TRACE(13);
                n_tasks = min(max(C.n_tasks, HS), kTasks);
                const long long Nr = (long long)(n_tasks - HS) * pl.nu_gu;
                const long long lo = c * Nr / G, hi = (c + 1) * Nr / G;
                n_units = hi - lo;
                if (rmaj) {  // unit g: row block g / n_routed of task HS + g mod n_routed
                    ti = HS + (int)(lo % (n_tasks - HS));
                    j = (int)(lo / (n_tasks - HS));
                } else {
                    ti = HS + (int)(lo / pl.nu_gu);
                    j = (int)(lo % pl.nu_gu);
                }
                jstep = 1;
                jwrap = pl.nu_gu;
                sh_blob = -1;
            }
            const bool tasks_inner = ph == 1 && rmaj;
            for (long long g = 0; g < n_units; ++g) {
                if (sh_blob >= 0)
                    issue_gu(sh_blob, sh_slot, j);
                else
                    issue_gu(C.tasks[ti].x, C.tasks[ti].z, j);
                if (tasks_inner) {
                    if (++ti == n_tasks) {
                        ti = HS;
                        ++j;
                    }
                    continue;
                }
                j += jstep;
                if (j == jwrap) {
                    j = 0;
                    ++ti;
                }
            }
        }
        if (rowrange) {
            // one unit per task: this CTA's rows of the task's down matrix and
            // their scales (the consumers read the task's codes from global
            // memory themselves, once written)
            const int n_rr = min(n_tasks, kDecRRMaxTasks);
            const int rot = pl.dn_rot ? c % n_rr : 0;  // the CTA's task order (so the CTAs read different matrices)
            for (int i = 0; i < n_rr; ++i) {
                const int ti = i + rot < n_rr ? i + rot : i + rot - n_rr;
                const int blob = idx_in(hdr, C.tasks[ti].z, 0, n_blobs, 612);
                const int ex = idx_in(hdr, C.tasks[ti].x, 0, E + HS, 608);
                const uint32_t wb = (uint32_t)rr_rows * rb_dn;
                uint8_t* dst = take(wb + (uint32_t)rr_rows * 4);
                bulk_g2s_hint(dst, p.pool + (size_t)blob * p.blob_bytes + 2 * (size_t)f * rb_gu + (size_t)rr_lo * rb_dn,
                              wb, &C.full[ps], pol_w);
                bulk_g2s(dst + pl.wbytes, p.scales + (size_t)ex * p.scale_rows + 2 * f + rr_lo, (uint32_t)rr_rows * 4,
                         &C.full[ps]);
                advance();
            }
        } else {
            const long long Nd = (long long)n_tasks * pl.nu_dn;
            const long long lo = c * Nd / G, hi = (c + 1) * Nd / G;
            int ti = (int)(lo / pl.nu_dn), j = (int)(lo % pl.nu_dn);
            for (long long g = lo; g < hi; ++g) {
                const int blob = idx_in(hdr, C.tasks[ti].z, 0, n_blobs, 612);
                const int ex = idx_in(hdr, C.tasks[ti].x, 0, E + HS, 608);
                const int r0 = j * pl.rd, rows = min(pl.rd, d - r0);  // multiples of 8
                const uint32_t bytes = (uint32_t)rows * rb_dn;
                uint64_t* bar = &C.full[ps];
                uint8_t* dst = take(bytes + rows * 4);
                bulk_g2s_hint(dst, p.pool + (size_t)blob * p.blob_bytes + 2 * (size_t)f * rb_gu + (size_t)r0 * rb_dn,
                              bytes, bar, pol_w);
                bulk_g2s(dst + pl.wbytes, p.scales + (size_t)ex * p.scale_rows + 2 * f + r0, rows * 4, bar);
                advance();
                if (++j == pl.nu_dn) {
                    j = 0;
                    ++ti;
                }
            }
        }
        DEC_TRACE(14);
        if (trace) trace[10] = t_empty;
        // drain: every copy issued must have landed before this thread (and so
        // the CTA and its shared memory) can retire
        for (int s = 0; s < nslot; ++s)
            if (issued > (uint32_t)s)
                mbar_wait_bounded(&C.full[s], ((issued - s + nslot - 1) / nslot - 1) & 1, hdr, 120 + s, 2 * p.wait_ns);
        DEC_TRACE(15);
        return;
    }

    // =====================================================================
    // consumers: warps 0..15, two groups of 8; unit u belongs to group u & 1
    // =====================================================================
    const int ctid = tid;
    const int grp = warp / kDecWarps, gw = warp % kDecWarps, gtid = ctid % kDecGrp;
    const int hs_grp = pl.hs_grp_bytes;  // staging bytes of one group

    // single token: this thread's router inputs x[4v .. 4v + 3], v = gtid + i * kDecGrp
    float4 xrr[TM == 1 ? kDecXr : 1];
    if constexpr (TM == 1) {
#pragma unroll
        for (int i = 0; i < kDecXr; ++i) {
            const int v = (ctid % kDecGrp) + i * kDecGrp;
            xrr[i] = v < d / 4 ? load_x4(x, (size_t)4 * v) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    // ---- 1. the router bias into shared memory (the router reads x as given) ----
    if (E <= kDecBiasCache)
        for (int e = ctid; e < E; e += kDecCons) C.bias_s[e] = __ldg(p.bias + e);
    // an HBM expert cache: every expert's slot (the producer reads the shared
    // task's slot only after the routing is published to it)
    if (p.slot_of) {
        if (E + HS <= kDecSlotCache)
            for (int e = ctid; e < E + HS; e += kDecCons) C.slot_s[e] = blob_slot(p, e, 607);
        if (HS && ctid == 0) C.tasks[0].z = blob_slot(p, E, 607);
    }
    named_sync(kDecBar, kDecCons);  // the bias cache is filled

    // unit index (identical sequence to the producer's) and its ring slot and
    // phase, advanced without divisions; unit u belongs to group u & 1
    uint32_t u = 0;
    int cs_slot = 0;
    uint32_t cs_phase = 0;
    unsigned long long t_full = 0;  // time thread 0 spent waiting for data (traced)
    auto next_unit = [&]() {
        ++u;
        if (++cs_slot == nslot) {
            cs_slot = 0;
            cs_phase ^= 1u;
        }
    };
    auto wait_full = [&]() -> const uint8_t* {
        const unsigned long long t0 = (trace && ctid == 0) ? global_timer_ns() : 0;
        mbar_wait_bounded(&C.full[cs_slot], cs_phase, hdr, 200 + cs_slot, 2 * p.wait_ns);
        if (trace && ctid == 0) t_full += global_timer_ns() - t0;
        return ring + (size_t)cs_slot * slot_bytes;
    };
    auto release = [&]() {  // the proxy fence orders the warp's reads before the next bulk copy
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&C.empty[cs_slot]);
    };
    const bool mine_even = grp == 0;
    auto mine = [&]() { return ((u & 1) == 0) == mine_even; };

    // ---- 2. quantise the T tokens into the permuted staging layout (while
    //         the router rows are on their way) ----
    for (int t = 0; t < T; ++t) {
        const XT* xt = x + (size_t)t * d;
        float v[16];
        float m = 0.0f;
        const int pc = ctid;  // d / 16 <= kDecCons pieces of 16 values
        if (pc < d / 16) {
            load16(xt, (size_t)pc * 16, v);
#pragma unroll
            for (int q = 0; q < 16; ++q) m = fmaxf(m, fabsf(v[q]));
        }
        m = cons_max(m, C.redf);
        const float s = m == 0.0f ? 0.0f : __fdiv_rn(m, 127.0f);
        const float rs = quant_recip(s);
        int cs = 0;
        if (pc < d / 16) {
            unsigned wds[4] = {0u, 0u, 0u, 0u};
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const int code = m == 0.0f ? 0 : quant_code_r(v[q], s, rs);
                cs += code;
                wds[q >> 2] |= ((unsigned)code & 0xFFu) << (8 * (q & 3));
            }
            xs[(size_t)t * NSUB * nch_gu + (pc % NSUB) * nch_gu + pc / NSUB] =
                permute16<WB>(make_uint4(wds[0], wds[1], wds[2], wds[3]));
        }
        cs = cons_sum_int(cs, C.redi);
        if (ctid == 0) {
            C.sx[t] = s;
            C.xcs[t] = cs;
        }
    }
    named_sync(kDecBar, kDecCons);
    if (ctid == 0) DEC_TRACE(1);
    for (int i = c * kDecCons + ctid; i < p.a_cap; i += G * kDecCons) amax_nxt[i] = 0u;
    for (int i = c * kDecCons + ctid; i < kDecMaxTasks; i += G * kDecCons) rows_nxt[i] = 0u;
    if (rowrange) {
        // single token: the h rows, code rows and scales of the call's S
        // assignments start as "not written", so that the gate/up -> down
        // hand-off needs no fence (a fence issued while the weight streams
        // saturate HBM takes microseconds): the requantiser polls the h values
        // and the down units poll the codes and scale.  The grid barrier below
        // orders these stores before every write of this call.
        const uint4 hn = make_uint4(kNotWritten, kNotWritten, kNotWritten, kNotWritten);
        const uint4 qn = make_uint4(kCodesNotWritten, kCodesNotWritten, kCodesNotWritten, kCodesNotWritten);
        for (int i = c * kDecCons + ctid; i < S * f / 4; i += G * kDecCons) reinterpret_cast<uint4*>(p.ws.h)[i] = hn;
        for (int i = c * kDecCons + ctid; i < S * f / 16; i += G * kDecCons) reinterpret_cast<uint4*>(p.ws.hq)[i] = qn;
        if (c == G - 1 && ctid < S) reinterpret_cast<uint32_t*>(p.ws.sh)[ctid] = kNotWritten;
    }

    // ---- 3. router units ----
    for (int ru = 0; ru < n_router_units; ++ru, next_unit()) {
        if (!mine()) continue;
        const int rows = min(pl.rr, n_my_router - ru * pl.rr);
        const float* wrow = reinterpret_cast<const float*>(wait_full());
        float acc[2][TM];
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
            for (int t = 0; t < TM; ++t) acc[i][t] = 0.0f;
        if constexpr (TM == 1) {  // the token's values were loaded into registers at the start
#pragma unroll
            for (int i = 0; i < kDecXr; ++i) {
                const int v = gtid + i * kDecGrp;
                if (v < d / 4) {
                    const float4 w0 = reinterpret_cast<const float4*>(wrow)[v];
                    const float4 w1 = rows > 1 ? reinterpret_cast<const float4*>(wrow + d)[v] : make_float4(0.f, 0.f, 0.f, 0.f);
                    acc[0][0] = fmaf(w0.x, xrr[i].x, acc[0][0]);
                    acc[0][0] = fmaf(w0.y, xrr[i].y, acc[0][0]);
                    acc[0][0] = fmaf(w0.z, xrr[i].z, acc[0][0]);
                    acc[0][0] = fmaf(w0.w, xrr[i].w, acc[0][0]);
                    acc[1][0] = fmaf(w1.x, xrr[i].x, acc[1][0]);
                    acc[1][0] = fmaf(w1.y, xrr[i].y, acc[1][0]);
                    acc[1][0] = fmaf(w1.z, xrr[i].z, acc[1][0]);
                    acc[1][0] = fmaf(w1.w, xrr[i].w, acc[1][0]);
                }
            }
        } else
        for (int v = gtid; v < d / 4; v += kDecGrp) {
            float4 wv[2];
            wv[0] = reinterpret_cast<const float4*>(wrow)[v];
            wv[1] = rows > 1 ? reinterpret_cast<const float4*>(wrow + d)[v] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int t = 0; t < TM; ++t)
                if (t < T) {
                    const float4 xv = load_x4(x, (size_t)t * d + 4 * v);
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        acc[i][t] = fmaf(wv[i].x, xv.x, acc[i][t]);
                        acc[i][t] = fmaf(wv[i].y, xv.y, acc[i][t]);
                        acc[i][t] = fmaf(wv[i].z, xv.z, acc[i][t]);
                        acc[i][t] = fmaf(wv[i].w, xv.w, acc[i][t]);
                    }
                }
        }
        release();
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
            for (int t = 0; t < TM; ++t) {
                const float v = warp_sum(acc[i][t]);
                if (lane == 0) C.part[grp][gw][i * TM + t] = v;
            }
        named_sync(2 + grp, kDecGrp);
        if (gtid < rows * T) {
            const int i = gtid / T, t = gtid % T;
            float v = 0.0f;
#pragma unroll
            for (int w = 0; w < kDecWarps; ++w) v += C.part[grp][w][i * TM + t];
            const int e = c + (ru * pl.rr + i) * G;
            reinterpret_cast<uint2*>(p.ws.logits)[(size_t)t * E + e] =
                route_pair(v, E <= kDecBiasCache ? C.bias_s[e] : __ldg(p.bias + e));
        }
        named_sync(2 + grp, kDecGrp);
    }
    // arrive at the grid barrier (logits of this CTA published).  One fence
    // per CTA and one for the last arrival: a fence costs microseconds once
    // the weight streams load HBM.
    named_sync(kDecBar, kDecCons);
    if (ctid == 0) {
        DEC_TRACE(2);
        fence_acq_rel_gpu();  // release: the CTA's logits, ordered by the barrier, before the arrival
        const unsigned ticket = atomicAdd(&hdr->b1_count, 1u);
        if (ticket == (unsigned)G - 1) {
            hdr->b1_count = 0u;  // read again only by the next launch
            fence_acq_rel_gpu();  // acquire every arrival's logits, release them with the flag
            st_relaxed_u32(&hdr->b1_gen, epoch + 1);
        }
    }

    // the pool blob of expert e (its own index, or its HBM cache slot)
    auto slot_e = [&](int e) -> int {
        if (!p.slot_of) return e;
        return E + HS <= kDecSlotCache ? C.slot_s[e] : blob_slot(p, e, 606);
    };

    // One token: the h rows of the call are preset to "not written" before the
    // grid barrier by other CTAs, so an h value computed before the barrier
    // (the first shared-expert unit) is held in a register and stored once
    // the barrier has passed -- stored earlier, a CTA that presets later could
    // overwrite it.
    bool defer_h = rowrange;
    float h_held = 0.0f;
    float* h_held_at = nullptr;

    // ---- per-warp gate/up bookkeeping ----
    // Rows finished per task are counted in registers and published once, at
    // the end of the gate/up phase: a fence and an atomic with a returned
    // value per task switch stalled each warp for microseconds while HBM was
    // saturated.  A warp's units span at most a few tasks; a fifth one
    // publishes the oldest early.
    constexpr int kPend = 4;
    int pend_task[kPend], pend_cnt[kPend], n_pend = 0;
    int cur_task = -1, cur_cnt = 0, cur_n = 0;
    int xoff[TM];    // staged-row offsets (uint4) of the current task's tokens
    int t_asg[TM];   // their assignment ids
    int t_cs[TM];    // their code sums
    float t_sx[TM];  // their scales
    float amax[TM];
#pragma unroll
    for (int i = 0; i < TM; ++i) {
        amax[i] = 0.0f;
        xoff[i] = 0;
        t_asg[i] = 0;
        t_cs[i] = 0;
        t_sx[i] = 0.0f;
    }
    auto publish = [&](int n_keep) {  // publish all but the newest n_keep pending counts
        if (n_pend <= n_keep) return;  // (warp-uniform)
        fence_acq_rel_gpu();           // this warp's h stores and maxima before its counts
        __syncwarp();
        if (lane == 0)
            for (int i = 0; i < n_pend - n_keep; ++i) red_add_u32(rows_cur + pend_task[i], (uint32_t)pend_cnt[i]);
        for (int i = 0; i < n_keep; ++i) {
            pend_task[i] = pend_task[n_pend - n_keep + i];
            pend_cnt[i] = pend_cnt[n_pend - n_keep + i];
        }
        n_pend = n_keep;
    };
    auto flush_gu = [&]() {  // close the current task: maxima now, the row count later
        if (cur_task < 0 || cur_cnt == 0) return;
        if (rowrange) {  // single token: the requantiser reads the h values themselves
            cur_cnt = 0;
            return;
        }
#pragma unroll
        for (int i = 0; i < TM; ++i)
            if (i < cur_n && lane == i) atomicMax(amax_cur + t_asg[i], __float_as_uint(amax[i]));
        if (n_pend == kPend) publish(0);
        pend_task[n_pend] = cur_task;
        pend_cnt[n_pend] = cur_cnt;
        ++n_pend;
        cur_cnt = 0;
#pragma unroll
        for (int i = 0; i < TM; ++i) amax[i] = 0.0f;
    };
    auto gu_unit = [&](int ti, int j) {
        if (ti != cur_task) {
            flush_gu();
            cur_task = ti;
            cur_n = C.tasks[ti].y;
#pragma unroll
            for (int i = 0; i < TM; ++i)
                if (i < cur_n) {
                    t_asg[i] = idx_in(hdr, C.ttok[ti][i], 0, T * S, 613);
                    const int tok = t_asg[i] / S;
                    xoff[i] = tok * NSUB * nch_gu;
                    t_cs[i] = C.xcs[tok];
                    t_sx[i] = C.sx[tok];
                }
        }
        const uint8_t* slot = wait_full();
        const int r = j * kDecWarps + gw;
        const int n = cur_n;
        bool released = false;
        if (r < f) {
            const uint8_t* grow = slot + (size_t)gw * rb_gu;
            const uint8_t* urow = slot + (size_t)(kDecWarps + gw) * rb_gu;
            const float* ssc = reinterpret_cast<const float*>(slot + pl.wbytes);
            float sg, su;
            int ag[TM], au[TM];
#pragma unroll
            for (int i = 0; i < TM; ++i) ag[i] = au[i] = 0;
            if constexpr (NG > 0) {
                uint4 wg[NG], wu[NG];
#pragma unroll
                for (int i = 0; i < NG; ++i) {
                    wg[i] = *reinterpret_cast<const uint4*>(grow + (size_t)(lane + 32 * i) * 16);
                    wu[i] = *reinterpret_cast<const uint4*>(urow + (size_t)(lane + 32 * i) * 16);
                }
                sg = ssc[gw];
                su = ssc[kDecWarps + gw];
                // the warp's rows are in registers: hand the slot back before the dots
                release();
                released = true;
                if constexpr (TM == 1) {
                    int g0 = 0, g1 = 0, u0 = 0, u1 = 0;
#pragma unroll
                    for (int i = 0; i < NG; ++i) {
                        uint4 xv[NSUB];
#pragma unroll
                        for (int sb = 0; sb < NSUB; ++sb) xv[sb] = xs[sb * nch_gu + lane + 32 * i];
                        dot_chunk_regs<WB>(wg[i], xv, g0, g1);
                        dot_chunk_regs<WB>(wu[i], xv, u0, u1);
                    }
                    ag[0] = g0 + g1;
                    au[0] = u0 + u1;
                } else {
#pragma unroll
                    for (int i = 0; i < NG; ++i)
#pragma unroll
                        for (int t = 0; t < TM; ++t)
                            if (t < n) {
                                ag[t] = dot_chunk<WB>(wg[i], xs + xoff[t], nch_gu, lane + 32 * i, ag[t]);
                                au[t] = dot_chunk<WB>(wu[i], xs + xoff[t], nch_gu, lane + 32 * i, au[t]);
                            }
                }
            } else {
                for (int cc = lane; cc < nch_gu; cc += 32) {
                    const uint4 wg = *reinterpret_cast<const uint4*>(grow + (size_t)cc * 16);
                    const uint4 wu = *reinterpret_cast<const uint4*>(urow + (size_t)cc * 16);
#pragma unroll
                    for (int t = 0; t < TM; ++t)
                        if (t < n) {
                            ag[t] = dot_chunk<WB>(wg, xs + xoff[t], nch_gu, cc, ag[t]);
                            au[t] = dot_chunk<WB>(wu, xs + xoff[t], nch_gu, cc, au[t]);
                        }
                }
                sg = ssc[gw];
                su = ssc[kDecWarps + gw];
            }
#pragma unroll
            for (int i = 0; i < TM; ++i)
                if (i < n) {
                    const int Gv = __reduce_add_sync(kFull, ag[i]) - code_offset<WB>() * t_cs[i];
                    const int Uv = __reduce_add_sync(kFull, au[i]) - code_offset<WB>() * t_cs[i];
                    if (lane == i) {
                        const float g = __fmul_rn((float)Gv, __fmul_rn(sg, t_sx[i]));
                        const float uu = __fmul_rn((float)Uv, __fmul_rn(su, t_sx[i]));
                        const float h = __fmul_rn(__fdiv_rn(g, __fadd_rn(1.0f, expf(-g))), uu);
                        // (the h-skip test hook exists only on the row-range path)
                        if (TM > 1 || ND == 0 || cur_task != p.skip_h_task) {
                            float* dst = p.ws.h + (size_t)t_asg[i] * f + r;
                            if (defer_h) {  // before the grid barrier: held until it has passed
                                h_held = h;
                                h_held_at = dst;
                            } else {
                                st_relaxed_f32(dst, h);
                            }
                        }
                        amax[i] = fmaxf(amax[i], fabsf(h));
                    }
                }
        }
        if (!released) release();
        ++cur_cnt;
    };

    // ---- 4-5. gate/up units, with the grid barrier and the routing
    //      between them.  The group that does not own this CTA's last router
    //      unit runs the first shared-expert unit before the routing (its rows
    //      were copied with the router rows; running gu_unit once there brings
    //      its code into the instruction cache while HBM is otherwise idle);
    //      the remaining shared units and the routed units follow the routing.
    //      One call site of gu_unit for every unit: a second inlined copy would
    //      start cold, with its fetches on the critical path after the routing.
    int n_tasks = HS;
    const int n_sh_first = min(n_sh_units, 1);
#pragma unroll 1
    for (int ph = 0; ph < 3; ++ph) {
        long long n_units = n_sh_first;
        int ti = 0, j = c, jstep = G, jwrap = 0x7fffffff;  // shared: units c, c + G, ... of task 0
        if (ph == 1) {
            // ---- 4. grid barrier, then every CTA derives the routing ----
            if (ctid == 0) flag_wait_bounded(&hdr->b1_gen, epoch + 1, hdr, 300, p.wait_ns);
            named_sync(kDecBar, kDecCons);
            if (ctid == 0) DEC_TRACE(4);
            defer_h = false;
            if (h_held_at) st_relaxed_f32(h_held_at, h_held);  // every preset of the call is ordered before this
            if (c == 0 && ctid == 0) hdr->epoch = epoch + 1;
            if (warp < T) {
                int my_e;
                float my_w;
                if (E <= kDecBiasCache) {
                    topk_warp_small(reinterpret_cast<const uint2*>(p.ws.logits) + (size_t)warp * E, E, k, p.routed_scale,
                                    p.topp, my_e, my_w, trace && warp == 0 ? trace + 18 : nullptr);
                } else {
                    float* scr = reinterpret_cast<float*>(hsb) + (size_t)warp * 2 * E;
                    topk_warp(reinterpret_cast<const uint2*>(p.ws.logits) + (size_t)warp * E, E, k, p.routed_scale,
                              p.topp, scr, scr + E, my_e, my_w);
                }
                if (lane < k) {
                    if (my_e != -1) my_e = idx_in(hdr, my_e, 0, E, 618);  // -1: dropped by the truncation
                    C.idx[warp][lane] = my_e;
                    C.w[warp][lane] = my_w;
                    if (c == 0) {
                        p.ws.idx[warp * k + lane] = my_e;
                        p.ws.w[warp * k + lane] = my_w;
                        if (p.idx_out) p.idx_out[warp * k + lane] = my_e;
                        if (p.w_out) p.w_out[warp * k + lane] = my_w;
                    }
                }
            }
            named_sync(kDecBar, kDecCons);
            if (ctid == 0) DEC_TRACE(11);
            // bucket: sort the T*k assignments by (expert, token, slot); one task per expert
            const int A = T * k;
            if (T == 1) {  // one token: the k experts, each a task with that token, by ascending expert
                if (warp == 0) {  // (a slot the truncation dropped sorts last and makes no task)
                    const int e = lane < k && C.idx[0][lane] >= 0 ? C.idx[0][lane] : 0x7fffffff;
                    int rank = 0;
                    for (int jj = 0; jj < k; ++jj) rank += __shfl_sync(kFull, e, jj) < e;
                    const bool kept = e != 0x7fffffff;
                    if (kept) {
                        C.ttok[HS + rank][0] = lane;  // assignment id: token 0, slot lane
                        C.tasks[HS + rank] = make_int4(e, 1, slot_e(e), 0);
                    }
                    const int m = __popc(__ballot_sync(kFull, kept));
                    if (lane == 0) C.n_tasks = HS + m;
                }
            } else if (ctid < A) {
                // a slot the truncation dropped (-1) sorts last, as expert E
                const int ea = C.idx[ctid / k][ctid % k] < 0 ? E : C.idx[ctid / k][ctid % k];
                int pos = 0, a2 = 0;
                for (int t2 = 0; t2 < T; ++t2)
                    for (int j2 = 0; j2 < k; ++j2, ++a2) {
                        const int e2 = C.idx[t2][j2] < 0 ? E : C.idx[t2][j2];
                        pos += (e2 < ea) || (e2 == ea && a2 < ctid);
                    }
                C.sorted[pos] = ctid;
                C.sorted_e[pos] = ea;
            }
            named_sync(kDecBar, kDecCons);
            if (T > 1 && ctid < A && C.sorted_e[ctid] < E) {
                const int a = C.sorted[ctid];
                const int ea = C.sorted_e[ctid];
                int tq = -1, rank = 0, n = 0;
                for (int q = 0; q <= ctid; ++q) {
                    const int eq = C.sorted_e[q];
                    tq += eq != (q == 0 ? -1 : C.sorted_e[q - 1]);
                    rank += (eq == ea) && q < ctid;
                }
                for (int q = 0; q < A; ++q) n += C.sorted_e[q] == ea;
                C.ttok[HS + tq][rank] = (a / k) * S + (a % k);
                if (rank == 0) C.tasks[HS + tq] = make_int4(ea, n, slot_e(ea), 0);
                if (ctid == A - 1 || C.sorted_e[ctid + 1] == E) C.n_tasks = HS + tq + 1;  // the last kept one
            }
            named_sync(kDecBar, kDecCons);
            if (ctid == 0) {
                mbar_arrive(&C.route_ready);  // the producer may issue routed rows
                DEC_TRACE(5);
            }
            n_tasks = min(max(C.n_tasks, HS), kTasks);
            n_units = n_sh_units - n_sh_first;
            j = c + n_sh_first * G;
        } else if (ph == 2) {
            if (ctid == 0) DEC_TRACE(3);
            const long long Nr = (long long)(n_tasks - HS) * pl.nu_gu;
            const long long lo = c * Nr / G, hi = (c + 1) * Nr / G;
            n_units = hi - lo;
            if (rmaj) {  // the producer's order: row block first, tasks inner
                ti = HS + (int)(lo % (n_tasks - HS));
                j = (int)(lo / (n_tasks - HS));
            } else {
                ti = HS + (int)(lo / pl.nu_gu);
                j = (int)(lo % pl.nu_gu);
            }
            jstep = 1;
            jwrap = pl.nu_gu;
        }
        const bool tasks_inner = ph == 2 && rmaj;
        for (long long g = 0; g < n_units; ++g, next_unit()) {
            if (mine()) gu_unit(ti, j);
            if (tasks_inner) {
                if (++ti == n_tasks) {
                    ti = HS;
                    ++j;
                }
                continue;
            }
            j += jstep;
            if (j == jwrap) {
                j = 0;
                ++ti;
            }
        }
    }
    flush_gu();
    publish(0);
    if (ctid == 0) DEC_TRACE(6);

    // ---- 6r. single token: row-range down with a local combine ----
    if constexpr (TM == 1 && ND > 0) {
        if (rowrange) {
            // requantise the tasks this CTA is designated for (task ti -> CTA
            // ti % G): poll the task's h values until every one is written,
            // max |h| over the row, then the codes and the scale, with relaxed
            // stores that the down units poll in turn (no count, no fence)
            for (int ti = c; ti < n_tasks; ti += G) {
                const int a = idx_in(hdr, C.ttok[ti][0], 0, S, 615);
                const int pc = ctid;
                float4 hv4[4];
                float m = 0.0f;
                if (pc < f / 16) {
                    const float* src = p.ws.h + (size_t)a * f + pc * 16;
                    const uint64_t t0 = global_timer_ns();
                    for (;;) {
                        bool ok = true;
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4) {
                            hv4[q4] = ld_relaxed_f4(src + 4 * q4);
                            ok = ok && __float_as_uint(hv4[q4].x) != kNotWritten && __float_as_uint(hv4[q4].y) != kNotWritten &&
                                 __float_as_uint(hv4[q4].z) != kNotWritten && __float_as_uint(hv4[q4].w) != kNotWritten;
                        }
                        if (ok) break;
                        if (global_timer_ns() - t0 > p.wait_ns || ld_volatile_status(hdr) != 0) {
                            set_status(hdr, MOE_ETIMEOUT, 410);
                            break;
                        }
                    }
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        m = fmaxf(fmaxf(fmaxf(m, fabsf(hv4[q4].x)), fmaxf(fabsf(hv4[q4].y), fabsf(hv4[q4].z))),
                                  fabsf(hv4[q4].w));
                }
                m = cons_max(m, C.redf);
                if (ctid == 0 && ti == c) DEC_TRACE(16);
                const float sh = m == 0.0f ? 0.0f : __fdiv_rn(m, 127.0f);
                const float rh = quant_recip(sh);
                if (pc < f / 16) {
                    unsigned wds[4] = {0u, 0u, 0u, 0u};
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const float hs4[4] = {hv4[q4].x, hv4[q4].y, hv4[q4].z, hv4[q4].w};
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const int code = m == 0.0f ? 0 : quant_code_r(hs4[q], sh, rh);
                            wds[q4] |= ((unsigned)code & 0xFFu) << (8 * q);
                        }
                    }
                    st_relaxed_u4(reinterpret_cast<uint4*>(p.ws.hq + (size_t)a * f) + (pc % NSUB) * nch_dn + pc / NSUB,
                                  permute16<WB>(make_uint4(wds[0], wds[1], wds[2], wds[3])));
                }
                if (ctid == 0) {
                    st_relaxed_f32(p.ws.sh + a, sh);
                    if (ti == c) DEC_TRACE(17);
                }
            }
            if (ctid == 0) DEC_TRACE(7);
            // stage the codes of every task at once: each consumer thread
            // polls up to kDecRRChunks 16-byte chunks (and one thread per
            // task the scale) until written, into shared memory; then one
            // down unit per task in the CTA's task order, with nothing but
            // its weight rows to wait for.  y of (assignment, row) stays in
            // shared memory for the combine.
            constexpr int RRW = kDecNQ * kDecWarps;
            const int n_rr = min(n_tasks, kDecRRMaxTasks);
            const int cpt = f / 16;      // code chunks per task
            const int nq = n_rr * cpt;   // <= kDecRRChunks * kDecCons (the plan checks)
            uint4* stage = reinterpret_cast<uint4*>(hsb);               // [n_rr][f] codes
            float* ys = reinterpret_cast<float*>(hsb + (size_t)S * f);  // [S][RRW]
            {
                uint4 cv[kDecRRChunks];
                float shv = 0.0f;
                const uint64_t t0 = global_timer_ns();
                for (;;) {
                    uint32_t bad = 0u;
#pragma unroll
                    for (int r = 0; r < kDecRRChunks; ++r) {
                        const int q = ctid + r * kDecCons;
                        if (q < nq) {
                            const int a = idx_in(hdr, C.ttok[q / cpt][0], 0, S, 615);
                            cv[r] = ld_relaxed_u4(reinterpret_cast<const uint4*>(p.ws.hq + (size_t)a * f) + q % cpt);
                            bad |= has_byte_80(cv[r].x) | has_byte_80(cv[r].y) | has_byte_80(cv[r].z) | has_byte_80(cv[r].w);
                        }
                    }
                    if (ctid < n_rr) {
                        shv = ld_relaxed_f32(p.ws.sh + idx_in(hdr, C.ttok[ctid][0], 0, S, 615));
                        bad |= __float_as_uint(shv) == kNotWritten;
                    }
                    if (bad == 0u) break;
                    if (global_timer_ns() - t0 > p.wait_ns || ld_volatile_status(hdr) != 0) {
                        set_status(hdr, MOE_ETIMEOUT, 420);
                        break;
                    }
                    __nanosleep(64);
                }
#pragma unroll
                for (int r = 0; r < kDecRRChunks; ++r) {
                    const int q = ctid + r * kDecCons;
                    if (q < nq) stage[q] = cv[r];
                }
                if (ctid < n_rr) C.rsh[ctid] = shv;
            }
            named_sync(kDecBar, kDecCons);  // every task's codes and scale are staged
            if (ctid == 0) DEC_TRACE(20);
            const int rot = pl.dn_rot ? c % n_rr : 0;
            int n_done = 0;  // down units group 0 has finished (traced)
            for (int i = 0; i < n_rr; ++i, next_unit()) {
                if (!mine()) continue;
                const int ti = i + rot < n_rr ? i + rot : i + rot - n_rr;
                const uint8_t* slot = wait_full();
                const int a = idx_in(hdr, C.ttok[ti][0], 0, S, 615);
                const uint4* st = stage + (size_t)ti * cpt;
                uint4 hrr[ND][NSUB];
#pragma unroll
                for (int i2 = 0; i2 < ND; ++i2)
#pragma unroll
                    for (int sb = 0; sb < NSUB; ++sb) hrr[i2][sb] = st[sb * nch_dn + lane + 32 * i2];
                const float shv = C.rsh[ti];
                int csl = 0;  // the code sum, for the offset-binary correction
#pragma unroll
                for (int i = 0; i < ND; ++i)
#pragma unroll
                    for (int sb = 0; sb < NSUB; ++sb) {
                        csl = __dp4a((int)hrr[i][sb].x, 0x01010101, csl);
                        csl = __dp4a((int)hrr[i][sb].y, 0x01010101, csl);
                        csl = __dp4a((int)hrr[i][sb].z, 0x01010101, csl);
                        csl = __dp4a((int)hrr[i][sb].w, 0x01010101, csl);
                    }
                const int cs = __reduce_add_sync(kFull, csl);
                const float* sd = reinterpret_cast<const float*>(slot + pl.wbytes);
                uint4 wv[kDecNQ][ND];
                float sdr[kDecNQ];
#pragma unroll
                for (int q = 0; q < kDecNQ; ++q) {
                    const int rl = q * kDecWarps + gw;
                    const bool ok = rl < rr_rows;
#pragma unroll
                    for (int i = 0; i < ND; ++i)
                        wv[q][i] = ok ? *reinterpret_cast<const uint4*>(slot + (size_t)rl * rb_dn + (size_t)(lane + 32 * i) * 16)
                                      : make_uint4(0u, 0u, 0u, 0u);
                    sdr[q] = ok ? sd[rl] : 0.0f;
                }
                release();
#pragma unroll
                for (int q = 0; q < kDecNQ; ++q) {
                    int a0 = 0, a1 = 0;
#pragma unroll
                    for (int i = 0; i < ND; ++i) dot_chunk_regs<WB>(wv[q][i], hrr[i], a0, a1);
                    const int D = __reduce_add_sync(kFull, a0 + a1) - code_offset<WB>() * cs;
                    const int rl = q * kDecWarps + gw;
                    if (lane == 0 && rl < rr_rows) ys[a * RRW + rl] = __fmul_rn((float)D, __fmul_rn(sdr[q], shv));
                }
                if (n_done == 0 && ctid == 0) DEC_TRACE(22);
                ++n_done;
            }
            named_sync(kDecBar, kDecCons);  // every y of this CTA's rows is in shared memory
            if (ctid == 0) DEC_TRACE(21);
            for (int rl = ctid; rl < rr_rows; rl += kDecCons) {
                float o = 0.0f;
                for (int jj = 0; jj < k; ++jj)
                    if (C.idx[0][jj] >= 0) o = fmaf(C.w[0][jj], ys[jj * RRW + rl], o);
                if (HS) o += ys[k * RRW + rl];
                float* dst = p.out + rr_lo + rl;
                *dst = p.accumulate ? *dst + o : o;
            }
            if (ctid == 0) {
                DEC_TRACE(8);
                if (trace) trace[9] = t_full;
            }
            return;
        }
    }

    // ---- 6. down units ----
    uint8_t* hsg = hsb + (size_t)grp * hs_grp;  // this group's staged h codes
    uint4 hr[ND > 0 ? ND : 1][NSUB];             // single token: the lane's h chunks
    const long long Nd = (long long)n_tasks * pl.nu_dn;
    const long long dlo = c * Nd / G, dhi = (c + 1) * Nd / G;
    int dti = (int)(dlo / pl.nu_dn), dj = (int)(dlo % pl.nu_dn);
    for (long long g = dlo; g < dhi; ++g, next_unit()) {
        const int ti = dti, j = dj;
        if (++dj == pl.nu_dn) {
            dj = 0;
            ++dti;
        }
        if (!mine()) continue;
        const int n = C.tasks[ti].y;
        if (ti != C.hq_task[grp]) {  // requantise and stage this task's h (the whole group agrees on ti)
            named_sync(2 + grp, kDecGrp);
            if (gtid == 0) flag_wait_bounded(rows_cur + ti, (uint32_t)(pl.nu_gu * kDecWarps), hdr, 400, p.wait_ns);
            named_sync(2 + grp, kDecGrp);
            for (int i = 0; i < n; ++i) {
                const int a = idx_in(hdr, C.ttok[ti][i], 0, T * S, 614);
                const float m = __uint_as_float(__ldcg(amax_cur + a));
                const float sh = m == 0.0f ? 0.0f : __fdiv_rn(m, 127.0f);
                const float rh = quant_recip(sh);
                const float* hrow = p.ws.h + (size_t)a * f;
                uint4* hst = reinterpret_cast<uint4*>(hsg) + (size_t)i * NSUB * nch_dn;
                int cs = 0;
                for (int pc = gtid; pc < f / 16; pc += kDecGrp) {
                    unsigned wds[4] = {0u, 0u, 0u, 0u};
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const float4 hv = __ldcg(reinterpret_cast<const float4*>(hrow + pc * 16 + 4 * q4));
                        const float hs4[4] = {hv.x, hv.y, hv.z, hv.w};
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const int code = m == 0.0f ? 0 : quant_code_r(hs4[q], sh, rh);
                            cs += code;
                            wds[q4] |= ((unsigned)code & 0xFFu) << (8 * q);
                        }
                    }
                    hst[(pc % NSUB) * nch_dn + pc / NSUB] = permute16<WB>(make_uint4(wds[0], wds[1], wds[2], wds[3]));
                }
                cs = grp_sum_int(cs, C.redi, grp);
                if (gtid == 0) {
                    C.hcs[grp][i] = cs;
                    C.hsh[grp][i] = sh;
                }
            }
            if (gtid == 0) {
                if (C.hq_task[0] < 0 && C.hq_task[1] < 0) DEC_TRACE(7);
                C.hq_task[grp] = ti;
            }
            named_sync(2 + grp, kDecGrp);
            if constexpr (TM == 1 && ND > 0) {
#pragma unroll
                for (int i = 0; i < ND; ++i)
#pragma unroll
                    for (int sb = 0; sb < NSUB; ++sb) hr[i][sb] = reinterpret_cast<const uint4*>(hsg)[sb * nch_dn + lane + 32 * i];
            }
        }
        const uint8_t* slot = wait_full();
        const float* sd = reinterpret_cast<const float*>(slot + pl.wbytes);  // this unit's row scales
        const int nq = pl.rd / kDecWarps;
        if constexpr (TM == 1 && ND > 0) {
            // single token: the warp's kDecNQ rows into registers, the slot back
            // to the producer, then independent dot chains per row
            uint4 wv[kDecNQ][ND];
            float sdr[kDecNQ];
#pragma unroll
            for (int q = 0; q < kDecNQ; ++q) {
                const int rl = q * kDecWarps + gw;
                const bool ok = j * pl.rd + rl < d;
#pragma unroll
                for (int i = 0; i < ND; ++i)
                    wv[q][i] = ok ? *reinterpret_cast<const uint4*>(slot + (size_t)rl * rb_dn + (size_t)(lane + 32 * i) * 16)
                                  : make_uint4(0u, 0u, 0u, 0u);
                sdr[q] = ok ? sd[rl] : 0.0f;
            }
            release();
            int dv[kDecNQ];
#pragma unroll
            for (int q = 0; q < kDecNQ; ++q) {
                int a0 = 0, a1 = 0;
#pragma unroll
                for (int i = 0; i < ND; ++i) dot_chunk_regs<WB>(wv[q][i], hr[i], a0, a1);
                dv[q] = a0 + a1;
            }
            const int a = idx_in(hdr, C.ttok[ti][0], 0, T * S, 616);
#pragma unroll
            for (int q = 0; q < kDecNQ; ++q) {
                const int D = __reduce_add_sync(kFull, dv[q]) - code_offset<WB>() * C.hcs[grp][0];
                const int r = j * pl.rd + q * kDecWarps + gw;
                if (lane == q && r < d) p.ws.ybuf[(size_t)a * d + r] = __fmul_rn((float)D, __fmul_rn(sdr[q], C.hsh[grp][0]));
            }
            continue;
        }
        for (int q = 0; q < nq; ++q) {
            const int rl = q * kDecWarps + gw, r = j * pl.rd + rl;
            if (r >= d) break;
            const uint8_t* wrow = slot + (size_t)rl * rb_dn;
            int acc[TM];
#pragma unroll
            for (int i = 0; i < TM; ++i) acc[i] = 0;
            if constexpr (TM == 1 && ND > 0) {
                int a0 = 0, a1 = 0;
#pragma unroll
                for (int i = 0; i < ND; ++i)
                    dot_chunk_regs<WB>(*reinterpret_cast<const uint4*>(wrow + (size_t)(lane + 32 * i) * 16), hr[i], a0,
                                       a1);
                acc[0] = a0 + a1;
            } else {
                for (int cc = lane; cc < nch_dn; cc += 32) {
                    const uint4 wv = *reinterpret_cast<const uint4*>(wrow + (size_t)cc * 16);
#pragma unroll
                    for (int i = 0; i < TM; ++i)
                        if (i < n)
                            acc[i] = dot_chunk<WB>(wv, reinterpret_cast<const uint4*>(hsg) + (size_t)i * NSUB * nch_dn,
                                                   nch_dn, cc, acc[i]);
                }
            }
            const float sdr = sd[rl];
#pragma unroll
            for (int i = 0; i < TM; ++i)
                if (i < n) {
                    const int D = __reduce_add_sync(kFull, acc[i]) - code_offset<WB>() * C.hcs[grp][i];
                    if (lane == i) {
                        const int a = idx_in(hdr, C.ttok[ti][i], 0, T * S, 617);
                        p.ws.ybuf[(size_t)a * d + r] = __fmul_rn((float)D, __fmul_rn(sdr, C.hsh[grp][i]));
                    }
                }
        }
        release();
    }

    // ---- 7. sign off this CTA's row blocks; the CTA completing one combines it ----
    named_sync(kDecBar, kDecCons);  // every down output of this CTA is written
    for (long long base = dlo; base < dhi; base += kDecCons) {
        if (ctid == 0) C.n_last = 0;
        named_sync(kDecBar, kDecCons);
        const long long g = base + ctid;
        if (g < dhi) {
            const int rb = (int)(g % pl.nu_dn);
            __threadfence();  // release: the CTA's stores (ordered by the barrier) before the arrival
            if (atomicAdd(p.ws.rb_ctr + rb, 1u) == (unsigned)(n_tasks - 1)) {
                p.ws.rb_ctr[rb] = 0u;
                C.last_rb[atomicAdd(&C.n_last, 1)] = rb;
            }
        }
        named_sync(kDecBar, kDecCons);
        const int n_last = C.n_last;
        if (n_last > 0) __threadfence();  // acquire: the other CTAs' down outputs
        for (int li = 0; li < n_last; ++li) {
            const int rb = C.last_rb[li];
            const int r0 = rb * pl.rd, rows = min(pl.rd, d - r0);
            for (int i = ctid; i < T * rows; i += kDecCons) {
                const int t = i / rows, r = r0 + i % rows;
                float o = 0.0f;
                for (int jj = 0; jj < k; ++jj)
                    if (C.idx[t][jj] >= 0) o = fmaf(C.w[t][jj], __ldcg(p.ws.ybuf + ((size_t)t * S + jj) * d + r), o);
                if (HS) o += __ldcg(p.ws.ybuf + ((size_t)t * S + k) * d + r);
                float* dst = p.out + (size_t)t * d + r;
                *dst = p.accumulate ? *dst + o : o;
            }
        }
        named_sync(kDecBar, kDecCons);
    }
    if (ctid == 0) {
        DEC_TRACE(8);
        if (trace) trace[9] = t_full;
    }
#undef DEC_TRACE
}

}  // namespace moe
