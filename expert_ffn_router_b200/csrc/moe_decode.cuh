// The whole MoE layer for decode-sized batches (T <= 8) in one persistent,
// cooperatively launched kernel: one CTA per SM, 8 consumer warps and one
// producer warp.
//
// The producer streams every weight row the CTA needs -- its router rows, its
// share of the shared expert's gate/up rows, then (once the routing is known)
// its share of the routed gate/up rows and of all down rows -- into a ring of
// shared-memory slots with 1-D bulk copies (cp.async.bulk, completion counted
// on an mbarrier per slot).  The consumers work through the same unit
// sequence:
//   1. quantise the T tokens (every CTA, into its own shared memory);
//   2. router units: logits of this CTA's experts -> workspace; arrive at the
//      one grid barrier;
//   3. shared-expert gate/up units (need no routing) while the barrier fills;
//   4. after the barrier every CTA reads all logits and derives the same
//      top-k routing and the same expert task list (no second barrier);
//   5. routed gate/up units; the warp that completes a task's last row
//      requantises its h and publishes the task as ready (release flag);
//   6. down units (waiting, bounded, for their task's ready flag); the warp
//      that completes a row block's last contribution combines it.
// Each expert selected by several tokens is streamed once: a task is one
// expert with all its tokens.  Every wait is bounded (MOE_ETIMEOUT).
#pragma once

#include <float.h>

#include "moe_common.cuh"

namespace moe {

constexpr int kDecWarps = 8;
constexpr int kDecThreads = (kDecWarps + 1) * 32;
constexpr int kDecCons = kDecWarps * 32;
constexpr int kDecMaxSlots = 4;
constexpr int kDecMaxT = 8;
constexpr int kDecMaxK = 32;
constexpr int kDecMaxTasks = kDecMaxT * kDecMaxK + 1;
constexpr int kDecBar = 1;  // named barrier of the consumer warps

struct DecPlan {
    int slot_bytes, nslot;
    int rd;            // down rows per unit (multiple of kDecWarps)
    int rr;            // router rows per unit (1 or 2)
    int nu_gu, nu_dn;  // units per task
    int xs_off, hs_off, ring_off, smem_bytes;
};

struct DecCtl {
    uint64_t full[kDecMaxSlots];
    uint64_t empty[kDecMaxSlots];
    uint64_t route_ready;
    uint32_t epoch;
    int n_tasks;
    int hq_task;
    float sx[kDecMaxT];
    int xcs[kDecMaxT];
    int idx[kDecMaxT][kDecMaxK];
    float w[kDecMaxT][kDecMaxK];
    int4 tasks[kDecMaxTasks];  // (blob, n tokens, -, -)
    int ttok[kDecMaxTasks][kDecMaxT];
    int sorted[kDecMaxT * kDecMaxK];
    int hcs[kDecMaxT];
    float hsh[kDecMaxT];
    float redf[kDecWarps];
    int redi[kDecWarps];
    float part[kDecWarps][2 * kDecMaxT];
};

// --- consumer-only reductions (named barrier, 256 threads) -----------------
__device__ __forceinline__ float cons_max(float v, float* red) {
    v = warp_max(v);
    named_sync(kDecBar, kDecCons);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    named_sync(kDecBar, kDecCons);
    float r = red[0];
#pragma unroll
    for (int i = 1; i < kDecWarps; ++i) r = fmaxf(r, red[i]);
    return r;
}
__device__ __forceinline__ int cons_sum_int(int v, int* red) {
    v = __reduce_add_sync(kFull, v);
    named_sync(kDecBar, kDecCons);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    named_sync(kDecBar, kDecCons);
    int r = 0;
#pragma unroll
    for (int i = 0; i < kDecWarps; ++i) r += red[i];
    return r;
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

// Top-k of one token by one warp from a logits row in global memory; lane j
// (< k) returns slot j's expert and weight.  Same rule as topk_token.
__device__ __forceinline__ void topk_warp(const float* lrow, const float* bias, int E, int k, float scale,
                                          float* s_sm, float* sel_sm, int& my_e, float& my_w) {
    const int lane = threadIdx.x & 31;
    for (int e = lane; e < E; e += 32) {
        const float lg = __ldcg(lrow + e);
        const float s = __fdiv_rn(1.0f, __fadd_rn(1.0f, expf(-lg)));
        s_sm[e] = s;
        sel_sm[e] = __fadd_rn(s, __ldg(bias + e));
    }
    __syncwarp();
    float ssum = 0.0f, my_s = 0.0f;
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
        }
        ssum = __fadd_rn(ssum, sj);
        __syncwarp();
        if (lane == 0) sel_sm[be] = -INFINITY;
        __syncwarp();
    }
    my_w = lane < k ? __fmul_rn(__fdiv_rn(my_s, ssum), scale) : 0.0f;
}

template <int WB, int TM, typename XT>
__global__ void __launch_bounds__(kDecThreads, 1) k_decode(const Params p, const DecPlan pl, const XT* __restrict__ x) {
    constexpr int NSUB = 8 / WB;
    extern __shared__ __align__(128) uint8_t dec_smem[];
    DecCtl& C = *reinterpret_cast<DecCtl*>(dec_smem);
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

    if (tid == 0) {
        for (int i = 0; i < nslot; ++i) {
            mbar_init(&C.full[i], 1);
            mbar_init(&C.empty[i], kDecWarps);
        }
        mbar_init(&C.route_ready, 1);
        fence_mbar_init();
        C.epoch = __ldcg(&hdr->epoch);
        C.hq_task = -1;
    }
    __syncthreads();  // the only CTA-wide barrier: producer and consumers part here
    const uint32_t epoch = C.epoch;
    const int n_my_router = c < E ? (E - c + G - 1) / G : 0;  // experts c, c+G, ...
    const int n_router_units = (n_my_router + pl.rr - 1) / pl.rr;
    const int n_sh_units = HS && c < pl.nu_gu ? (pl.nu_gu - c + G - 1) / G : 0;  // shared units c, c+G, ...

    // =====================================================================
    // producer: lane 0 of warp kDecWarps
    // =====================================================================
    if (warp == kDecWarps) {
        if (lane != 0) return;
        uint32_t u = 0;
        auto take = [&](uint32_t bytes) -> uint8_t* {
            const int s = u % nslot;
            const uint32_t round = u / nslot;
            if (round > 0) mbar_wait_bounded(&C.empty[s], (round - 1) & 1, hdr, 100 + s);
            mbar_arrive_expect_tx(&C.full[s], bytes);
            return ring + (size_t)s * slot_bytes;
        };
        const int n_blobs = E + HS;
        auto issue_gu = [&](int blob, int j) {
            blob = min(max(blob, 0), n_blobs - 1);  // never copy outside the pool, whatever happened
            const int r0 = j * kDecWarps, rows = min(kDecWarps, f - r0);
            const uint32_t bytes = (uint32_t)rows * rb_gu;
            const uint8_t* base = p.pool + (size_t)blob * p.blob_bytes;
            uint8_t* dst = take(2 * bytes);
            bulk_g2s(dst, base + (size_t)r0 * rb_gu, bytes, &C.full[u % nslot]);
            bulk_g2s(dst + (size_t)kDecWarps * rb_gu, base + ((size_t)f + r0) * rb_gu, bytes, &C.full[u % nslot]);
            ++u;
        };
        for (int ru = 0; ru < n_router_units; ++ru) {
            const int rows = min(pl.rr, n_my_router - ru * pl.rr);
            uint8_t* dst = take((uint32_t)rows * d * 4);
            for (int i = 0; i < rows; ++i) {
                const int e = c + (ru * pl.rr + i) * G;
                bulk_g2s(dst + (size_t)i * d * 4, p.w_router + (size_t)e * d, (uint32_t)d * 4, &C.full[u % nslot]);
            }
            ++u;
        }
        for (int i = 0; i < n_sh_units; ++i) issue_gu(E, c + i * G);
        mbar_wait_bounded(&C.route_ready, 0, hdr, 110);
        const int n_tasks = min(max(C.n_tasks, HS), kDecMaxTasks);
        const long long Nr = (long long)(n_tasks - HS) * pl.nu_gu;
        for (long long g = c * Nr / G; g < (c + 1) * Nr / G; ++g)
            issue_gu(C.tasks[HS + (int)(g / pl.nu_gu)].x, (int)(g % pl.nu_gu));
        const long long Nd = (long long)n_tasks * pl.nu_dn;
        for (long long g = c * Nd / G; g < (c + 1) * Nd / G; ++g) {
            const int blob = min(max(C.tasks[(int)(g / pl.nu_dn)].x, 0), n_blobs - 1), j = (int)(g % pl.nu_dn);
            const int r0 = j * pl.rd, rows = min(pl.rd, d - r0);
            const uint32_t bytes = (uint32_t)rows * rb_dn;
            uint8_t* dst = take(bytes);
            bulk_g2s(dst, p.pool + (size_t)blob * p.blob_bytes + 2 * (size_t)f * rb_gu + (size_t)r0 * rb_dn, bytes,
                     &C.full[u % nslot]);
            ++u;
        }
        // drain: every copy issued must have landed before this thread (and so
        // the CTA and its shared memory) can retire
        for (int s = 0; s < nslot; ++s)
            if (u > (uint32_t)s) mbar_wait_bounded(&C.full[s], ((u - s + nslot - 1) / nslot - 1) & 1, hdr, 120 + s);
        return;
    }

    // =====================================================================
    // consumers: warps 0..7, ctid = threadIdx.x
    // =====================================================================
    const int ctid = tid;
    // ---- 1. quantise the T tokens into the permuted staging layout ----
    for (int t = 0; t < T; ++t) {
        const XT* xt = x + (size_t)t * d;
        float m = 0.0f;
        for (int col = ctid; col < d; col += kDecCons) m = fmaxf(m, fabsf(load_x(xt, col)));
        m = cons_max(m, C.redf);
        const float s = m == 0.0f ? 0.0f : __fdiv_rn(m, 127.0f);
        int cs = 0;
        uint4* xst = xs + (size_t)t * NSUB * nch_gu;
        for (int pc = ctid; pc < d / 16; pc += kDecCons) {
            float v[16];
            load16(xt, (size_t)pc * 16, v);
            unsigned wds[4] = {0u, 0u, 0u, 0u};
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const int code = m == 0.0f ? 0 : quant_code(v[q], s);
                cs += code;
                wds[q >> 2] |= ((unsigned)code & 0xFFu) << (8 * (q & 3));
            }
            xst[(pc % NSUB) * nch_gu + pc / NSUB] = permute16<WB>(make_uint4(wds[0], wds[1], wds[2], wds[3]));
        }
        cs = cons_sum_int(cs, C.redi);
        if (ctid == 0) {
            C.sx[t] = s;
            C.xcs[t] = cs;
        }
    }
    named_sync(kDecBar, kDecCons);

    uint32_t u = 0;  // unit counter, identical sequence to the producer's
    auto wait_full = [&]() -> const uint8_t* {
        const int s = u % nslot;
        mbar_wait_bounded(&C.full[s], (u / nslot) & 1, hdr, 200 + s);
        return ring + (size_t)s * slot_bytes;
    };
    auto release = [&]() {
        __syncwarp();
        if (lane == 0) mbar_arrive(&C.empty[u % nslot]);
        ++u;
    };

    // ---- 2. router units ----
    for (int ru = 0; ru < n_router_units; ++ru) {
        const int rows = min(pl.rr, n_my_router - ru * pl.rr);
        const float* wrow = reinterpret_cast<const float*>(wait_full());
        float acc[2][TM];
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
            for (int t = 0; t < TM; ++t) acc[i][t] = 0.0f;
        for (int v = ctid; v < d / 4; v += kDecCons) {
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
                if (lane == 0) C.part[warp][i * TM + t] = v;
            }
        named_sync(kDecBar, kDecCons);
        if (ctid < rows * T) {
            const int i = ctid / T, t = ctid % T;
            float v = 0.0f;
#pragma unroll
            for (int w = 0; w < kDecWarps; ++w) v += C.part[w][i * TM + t];
            const int e = c + (ru * pl.rr + i) * G;
            p.ws.logits[(size_t)t * E + e] = v;
        }
        named_sync(kDecBar, kDecCons);
    }
    // arrive at the grid barrier (logits of this CTA published)
    __threadfence();
    named_sync(kDecBar, kDecCons);
    if (ctid == 0) {
        const unsigned ticket = atomicAdd(&hdr->b1_count, 1u);
        if (ticket == (unsigned)G - 1) {
            hdr->b1_count = 0u;
            __threadfence();
            st_release_u32(&hdr->b1_gen, epoch + 1);
        }
    }

    // ---- per-warp gate/up bookkeeping ----
    int cur_task = -1, cur_cnt = 0;
    float amax[TM];
#pragma unroll
    for (int i = 0; i < TM; ++i) amax[i] = 0.0f;

    auto requant = [&](int ti) {  // one warp: h of task ti -> hq, sh; publish
        const int n = C.tasks[ti].y;
        for (int i = 0; i < n; ++i) {
            const int a = C.ttok[ti][i];
            const float m = __uint_as_float(__ldcg(p.ws.amax + a));
            const float sh = m == 0.0f ? 0.0f : __fdiv_rn(m, 127.0f);
            const float* hrow = p.ws.h + (size_t)a * f;
            int8_t* qrow = p.ws.hq + (size_t)a * f;
            for (int cc = lane * 4; cc < f; cc += 128) {
                const float4 hv = __ldcg(reinterpret_cast<const float4*>(hrow + cc));
                char4 q = make_char4(0, 0, 0, 0);
                if (m != 0.0f)
                    q = make_char4((signed char)quant_code(hv.x, sh), (signed char)quant_code(hv.y, sh),
                                   (signed char)quant_code(hv.z, sh), (signed char)quant_code(hv.w, sh));
                *reinterpret_cast<char4*>(qrow + cc) = q;
            }
            __syncwarp();  // every lane has read amax[a]
            if (lane == 0) {
                p.ws.sh[a] = sh;
                p.ws.amax[a] = 0u;  // ready for the next call
            }
        }
        __threadfence();
        __syncwarp();
        if (lane == 0) {
            p.ws.task_ctr[ti] = 0u;
            st_release_u32(p.ws.ready + ti, epoch + 1);
        }
    };
    auto flush_gu = [&]() {
        if (cur_task < 0 || cur_cnt == 0) return;
        const int n = C.tasks[cur_task].y;
#pragma unroll
        for (int i = 0; i < TM; ++i)
            if (i < n && lane == i) atomicMax(p.ws.amax + C.ttok[cur_task][i], __float_as_uint(amax[i]));
        __threadfence();
        __syncwarp();
        unsigned last = 0;
        if (lane == 0) {
            const unsigned t0 = atomicAdd(p.ws.task_ctr + cur_task, (unsigned)cur_cnt);
            last = t0 + cur_cnt == (unsigned)(pl.nu_gu * kDecWarps);
        }
        last = __shfl_sync(kFull, last, 0);
        if (last) {
            __threadfence();
            requant(cur_task);
        }
        cur_cnt = 0;
#pragma unroll
        for (int i = 0; i < TM; ++i) amax[i] = 0.0f;
    };
    auto gu_unit = [&](int ti, int j) {
        if (ti != cur_task) {
            flush_gu();
            cur_task = ti;
        }
        const uint8_t* slot = wait_full();
        const int r = j * kDecWarps + warp;
        const int4 tk = C.tasks[ti];
        const int n = tk.y;
        if (r < f) {
            const uint8_t* grow = slot + (size_t)warp * rb_gu;
            const uint8_t* urow = slot + (size_t)(kDecWarps + warp) * rb_gu;
            int ag[TM], au[TM];
#pragma unroll
            for (int i = 0; i < TM; ++i) ag[i] = au[i] = 0;
            for (int cc = lane; cc < nch_gu; cc += 32) {
                const uint4 wg = *reinterpret_cast<const uint4*>(grow + (size_t)cc * 16);
                const uint4 wu = *reinterpret_cast<const uint4*>(urow + (size_t)cc * 16);
#pragma unroll
                for (int i = 0; i < TM; ++i)
                    if (i < n) {
                        const uint4* xt = xs + (size_t)(C.ttok[ti][i] / S) * NSUB * nch_gu;
                        ag[i] = dot_chunk<WB>(wg, xt, nch_gu, cc, ag[i]);
                        au[i] = dot_chunk<WB>(wu, xt, nch_gu, cc, au[i]);
                    }
            }
            const float* sc = p.scales + (size_t)tk.x * p.scale_rows;
            const float sg = __ldg(sc + r), su = __ldg(sc + f + r);
#pragma unroll
            for (int i = 0; i < TM; ++i)
                if (i < n) {
                    const int a = C.ttok[ti][i], tok = a / S;
                    const int Gv = __reduce_add_sync(kFull, ag[i]) - code_offset<WB>() * C.xcs[tok];
                    const int Uv = __reduce_add_sync(kFull, au[i]) - code_offset<WB>() * C.xcs[tok];
                    if (lane == i) {
                        const float g = __fmul_rn((float)Gv, __fmul_rn(sg, C.sx[tok]));
                        const float uu = __fmul_rn((float)Uv, __fmul_rn(su, C.sx[tok]));
                        const float h = __fmul_rn(__fdiv_rn(g, __fadd_rn(1.0f, expf(-g))), uu);
                        p.ws.h[(size_t)a * f + r] = h;
                        amax[i] = fmaxf(amax[i], fabsf(h));
                    }
                }
        }
        release();
        ++cur_cnt;
    };

    // ---- 3. shared-expert gate/up units (no routing needed) ----
    for (int i = 0; i < n_sh_units; ++i) {
        if (i == 0) {  // the shared task's description, known before routing
            if (ctid < T) C.ttok[0][ctid] = ctid * S + k;
            if (ctid == 0) C.tasks[0] = make_int4(E, T, 0, 0);
            named_sync(kDecBar, kDecCons);
        }
        gu_unit(0, c + i * G);
    }

    // ---- 4. grid barrier, then every CTA derives the routing ----
    if (ctid == 0) flag_wait_bounded(&hdr->b1_gen, epoch + 1, hdr, 300);
    named_sync(kDecBar, kDecCons);
    if (c == 0 && ctid == 0) hdr->epoch = epoch + 1;
    if (warp < T) {
        float* scr = reinterpret_cast<float*>(hsb) + (size_t)warp * 2 * E;
        int my_e;
        float my_w;
        topk_warp(p.ws.logits + (size_t)warp * E, p.bias, E, k, p.routed_scale, scr, scr + E, my_e, my_w);
        if (lane < k) {
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
    // bucket: sort the T*k assignments by (expert, token, slot); one task per expert
    const int A = T * k;
    if (ctid < A) {
        const int ea = C.idx[ctid / k][ctid % k];
        int pos = 0;
        for (int a2 = 0; a2 < A; ++a2) {
            const int e2 = C.idx[a2 / k][a2 % k];
            pos += (e2 < ea) || (e2 == ea && a2 < ctid);
        }
        C.sorted[pos] = ctid;
    }
    if (HS && ctid < T) C.ttok[0][ctid] = ctid * S + k;
    if (HS && ctid == 0) C.tasks[0] = make_int4(E, T, 0, 0);
    named_sync(kDecBar, kDecCons);
    if (ctid < A) {
        const int a = C.sorted[ctid];
        const int ea = C.idx[a / k][a % k];
        int ti = -1, rank = 0, n = 0;
        for (int q = 0; q <= ctid; ++q) {
            const int aq = C.sorted[q];
            const int eq = C.idx[aq / k][aq % k];
            const int ep = q == 0 ? -1 : C.idx[C.sorted[q - 1] / k][C.sorted[q - 1] % k];
            ti += eq != ep;
            rank += (eq == ea) && q < ctid;
        }
        for (int q = 0; q < A; ++q) {
            const int aq = C.sorted[q];
            n += C.idx[aq / k][aq % k] == ea;
        }
        C.ttok[HS + ti][rank] = (a / k) * S + (a % k);
        if (rank == 0) C.tasks[HS + ti] = make_int4(ea, n, 0, 0);
        if (ctid == A - 1) C.n_tasks = HS + ti + 1;
    }
    named_sync(kDecBar, kDecCons);
    if (ctid == 0) mbar_arrive(&C.route_ready);  // the producer may issue routed rows
    const int n_tasks = min(max(C.n_tasks, HS), kDecMaxTasks);

    // ---- 5. routed gate/up units ----
    {
        const long long Nr = (long long)(n_tasks - HS) * pl.nu_gu;
        for (long long g = c * Nr / G; g < (c + 1) * Nr / G; ++g)
            gu_unit(HS + (int)(g / pl.nu_gu), (int)(g % pl.nu_gu));
        flush_gu();
    }

    // ---- 6. down units + combine ----
    const long long Nd = (long long)n_tasks * pl.nu_dn;
    for (long long g = c * Nd / G; g < (c + 1) * Nd / G; ++g) {
        const int ti = (int)(g / pl.nu_dn), j = (int)(g % pl.nu_dn);
        const int4 tk = C.tasks[ti];
        const int n = tk.y;
        if (ti != C.hq_task) {  // stage this task's h codes (all consumer warps agree on ti)
            named_sync(kDecBar, kDecCons);
            if (ctid == 0) flag_wait_bounded(p.ws.ready + ti, epoch + 1, hdr, 400);
            named_sync(kDecBar, kDecCons);
            for (int i = 0; i < n; ++i) {
                const int a = C.ttok[ti][i];
                int cs = stage_row<WB>(p.ws.hq + (size_t)a * f, f,
                                       reinterpret_cast<uint4*>(hsb) + (size_t)i * NSUB * nch_dn);
                cs = cons_sum_int(cs, C.redi);
                if (ctid == 0) {
                    C.hcs[i] = cs;
                    C.hsh[i] = __ldcg(p.ws.sh + a);
                }
            }
            if (ctid == 0) C.hq_task = ti;
            named_sync(kDecBar, kDecCons);
        }
        const uint8_t* slot = wait_full();
        const float* sd = p.scales + (size_t)tk.x * p.scale_rows + 2 * f;
        for (int q = 0; q < pl.rd / kDecWarps; ++q) {
            const int rl = q * kDecWarps + warp, r = j * pl.rd + rl;
            if (r >= d) break;
            const uint8_t* wrow = slot + (size_t)rl * rb_dn;
            int acc[TM];
#pragma unroll
            for (int i = 0; i < TM; ++i) acc[i] = 0;
            for (int cc = lane; cc < nch_dn; cc += 32) {
                const uint4 wv = *reinterpret_cast<const uint4*>(wrow + (size_t)cc * 16);
#pragma unroll
                for (int i = 0; i < TM; ++i)
                    if (i < n) acc[i] = dot_chunk<WB>(wv, reinterpret_cast<const uint4*>(hsb) + (size_t)i * NSUB * nch_dn,
                                                      nch_dn, cc, acc[i]);
            }
            const float sdr = __ldg(sd + r);
#pragma unroll
            for (int i = 0; i < TM; ++i)
                if (i < n) {
                    const int D = __reduce_add_sync(kFull, acc[i]) - code_offset<WB>() * C.hcs[i];
                    if (lane == i) {
                        const int a = C.ttok[ti][i];
                        p.ws.ybuf[(size_t)a * d + r] = __fmul_rn((float)D, __fmul_rn(sdr, C.hsh[i]));
                    }
                }
        }
        release();
        // row block j: the warp bringing its last contribution combines it
        __threadfence();
        __syncwarp();
        unsigned last = 0;
        if (lane == 0) last = atomicAdd(p.ws.rb_ctr + j, 1u) == (unsigned)(n_tasks * kDecWarps - 1);
        last = __shfl_sync(kFull, last, 0);
        if (last) {
            __threadfence();
            const int r0 = j * pl.rd, rows = min(pl.rd, d - r0);
            for (int i = lane; i < T * rows; i += 32) {
                const int t = i / rows, r = r0 + i % rows;
                float o = 0.0f;
                for (int jj = 0; jj < k; ++jj)
                    o = fmaf(C.w[t][jj], __ldcg(p.ws.ybuf + ((size_t)t * S + jj) * d + r), o);
                if (HS) o += __ldcg(p.ws.ybuf + ((size_t)t * S + k) * d + r);
                float* dst = p.out + (size_t)t * d + r;
                *dst = p.accumulate ? *dst + o : o;
            }
            if (lane == 0) p.ws.rb_ctr[j] = 0u;
        }
    }
}

}  // namespace moe
