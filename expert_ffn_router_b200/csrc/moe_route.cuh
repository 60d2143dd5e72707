// Steps a0-a2 of the layer: activation quantiser, DeepSeek-V3-style sigmoid
// router with selection bias and lower-index tie-break, and the bucketing of
// (token, slot) assignments by expert into tasks for the expert kernels.
#pragma once

#include <float.h>

#include "moe_common.cuh"

namespace moe {

// a0 for one token by a whole CTA: s = max|x| / 127; codes by round half to
// even of x / s; writes codes, scale and the sum of the codes.
template <typename XT>
__device__ void quantize_token(const XT* x, int d, int8_t* xq, float* sx, int32_t* xcs, float* redf,
                               int* redi) {
    float m = 0.0f;
    for (int c = threadIdx.x; c < d; c += kThreads) m = fmaxf(m, fabsf(load_x(x, c)));
    m = block_max(m, redf);
    const float s = m == 0.0f ? 0.0f : __fdiv_rn(m, 127.0f);
    const float r = quant_recip(s);
    int cs = 0;
    // d is a multiple of 32: each thread writes 4 codes at a time
    for (int c = threadIdx.x * 4; c < d; c += kThreads * 4) {
        float4 v = load_x4(x, c);
        int q0 = 0, q1 = 0, q2 = 0, q3 = 0;
        if (m != 0.0f) {
            q0 = quant_code_r(v.x, s, r);
            q1 = quant_code_r(v.y, s, r);
            q2 = quant_code_r(v.z, s, r);
            q3 = quant_code_r(v.w, s, r);
        }
        cs += q0 + q1 + q2 + q3;
        *reinterpret_cast<char4*>(xq + c) = make_char4((signed char)q0, (signed char)q1, (signed char)q2,
                                                       (signed char)q3);
    }
    cs = block_sum_int(cs, redi);
    if (threadIdx.x == 0) {
        *sx = s;
        if (xcs) *xcs = cs;
    }
}

// Copy n16 16-byte chunks from src -- pinned host memory mapped into the
// device's address space -- to device memory, four independent loads in
// flight per thread (plain coherent loads: no read-only-cache path on host
// memory).
__global__ void __launch_bounds__(kThreads) k_stage_in(const uint4* src, uint4* dst, long long n16) {
    const long long stride = (long long)gridDim.x * kThreads;
    long long i = (long long)blockIdx.x * kThreads + threadIdx.x;
    for (; i + 3 * stride < n16; i += 4 * stride) {
        const uint4 a = src[i], b = src[i + stride], c = src[i + 2 * stride], e = src[i + 3 * stride];
        dst[i] = a;
        dst[i + stride] = b;
        dst[i + 2 * stride] = c;
        dst[i + 3 * stride] = e;
    }
    for (; i < n16; i += stride) dst[i] = src[i];
}

template <typename XT>
__global__ void __launch_bounds__(kThreads) k_quantize(const XT* __restrict__ x, int T, int d,
                                                        int8_t* __restrict__ xq, float* __restrict__ sx,
                                                        int32_t* __restrict__ xcs) {
    __shared__ float redf[kWarps];
    __shared__ int redi[kWarps];
    for (int t = blockIdx.x; t < T; t += gridDim.x)
        quantize_token(x + (size_t)t * d, d, xq + (size_t)t * d, sx + t, xcs ? xcs + t : nullptr, redf, redi);
}

// Sum of each token's int8 codes (the offset-binary correction of the dots).
__global__ void __launch_bounds__(kThreads) k_sum_codes(const int8_t* __restrict__ xq, int T, int d,
                                                         int32_t* __restrict__ xcs) {
    __shared__ int redi[kWarps];
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        int s = 0;
        for (int c = threadIdx.x * 16; c < d; c += kThreads * 16)
            s += sum16(__ldcg(reinterpret_cast<const uint4*>(xq + (size_t)t * d + c)));
        s = block_sum_int(s, redi);
        if (threadIdx.x == 0) xcs[t] = s;
    }
}

// Top-k of one token by one warp.  s_sm / sel_sm: this warp's E-float shared
// scratch.  Logits are the sum of `ksplit` partial planes, added in order.
static __device__ void topk_token(const Params& p, int t, float* s_sm, float* sel_sm) {
    const int lane = threadIdx.x & 31;
    const int E = p.m.E, k = p.m.k, T = p.m.T;
    for (int e = lane; e < E; e += 32) {
        float lg = __ldcg(p.ws.logits + (size_t)t * E + e);
        for (int ks = 1; ks < p.ksplit; ++ks) lg += __ldcg(p.ws.logits + ((size_t)ks * T + t) * E + e);
        const float s = __fdiv_rn(1.0f, __fadd_rn(1.0f, expf(-lg)));
        s_sm[e] = s;
        sel_sm[e] = __fadd_rn(s, __ldg(p.bias + e));
    }
    __syncwarp();
    float ssum = 0.0f, my_s = 0.0f, cex = 0.0f, cin = 0.0f;
    int my_e = 0;
    for (int j = 0; j < k; ++j) {
        float bv = -FLT_MAX;
        int be = 0x7fffffff;
        for (int e = lane; e < E; e += 32) {
            const float v = sel_sm[e];
            if (v > bv) {  // ascending e, strict: the lower index keeps ties
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
    const float norm = topp_keep(p.topp, k, ssum, cex, cin, kept);
    if (lane < k) {  // a slot the truncation drops selects no expert: -1, weight 0
        const float w = kept ? __fmul_rn(__fdiv_rn(my_s, norm), p.routed_scale) : 0.0f;
        const int e = kept ? my_e : -1;
        p.ws.idx[(size_t)t * k + lane] = e;
        p.ws.w[(size_t)t * k + lane] = w;
        if (p.idx_out) p.idx_out[(size_t)t * k + lane] = e;
        if (p.w_out) p.w_out[(size_t)t * k + lane] = w;
    }
}

// a2 by one CTA: group the T*k (token, slot) assignments by expert, stable in
// (token, slot) order, append the shared expert's T assignments first, cut
// each expert's list into tasks of at most CH tokens, publish the work-item
// counts and zero the per-call counters of the expert kernels.  For
// tensor-core tasks (p.tc) task.w is the task's first row in the padded
// operand buffers (the sum of tc_npad over the tasks before it).
// The routing indices pass through shared memory kBucketStage at a time; the
// stable placement of a stage is split over the warps (each warp a contiguous
// slice, its per-expert start found by a scan over the warps' histograms).
// smem: bucket_smem_ints(E) ints.
constexpr int kBucketStage = 4096;
__host__ __device__ constexpr int bucket_smem_ints(int E) { return 5 * E + kWarps + kWarps * E + kBucketStage; }

static __device__ void bucket_cta(const Params& p, int* smem) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int E = p.m.E, k = p.m.k, T = p.m.T, S = p.m.S, CH = p.CH;
    const int A = T * k;
    int* cnt = smem;
    int* off = smem + E;
    int* tb = smem + 2 * E;
    int* off0 = smem + 3 * E;
    int* prow = smem + 4 * E;
    int* red = smem + 5 * E;
    int* hist = red + kWarps;      // [kWarps][E]
    int* stage = hist + kWarps * E;  // [kBucketStage]
    WsHeader* hdr = p.ws.hdr;
    // one stage of routing indices into shared memory, four loads in flight per thread
    auto load_stage = [&](int base, int nb) {
        for (int i0 = 0; i0 < nb; i0 += 4 * kThreads) {
            int v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + tid + u * kThreads;
                v[u] = i < nb ? __ldcg(p.ws.idx + base + i) : 0;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int i = i0 + tid + u * kThreads;
                if (i < nb) {
                    if (v[u] == -1) {
                        v[u] = E;  // a slot the truncation dropped: no assignment
                    } else if (v[u] < 0 || v[u] >= E) {
                        set_status(hdr, MOE_EDEVICE, base + i);
                        v[u] = 0;
                    }
                    stage[i] = v[u];
                }
            }
        }
    };
    for (int e = tid; e < E; e += kThreads) cnt[e] = 0;
    __syncthreads();
    for (int base = 0; base < A; base += kBucketStage) {
        const int nb = min(kBucketStage, A - base);
        load_stage(base, nb);
        __syncthreads();
        for (int i = tid; i < nb; i += kThreads)
            if (stage[i] < E) atomicAdd(&cnt[stage[i]], 1);
        __syncthreads();
    }
    for (int e = tid; e < E; e += kThreads) {
        off[e] = cnt[e];
        tb[e] = (cnt[e] + CH - 1) / CH;
        prow[e] = (cnt[e] / CH) * tc_npad(CH) + (cnt[e] % CH ? tc_npad(cnt[e] % CH) : 0);
    }
    __syncthreads();
    block_exscan(off, E, red);
    const int n_routed_tasks = block_exscan(tb, E, red);
    const int routed_rows = p.tc ? block_exscan(prow, E, red) : 0;
    for (int e = tid; e < E; e += kThreads) off0[e] = off[e];
    __syncthreads();
    const int asg_base = p.m.has_shared ? T : 0;
    const int n_sh_tasks = p.m.has_shared ? (T + CH - 1) / CH : 0;
    const int sh_rows = p.m.has_shared ? (T / CH) * tc_npad(CH) + (T % CH ? tc_npad(T % CH) : 0) : 0;
    // stable placement: warp w takes the contiguous slice [w * per, (w + 1) * per) of a stage
    for (int base = 0; base < A; base += kBucketStage) {
        const int nb = min(kBucketStage, A - base);
        if (A > kBucketStage) {  // the stage from the counting pass was overwritten
            load_stage(base, nb);
        }
        for (int i = tid; i < kWarps * E; i += kThreads) hist[i] = 0;
        __syncthreads();
        const int per = (nb + 32 * kWarps - 1) / (32 * kWarps) * 32;
        const int lo = warp * per, hi = min(nb, lo + per);
        for (int b = lo; b < hi; b += 32) {  // per-warp histogram of the slice
            const int e = b + lane < hi ? stage[b + lane] : E;
            const unsigned peers = __match_any_sync(kFull, e);
            if (e < E && (peers & lanemask_lt()) == 0) hist[warp * E + e] += __popc(peers);
            __syncwarp();
        }
        __syncthreads();
        for (int e = tid; e < E; e += kThreads) {  // each warp's first position per expert, in warp order
            int run = off[e];
#pragma unroll
            for (int w = 0; w < kWarps; ++w) {
                const int h = hist[w * E + e];
                hist[w * E + e] = run;
                run += h;
            }
            off[e] = run;
        }
        __syncthreads();
        for (int b = lo; b < hi; b += 32) {
            const int a = base + b + lane;
            const int e = b + lane < hi ? stage[b + lane] : E;
            const unsigned peers = __match_any_sync(kFull, e);
            const int rank = __popc(peers & lanemask_lt());
            if (e < E) p.ws.asg[asg_base + hist[warp * E + e] + rank] = (a / k) * S + (a % k);
            __syncwarp();
            if (e < E && rank == 0) hist[warp * E + e] += __popc(peers);
            __syncwarp();
        }
        __syncthreads();
    }
    if (p.m.has_shared)
        for (int t = tid; t < T; t += kThreads) p.ws.asg[t] = t * S + k;
    for (int c = tid; c < n_sh_tasks; c += kThreads)
        p.ws.tasks[c] = make_int4(E, c * CH, min(CH, T - c * CH), p.tc ? c * tc_npad(CH) : 0);
    for (int e = tid; e < E; e += kThreads) {
        const int n = cnt[e];
        for (int c = 0; c * CH < n; ++c)
            p.ws.tasks[n_sh_tasks + tb[e] + c] = make_int4(e, asg_base + off0[e] + c * CH, min(CH, n - c * CH),
                                                           p.tc ? sh_rows + prow[e] + c * tc_npad(CH) : 0);
    }
    const int n_tasks = n_sh_tasks + n_routed_tasks;
    for (int i = tid; i < n_tasks; i += kThreads) p.ws.task_ctr[i] = 0;
    for (int i = tid; i < T * S; i += kThreads) p.ws.amax[i] = 0u;
    for (int i = tid; i < p.nrb4; i += kThreads) p.ws.rb_ctr[i] = 0u;
    if (tid == 0) {
        hdr->n_tasks = n_tasks;
        hdr->tc_rows = sh_rows + routed_rows;
        hdr->n_asg = T * S;
        hdr->n_items3 = n_tasks * p.nrb3;
        hdr->n_items4 = n_tasks * p.nrb4;
    }
}

// Router GEMV for up to TM tokens.  CTA b computes the logits of experts 2b and
// 2b+1 for every token (each thread a slice of d, weights streamed once); CTAs
// b < T also quantise token b.  The last CTA to finish runs the top-k of every
// token (one warp per token) and, if `bucket`, the bucketing.
// Dynamic smem: max(2 * kWarps * E floats, bucket_smem_ints(E) ints).
template <int TM, int NV, typename XT>
__global__ void __launch_bounds__(kThreads) k_route_small(const Params p, const XT* __restrict__ x,
                                                          int do_quant, int bucket) {
    extern __shared__ float dsm[];
    __shared__ float redf[kWarps];
    __shared__ int redi[kWarps];
    __shared__ float part[kWarps][2 * TM];
    __shared__ int s_last;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int d = p.m.d, E = p.m.E, T = p.m.T;
    if (do_quant)
        for (int t = blockIdx.x; t < T; t += gridDim.x)
            quantize_token(x + (size_t)t * d, d, p.ws.xq + (size_t)t * d, p.ws.sx + t, p.ws.xcs + t, redf, redi);

    const int e0 = blockIdx.x * 2;
    const int nv = d / 4;
    float acc[2][TM];
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int t = 0; t < TM; ++t) acc[j][t] = 0.0f;
    float4 wv[2][NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int v = tid + i * kThreads;
#pragma unroll
        for (int j = 0; j < 2; ++j)
            wv[j][i] = (v < nv && e0 + j < E) ? ld_stream_f4(p.w_router + (size_t)(e0 + j) * d + 4 * v)
                                              : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int v = tid + i * kThreads;
        if (v < nv) {
#pragma unroll
            for (int t = 0; t < TM; ++t) {
                if (t < T) {
                    const float4 xv = load_x4(x, (size_t)t * d + 4 * v);
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        acc[j][t] = fmaf(wv[j][i].x, xv.x, acc[j][t]);
                        acc[j][t] = fmaf(wv[j][i].y, xv.y, acc[j][t]);
                        acc[j][t] = fmaf(wv[j][i].z, xv.z, acc[j][t]);
                        acc[j][t] = fmaf(wv[j][i].w, xv.w, acc[j][t]);
                    }
                }
            }
        }
    }
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int t = 0; t < TM; ++t) {
            const float v = warp_sum(acc[j][t]);
            if (lane == 0) part[warp][j * TM + t] = v;
        }
    __syncthreads();
    if (tid < 2 * TM) {
        const int j = tid / TM, t = tid % TM;
        if (t < T && e0 + j < E) {
            float v = 0.0f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) v += part[w][tid];
            p.ws.logits[(size_t)t * E + e0 + j] = v;
        }
    }
    // last-arriving CTA: top-k (+ bucketing) over every token
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const unsigned ticket = atomicAdd(&p.ws.hdr->route_ctr, 1u);
        s_last = ticket == gridDim.x - 1;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (tid == 0) p.ws.hdr->route_ctr = 0u;
    for (int t = warp; t < T; t += kWarps) topk_token(p, t, dsm + warp * 2 * E, dsm + warp * 2 * E + E);
    __threadfence();
    __syncthreads();
    if (bucket) bucket_cta(p, reinterpret_cast<int*>(dsm));
}

// Router for many tokens: fp32 tiled GEMM logits[ks][T][E] over a 1/ksplit
// slice of d per blockIdx.z (the top-k adds the slices in order).
// 64 x 64 tile, 32-column k-step, 4 x 4 outputs per thread.
template <typename XT>
__global__ void __launch_bounds__(kThreads) k_router_tiled(const Params p, const XT* __restrict__ x) {
    // 64 tokens x 64 experts per CTA over a slice of d (blockIdx.z), 32
    // columns per step; the next step's tiles are loaded into registers while
    // the current step's FMAs run (two shared buffers).  Each thread owns a
    // 4 x 4 block of outputs; sums run in ascending column order per slice.
    __shared__ __align__(16) float xs[2][32][64 + 4];
    __shared__ __align__(16) float wsm[2][32][64 + 4];
    const int tid = threadIdx.x;
    const int d = p.m.d, E = p.m.E, T = p.m.T;
    const int t0 = blockIdx.y * 64, e0 = blockIdx.x * 64;
    const int ksteps = d / 32;
    const int per = (ksteps + p.ksplit - 1) / p.ksplit;
    const int kb = blockIdx.z * per, ke = min(ksteps, kb + per);
    const int ty = tid / 16, tx = tid % 16;
    float acc[4][4] = {};
    float4 xr[2], wr[2];  // this thread's share of one step's tiles: rows r = i / 8, columns (i % 8) * 4
    auto load = [&](int ks) {
        const int c0 = ks * 32;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int i = tid + u * kThreads, r = i / 8, c4 = (i % 8) * 4;
            xr[u] = t0 + r < T ? load_x4(x, (size_t)(t0 + r) * d + c0 + c4) : make_float4(0.f, 0.f, 0.f, 0.f);
            wr[u] = e0 + r < E ? __ldg(reinterpret_cast<const float4*>(p.w_router + (size_t)(e0 + r) * d + c0 + c4))
                               : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    };
    auto store = [&](int buf) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int i = tid + u * kThreads, r = i / 8, c4 = (i % 8) * 4;
            xs[buf][c4 + 0][r] = xr[u].x;
            xs[buf][c4 + 1][r] = xr[u].y;
            xs[buf][c4 + 2][r] = xr[u].z;
            xs[buf][c4 + 3][r] = xr[u].w;
            wsm[buf][c4 + 0][r] = wr[u].x;
            wsm[buf][c4 + 1][r] = wr[u].y;
            wsm[buf][c4 + 2][r] = wr[u].z;
            wsm[buf][c4 + 3][r] = wr[u].w;
        }
    };
    int buf = 0;
    if (kb < ke) {
        load(kb);
        store(0);
    }
    __syncthreads();
    for (int ks = kb; ks < ke; ++ks) {
        if (ks + 1 < ke) load(ks + 1);  // in flight during the FMAs below
#pragma unroll 8
        for (int c = 0; c < 32; ++c) {
            const float4 av = *reinterpret_cast<const float4*>(&xs[buf][c][ty * 4]);
            const float4 bv = *reinterpret_cast<const float4*>(&wsm[buf][c][tx * 4]);
            const float a[4] = {av.x, av.y, av.z, av.w}, b[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        if (ks + 1 < ke) store(buf ^ 1);
        __syncthreads();
        buf ^= 1;
    }
    float* dst = p.ws.logits + (size_t)blockIdx.z * T * E;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int t = t0 + ty * 4 + i;
        if (t >= T) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int e = e0 + tx * 4 + j;
            if (e < E) dst[(size_t)t * E + e] = acc[i][j];
        }
    }
}

// Top-k of many tokens: one warp per token.  Dynamic smem 2 * kWarps * E floats.
__global__ void __launch_bounds__(kThreads) k_topk(const Params p) {
    extern __shared__ float dsm[];
    const int warp = threadIdx.x >> 5;
    const int t = blockIdx.x * kWarps + warp;
    if (t < p.m.T) topk_token(p, t, dsm + warp * 2 * p.m.E, dsm + warp * 2 * p.m.E + p.m.E);
}

// Top-k of many tokens for E <= 256: one warp per token, lane l holding
// experts l + 32 i in registers.  The logits are the ksplit partial planes
// added in plane order (as topk_token adds them), every plane's loads in
// flight together; each of the k rounds takes the largest selection value
// (lowest index on ties) with two warp reductions.  Same rule and arithmetic
// as topk_token.  With `bucket`, the last CTA to finish runs the bucketing.
// Dynamic smem: bucket_smem_ints(E) ints if `bucket`.
__global__ void __launch_bounds__(kThreads) k_topk_small(const Params p, int bucket) {
    extern __shared__ int bsm[];
    __shared__ int s_last;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int E = p.m.E, k = p.m.k, T = p.m.T;
    const int t = blockIdx.x * kWarps + warp;
    if (t < T) {
        float lg[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) lg[i] = lane + 32 * i < E ? __ldcg(p.ws.logits + (size_t)t * E + lane + 32 * i) : 0.0f;
        for (int ks = 1; ks < p.ksplit; ++ks) {
            float v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                v[i] = lane + 32 * i < E ? __ldcg(p.ws.logits + ((size_t)ks * T + t) * E + lane + 32 * i) : 0.0f;
#pragma unroll
            for (int i = 0; i < 8; ++i) lg[i] += v[i];
        }
        float sv[8];
        unsigned key[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = lane + 32 * i;
            sv[i] = 0.0f;
            key[i] = 0u;  // below every real key
            if (e < E) {
                sv[i] = __fdiv_rn(1.0f, __fadd_rn(1.0f, expf(-lg[i])));
                key[i] = float_key(__fadd_rn(sv[i], __ldg(p.bias + e)));
            }
        }
        float ssum = 0.0f, my_s = 0.0f, cex = 0.0f, cin = 0.0f;
        int my_e = 0;
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
        const float norm = topp_keep(p.topp, k, ssum, cex, cin, kept);
        if (lane < k) {  // a slot the truncation drops selects no expert: -1, weight 0
            const float w = kept ? __fmul_rn(__fdiv_rn(my_s, norm), p.routed_scale) : 0.0f;
            const int e = kept ? my_e : -1;
            p.ws.idx[(size_t)t * k + lane] = e;
            p.ws.w[(size_t)t * k + lane] = w;
            if (p.idx_out) p.idx_out[(size_t)t * k + lane] = e;
            if (p.w_out) p.w_out[(size_t)t * k + lane] = w;
        }
    }
    if (!bucket) return;
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        s_last = atomicAdd(&p.ws.hdr->route_ctr, 1u) == gridDim.x - 1;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (tid == 0) p.ws.hdr->route_ctr = 0u;
    bucket_cta(p, bsm);
}

// Bucketing alone (one CTA).  Dynamic smem bucket_smem_ints(E) ints.
__global__ void __launch_bounds__(kThreads) k_bucket(const Params p) {
    extern __shared__ int ism[];
    bucket_cta(p, ism);
}

// Plan of the single-expert entry points: the tokens 0..T-1 of one expert in
// tasks of at most CH tokens (assignment id = token), counters zeroed.
__global__ void __launch_bounds__(kThreads) k_plan_single(const Params p, int blob) {
    const int T = p.m.T, CH = p.CH;
    const int n_tasks = (T + CH - 1) / CH;
    for (int t = threadIdx.x; t < T; t += kThreads) {
        p.ws.asg[t] = t;
        p.ws.amax[t] = 0u;
    }
    for (int c = threadIdx.x; c < n_tasks; c += kThreads) {
        p.ws.tasks[c] = make_int4(blob, c * CH, min(CH, T - c * CH), p.tc ? c * tc_npad(CH) : 0);
        p.ws.task_ctr[c] = 0u;
    }
    for (int i = threadIdx.x; i < p.nrb4; i += kThreads) p.ws.rb_ctr[i] = 0u;
    if (threadIdx.x == 0) {
        p.ws.hdr->n_tasks = n_tasks;
        p.ws.hdr->tc_rows = (T / CH) * tc_npad(CH) + (T % CH ? tc_npad(T % CH) : 0);
        p.ws.hdr->n_asg = T;
        p.ws.hdr->n_items3 = n_tasks * p.nrb3;
        p.ws.hdr->n_items4 = n_tasks * p.nrb4;
    }
}

// Parameter-free RMSNorm (one CTA per token): x_in = x / sqrt(mean(x^2) + eps).
template <typename XT>
__global__ void __launch_bounds__(kThreads) k_rmsnorm(const XT* __restrict__ x, int T, int d, float eps,
                                                       float* __restrict__ x_in, float* __restrict__ x_copy) {
    __shared__ float redf[kWarps];
    for (int t = blockIdx.x; t < T; t += gridDim.x) {
        const XT* xt = x + (size_t)t * d;
        float ss = 0.0f;
        for (int c = threadIdx.x; c < d; c += kThreads) {
            const float v = load_x(xt, c);
            ss = fmaf(v, v, ss);
        }
        ss = block_sum(ss, redf);
        const float r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(ss, (float)d), eps)));
        for (int c = threadIdx.x; c < d; c += kThreads) {
            const float v = load_x(xt, c);
            x_in[(size_t)t * d + c] = v * r;
            if (x_copy) x_copy[(size_t)t * d + c] = v;
        }
    }
}

}  // namespace moe
