// Steps a3-a6 for decode-sized batches: the fused gate/up GEMV and the down
// GEMV + weighted combine.  Both walk a list of work items (task, row block);
// a task is one expert with up to CH of its tokens, so each expert's weights
// stream from HBM once per call however many tokens picked it.
#pragma once

#include "moe_common.cuh"

namespace moe {

// Stage the int8 rows of a task's tokens into the permuted shared layout.
// Returns true after a restage (the caller syncs); rows come from `src`
// (row r of token slot i at src + key_i * ld).  s_key caches what is staged.
// ---------------------------------------------------------------------------
// a3: gate/up.  Item = (task, RB3 = 8 * RPW rows of f).  Each warp takes RPW
// rows; for a row r it streams gate row r and up row r (16-byte chunks per
// lane), dots them with every staged token, reduces across the warp and forms
// h = SiLU(g) * u.  Per-token max |h| goes to amax[asg] (atomicMax on the
// float bits, order-free).  The CTA that completes a task's last item
// requantises h of that task into hq / sh (int8 rule of the layer).
// ---------------------------------------------------------------------------
template <int WB, int CH, int NCL, int RPW, bool DBG>
__global__ void __launch_bounds__(kThreads) k_gate_up(const Params p) {
    constexpr int NSUB = 8 / WB;
    extern __shared__ uint4 xs[];  // [CH][NSUB][nch]
    __shared__ int s_tok[CH], s_asg[CH], s_cs[CH], s_n, s_last;
    __shared__ float s_sx[CH];
    __shared__ unsigned s_amax[CH];
    __shared__ int redi[kWarps];
    __shared__ float redf[kWarps];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int d = p.m.d, f = p.m.f, S = p.m.S;
    const int rowbytes = d * WB / 8, nch = rowbytes / 16;
    const int n_items = p.ws.hdr->n_items3;
    if (tid == 0) s_n = -1;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        const int ti = item / p.nrb3, rb = item % p.nrb3;
        const int4 task = p.ws.tasks[ti];
        const int n = idx_in(p.ws.hdr, task.z, 0, CH + 1, 621);
        __syncthreads();  // previous item done with the staged rows
        if (warp == 0) {
            int a = -1, tok = -1;
            if (lane < n) {
                a = idx_in(p.ws.hdr, p.ws.asg[idx_in(p.ws.hdr, task.y + lane, 0, p.a_cap, 622)], 0, p.a_cap, 623);
                tok = a / S;
            }
            const bool same = __all_sync(kFull, s_n == n && (lane >= n || s_tok[lane] == tok));
            __syncwarp();
            if (lane < CH) {
                s_asg[lane] = a;
                s_amax[lane] = 0u;
                if (!same) s_tok[lane] = tok;
            }
            if (lane == 0 && !same) s_n = -2 - n;
        }
        __syncthreads();
        if (s_n < -1) {  // restage this task's activation rows
            const int nn = -2 - s_n;
            for (int i = 0; i < nn; ++i) {
                const int tok = s_tok[i];
                stage_row<WB>(p.ws.xq + (size_t)tok * d, d, xs + (size_t)i * NSUB * nch);
                if (tid == 0) {
                    s_sx[i] = p.ws.sx[tok];
                    s_cs[i] = p.ws.xcs[tok];
                }
            }
            __syncthreads();
            if (tid == 0) s_n = nn;
        }
        const int bx = idx_in(p.ws.hdr, task.x, 0, p.m.E + p.m.has_shared, 624);
        const uint8_t* blob = p.pool + (size_t)blob_slot(p, bx, 625) * p.blob_bytes;
        const float* sc = p.scales + (size_t)bx * p.scale_rows;
        float amax[CH];
#pragma unroll
        for (int t = 0; t < CH; ++t) amax[t] = 0.0f;
#pragma unroll 1
        for (int rr = 0; rr < RPW; ++rr) {
            const int r = rb * (kWarps * RPW) + rr * kWarps + warp;
            if (r >= f) break;
            const uint8_t* grow = blob + (size_t)r * rowbytes;
            const uint8_t* urow = blob + ((size_t)f + r) * rowbytes;
            uint4 wg[NCL], wu[NCL];
#pragma unroll
            for (int i = 0; i < NCL; ++i) {
                const int c = lane + 32 * i;
                if (c < nch) {
                    wg[i] = ld_stream(grow + (size_t)c * 16);
                    wu[i] = ld_stream(urow + (size_t)c * 16);
                }
            }
            int ag[CH], au[CH];
#pragma unroll
            for (int t = 0; t < CH; ++t) ag[t] = au[t] = 0;
#pragma unroll
            for (int i = 0; i < NCL; ++i) {
                const int c = lane + 32 * i;
                if (c < nch) {
#pragma unroll
                    for (int t = 0; t < CH; ++t)
                        if (t < n) {
                            const uint4* xt = xs + (size_t)t * NSUB * nch;
                            ag[t] = dot_chunk<WB>(wg[i], xt, nch, c, ag[t]);
                            au[t] = dot_chunk<WB>(wu[i], xt, nch, c, au[t]);
                        }
                }
            }
            const float sg = __ldg(sc + r), su = __ldg(sc + f + r);
#pragma unroll
            for (int t = 0; t < CH; ++t) {
                if (t < n) {
                    const int G = __reduce_add_sync(kFull, ag[t]) - code_offset<WB>() * s_cs[t];
                    const int U = __reduce_add_sync(kFull, au[t]) - code_offset<WB>() * s_cs[t];
                    if (lane == t) {
                        const float g = __fmul_rn((float)G, __fmul_rn(sg, s_sx[t]));
                        const float u = __fmul_rn((float)U, __fmul_rn(su, s_sx[t]));
                        const float h = __fmul_rn(__fdiv_rn(g, __fadd_rn(1.0f, expf(-g))), u);
                        const int a = s_asg[t];
                        p.ws.h[(size_t)a * f + r] = h;
                        amax[t] = fmaxf(amax[t], fabsf(h));
                        if (DBG && p.dbg_acc_gu) {
                            p.dbg_acc_gu[(size_t)a * 2 * f + r] = G;
                            p.dbg_acc_gu[(size_t)a * 2 * f + f + r] = U;
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int t = 0; t < CH; ++t)
            if (t < n && lane == t) atomicMax(&s_amax[t], __float_as_uint(amax[t]));
        __syncthreads();
        if (tid < n) atomicMax(&p.ws.amax[s_asg[tid]], s_amax[tid]);
        __syncthreads();
        if (tid == 0) {
            __threadfence();
            s_last = atomicAdd(&p.ws.task_ctr[ti], 1u) == (unsigned)(p.nrb3 - 1);
        }
        __syncthreads();
        if (s_last) {  // every item of this task is done: requantise its h
            __threadfence();
            if (tid == 0) p.ws.task_ctr[ti] = 0u;
            for (int t = 0; t < n; ++t) {
                const int a = s_asg[t];
                const float m = __uint_as_float(__ldcg(p.ws.amax + a));
                const float sh = m == 0.0f ? 0.0f : __fdiv_rn(m, 127.0f);
                const float rh = quant_recip(sh);
                const float* hrow = p.ws.h + (size_t)a * f;
                int8_t* qrow = p.ws.hq + (size_t)a * f;
                for (int c = tid * 4; c < f; c += kThreads * 4) {
                    const float4 hv = __ldcg(reinterpret_cast<const float4*>(hrow + c));
                    char4 q = make_char4(0, 0, 0, 0);
                    if (m != 0.0f)
                        q = make_char4((signed char)quant_code_r(hv.x, sh, rh), (signed char)quant_code_r(hv.y, sh, rh),
                                       (signed char)quant_code_r(hv.z, sh, rh), (signed char)quant_code_r(hv.w, sh, rh));
                    *reinterpret_cast<char4*>(qrow + c) = q;
                    if (DBG && p.dbg_hq) *reinterpret_cast<char4*>(p.dbg_hq + (size_t)a * f + c) = q;
                }
                if (tid == 0) {
                    p.ws.sh[a] = sh;
                    if (DBG && p.dbg_sh) p.dbg_sh[a] = sh;
                }
            }
            __syncthreads();  // every thread has read amax of the task's tokens
            if (tid < n) p.ws.amax[s_asg[tid]] = 0u;  // leave the workspace zeroed for the next call
        }
    }
    (void)redi;
    (void)redf;
}

// ---------------------------------------------------------------------------
// a4 + a6: down.  Item = (task, RB4 = 8 * RPW rows of d).  The task's hq rows
// are staged (permuted) with their code sums; each warp streams RPW down rows
// at once and writes y = D * (s_row * s_h) for every token, either straight to
// the output (single-expert entry points) or to the per-assignment slot
// buffer.  The CTA that completes the last item of a row block combines that
// block for every token in a fixed order: out = sum_j w_j y_j + y_shared.
// ---------------------------------------------------------------------------
template <int WB, int CH, int NCL, int RPW, bool DBG>
__global__ void __launch_bounds__(kThreads) k_down(const Params p) {
    constexpr int NSUB = 8 / WB;
    constexpr int RB = kWarps * RPW;
    extern __shared__ uint4 xs[];  // [CH][NSUB][nch]
    __shared__ int s_asg[CH], s_cs[CH], s_key, s_last;
    __shared__ float s_sh[CH];
    __shared__ int redi[kWarps];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int d = p.m.d, f = p.m.f, S = p.m.S, k = p.m.k, T = p.m.T;
    const int rowbytes = f * WB / 8, nch = rowbytes / 16;
    const int n_items = p.ws.hdr->n_items4;
    const int n_tasks = p.ws.hdr->n_tasks;
    if (tid == 0) s_key = -1;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        const int ti = item / p.nrb4, rb = item % p.nrb4;
        const int4 task = p.ws.tasks[ti];
        const int n = idx_in(p.ws.hdr, task.z, 0, CH + 1, 631);
        __syncthreads();
        if (s_key != ti) {  // stage this task's h codes
            if (tid < n)
                s_asg[tid] = idx_in(p.ws.hdr, p.ws.asg[idx_in(p.ws.hdr, task.y + tid, 0, p.a_cap, 632)], 0, p.a_cap, 633);
            __syncthreads();
            for (int i = 0; i < n; ++i) {
                const int a = s_asg[i];
                const int8_t* src = p.hq_in ? p.hq_in + (size_t)a * f : p.ws.hq + (size_t)a * f;
                int cs = stage_row<WB>(src, f, xs + (size_t)i * NSUB * nch);
                cs = block_sum_int(cs, redi);
                if (tid == 0) {
                    s_cs[i] = cs;
                    s_sh[i] = p.sh_in ? p.sh_in[a] : __ldcg(p.ws.sh + a);
                }
            }
            if (tid == 0) s_key = ti;
            __syncthreads();
        }
        const int bx = idx_in(p.ws.hdr, task.x, 0, p.m.E + p.m.has_shared, 634);
        const uint8_t* wd = p.pool + (size_t)blob_slot(p, bx, 635) * p.blob_bytes + 2 * (size_t)f * (d * WB / 8);
        const float* sd = p.scales + (size_t)bx * p.scale_rows + 2 * f;
        const int r0 = rb * RB + warp * RPW;
        uint4 wv[RPW][NCL];
#pragma unroll
        for (int j = 0; j < RPW; ++j)
#pragma unroll
            for (int i = 0; i < NCL; ++i) {
                const int c = lane + 32 * i;
                if (r0 + j < d && c < nch) wv[j][i] = ld_stream(wd + (size_t)(r0 + j) * rowbytes + (size_t)c * 16);
            }
        int acc[RPW][CH];
#pragma unroll
        for (int j = 0; j < RPW; ++j)
#pragma unroll
            for (int t = 0; t < CH; ++t) acc[j][t] = 0;
#pragma unroll
        for (int i = 0; i < NCL; ++i) {
            const int c = lane + 32 * i;
            if (c < nch) {
#pragma unroll
                for (int t = 0; t < CH; ++t)
                    if (t < n) {
                        const uint4* xt = xs + (size_t)t * NSUB * nch;
#pragma unroll
                        for (int j = 0; j < RPW; ++j) acc[j][t] = dot_chunk<WB>(wv[j][i], xt, nch, c, acc[j][t]);
                    }
            }
        }
#pragma unroll
        for (int j = 0; j < RPW; ++j) {
            const int r = r0 + j;
            if (r >= d) break;
            const float sdr = __ldg(sd + r);
#pragma unroll
            for (int t = 0; t < CH; ++t)
                if (t < n) {
                    const int D = __reduce_add_sync(kFull, acc[j][t]) - code_offset<WB>() * s_cs[t];
                    if (lane == t) {
                        const int a = s_asg[t];
                        const float y = __fmul_rn((float)D, __fmul_rn(sdr, s_sh[t]));
                        if (p.direct_out) p.out[(size_t)a * d + r] = y;
                        else p.ws.ybuf[(size_t)a * d + r] = y;
                        if (DBG && p.dbg_acc_d) p.dbg_acc_d[(size_t)a * d + r] = D;
                    }
                }
        }
        if (p.direct_out) continue;
        __syncthreads();
        if (tid == 0) {
            __threadfence();
            s_last = atomicAdd(&p.ws.rb_ctr[rb], 1u) == (unsigned)(n_tasks - 1);
        }
        __syncthreads();
        if (s_last) {  // all tasks wrote this row block: combine it
            __threadfence();
            if (tid == 0) p.ws.rb_ctr[rb] = 0u;
            const int rows = min(RB, d - rb * RB);
            for (int i = tid; i < T * rows; i += kThreads) {
                const int t = i / rows, r = rb * RB + i % rows;
                float o = 0.0f;
                for (int j = 0; j < k; ++j)  // (a slot the truncation dropped has no output)
                    if (__ldcg(p.ws.idx + (size_t)t * k + j) >= 0)
                        o = fmaf(__ldcg(p.ws.w + (size_t)t * k + j), __ldcg(p.ws.ybuf + ((size_t)t * S + j) * d + r), o);
                if (p.m.has_shared) o += __ldcg(p.ws.ybuf + ((size_t)t * S + k) * d + r);
                float* dst = p.out + (size_t)t * d + r;
                *dst = p.accumulate ? *dst + o : o;
            }
        }
    }
}

}  // namespace moe
