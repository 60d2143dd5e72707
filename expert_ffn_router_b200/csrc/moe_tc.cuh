// Steps a3-a6 on the 5th-generation tensor cores (tcgen05, sm_100a): the
// int8 grouped GEMM for batches whose experts see many tokens (prefill,
// long verify batches).  An expert's packed weights stream from HBM once per
// task of up to kTcNT tokens; the integer products run as
// tcgen05.mma.kind::i8 with int32 accumulators in tensor memory (TMEM).
//
// Operands (one MMA: M = 128 weight rows, N = the task's padded tokens,
// K = 32 codes):
//  A  weight codes.  A TMA box of 128 rows x 64 packed bytes (64-byte swizzle)
//     lands in shared memory; the unpack warps split each 32-bit word into
//     offset-binary bytes (u = c + 8 for int4, c + 2 for int2, the same masks
//     as the dp4a kernels; int8 bytes with the sign bit flipped, c + 128) and
//     store them to TMEM, from where the MMA reads A.
//     Unsigned A times signed activations gives sum(u x) = sum(c x) + off sum(x);
//     the epilogue subtracts off * sum(x).
//  B  int8 activations (or requantised h) of the task's tokens, in the
//     canonical K-major no-swizzle layout of 8-row x 16-byte core matrices,
//     with each 16-byte K group in the byte order the unpack produces
//     (permute16).  The gather kernel (x) or the requantisation kernel (h)
//     writes it per task and K chunk, so one bulk copy brings a chunk's B into
//     shared memory.
//
// An M = 128, K = 32 MMA issued back to back takes ~97 SM cycles for any
// N <= 128 when each one accumulates into the previous one's tile, ~54 when
// two tiles alternate (as here), ~68 with two commits per eight MMAs
// (microbenchmark on B200), while an SM's share of HBM bandwidth delivers
// one int4 A step (2 KB of packed codes) in ~90 cycles: the MMA stream keeps
// up with HBM only while it does not stall.  Persistent, two CTAs per SM (their
// MMA streams interleave on the SM's tensor pipe), 448 threads each:
//  warp 0      TMA producer: per K chunk two A boxes + the B chunk into a
//              ring of shared-memory slots (full / empty mbarriers);
//  warp 1      TMEM allocator and MMA issuer (one thread): per chunk
//              KC/32 K-steps x 2 tiles; tcgen05.commit releases the slot and
//              the TMEM A buffer, a commit per unit hands an accumulator
//              buffer to the epilogue;
//  warps 2-9   unpack A into a ring of TMEM A buffers (two warps per TMEM
//              lane quarter, each half of a row's chunk);
//  warps 10-13 epilogue (tcgen05.ld of the accumulators, one warp per lane
//              quarter), so the MMAs of a unit overlap the previous unit's
//              epilogue.
// A unit is (task, row block): two 128-row A tiles sharing one B --
//  gate/up (EPI 0): gate rows and up rows [128 rb, 128 rb + 128) of f;
//                   epilogue h = SiLU(g) u and the per-token max |h|
//                   (requantisation is a separate kernel);
//  down    (EPI 1): rows [256 rb, 256 rb + 256) of d as two tiles; epilogue
//                   y = acc (s_row s_h) to the per-assignment buffer (the
//                   combine is a separate kernel) or straight to the output.
// TMEM columns (CPS = 1, one CTA per SM): two accumulator buffers [128 b, 128 b + 128)
// (tile 0 at +0, tile 1 at +64, N <= 64), then the A buffers from column 256
// (2 x KC/4 columns each: eight buffers for int8, four for int4, two for
// int2); two CTAs per SM: 256 columns each, one accumulator buffer and A
// buffers from column 128 (four for int8, two for int4, one for int2).  Every wait is bounded
// (kWaitLimitNs); on a timeout the CTA records MOE_ETIMEOUT, lets its copies
// and MMAs drain and exits.
#pragma once

#include <cuda.h>

#include "moe_common.cuh"

namespace moe {

constexpr int kTcThreads = 448;
constexpr int kTcUnpack = 256;                 // warps 2-9
constexpr int kTcEpiWarp0 = 10;                // warps 10-13
constexpr int kTcEpi = 128;
// A weight box: 128 rows x tc_box_w bytes of packed codes, one box per tile
// per ring slot.  Rows loaded 128 bytes (two chunks of 64 bytes) at a time
// with the 128-byte swizzle arrive whole instead of through promoted L2 lines
// that may be evicted before their chunk is loaded, but a slot is then
// released only after both chunks.  Measured on B200 (two CTAs per SM): the
// down kernels and int8 weights gain (T = 512, int4 down: 285 us instead of
// 307; int8 gate/up at T = 8: 264 instead of 270), the int4 gate/up kernel
// loses (519 instead of 506), so it keeps 64-byte boxes, as does int2, whose
// operand-B chunks are four times larger (two-chunk slots would not fit
// twice in a CTA's shared memory).
__host__ __device__ constexpr int tc_box_w(int wb, int epi) { return wb == 2 || (wb == 4 && epi == 0) ? 64 : 128; }
__host__ __device__ constexpr int tc_cpl(int wb, int epi) { return tc_box_w(wb, epi) / 64; }  // chunks per slot
__host__ __device__ constexpr int tc_box_bytes(int wb, int epi) { return 128 * tc_box_w(wb, epi); }
__host__ __device__ constexpr int tc_slot_a(int wb, int epi) { return 2 * tc_box_bytes(wb, epi); }  // both tiles
constexpr int kTcMaxSlots = 8;
constexpr int kTcMaxAB = 8;                    // TMEM A buffers: 256 columns / (2 tiles x KC/4), KC = 64 for int8

// Dynamic shared memory: [slots][control block], slots 1024-byte aligned.
struct TcCtl {
    uint64_t full[kTcMaxSlots], empty[kTcMaxSlots];
    uint64_t afull[kTcMaxAB], afree[kTcMaxAB], accfull[2], accempty[2], drain;
    uint32_t tmem_base;
    int asg[kTcNT];
    float sx[kTcNT];
    int cs[kTcNT];
};

__host__ __device__ constexpr int tc_slot_bytes(int nt_max, int wb, int epi) {
    return (tc_slot_a(wb, epi) + tc_cpl(wb, epi) * nt_max * tc_kc(wb) + 1023) / 1024 * 1024;
}
__host__ __device__ constexpr size_t tc_smem_bytes(int ns, int nt_max, int wb, int epi) {
    return 1024 + (size_t)ns * tc_slot_bytes(nt_max, wb, epi) + sizeof(TcCtl);
}

// Same as mbar_wait_bounded, but also gives up when another wait of the call
// has already failed (the status word is set).
__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity, WsHeader* hdr, int site) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 255u) == 255u) {
            if (ld_volatile_status(hdr) != 0) return false;
            if (global_timer_ns() - t0 > kWaitLimitNs) {
                set_status(hdr, MOE_ETIMEOUT, site);
                return false;
            }
        }
    }
}

// Unpack one thread's share of one A tile of a chunk into TMEM.  Row `row` of
// the box: BW packed bytes, 64-byte rows with the 64-byte swizzle
// (16-byte unit j of row r at unit j ^ ((r >> 1) & 3)) or 128-byte rows with
// the 128-byte swizzle (unit j at j ^ (r & 7)); the chunk is half `hc` of a
// 128-byte row (units 4hc .. 4hc + 3), and half `hh` of the chunk takes its
// units 2hh and 2hh+1.
template <int BW>
__device__ __forceinline__ int tc_unit(int row, int hc, int u) {
    return BW == 64 ? u ^ ((row >> 1) & 3) : (4 * hc + u) ^ (row & 7);
}
template <int WB, int BW>
__device__ __forceinline__ void tc_unpack_tile(const uint8_t* box, int row, int hh, int hc, uint32_t taddr) {
    const uint8_t* rp = box + row * BW;
    if (WB == 8) {  // one code per byte: flip each sign bit
        uint32_t w[8];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const uint4 v = *reinterpret_cast<const uint4*>(rp + (tc_unit<BW>(row, hc, 2 * hh + j) << 4));
            w[4 * j] = v.x ^ 0x80808080u;
            w[4 * j + 1] = v.y ^ 0x80808080u;
            w[4 * j + 2] = v.z ^ 0x80808080u;
            w[4 * j + 3] = v.w ^ 0x80808080u;
        }
        tmem_st8(taddr, w);
    } else if (WB == 4) {
        uint32_t w[16];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const uint4 v = *reinterpret_cast<const uint4*>(rp + (tc_unit<BW>(row, hc, 2 * hh + j) << 4));
            const uint32_t in[4] = {v.x ^ 0x88888888u, v.y ^ 0x88888888u, v.z ^ 0x88888888u, v.w ^ 0x88888888u};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                w[8 * j + 2 * i] = in[i] & 0x0F0F0F0Fu;
                w[8 * j + 2 * i + 1] = (in[i] >> 4) & 0x0F0F0F0Fu;
            }
        }
        tmem_st16(taddr, w);
    } else {
        uint32_t w[32];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const uint4 v = *reinterpret_cast<const uint4*>(rp + (tc_unit<BW>(row, hc, 2 * hh + j) << 4));
            const uint32_t in[4] = {v.x ^ 0xAAAAAAAAu, v.y ^ 0xAAAAAAAAu, v.z ^ 0xAAAAAAAAu, v.w ^ 0xAAAAAAAAu};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int s = 0; s < 4; ++s) w[16 * j + 4 * i + s] = (in[i] >> (2 * s)) & 0x03030303u;
        }
        tmem_st32(taddr, w);
    }
}

// Byte offset of 16-byte K group `kg` (K columns 16 kg .. 16 kg + 15) of
// padded row j in a task's B buffer, laid out [K group][row][16 bytes]: K
// chunk c (KC columns) is the npad * KC bytes at c * npad * KC, and within it
// the core matrix of rows 8i..8i+7 and K group g sits at (g * npad + 8i) * 16.
__device__ __forceinline__ size_t tc_b_offset(int kg, int j, int npad) {
    return ((size_t)kg * npad + j) * 16;
}

// CPS: CTAs per SM.  One CTA (CPS = 1) owns all 512 TMEM columns: two
// accumulator buffers (the epilogue of a unit overlaps the next unit's MMAs)
// and 256 columns of A buffers.  Two CTAs (CPS = 2, what the library
// launches) own 256 columns each: one accumulator buffer and 128 columns of
// A buffers (one for int2); the SM's tensor pipe then interleaves the two
// CTAs' MMA streams, so neither CTA's serial waits (slot, A buffer,
// accumulator hand-offs) leave it idle.  Measured on B200, two CTAs beat one
// for every width: at T = 512 (int4) the gate/up kernel takes 505 us instead
// of 611, on the int2 stack 156 us instead of 167, although an int2 CTA then
// unpacks a chunk only after the previous one's MMAs have completed.
template <int WB, int EPI, int CPS>
__global__ void __launch_bounds__(kTcThreads, CPS)
    k_tc(const Params p, const __grid_constant__ CUtensorMap tmA, int ns, int nt_max) {
    constexpr int KC = tc_kc(WB);           // K columns per chunk
    constexpr int ACOLS = KC / 4;           // TMEM columns of one tile's A chunk
    constexpr int KSTEPS = KC / 32;
    constexpr uint32_t TCOLS = 512 / CPS;   // TMEM columns this CTA allocates
    constexpr uint32_t NACC = 2 / CPS;      // accumulator buffers of 128 columns
    constexpr uint32_t ABASE = 128 * NACC;  // first A-buffer column
    constexpr int NAB = (int)(TCOLS - ABASE) / (2 * ACOLS);  // TMEM A buffers
    static_assert(NAB >= 1 && NAB <= kTcMaxAB, "TcCtl holds kTcMaxAB A-buffer barriers");
    constexpr int OFF = code_offset<WB>();
    constexpr int BW = tc_box_w(WB, EPI), CPL = tc_cpl(WB, EPI), BOX = tc_box_bytes(WB, EPI);
    constexpr int SLOT_A = tc_slot_a(WB, EPI);
    extern __shared__ uint8_t tc_raw[];
    uint8_t* base = tc_raw + ((1024 - (smem_u32(tc_raw) & 1023u)) & 1023u);
    const int slot_bytes = tc_slot_bytes(nt_max, WB, EPI);
    TcCtl* ctl = reinterpret_cast<TcCtl*>(base + (size_t)ns * slot_bytes);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    WsHeader* hdr = p.ws.hdr;
    const int d = p.m.d, f = p.m.f;
    const int K = EPI == 0 ? d : f;
    const int nch = (K + KC - 1) / KC;
    const int kpad = nch * KC;
    const int nrb = EPI == 0 ? (f + 127) / 128 : (d + 255) / 256;
    const int n_units = hdr->n_tasks * nrb;
    const uint8_t* bbuf = EPI == 0 ? p.ws.xb : p.ws.hb;

    if (tid == 0) {
        for (int i = 0; i < ns; ++i) {
            mbar_init(&ctl->full[i], 1);
            mbar_init(&ctl->empty[i], 1);
        }
        for (int i = 0; i < NAB; ++i) {
            mbar_init(&ctl->afull[i], kTcUnpack / 32);  // one arrival per unpack warp
            mbar_init(&ctl->afree[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&ctl->accfull[i], 1);
            mbar_init(&ctl->accempty[i], kTcEpi / 32);  // one arrival per epilogue warp
        }
        mbar_init(&ctl->drain, 1);
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(&ctl->tmem_base, TCOLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = ctl->tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_first();
            int slot = 0;
            uint32_t ph = 0, issued = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
                const int ti = u / nrb, rb = u - ti * nrb;
                const int4 task = p.ws.tasks[ti];
                const int npad = tc_npad(idx_in(hdr, task.z, 1, kTcNT + 1, 641));
                const uint32_t bbytes = (uint32_t)npad * KC;
                const int bx = blob_slot(p, idx_in(hdr, task.x, 0, p.m.E + p.m.has_shared, 642), 649);
                int y0, y1;  // rows of the pool map (the task's blob: its expert, or its cache slot)
                if (EPI == 0) {
                    y0 = bx * 3 * f + rb * 128;
                    y1 = y0 + f;
                } else {
                    y0 = bx * 3 * d + 2 * d + rb * 256;
                    y1 = y0 + 128;
                }
                const uint8_t* bsrc =
                    bbuf + (size_t)idx_in(hdr, task.w, 0, (int)tc_rows_bound(p.m) - npad + 1, 643) * kpad;
                // one slot per CPL chunks (the unit's last slot may hold
                // fewer): both tiles' boxes and the chunks' operand B
                for (int c = 0; c < nch; c += CPL) {
                    if (!tc_wait(&ctl->empty[slot], ph ^ 1u, hdr, 0x7101)) {
                        ok = false;
                        break;
                    }
                    const uint32_t nc = (uint32_t)min(CPL, nch - c);
                    uint8_t* sp = base + (size_t)slot * slot_bytes;
                    mbar_arrive_expect_tx(&ctl->full[slot], SLOT_A + nc * bbytes);
                    tma_load_2d(sp, &tmA, c * 64, y0, &ctl->full[slot], pol);
                    tma_load_2d(sp + BOX, &tmA, c * 64, y1, &ctl->full[slot], pol);
                    bulk_g2s(sp + SLOT_A, bsrc + (size_t)c * bbytes, nc * bbytes, &ctl->full[slot]);
                    ++issued;
                    if (++slot == ns) {
                        slot = 0;
                        ph ^= 1u;
                    }
                }
            }
            // drain: every issued copy has landed before the CTA exits
            for (int s = 0; s < ns; ++s) {
                const uint32_t n_s = issued / ns + ((uint32_t)s < issued % ns ? 1u : 0u);
                if (n_s) mbar_wait_bounded(&ctl->full[s], (n_s - 1) & 1u, hdr, 0x7102);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int slot = 0, ab = 0;
            uint32_t ph = 0, abph = 0, uidx = 0;
            bool ok = true, issued = false;
            for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++uidx) {
                const int ti = u / nrb;
                const int npad = tc_npad(idx_in(hdr, p.ws.tasks[ti].z, 1, kTcNT + 1, 644));
                const uint32_t idesc = tc_idesc_u8s8(npad);
                const uint32_t lbo = (uint32_t)npad * 16;
                const uint32_t buf = uidx % NACC;
                const uint32_t dcol = tbase + 128 * buf;
                if (!tc_wait(&ctl->accempty[buf], ((uidx / NACC) & 1u) ^ 1u, hdr, 0x7103)) break;
                tc_fence_after();
                for (int c = 0; c < nch; ++c) {
                    if (!tc_wait(&ctl->full[slot], ph, hdr, 0x7104) || !tc_wait(&ctl->afull[ab], abph, hdr, 0x7105)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int hc = c % CPL;  // which chunk of the slot
                    const uint32_t bsm = smem_u32(base + (size_t)slot * slot_bytes + SLOT_A) + hc * npad * KC;
                    const uint32_t acol = tbase + ABASE + ab * 2 * ACOLS;
#pragma unroll
                    for (int ks = 0; ks < KSTEPS; ++ks) {
                        const uint64_t bdesc = smem_desc(bsm + ks * 2 * lbo, lbo, 128);
                        const uint32_t acc = (c | ks) != 0;
                        tc_mma_i8_ts(dcol, acol + ks * 8, bdesc, idesc, acc);
                        tc_mma_i8_ts(dcol + 64, acol + ACOLS + ks * 8, bdesc, idesc, acc);
                    }
                    issued = true;
                    if (hc == CPL - 1 || c == nch - 1) {  // the slot's last chunk
                        tc_commit(&ctl->empty[slot]);
                        if (++slot == ns) {
                            slot = 0;
                            ph ^= 1u;
                        }
                    }
                    tc_commit(&ctl->afree[ab]);
                    if (++ab == NAB) {
                        ab = 0;
                        abph ^= 1u;
                    }
                }
                if (ok) tc_commit(&ctl->accfull[buf]);
            }
            // drain: every MMA issued has completed before TMEM is released
            if (issued) {
                tc_commit(&ctl->drain);
                mbar_wait_bounded(&ctl->drain, 0, hdr, 0x7106);
            }
        }
    } else if (warp < kTcEpiWarp0) {
        // ------------------------------------------------------------ unpack
        // A failed wait (timeout, or another wait of the call failed) makes
        // `ok` false for the whole warp; the warp then skips the tensor-memory
        // work but still arrives on every mbarrier.
        const int ew = warp - 2;
        const int q = warp & 3;            // TMEM lane quarter this warp may access
        const int hh = ew >> 2;            // which half of a chunk row
        const int row = 32 * q + lane;     // row of the 128-row tiles
        const uint32_t tlane = tbase + ((uint32_t)(32 * q) << 16);
        int slot = 0, ab = 0;
        uint32_t ph = 0, abph = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
            for (int c = 0; c < nch; ++c) {
                const int hc = c % CPL;  // which chunk of the slot
                if (ok) ok = tc_wait(&ctl->full[slot], ph, hdr, 0x7107) && tc_wait(&ctl->afree[ab], abph ^ 1u, hdr, 0x7108);
                ok = __all_sync(kFull, ok);
                if (ok) {
                    tc_fence_after();
                    const uint8_t* sp = base + (size_t)slot * slot_bytes;
                    const uint32_t acol = tlane + ABASE + ab * 2 * ACOLS + hh * (ACOLS / 2);
                    tc_unpack_tile<WB, BW>(sp, row, hh, hc, acol);
                    tc_unpack_tile<WB, BW>(sp + BOX, row, hh, hc, acol + ACOLS);
                    tmem_st_wait();
                }
                // this warp's reads of the slot (generic proxy) before the
                // producer's next TMA load into it (async proxy), which the
                // MMA's commit of the slot's last chunk lets it issue
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl->afull[ab]);
                if (hc == CPL - 1 || c == nch - 1) {  // the slot's last chunk
                    if (++slot == ns) {
                        slot = 0;
                        ph ^= 1u;
                    }
                }
                if (++ab == NAB) {
                    ab = 0;
                    abph ^= 1u;
                }
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int etid = tid - 32 * kTcEpiWarp0;
        const int q = warp & 3;
        const int row = 32 * q + lane;
        const uint32_t tlane = tbase + ((uint32_t)(32 * q) << 16);
        uint32_t uidx = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < n_units; u += gridDim.x, ++uidx) {
            const int ti = u / nrb, rb = u - ti * nrb;
            const int4 task = p.ws.tasks[ti];
            const int n = idx_in(hdr, task.z, 1, kTcNT + 1, 645), npad = tc_npad(n);
            const int bx = idx_in(hdr, task.x, 0, p.m.E + p.m.has_shared, 648);
            const uint32_t buf = uidx % NACC;
            named_sync(2, kTcEpi);  // the previous unit's metadata is no longer read
            if (etid < n) {
                const int a = idx_in(hdr, p.ws.asg[idx_in(hdr, task.y + etid, 0, p.a_cap, 646)], 0, p.a_cap, 647);
                ctl->asg[etid] = a;
                if (EPI == 0) {
                    const int tok = a / p.m.S;
                    ctl->sx[etid] = p.ws.sx[tok];
                    ctl->cs[etid] = p.ws.xcs[tok];
                } else {
                    ctl->sx[etid] = p.sh_in ? p.sh_in[a] : __ldcg(p.ws.sh + a);
                    ctl->cs[etid] = __ldcg(p.ws.hcs + a);
                }
            }
            named_sync(2, kTcEpi);
            if (ok) ok = tc_wait(&ctl->accfull[buf], (uidx / NACC) & 1u, hdr, 0x7109);
            ok = __all_sync(kFull, ok);
            tc_fence_after();
            const uint32_t dcol = tlane + 128 * buf;
            if (ok && EPI == 0) {
                const int r = rb * 128 + row;
                const bool rv = r < f;
                const float sg = rv ? __ldg(p.scales + (size_t)bx * p.scale_rows + r) : 0.0f;
                const float su = rv ? __ldg(p.scales + (size_t)bx * p.scale_rows + f + r) : 0.0f;
                for (int tg = 0; tg * 8 < npad; ++tg) {
                    int G[8], U[8];
                    tmem_ld8(dcol + tg * 8, G);
                    tmem_ld8(dcol + 64 + tg * 8, U);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int t = tg * 8 + j;
                        if (t >= n) break;
                        const int a = ctl->asg[t];
                        const float sx = ctl->sx[t];
                        const int gi = G[j] - OFF * ctl->cs[t];
                        const int ui = U[j] - OFF * ctl->cs[t];
                        const float gv = __fmul_rn((float)gi, __fmul_rn(sg, sx));
                        const float uv = __fmul_rn((float)ui, __fmul_rn(su, sx));
                        const float h = __fmul_rn(__fdiv_rn(gv, __fadd_rn(1.0f, expf(-gv))), uv);
                        if (rv) {
                            p.ws.h[(size_t)a * f + r] = h;
                            if (p.dbg_acc_gu) {
                                p.dbg_acc_gu[(size_t)a * 2 * f + r] = gi;
                                p.dbg_acc_gu[(size_t)a * 2 * f + f + r] = ui;
                            }
                        }
                        const unsigned m = __reduce_max_sync(kFull, rv ? __float_as_uint(fabsf(h)) : 0u);
                        if (lane == 0 && m != 0u) atomicMax(&p.ws.amax[a], m);
                    }
                }
            } else if (ok) {
                const int r0 = rb * 256 + row;
                const float* sd = p.scales + (size_t)bx * p.scale_rows + 2 * f;
                const float s0 = r0 < d ? __ldg(sd + r0) : 0.0f;
                const float s1 = r0 + 128 < d ? __ldg(sd + r0 + 128) : 0.0f;
                float* dst = p.direct_out ? p.out : p.ws.ybuf;
                for (int tg = 0; tg * 8 < npad; ++tg) {
                    int D0[8], D1[8];
                    tmem_ld8(dcol + tg * 8, D0);
                    tmem_ld8(dcol + 64 + tg * 8, D1);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int t = tg * 8 + j;
                        if (t >= n) break;
                        const int a = ctl->asg[t];
                        const float sh = ctl->sx[t];
                        const int d0 = D0[j] - OFF * ctl->cs[t];
                        const int d1 = D1[j] - OFF * ctl->cs[t];
                        if (r0 < d) {
                            dst[(size_t)a * d + r0] = __fmul_rn((float)d0, __fmul_rn(s0, sh));
                            if (p.dbg_acc_d) p.dbg_acc_d[(size_t)a * d + r0] = d0;
                        }
                        if (r0 + 128 < d) {
                            dst[(size_t)a * d + r0 + 128] = __fmul_rn((float)d1, __fmul_rn(s1, sh));
                            if (p.dbg_acc_d) p.dbg_acc_d[(size_t)a * d + r0 + 128] = d1;
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->accempty[buf]);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        tmem_dealloc(tbase, TCOLS);
    }
}

// The task whose padded rows hold row R (tasks are in row order, task.w
// ascending): a binary search over the tasks' first rows, in shared memory
// when the CTA has staged them (tw_s), else in global memory.  Staging turns
// the search's dependent global loads (several L2 round trips per row) into
// one coalesced load per CTA.
constexpr int kTcTaskCache = 2048;
__device__ __forceinline__ int tc_task_of_row(const Params& p, const int* tw_s, int n_tasks, int R) {
    int lo = 0, hi = n_tasks - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        const int w = tw_s ? tw_s[mid] : __ldg(&p.ws.tasks[mid].w);
        if (w <= R) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}
// Stages the tasks' first rows in shared memory if they fit (all threads of
// the CTA call it); returns the staged array or nullptr.
__device__ __forceinline__ const int* tc_stage_task_rows(const Params& p, int* tw_s, int n_tasks) {
    const bool cached = n_tasks <= kTcTaskCache;
    if (cached)
        for (int i = threadIdx.x; i < n_tasks; i += blockDim.x) tw_s[i] = __ldg(&p.ws.tasks[i].w);
    __syncthreads();
    return cached ? tw_s : nullptr;
}

// a4's input rule on the tensor-core path: requantise each assignment's h
// (max |h| from the gate/up epilogue) into the down operand B, in the MMA
// layout, with its scale and code sum; leaves the maxima zeroed.  One warp per
// padded row of the call, as in the gather.
template <int WB>
__global__ void __launch_bounds__(kThreads) k_tc_requant(const Params p) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int f = p.m.f;
    const int n_tasks = p.ws.hdr->n_tasks, rows = p.ws.hdr->tc_rows;
    const int kpad = tc_kpad(f, WB), npk = kpad / 16;
    __shared__ int tw_s[kTcTaskCache];
    const int* tw = tc_stage_task_rows(p, tw_s, n_tasks);
    for (int R = blockIdx.x * kWarps + warp; R < rows; R += gridDim.x * kWarps) {
        const int lo = tc_task_of_row(p, tw, n_tasks, R);
        const int4 task = __ldg(p.ws.tasks + lo);
        const int j = idx_in(p.ws.hdr, R - task.w, 0, kTcNT + 16, 651), npad = tc_npad(task.z);
        const bool live = j < task.z;
        const int a = live ? idx_in(p.ws.hdr, __ldg(p.ws.asg + idx_in(p.ws.hdr, task.y + j, 0, p.a_cap, 652)), 0,
                                    p.a_cap, 653)
                           : 0;
        const float m = live ? __uint_as_float(__ldcg(p.ws.amax + a)) : 0.0f;
        const float sh = m == 0.0f ? 0.0f : __fdiv_rn(m, 127.0f);
        const float rh = quant_recip(sh);
        const float* hrow = p.ws.h + (size_t)a * f;
        uint8_t* out = p.ws.hb + (size_t)task.w * kpad;
        int cs = 0;
#pragma unroll 2
        for (int kg = lane; kg < npk; kg += 32) {
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (m != 0.0f && kg * 16 < f) {
                const float4* hp = reinterpret_cast<const float4*>(hrow + kg * 16);
                uint32_t wv[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float4 hv = __ldcg(hp + i);
                    wv[i] = (uint32_t)(quant_code_r(hv.x, sh, rh) & 0xFF) |
                            ((uint32_t)(quant_code_r(hv.y, sh, rh) & 0xFF) << 8) |
                            ((uint32_t)(quant_code_r(hv.z, sh, rh) & 0xFF) << 16) |
                            ((uint32_t)(quant_code_r(hv.w, sh, rh) & 0xFF) << 24);
                }
                v = make_uint4(wv[0], wv[1], wv[2], wv[3]);
            }
            cs += sum16(v);
            if (live && p.dbg_hq && kg * 16 < f) *reinterpret_cast<uint4*>(p.dbg_hq + (size_t)a * f + kg * 16) = v;
            *reinterpret_cast<uint4*>(out + tc_b_offset(kg, j, npad)) = permute16<WB>(v);
        }
        cs = __reduce_add_sync(kFull, cs);
        if (live && lane == 0) {
            p.ws.sh[a] = sh;
            p.ws.hcs[a] = cs;
            if (p.dbg_sh) p.dbg_sh[a] = sh;
            p.ws.amax[a] = 0u;  // every lane has read it (the reduction above synchronised the warp)
        }
    }
}

// Build the operand B of every task from int8 rows (row key = assignment id /
// key_div of `src`, `ld` bytes apart): K columns [0, K) zero-padded to kpad,
// rows padded to tc_npad, in the MMA layout with permute16 byte order.  One
// warp per padded row of the call (hdr->tc_rows); a row finds its task by
// binary search over the tasks' first rows (task.w, ascending).
template <int WB>
__global__ void __launch_bounds__(kThreads) k_tc_gather(const Params p, const int8_t* __restrict__ src, int ld,
                                                        int key_div, int K, int kpad, uint8_t* __restrict__ dst) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_tasks = p.ws.hdr->n_tasks, rows = p.ws.hdr->tc_rows;
    const int npk = kpad / 16;
    __shared__ int tw_s[kTcTaskCache];
    const int* tw = tc_stage_task_rows(p, tw_s, n_tasks);
    for (int R = blockIdx.x * kWarps + warp; R < rows; R += gridDim.x * kWarps) {
        const int lo = tc_task_of_row(p, tw, n_tasks, R);
        const int4 task = __ldg(p.ws.tasks + lo);
        const int j = idx_in(p.ws.hdr, R - task.w, 0, kTcNT + 16, 654), npad = tc_npad(task.z);
        const int key = j < task.z ? idx_in(p.ws.hdr, __ldg(p.ws.asg + idx_in(p.ws.hdr, task.y + j, 0, p.a_cap, 655)),
                                            0, p.a_cap, 656) / key_div
                                   : -1;
        const int8_t* row = src + (size_t)(key < 0 ? 0 : key) * ld;
        uint8_t* out = dst + (size_t)task.w * kpad;
#pragma unroll 4
        for (int kg = lane; kg < npk; kg += 32) {
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (key >= 0 && kg * 16 < K) v = __ldcg(reinterpret_cast<const uint4*>(row + kg * 16));
            *reinterpret_cast<uint4*>(out + tc_b_offset(kg, j, npad)) = permute16<WB>(v);
        }
    }
}

// a6 over the whole grid: out[t] (+)= sum_j w_tj y_(t,j) + y_(t,shared),
// summed in slot order (the same order as the row-block combine of k_down).
__global__ void __launch_bounds__(kThreads) k_combine(const Params p) {
    const int d = p.m.d, S = p.m.S, k = p.m.k, T = p.m.T;
    const int nq = d / 4;
    for (size_t i = (size_t)blockIdx.x * kThreads + threadIdx.x; i < (size_t)T * nq; i += (size_t)gridDim.x * kThreads) {
        const int t = (int)(i / nq), c4 = (int)(i - (size_t)t * nq) * 4;
        float4 o = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        for (int j = 0; j < k; ++j) {
            if (__ldcg(p.ws.idx + (size_t)t * k + j) < 0) continue;  // dropped by the truncation: no output
            const float w = __ldcg(p.ws.w + (size_t)t * k + j);
            const float4 y = __ldcg(reinterpret_cast<const float4*>(p.ws.ybuf + ((size_t)t * S + j) * d + c4));
            o.x = fmaf(w, y.x, o.x);
            o.y = fmaf(w, y.y, o.y);
            o.z = fmaf(w, y.z, o.z);
            o.w = fmaf(w, y.w, o.w);
        }
        if (p.m.has_shared) {
            const float4 y = __ldcg(reinterpret_cast<const float4*>(p.ws.ybuf + ((size_t)t * S + k) * d + c4));
            o.x += y.x;
            o.y += y.y;
            o.z += y.z;
            o.w += y.w;
        }
        float4* dp = reinterpret_cast<float4*>(p.out + (size_t)t * d + c4);
        if (p.accumulate) {
            const float4 b = *dp;
            o.x += b.x;
            o.y += b.y;
            o.z += b.z;
            o.w += b.w;
        }
        *dp = o;
    }
}

}  // namespace moe
