// Instantiations, shared-memory plan and cooperative launch of the persistent
// decode kernel.
#include <algorithm>
#include <mutex>

#include "moe_decode.cuh"
#include "moe_launch.h"

namespace moe {

// Per-device facts the plan and the launch need, queried once per device.
struct DevFacts {
    int optin = 0, sms = 0;
};
static std::mutex g_dev_mu;
static DevFacts g_dev[64];
static bool dev_facts(DevFacts* out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DevFacts& f = g_dev[dev];
    if (f.sms == 0) {
        if (cudaDeviceGetAttribute(&f.optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&f.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            f = DevFacts{};
            return false;
        }
    }
    *out = f;
    return true;
}

// Tokens the kernel instance for T tokens is compiled for (its shared control
// block is sized for them).
static size_t ctl_bytes(int T) {
    if (T <= 1) return sizeof(DecCtl<1>);
    if (T <= 2) return sizeof(DecCtl<2>);
    if (T <= 4) return sizeof(DecCtl<4>);
    return sizeof(DecCtl<8>);
}

bool decode_plan(const Dims& m, DecPlan* pl) {
    if (m.T < 1 || m.T > kDecMaxT || m.k > kDecMaxK) return false;
    DevFacts df;
    if (!dev_facts(&df)) return false;
    const int optin = df.optin;
    const int rb_gu = m.d * m.wb / 8, rb_dn = m.f * m.wb / 8;
    if (m.d > 16 * kDecCons) return false;  // the quantiser holds one 16-value piece per consumer thread
    int wbytes = std::max(2 * kDecWarps * rb_gu, kDecWarps * rb_dn);
    wbytes = std::max(wbytes, m.d * 4);
    wbytes = (int)align_up((size_t)wbytes, 128);
    DecPlan q{};
    q.wbytes = wbytes;
    q.rr = std::min(2, wbytes / (m.d * 4));
    q.rd = (wbytes / rb_dn) / kDecWarps * kDecWarps;
    // row scales of a unit follow its weights: 2 x 8 (gate/up) or rd (down) floats
    const int slot = (int)align_up((size_t)wbytes + 4 * std::max(2 * kDecWarps, q.rd), 128);
    q.slot_bytes = slot;
    q.nu_gu = (m.f + kDecWarps - 1) / kDecWarps;
    q.nu_dn = (m.d + q.rd - 1) / q.rd;
    const int ctl = (int)align_up(ctl_bytes(m.T), 128);
    const int xs = (int)align_up((size_t)m.T * m.d, 128);
    q.hs_grp_bytes = (int)align_up((size_t)m.T * m.f, 128);
    // single-token down by output-row ranges: every CTA's rows (whole quads)
    // of one task fit a unit with f bytes to spare (the set of shapes this
    // path has been measured and tested on), and the consumers stage every
    // task's codes at once
    const int sms = df.sms;
    const int rr_rows_max = sms > 0 ? (m.d / 4 + sms - 1) / sms * 4 : 1 << 30;
    const bool rr_shape = m.T == 1 && m.k + m.has_shared <= kDecRRMaxTasks && m.d % 4 == 0 && m.f % 16 == 0 &&
                          m.S * (m.f / 16) <= kDecRRChunks * kDecCons && q.rd == kDecNQ * kDecWarps &&
                          rr_rows_max <= kDecRRMaxRows && rr_rows_max * rb_dn <= wbytes - m.f;
    // h staging of both consumer groups (the same bytes serve the top-k
    // scratch); on the row-range path the codes of every task, then the
    // per-row outputs of every assignment
    const size_t hs_base = std::max((size_t)kDecGroups * q.hs_grp_bytes, (size_t)8 * m.T * m.E);
    const size_t hs_rr = std::max(hs_base, (size_t)m.S * m.f + (size_t)m.S * kDecNQ * kDecWarps * 4);
    // an even slot count: the two consumer groups take alternate units, so
    // each group then owns the slots of its parity and waits on consecutive
    // phases of each (an odd count would let a group reach a slot two rounds
    // ahead, where a parity wait cannot tell the phases apart)
    auto slots_for = [&](size_t hs) {
        const int room = optin - ctl - xs - (int)align_up(hs, 128) - 1024;  // keep 1 KB for static shared memory
        return std::min(kDecMaxSlots, room / slot) / 2 * 2;
    };
    // the row-range path only where it keeps the full ring
    q.rowrange = rr_shape && slots_for(hs_rr) == kDecMaxSlots;
    const int hs = (int)align_up(q.rowrange ? hs_rr : hs_base, 128);
    q.nslot = slots_for((size_t)hs);
    if (q.nslot < 2) return false;
    q.dn_rot = 1;
    q.gu_rmaj = 1;
    q.xs_off = ctl;
    q.hs_off = ctl + xs;
    q.ring_off = ctl + xs + hs;
    q.smem_bytes = q.ring_off + q.nslot * slot;
    *pl = q;
    return true;
}

template <int WB, int TM, int NG, int ND, typename XT>
static cudaError_t go(const Params& p, const DecPlan& pl, const void* x, cudaStream_t s) {
    auto fn = k_decode<WB, TM, NG, ND, XT>;
    cudaError_t e = allow_smem((const void*)fn, pl.smem_bytes);
    if (e != cudaSuccess) return e;
    DevFacts df;
    if (!dev_facts(&df)) return cudaErrorInvalidDevice;
    const int sms = df.sms;
    // one CTA per SM must fit (checked once per kernel, device and size: the
    // occupancy query costs microseconds of host time per call)
    if (blocks_per_sm((const void*)fn, pl.smem_bytes, kDecThreads) < 1) return cudaErrorCooperativeLaunchTooLarge;
    const XT* xp = static_cast<const XT*>(x);
    void* args[] = {(void*)&p, (void*)&pl, (void*)&xp};
    return cudaLaunchCooperativeKernel((const void*)fn, dim3(sms), dim3(kDecThreads), args, pl.smem_bytes, s);
}

template <int WB, int NG, int ND, typename XT>
static cudaError_t by_t(const Params& p, const DecPlan& pl, const void* x, cudaStream_t s) {
    const int T = p.m.T;
    if (T <= 1) return go<WB, 1, NG, ND, XT>(p, pl, x, s);
    if (T <= 2) return go<WB, 2, NG, ND, XT>(p, pl, x, s);
    if (T <= 4) return go<WB, 4, NG, ND, XT>(p, pl, x, s);
    return go<WB, 8, NG, ND, XT>(p, pl, x, s);
}

// Fully unrolled rows for the GLM-5.2 expert shape (d = 6144, f = 2048):
// 6 (int4) or 3 (int2) 16-byte chunks per lane of a gate/up row, 2 or 1 of a
// down row; any other shape (and int8 experts) takes the runtime loop.
template <int WB, typename XT>
static cudaError_t by_shape(const Params& p, const DecPlan& pl, const void* x, cudaStream_t s) {
    const int nch_gu = p.m.d * WB / 8 / 16, nch_dn = p.m.f * WB / 8 / 16;
    if constexpr (WB == 8) return by_t<WB, 0, 0, XT>(p, pl, x, s);
    constexpr int NG = WB == 4 ? 6 : 3, ND = WB == 4 ? 2 : 1;
    if (nch_gu == 32 * NG && nch_dn == 32 * ND && pl.rd == kDecNQ * kDecWarps) return by_t<WB, NG, ND, XT>(p, pl, x, s);
    return by_t<WB, 0, 0, XT>(p, pl, x, s);
}

cudaError_t launch_decode(const Params& p, const DecPlan& pl, const void* x, bool bf16, cudaStream_t s) {
    if (p.m.wb == 8)
        return bf16 ? by_shape<8, __nv_bfloat16>(p, pl, x, s) : by_shape<8, float>(p, pl, x, s);
    if (p.m.wb == 4)
        return bf16 ? by_shape<4, __nv_bfloat16>(p, pl, x, s) : by_shape<4, float>(p, pl, x, s);
    return bf16 ? by_shape<2, __nv_bfloat16>(p, pl, x, s) : by_shape<2, float>(p, pl, x, s);
}

}  // namespace moe
