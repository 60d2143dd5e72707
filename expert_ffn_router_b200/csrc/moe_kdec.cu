// Instantiations, shared-memory plan and cooperative launch of the persistent
// decode kernel.
#include <algorithm>

#include "moe_decode.cuh"
#include "moe_launch.h"

namespace moe {

bool decode_plan(const Dims& m, DecPlan* pl) {
    if (m.T < 1 || m.T > kDecMaxT || m.k > kDecMaxK) return false;
    int dev = 0, optin = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) return false;
    const int rb_gu = m.d * m.wb / 8, rb_dn = m.f * m.wb / 8;
    int slot = std::max(2 * kDecWarps * rb_gu, kDecWarps * rb_dn);
    slot = std::max(slot, m.d * 4);
    slot = (int)align_up((size_t)slot, 128);
    DecPlan q{};
    q.slot_bytes = slot;
    q.rr = std::min(2, slot / (m.d * 4));
    q.rd = (slot / rb_dn) / kDecWarps * kDecWarps;
    q.nu_gu = (m.f + kDecWarps - 1) / kDecWarps;
    q.nu_dn = (m.d + q.rd - 1) / q.rd;
    const int ctl = (int)align_up(sizeof(DecCtl), 128);
    const int xs = (int)align_up((size_t)m.T * m.d, 128);
    const int hs = (int)align_up(std::max((size_t)m.T * m.f, (size_t)8 * m.T * m.E), 128);
    const int room = optin - ctl - xs - hs - 1024;  // keep 1 KB for static shared memory
    q.nslot = std::min(kDecMaxSlots, room / slot);
    if (q.nslot < 2) return false;
    q.xs_off = ctl;
    q.hs_off = ctl + xs;
    q.ring_off = ctl + xs + hs;
    q.smem_bytes = q.ring_off + q.nslot * slot;
    *pl = q;
    return true;
}

template <int WB, int TM, typename XT>
static cudaError_t go(const Params& p, const DecPlan& pl, const void* x, cudaStream_t s) {
    auto fn = k_decode<WB, TM, XT>;
    cudaError_t e = allow_smem((const void*)fn, pl.smem_bytes);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0, per_sm = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kDecThreads, pl.smem_bytes);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) return cudaErrorCooperativeLaunchTooLarge;
    const XT* xp = static_cast<const XT*>(x);
    void* args[] = {(void*)&p, (void*)&pl, (void*)&xp};
    return cudaLaunchCooperativeKernel((const void*)fn, dim3(sms), dim3(kDecThreads), args, pl.smem_bytes, s);
}

template <int WB, typename XT>
static cudaError_t by_t(const Params& p, const DecPlan& pl, const void* x, cudaStream_t s) {
    const int T = p.m.T;
    if (T <= 1) return go<WB, 1, XT>(p, pl, x, s);
    if (T <= 2) return go<WB, 2, XT>(p, pl, x, s);
    if (T <= 4) return go<WB, 4, XT>(p, pl, x, s);
    return go<WB, 8, XT>(p, pl, x, s);
}

cudaError_t launch_decode(const Params& p, const DecPlan& pl, const void* x, bool bf16, cudaStream_t s) {
    if (p.m.wb == 4)
        return bf16 ? by_t<4, __nv_bfloat16>(p, pl, x, s) : by_t<4, float>(p, pl, x, s);
    return bf16 ? by_t<2, __nv_bfloat16>(p, pl, x, s) : by_t<2, float>(p, pl, x, s);
}

}  // namespace moe
