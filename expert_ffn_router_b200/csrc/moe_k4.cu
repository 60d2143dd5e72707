// Instantiations and launcher of the down + combine kernel.
#include "moe_expert.cuh"
#include "moe_launch.h"

namespace moe {

template <int WB, int CH, int NCL, bool DBG>
static cudaError_t go4(const Params& p, cudaStream_t s) {
    constexpr int RPW = rpw4(NCL);
    auto fn = k_down<WB, CH, NCL, RPW, DBG>;
    const size_t smem = (size_t)CH * p.m.f;
    cudaError_t e = allow_smem((const void*)fn, smem);
    if (e != cudaSuccess) return e;
    fn<<<persistent_grid((const void*)fn, smem), kThreads, smem, s>>>(p);
    return cudaGetLastError();
}

template <int WB, int CH, bool DBG>
static cudaError_t by_ncl(const Params& p, int ncl, cudaStream_t s) {
    switch (ncl) {
        case 1: return go4<WB, CH, 1, DBG>(p, s);
        case 2: return go4<WB, CH, 2, DBG>(p, s);
        case 4: return go4<WB, CH, 4, DBG>(p, s);
        case 8: return go4<WB, CH, 8, DBG>(p, s);
        case 12:  // rows of 6 KB and 8 KB: int8 experts only
            if constexpr (WB == 8) return go4<WB, CH, 12, DBG>(p, s);
            return cudaErrorInvalidValue;
        case 16:
            if constexpr (WB == 8) return go4<WB, CH, 16, DBG>(p, s);
            return cudaErrorInvalidValue;
        default: return cudaErrorInvalidValue;
    }
}

template <int WB>
static cudaError_t by_ch(const Params& p, int ncl, bool dbg, cudaStream_t s) {
    if (dbg) return by_ncl<WB, 8, true>(p, ncl, s);
    switch (p.CH) {
        case 1: return by_ncl<WB, 1, false>(p, ncl, s);
        case 2: return by_ncl<WB, 2, false>(p, ncl, s);
        case 4: return by_ncl<WB, 4, false>(p, ncl, s);
        case 8: return by_ncl<WB, 8, false>(p, ncl, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_down(const Params& p, const ExpertTiling& tl, bool dbg, cudaStream_t s) {
    if (p.m.wb == 8) return by_ch<8>(p, tl.ncl4, dbg, s);
    return p.m.wb == 4 ? by_ch<4>(p, tl.ncl4, dbg, s) : by_ch<2>(p, tl.ncl4, dbg, s);
}

}  // namespace moe
