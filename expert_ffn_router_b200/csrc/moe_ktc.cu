// Host side of the tensor-core expert path: tensor maps over the expert pool,
// shared-memory plan, and the launches of the gather, gate/up, down and
// combine kernels (moe_tc.cuh).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>
#include <set>
#include <utility>

#include "moe_launch.h"
#include "moe_tc.cuh"

namespace moe {

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// 2-D uint8 view of the pool: `rows` rows of `rowbytes` bytes; box of
// tc_box_w(wb, stage) bytes x 128 rows with the swizzle of that width (64 or
// 128 bytes), zero fill outside the tensor.
static cudaError_t make_pool_map(CUtensorMap* tm, const void* pool, uint64_t rowbytes, uint64_t rows, int wb,
                                 int stage) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {rowbytes, rows};
    const cuuint64_t strides[1] = {rowbytes};
    const int bw = tc_box_w(wb, stage);
    const cuuint32_t box[2] = {(cuuint32_t)bw, 128};
    const cuuint32_t estr[2] = {1, 1};
    const CUtensorMapSwizzle sw = bw == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
    const CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(pool), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Shared memory of one CTA when `cps` CTAs share an SM (228 KB per SM, 1 KB
// of it reserved per CTA), and the slot count that fills it.  Each CTA also
// takes at least kTcSmemFloor[cps - 1], so that no more than `cps` CTAs fit
// on an SM: their TMEM allocations (512 / cps columns) then always fit too.
constexpr size_t kTcSmemBudget[2] = {227 * 1024, 113 * 1024};
constexpr size_t kTcSmemFloor[2] = {120 * 1024, 78 * 1024};

static int tc_slots(int nt_max, int wb, int cps, int epi) {
    const size_t room = kTcSmemBudget[cps - 1] - 1024 - sizeof(TcCtl);
    return (int)std::min<size_t>(kTcMaxSlots, room / tc_slot_bytes(nt_max, wb, epi));
}

// CTAs per SM of the launches (k_tc's CPS).
constexpr int kTcCps = 2;

bool tc_shape_ok(const Dims& m) {
    // every assignment's token count fits the task split, and the slot ring
    // holds at least two chunks
    return tc_slots(kTcNT, m.wb, kTcCps, 0) >= 2 && tc_slots(kTcNT, m.wb, kTcCps, 1) >= 2 && m.d <= 8192 &&
           m.f <= 8192;
}

// Two CTAs per SM need the SM's whole shared memory as such (the carveout the
// driver picks by default may leave room for one); set once per kernel and
// device.  Without it the launch stays correct: the kernel's CTAs never wait
// on one another, so CTAs that do not fit run after the first ones exit.
static cudaError_t prefer_shared(const void* fn) {
    static std::mutex mu;
    static std::set<std::pair<int, const void*>> done;
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lk(mu);
    if (done.count({dev, fn})) return cudaSuccess;
    const cudaError_t e =
        cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e == cudaSuccess) done.insert({dev, fn});
    return e;
}

template <int WB, int EPI, int CPS>
static cudaError_t launch_tc_t(const Params& p, const CUtensorMap& tm, int nt_max, cudaStream_t s) {
    const int ns = tc_slots(nt_max, WB, CPS, EPI);
    const size_t smem = std::max(tc_smem_bytes(ns, nt_max, WB, EPI), kTcSmemFloor[CPS - 1]);
    auto fn = k_tc<WB, EPI, CPS>;
    cudaError_t e = allow_smem((const void*)fn, smem);
    if (e == cudaSuccess && CPS > 1) e = prefer_shared((const void*)fn);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    fn<<<CPS * sms, kTcThreads, smem, s>>>(p, tm, ns, nt_max);
    return cudaGetLastError();
}

cudaError_t launch_tc_expert(const Params& p, int stage, int nt_max, cudaStream_t s) {
    const int E1 = p.slot_of ? p.n_slots : p.m.E + p.m.has_shared;  // blobs the pool holds
    CUtensorMap tm;
    const int wb = p.m.wb;
    cudaError_t e;
    if (stage == 0)
        e = make_pool_map(&tm, p.pool, (uint64_t)p.m.d * wb / 8, (uint64_t)3 * p.m.f * E1, wb, 0);
    else
        e = make_pool_map(&tm, p.pool, (uint64_t)p.m.f * wb / 8, (uint64_t)3 * p.m.d * E1, wb, 1);
    if (e != cudaSuccess) return e;
    constexpr int C = kTcCps;
    if (wb == 8) return stage == 0 ? launch_tc_t<8, 0, C>(p, tm, nt_max, s) : launch_tc_t<8, 1, C>(p, tm, nt_max, s);
    if (wb == 4) return stage == 0 ? launch_tc_t<4, 0, C>(p, tm, nt_max, s) : launch_tc_t<4, 1, C>(p, tm, nt_max, s);
    return stage == 0 ? launch_tc_t<2, 0, C>(p, tm, nt_max, s) : launch_tc_t<2, 1, C>(p, tm, nt_max, s);
}

cudaError_t launch_tc_requant(const Params& p, cudaStream_t s) {
    const int grid = (int)std::min<size_t>((tc_rows_bound(p.m) + kWarps - 1) / kWarps,
                                           (size_t)persistent_grid((const void*)k_tc_requant<4>, 0));
    if (p.m.wb == 8) k_tc_requant<8><<<grid, kThreads, 0, s>>>(p);
    else if (p.m.wb == 4) k_tc_requant<4><<<grid, kThreads, 0, s>>>(p);
    else k_tc_requant<2><<<grid, kThreads, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_tc_gather(const Params& p, const int8_t* src, int ld, int key_div, int K, uint8_t* dst,
                             cudaStream_t s) {
    const int kpad = tc_kpad(K, p.m.wb);
    // one warp per padded row; the row count is known on the device only
    const int grid = (int)std::min<size_t>((tc_rows_bound(p.m) + kWarps - 1) / kWarps,
                                           (size_t)persistent_grid((const void*)k_tc_gather<4>, 0));
    if (p.m.wb == 8) k_tc_gather<8><<<grid, kThreads, 0, s>>>(p, src, ld, key_div, K, kpad, dst);
    else if (p.m.wb == 4) k_tc_gather<4><<<grid, kThreads, 0, s>>>(p, src, ld, key_div, K, kpad, dst);
    else k_tc_gather<2><<<grid, kThreads, 0, s>>>(p, src, ld, key_div, K, kpad, dst);
    return cudaGetLastError();
}

cudaError_t launch_combine(const Params& p, cudaStream_t s) {
    const size_t n4 = (size_t)p.m.T * (p.m.d / 4);
    const int grid = (int)std::max<size_t>(1, std::min<size_t>((n4 + kThreads - 1) / kThreads,
                                                               (size_t)persistent_grid((const void*)k_combine, 0)));
    k_combine<<<grid, kThreads, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace moe
