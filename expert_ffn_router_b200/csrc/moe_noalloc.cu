// moe_route_static: the router of moe_route for up to kStaticMaxT tokens,
// with its scratch memory in a file-scope device array instead of a
// caller-provided workspace.
//
// Some callers cannot hand the library a workspace: a host framework that owns
// all device memory and forbids allocations after start-up, a serving loop
// that must not pay cudaMalloc's implicit device synchronisation, or a plugin
// interface with no way to request scratch space.  This entry point needs only
// the inputs and outputs.  Its scratch lives in g_route_scratch below, which
// every GPU that loads the library holds until the process exits.
#include <cuda_runtime.h>

#include <string>

#include "moe.h"
#include "moe_launch.h"

namespace moe {

constexpr int kStaticMaxT = 8;              // tokens per call
constexpr int kStaticMaxE = 1024;           // routed experts
constexpr int kStaticMaxK = 32;             // experts per token
constexpr size_t kStaticScratchBytes = 64 * 1024;

// Control word + logits [T][E] + top-k copies [T][k] (indices and weights).
static_assert(sizeof(WsHeader) + (size_t)kStaticMaxT * kStaticMaxE * 4 + 2 * (size_t)kStaticMaxT * kStaticMaxK * 4 <=
                  kStaticScratchBytes,
              "static router scratch too small");

static __device__ __align__(256) unsigned char g_route_scratch[kStaticScratchBytes];

// Device address of g_route_scratch on the current device.  In host code the
// array's name stands for a host-side shadow, never for the device memory
// itself, so the address is looked up with the device current.  The lookup is
// repeated on every call (it costs well under a microsecond of host time): an
// address kept from an earlier call would be stale after the caller resets the
// device, which unloads and reloads the library's module.
static moe_status scratch_for_current_device(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(MOE_ECUDA, std::string("moe_route_static: cudaGetDevice: ") + cudaGetErrorString(e));
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_route_scratch);
    if (e != cudaSuccess || !ptr)
        return fail(MOE_ECUDA, std::string("moe_route_static: cudaGetSymbolAddress: ") + cudaGetErrorString(e));
    *out = ptr;
    return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" moe_status moe_route_static(const moe_config* cfg, const void* x, moe_dtype dtype, int32_t T,
                                       const float* w_router, const float* bias, int32_t* topk_idx, float* topk_w,
                                       moe_stream_t stream) {
    moe_status st = check_cfg(cfg);
    if (st != MOE_OK) return st;
    if ((st = check_dtype(dtype)) != MOE_OK) return st;
    if (T < 0) return fail(MOE_EINVAL, "moe_route_static: T < 0");
    if (T > kStaticMaxT)
        return fail(MOE_EINVAL, "moe_route_static: T = " + std::to_string(T) + " exceeds its limit of " +
                                    std::to_string(kStaticMaxT) + " tokens per call");
    if (cfg->n_experts > kStaticMaxE || cfg->top_k > kStaticMaxK)
        return fail(MOE_EINVAL, "moe_route_static: more than 1024 experts or 32 per token");
    if (T == 0) return MOE_OK;
    if ((st = check_ptr(x, "x")) != MOE_OK) return st;
    if ((st = check_ptr(w_router, "w_router")) != MOE_OK) return st;
    if ((st = check_ptr(bias, "bias")) != MOE_OK) return st;
    if ((st = check_ptr(topk_idx, "topk_idx")) != MOE_OK) return st;
    if ((st = check_ptr(topk_w, "topk_w")) != MOE_OK) return st;
    void* base = nullptr;
    if ((st = scratch_for_current_device(&base)) != MOE_OK) return st;

    Params p{};
    p.m = Dims{cfg->d, cfg->f, cfg->n_experts, cfg->top_k, cfg->has_shared, cfg->wbits, T,
               cfg->top_k + cfg->has_shared};
    p.routed_scale = cfg->routed_scale;
    p.topp = cfg->topp;
    p.ksplit = 1;
    char* b = static_cast<char*>(base);
    p.ws.hdr = reinterpret_cast<WsHeader*>(b);
    p.ws.logits = reinterpret_cast<float*>(b + sizeof(WsHeader));
    p.ws.idx = reinterpret_cast<int32_t*>(b + sizeof(WsHeader) + (size_t)T * cfg->n_experts * 4);
    p.ws.w = reinterpret_cast<float*>(reinterpret_cast<char*>(p.ws.idx) + (size_t)T * cfg->top_k * 4);
    p.w_router = w_router;
    p.bias = bias;
    p.idx_out = topk_idx;
    p.w_out = topk_w;
    cudaStream_t s = (cudaStream_t)stream;
    // The array keeps whatever the last call left; its control word (the
    // router CTAs' arrival counter) must start at zero.
    cudaError_t e = cudaMemsetAsync(base, 0, sizeof(WsHeader), s);
    if (e == cudaSuccess) e = launch_router_any(p, x, dtype, 0, 0, s);
    if (e != cudaSuccess) return fail(MOE_ECUDA, std::string("moe_route_static: ") + cudaGetErrorString(e));
    return MOE_OK;
}
