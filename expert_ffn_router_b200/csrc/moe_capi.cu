// The C ABI of libmoe: argument validation, workspace carving and the launch
// sequence of each entry point.  Every step of the layer runs in this
// library's kernels; the host only checks arguments and enqueues launches.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <mutex>
#include <string>
#include <unordered_map>

#include "moe.h"
#include "moe_launch.h"
#include "moe_decode.cuh"
#include "moe_route.cuh"

namespace moe {

static thread_local std::string g_last_error;

moe_status fail(moe_status st, const std::string& msg) {
    g_last_error = msg;
    return st;
}

static moe_status cuda_fail(cudaError_t e, const char* where) {
    return fail(MOE_ECUDA, std::string(where) + ": " + cudaGetErrorString(e));
}

// ---------------------------------------------------------------------------
// cached device facts
// ---------------------------------------------------------------------------
static std::mutex g_mu;
static std::unordered_map<unsigned long long, int> g_grid;  // (device, func, smem) -> grid
static std::unordered_map<unsigned long long, size_t> g_smem;

static unsigned long long cache_key(int dev, const void* func, size_t smem) {
    return ((unsigned long long)(uintptr_t)func * 1000003ull) ^ ((unsigned long long)smem << 20) ^
           (unsigned long long)dev;
}

// Resident CTAs per SM of a kernel for a block size and dynamic shared memory
// (cached: the occupancy query costs microseconds of host time).
int blocks_per_sm(const void* func, size_t smem, int threads) {
    int dev = 0;
    cudaGetDevice(&dev);
    const unsigned long long key = cache_key(dev, func, smem) ^ ((unsigned long long)threads << 48);
    {
        std::lock_guard<std::mutex> lk(g_mu);
        auto it = g_grid.find(key);
        if (it != g_grid.end()) return it->second;
    }
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, func, threads, smem) != cudaSuccess) per_sm = 0;
    std::lock_guard<std::mutex> lk(g_mu);
    g_grid[key] = per_sm;
    return per_sm;
}

int persistent_grid(const void* func, size_t smem, int threads) {
    int dev = 0, sms = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return std::max(1, sms * std::max(1, blocks_per_sm(func, smem, threads)));
}

cudaError_t allow_smem(const void* func, size_t smem) {
    // dynamic + static shared memory above 48 KB needs the opt-in; static
    // usage of these kernels is a few hundred bytes
    if (smem + 4096 <= 48 * 1024) return cudaSuccess;
    int dev = 0;
    cudaGetDevice(&dev);
    const unsigned long long key = cache_key(dev, func, 0);
    {
        std::lock_guard<std::mutex> lk(g_mu);
        auto it = g_smem.find(key);
        if (it != g_smem.end() && it->second >= smem) return cudaSuccess;
    }
    cudaError_t e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) {
        std::lock_guard<std::mutex> lk(g_mu);
        g_smem[key] = smem;
    }
    return e;
}

static int round_ncl(int ncl, bool down) {
    if (ncl <= 1) return 1;
    if (ncl <= 2) return 2;
    if (ncl <= 4) return 4;
    if (!down && ncl <= 6) return 6;
    if (ncl <= 8) return 8;
    if (ncl <= 12) return 12;  // rows above 4 KB: int8 experts only
    return 16;
}

ExpertTiling expert_tiling(int d, int f, int wb) {
    ExpertTiling t{};
    const int nch3 = d * wb / 8 / 16, nch4 = f * wb / 8 / 16;
    t.ncl3 = round_ncl((nch3 + 31) / 32, false);
    t.rpw3 = rpw3();
    t.ncl4 = round_ncl((nch4 + 31) / 32, true);
    t.rpw4 = rpw4(t.ncl4);
    return t;
}

// ---------------------------------------------------------------------------
// validation
// ---------------------------------------------------------------------------
static bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

moe_status check_cfg(const moe_config* c) {
    if (!c) return fail(MOE_EINVAL, "cfg is NULL");
    if (c->d <= 0 || c->f <= 0 || c->d > 8192 || c->f > 8192)
        return fail(MOE_EINVAL, "d and f must be in [1, 8192]");
    if (c->wbits != 4 && c->wbits != 2 && c->wbits != 8) return fail(MOE_EINVAL, "wbits must be 4, 2 or 8");
    if ((c->d * c->wbits / 8) % 16 || (c->f * c->wbits / 8) % 16 || (c->d * c->wbits) % 8 || (c->f * c->wbits) % 8)
        return fail(MOE_EINVAL, "d*wbits/8 and f*wbits/8 must be multiples of 16 bytes");
    if (c->n_experts < 1 || c->n_experts > 1024) return fail(MOE_EINVAL, "n_experts must be in [1, 1024]");
    if (c->top_k < 1 || c->top_k > 32 || c->top_k > c->n_experts)
        return fail(MOE_EINVAL, "top_k must be in [1, min(n_experts, 32)]");
    if (c->has_shared != 0 && c->has_shared != 1) return fail(MOE_EINVAL, "has_shared must be 0 or 1");
    if (!(c->routed_scale == c->routed_scale)) return fail(MOE_EINVAL, "routed_scale is NaN");
    if (!(c->topp >= 0.0f && c->topp <= 1.0f)) return fail(MOE_EINVAL, "topp must be in [0, 1]");
    return MOE_OK;
}

// A cached pool (slot_of set) holds n_slots >= 1 blobs; its table is device memory.
static moe_status check_pool_slots(const moe_pool* pool) {
    if (!pool->slot_of) return MOE_OK;
    if (pool->n_slots < 1) return fail(MOE_EINVAL, "pool->n_slots must be >= 1 when pool->slot_of is set");
    if (reinterpret_cast<uintptr_t>(pool->slot_of) % 4) return fail(MOE_EALIGN, "pool->slot_of is not 4-byte aligned");
    return MOE_OK;
}

moe_status check_ptr(const void* p, const char* name, bool nullable) {
    if (!p) return nullable ? MOE_OK : fail(MOE_EINVAL, std::string(name) + " is NULL");
    if (!aligned16(p)) return fail(MOE_EALIGN, std::string(name) + " is not 16-byte aligned");
    return MOE_OK;
}

#define MOE_TRY(expr)                       \
    do {                                    \
        moe_status _st = (expr);            \
        if (_st != MOE_OK) return _st;      \
    } while (0)

static Dims dims_of(const moe_config* c, int T, int S) {
    return Dims{c->d, c->f, c->n_experts, c->top_k, c->has_shared, c->wbits, T, S};
}

static int pick_ch(int T) { return T <= 1 ? 1 : T <= 2 ? 2 : T <= 4 ? 4 : 8; }

static Dims layout_dims(const moe_config* c, size_t ws_bytes);

// Default of moe_config.tc_min_tokens: calls with at least this many tokens
// run the experts on the tensor-core path.  Measured on B200 at the GLM-5.2
// expert shape (one layer, 256 experts, top-8, int4; us per call, decode
// kernel vs tensor-core path): T = 1: 68 vs 136, T = 2: 137 vs 168, T = 3:
// 222 vs 214, T = 4: 301 vs 251, T = 8: 878 vs 364 -- the decode kernel's ring
// holds only two slots from three tokens on, while the tensor-core path keeps
// its weight tiles flowing.
constexpr int kTcDefaultMinTokens = 3;

static bool use_tc(const moe_config* c, int T) {
    const int thr = c->tc_min_tokens == 0 ? kTcDefaultMinTokens : c->tc_min_tokens;
    return thr > 0 && T >= thr && tc_shape_ok(dims_of(c, T, c->top_k + c->has_shared));
}

// Bound on the tokens of one tensor-core task in a call of T tokens.
static int tc_nt_max(int T) { return tc_npad(std::min(T, kTcNT)); }

static Params base_params(const moe_config* c, const Dims& m, void* ws, size_t ws_bytes, bool tc = false) {
    Params p{};
    p.m = m;
    p.wait_ns = kWaitLimitNs;
    p.skip_h_task = -1;
    p.routed_scale = c->routed_scale;
    p.topp = c->topp;
    p.blob_bytes = 3ll * c->d * c->f * c->wbits / 8;
    p.scale_rows = 2 * c->f + c->d;
    p.CH = pick_ch(m.T);
    const ExpertTiling tl = expert_tiling(c->d, c->f, c->wbits);
    p.rb3 = kWarps * tl.rpw3;
    p.nrb3 = (c->f + p.rb3 - 1) / p.rb3;
    p.rb4 = kWarps * tl.rpw4;
    p.nrb4 = (c->d + p.rb4 - 1) / p.rb4;
    if (tc) {  // tasks of up to kTcNT tokens; units of 128 gate/up rows, 256 down rows
        p.tc = 1;
        p.CH = kTcNT;
        p.rb3 = 128;
        p.nrb3 = (c->f + 127) / 128;
        p.rb4 = 256;
        p.nrb4 = (c->d + 255) / 256;
    }
    p.ksplit = 1;
    const Dims l = layout_dims(c, ws_bytes);
    p.ws = ws_carve(l, ws);
    p.a_cap = l.T * l.S;
    return p;
}

// The workspace layout: that of its capacity, independent of the call's T.
static Dims layout_dims(const moe_config* c, size_t ws_bytes) {
    Dims l = dims_of(c, 1, c->top_k + c->has_shared);
    l.T = std::max(1, ws_capacity(l, ws_bytes));
    return l;
}

static moe_status check_ws(const moe_config* c, int T, void* ws, size_t ws_bytes) {
    MOE_TRY(check_ptr(ws, "ws"));
    Dims l = dims_of(c, std::max(1, T), c->top_k + c->has_shared);
    const size_t need = ws_carve(l, nullptr).bytes;
    if (ws_bytes < need)
        return fail(MOE_ENOSPACE, "workspace has " + std::to_string(ws_bytes) + " bytes, needs " + std::to_string(need));
    return MOE_OK;
}

// ---------------------------------------------------------------------------
// router launch sequence (a0 + a1 (+ a2))
// ---------------------------------------------------------------------------
template <int TM, typename XT>
static cudaError_t route_small_nv(Params& p, const XT* x, int do_quant, int bucket, cudaStream_t s) {
    const int E = p.m.E;
    const size_t smem = std::max((size_t)2 * kWarps * E * 4, (size_t)bucket_smem_ints(E) * 4);
    const int nv = p.m.d / 4;
    const int per = (nv + kThreads - 1) / kThreads;
    const int grid = (E + 1) / 2;
#define MOE_RS(NV)                                                                   \
    {                                                                                \
        auto fn = k_route_small<TM, NV, XT>;                                         \
        cudaError_t e = allow_smem((const void*)fn, smem);                           \
        if (e != cudaSuccess) return e;                                              \
        fn<<<grid, kThreads, smem, s>>>(p, x, do_quant, bucket);                     \
        return cudaGetLastError();                                                   \
    }
    if (per <= 2) MOE_RS(2)
    if (per <= 6) MOE_RS(6)
    MOE_RS(8)
#undef MOE_RS
}

template <typename XT>
static cudaError_t launch_router(Params& p, const XT* x, int do_quant, int bucket, cudaStream_t s) {
    const int T = p.m.T, E = p.m.E, d = p.m.d;
    if (T <= 8) {
        p.ksplit = 1;
        switch (T <= 1 ? 1 : T <= 2 ? 2 : T <= 4 ? 4 : 8) {
            case 1: return route_small_nv<1>(p, x, do_quant, bucket, s);
            case 2: return route_small_nv<2>(p, x, do_quant, bucket, s);
            case 4: return route_small_nv<4>(p, x, do_quant, bucket, s);
            default: return route_small_nv<8>(p, x, do_quant, bucket, s);
        }
    }
    cudaError_t e;
    if (do_quant) {
        k_quantize<XT><<<std::min(T, 65535), kThreads, 0, s>>>(x, T, d, p.ws.xq, p.ws.sx, p.ws.xcs);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // split d so that the tiled GEMM puts about four CTAs on each of the 148
    // SMs (slices of whole 32-column steps; measured on B200 at T = 512 and
    // 8192: four per SM beat two by ~10% of the router's time, eight lose)
    const int tiles = ((E + 63) / 64) * ((T + 63) / 64);
    const int ksteps = d / 32;
    int ks = std::max(1, std::min(std::min(ksteps, kRouterKsplitMax), (4 * 148 + tiles - 1) / tiles));
    const int per = (ksteps + ks - 1) / ks;
    ks = (ksteps + per - 1) / per;
    p.ksplit = ks;
    k_router_tiled<XT><<<dim3((E + 63) / 64, (T + 63) / 64, ks), kThreads, 0, s>>>(p, x);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (E <= 256) {  // register top-k; its last CTA buckets
        const size_t smem_b = bucket ? (size_t)bucket_smem_ints(E) * 4 : 0;
        if ((e = allow_smem((const void*)k_topk_small, smem_b)) != cudaSuccess) return e;
        k_topk_small<<<(T + kWarps - 1) / kWarps, kThreads, smem_b, s>>>(p, bucket);
        return cudaGetLastError();
    }
    const size_t smem_topk = (size_t)2 * kWarps * E * 4;
    if ((e = allow_smem((const void*)k_topk, smem_topk)) != cudaSuccess) return e;
    k_topk<<<(T + kWarps - 1) / kWarps, kThreads, smem_topk, s>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (bucket) {
        const size_t smem_b = (size_t)bucket_smem_ints(E) * 4;
        if ((e = allow_smem((const void*)k_bucket, smem_b)) != cudaSuccess) return e;
        k_bucket<<<1, kThreads, smem_b, s>>>(p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_router_any(Params& p, const void* x, moe_dtype dt, int do_quant, int bucket, cudaStream_t s) {
    if (dt == MOE_BF16) return launch_router(p, static_cast<const __nv_bfloat16*>(x), do_quant, bucket, s);
    return launch_router(p, static_cast<const float*>(x), do_quant, bucket, s);
}

moe_status check_dtype(moe_dtype dt) {
    return (dt == MOE_F32 || dt == MOE_BF16) ? MOE_OK : fail(MOE_EINVAL, "dtype must be MOE_F32 or MOE_BF16");
}

}  // namespace moe

using namespace moe;

// ---------------------------------------------------------------------------
// C ABI
// ---------------------------------------------------------------------------
extern "C" {

size_t moe_workspace_bytes(const moe_config* cfg, int32_t max_tokens) {
    if (check_cfg(cfg) != MOE_OK || max_tokens < 0) return 0;
    const int S = cfg->top_k + cfg->has_shared;
    return ws_carve(dims_of(cfg, std::max(1, (int)max_tokens), S), nullptr).bytes;
}

moe_status moe_workspace_init(void* ws, size_t ws_bytes, moe_stream_t stream) {
    MOE_TRY(check_ptr(ws, "ws"));
    if (ws_bytes < kCtrlBytes) return fail(MOE_ENOSPACE, "workspace smaller than its control words");
    // every counter of the kernels (control words, per-task and per-row-block
    // arrivals, running maxima) starts at zero and is left at zero by each call
    cudaError_t e = cudaMemsetAsync(ws, 0, ws_bytes, (cudaStream_t)stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_workspace_init");
}

moe_status moe_quantize(const moe_config* cfg, const void* x, moe_dtype dtype, int32_t T, int8_t* xq, float* sx,
                        moe_stream_t stream) {
    MOE_TRY(check_cfg(cfg));
    MOE_TRY(check_dtype(dtype));
    if (T < 0) return fail(MOE_EINVAL, "T < 0");
    if (T == 0) return MOE_OK;
    MOE_TRY(check_ptr(x, "x"));
    MOE_TRY(check_ptr(xq, "xq"));
    MOE_TRY(check_ptr(sx, "sx"));
    cudaStream_t s = (cudaStream_t)stream;
    const int grid = std::min((int)T, 65535);
    if (dtype == MOE_BF16)
        k_quantize<__nv_bfloat16><<<grid, kThreads, 0, s>>>(static_cast<const __nv_bfloat16*>(x), T, cfg->d, xq, sx,
                                                             nullptr);
    else
        k_quantize<float><<<grid, kThreads, 0, s>>>(static_cast<const float*>(x), T, cfg->d, xq, sx, nullptr);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_quantize");
}

moe_status moe_route(const moe_config* cfg, const void* x, moe_dtype dtype, int32_t T, const float* w_router,
                     const float* bias, int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes,
                     moe_stream_t stream) {
    MOE_TRY(check_cfg(cfg));
    MOE_TRY(check_dtype(dtype));
    if (T < 0) return fail(MOE_EINVAL, "T < 0");
    if (T == 0) return MOE_OK;
    MOE_TRY(check_ptr(x, "x"));
    MOE_TRY(check_ptr(w_router, "w_router"));
    MOE_TRY(check_ptr(bias, "bias"));
    MOE_TRY(check_ptr(topk_idx, "topk_idx"));
    MOE_TRY(check_ptr(topk_w, "topk_w"));
    const Dims m = dims_of(cfg, T, cfg->top_k + cfg->has_shared);
    MOE_TRY(check_ws(cfg, T, ws, ws_bytes));
    Params p = base_params(cfg, m, ws, ws_bytes);
    p.w_router = w_router;
    p.bias = bias;
    p.idx_out = topk_idx;
    p.w_out = topk_w;
    cudaError_t e = launch_router_any(p, x, dtype, 0, 0, (cudaStream_t)stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_route");
}

static moe_status expert_common(const moe_config* cfg, const moe_pool* pool, int32_t expert, int32_t T, float* y,
                                void* ws, size_t ws_bytes, Params* out_p) {
    MOE_TRY(check_cfg(cfg));
    if (!pool) return fail(MOE_EINVAL, "pool is NULL");
    MOE_TRY(check_ptr(pool->w, "pool->w"));
    MOE_TRY(check_pool_slots(pool));
    MOE_TRY(check_ptr(pool->s, "pool->s"));
    if (T < 0) return fail(MOE_EINVAL, "T < 0");
    if (expert < -1 || expert >= cfg->n_experts) return fail(MOE_EINVAL, "expert out of range");
    if (expert == -1 && !cfg->has_shared) return fail(MOE_EINVAL, "no shared expert in this config");
    MOE_TRY(check_ptr(y, "y"));
    const Dims m = dims_of(cfg, T, 1);
    MOE_TRY(check_ws(cfg, T, ws, ws_bytes));
    Params p = base_params(cfg, m, ws, ws_bytes);
    p.pool = pool->w;
    p.scales = pool->s;
    p.slot_of = pool->slot_of;
    p.n_slots = pool->n_slots;
    p.direct_out = 1;
    p.out = y;
    *out_p = p;
    return MOE_OK;
}

moe_status moe_expert_ffn(const moe_config* cfg, const moe_pool* pool, int32_t expert, const int8_t* xq,
                          const float* sx, int32_t T, float* y, int32_t* dbg_acc_gu, int8_t* dbg_hq, float* dbg_sh,
                          int32_t* dbg_acc_d, void* ws, size_t ws_bytes, moe_stream_t stream) {
    Params p;
    MOE_TRY(expert_common(cfg, pool, expert, T, y, ws, ws_bytes, &p));
    if (T == 0) return MOE_OK;
    MOE_TRY(check_ptr(xq, "xq"));
    MOE_TRY(check_ptr(sx, "sx"));
    MOE_TRY(check_ptr(dbg_acc_gu, "dbg_acc_gu", true));
    MOE_TRY(check_ptr(dbg_hq, "dbg_hq", true));
    MOE_TRY(check_ptr(dbg_sh, "dbg_sh", true));
    MOE_TRY(check_ptr(dbg_acc_d, "dbg_acc_d", true));
    const bool dbg = dbg_acc_gu || dbg_hq || dbg_sh || dbg_acc_d;
    const bool tc = use_tc(cfg, T);
    if (tc) p = base_params(cfg, p.m, ws, ws_bytes, true);
    else if (dbg) p.CH = 8;
    p.pool = pool->w;
    p.scales = pool->s;
    p.slot_of = pool->slot_of;
    p.n_slots = pool->n_slots;
    p.direct_out = 1;
    p.out = y;
    p.dbg_acc_gu = dbg_acc_gu;
    p.dbg_hq = dbg_hq;
    p.dbg_sh = dbg_sh;
    p.dbg_acc_d = dbg_acc_d;
    cudaStream_t s = (cudaStream_t)stream;
    const int blob = expert < 0 ? cfg->n_experts : expert;
    // the expert kernels read the activations from the workspace: copy them in
    cudaError_t e = cudaMemcpyAsync(p.ws.xq, xq, (size_t)T * cfg->d, cudaMemcpyDeviceToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(p.ws.sx, sx, (size_t)T * 4, cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "moe_expert_ffn copy");
    k_sum_codes<<<std::min((int)T, 65535), kThreads, 0, s>>>(p.ws.xq, T, cfg->d, p.ws.xcs);
    k_plan_single<<<1, kThreads, 0, s>>>(p, blob);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "moe_expert_ffn");
    if (tc) {
        e = launch_tc_gather(p, p.ws.xq, cfg->d, 1, cfg->d, p.ws.xb, s);
        if (e == cudaSuccess) e = launch_tc_expert(p, 0, tc_nt_max(T), s);
        if (e == cudaSuccess) e = launch_tc_requant(p, s);
        if (e == cudaSuccess) e = launch_tc_expert(p, 1, tc_nt_max(T), s);
        return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_expert_ffn (tensor cores)");
    }
    const ExpertTiling tl = expert_tiling(cfg->d, cfg->f, cfg->wbits);
    e = launch_gate_up(p, tl, dbg, s);
    if (e == cudaSuccess) e = launch_down(p, tl, dbg, s);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_expert_ffn");
}

moe_status moe_expert_down(const moe_config* cfg, const moe_pool* pool, int32_t expert, const int8_t* hq,
                           const float* sh, int32_t T, float* y, int32_t* dbg_acc_d, void* ws, size_t ws_bytes,
                           moe_stream_t stream) {
    Params p;
    MOE_TRY(expert_common(cfg, pool, expert, T, y, ws, ws_bytes, &p));
    if (T == 0) return MOE_OK;
    MOE_TRY(check_ptr(hq, "hq"));
    MOE_TRY(check_ptr(sh, "sh"));
    MOE_TRY(check_ptr(dbg_acc_d, "dbg_acc_d", true));
    const bool dbg = dbg_acc_d != nullptr;
    const bool tc = use_tc(cfg, T);
    if (tc) p = base_params(cfg, p.m, ws, ws_bytes, true);
    else if (dbg) p.CH = 8;
    p.pool = pool->w;
    p.scales = pool->s;
    p.slot_of = pool->slot_of;
    p.n_slots = pool->n_slots;
    p.direct_out = 1;
    p.out = y;
    p.hq_in = hq;
    p.sh_in = sh;
    p.dbg_acc_d = dbg_acc_d;
    cudaStream_t s = (cudaStream_t)stream;
    k_plan_single<<<1, kThreads, 0, s>>>(p, expert < 0 ? cfg->n_experts : expert);
    cudaError_t e = cudaGetLastError();
    if (tc) {
        if (e == cudaSuccess) {
            k_sum_codes<<<std::min((int)T, 65535), kThreads, 0, s>>>(hq, T, cfg->f, p.ws.hcs);
            e = cudaGetLastError();
        }
        if (e == cudaSuccess) e = launch_tc_gather(p, hq, cfg->f, 1, cfg->f, p.ws.hb, s);
        if (e == cudaSuccess) e = launch_tc_expert(p, 1, tc_nt_max(T), s);
        return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_expert_down (tensor cores)");
    }
    if (e == cudaSuccess) e = launch_down(p, expert_tiling(cfg->d, cfg->f, cfg->wbits), dbg, s);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_expert_down");
}

// The device-side address of pinned host memory (MOE_EINVAL if p is not host
// memory the device can address).
static moe_status host_mapped(const void* p, const char* name, const void** dev) {
    cudaPointerAttributes a{};
    const cudaError_t e = cudaPointerGetAttributes(&a, p);
    if (e != cudaSuccess) return cuda_fail(e, (std::string(name) + ": cudaPointerGetAttributes").c_str());
    if (a.type != cudaMemoryTypeHost || !a.devicePointer)
        return fail(MOE_EINVAL, std::string(name) + ": not pinned host memory mapped into the device's address space");
    if (!aligned16(a.devicePointer)) return fail(MOE_EALIGN, std::string(name) + " is not 16-byte aligned");
    *dev = a.devicePointer;
    return MOE_OK;
}

// Copy `bytes` (a multiple of 16) from mapped host memory into device memory.
static cudaError_t launch_stage_in(const void* src, void* dst, size_t bytes, cudaStream_t s) {
    const long long n16 = (long long)(bytes / 16);
    const long long per_cta = 4ll * kThreads;  // four chunks in flight per thread
    const int grid = (int)std::max(1ll, std::min((n16 + per_cta - 1) / per_cta, 4ll * 148));
    k_stage_in<<<grid, kThreads, 0, s>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst), n16);
    return cudaGetLastError();
}

moe_status moe_layer_ex(const moe_config* cfg, const moe_pool* pool, const float* w_router, const float* bias,
                        const void* x, moe_dtype dtype, int32_t T, float* out, int32_t accumulate,
                        int32_t* topk_idx_out, float* topk_w_out, void* ws, size_t ws_bytes, moe_stream_t stream,
                        moe_layer_opts* opts) {
    MOE_TRY(check_cfg(cfg));
    MOE_TRY(check_dtype(dtype));
    if (!pool) return fail(MOE_EINVAL, "pool is NULL");
    if (T < 0) return fail(MOE_EINVAL, "T < 0");
    if (opts) {
        opts->n_launches = 0;
        opts->path_ran = MOE_PATH_AUTO;
        if (opts->wait_limit_us < 0 || opts->test_skip_h < 0)
            return fail(MOE_EINVAL, "opts->wait_limit_us and opts->test_skip_h must be >= 0");
        if (opts->io_host & ~(MOE_IO_X_HOST | MOE_IO_OUT_HOST))
            return fail(MOE_EINVAL, "opts->io_host: unknown bits");
    }
    const int io = opts ? opts->io_host : 0;
    if (T == 0) return MOE_OK;
    MOE_TRY(check_ptr(pool->w, "pool->w"));
    MOE_TRY(check_pool_slots(pool));
    MOE_TRY(check_ptr(pool->s, "pool->s"));
    MOE_TRY(check_ptr(w_router, "w_router"));
    MOE_TRY(check_ptr(bias, "bias"));
    MOE_TRY(check_ptr(x, "x"));
    MOE_TRY(check_ptr(out, "out"));
    // the device-side addresses of host buffers (their own, with unified addressing)
    const void* x_host = nullptr;
    if (io & MOE_IO_X_HOST) MOE_TRY(host_mapped(x, "x", &x_host));
    if (io & MOE_IO_OUT_HOST) {
        const void* o = nullptr;
        MOE_TRY(host_mapped(out, "out", &o));
        out = static_cast<float*>(const_cast<void*>(o));
    }
    MOE_TRY(check_ptr(topk_idx_out, "topk_idx_out", true));
    MOE_TRY(check_ptr(topk_w_out, "topk_w_out", true));
    const Dims m = dims_of(cfg, T, cfg->top_k + cfg->has_shared);
    MOE_TRY(check_ws(cfg, T, ws, ws_bytes));
    Params p = base_params(cfg, m, ws, ws_bytes);
    p.pool = pool->w;
    p.scales = pool->s;
    p.slot_of = pool->slot_of;
    p.n_slots = pool->n_slots;
    p.w_router = w_router;
    p.bias = bias;
    p.out = out;
    p.accumulate = accumulate ? 1 : 0;
    p.idx_out = topk_idx_out;
    p.w_out = topk_w_out;
    p.trace = opts ? static_cast<unsigned long long*>(opts->trace) : nullptr;
    if (opts && opts->wait_limit_us > 0) p.wait_ns = (unsigned long long)opts->wait_limit_us * 1000ull;
    if (opts && opts->test_skip_h > 0) p.skip_h_task = opts->test_skip_h - 1;
    cudaStream_t s = (cudaStream_t)stream;
    const ExpertTiling tl = expert_tiling(cfg->d, cfg->f, cfg->wbits);
    auto mark = [&](int i) -> cudaError_t {
        if (opts && opts->events[i]) return cudaEventRecord((cudaEvent_t)opts->events[i], s);
        return cudaSuccess;
    };
    const int path = opts ? opts->path : MOE_PATH_AUTO;
    if (path != MOE_PATH_AUTO && path != MOE_PATH_MULTI && path != MOE_PATH_DECODE && path != MOE_PATH_TC)
        return fail(MOE_EINVAL, "opts->path must be MOE_PATH_AUTO, MOE_PATH_MULTI, MOE_PATH_DECODE or MOE_PATH_TC");
    DecPlan pl{};
    // AUTO: the tensor-core path from tc_min_tokens tokens on, else the
    // single-launch decode kernel where the shape fits it, else MULTI
    const bool auto_tc = path == MOE_PATH_AUTO && use_tc(cfg, T);
    const bool dec_ok = ((path == MOE_PATH_AUTO && !auto_tc) || path == MOE_PATH_DECODE) && decode_plan(m, &pl);
    // the h-skip hook acts only where the hand-off polls values (one token,
    // row-range down); elsewhere it would give wrong output instead of a timeout
    if (!(dec_ok && pl.rowrange)) p.skip_h_task = -1;
    if (path == MOE_PATH_DECODE && !dec_ok) return fail(MOE_EINVAL, "shape does not fit the single-launch decode path");
    if (path == MOE_PATH_TC && !tc_shape_ok(m)) return fail(MOE_EINVAL, "shape does not fit the tensor-core path");
    cudaError_t e = mark(0);
    if (e == cudaSuccess && x_host) {  // one read of x over the host link, into the workspace
        e = launch_stage_in(x_host, p.ws.xin, (size_t)T * cfg->d * (dtype == MOE_BF16 ? 2 : 4), s);
        x = p.ws.xin;
    }
    if (dec_ok) {
        if (e == cudaSuccess)
            e = launch_decode(p, pl, x, dtype == MOE_BF16, s);
        if (e == cudaSuccess) e = mark(3);  // [1] and [2] fall inside the one kernel: not recorded
        if (opts) {
            opts->n_launches = 1 + (x_host ? 1 : 0);
            opts->path_ran = MOE_PATH_DECODE;
        }
        return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_layer (decode)");
    }
    if (path == MOE_PATH_TC || auto_tc) {
        Params q = base_params(cfg, m, ws, ws_bytes, true);
        q.pool = p.pool;
        q.scales = p.scales;
        q.slot_of = p.slot_of;
        q.n_slots = p.n_slots;
        q.w_router = p.w_router;
        q.bias = p.bias;
        q.out = p.out;
        q.accumulate = p.accumulate;
        q.idx_out = p.idx_out;
        q.w_out = p.w_out;
        if (e == cudaSuccess) e = launch_router_any(q, x, dtype, 1, 1, s);
        if (e == cudaSuccess) e = launch_tc_gather(q, q.ws.xq, cfg->d, m.S, cfg->d, q.ws.xb, s);
        if (e == cudaSuccess) e = mark(1);
        if (e == cudaSuccess) e = launch_tc_expert(q, 0, tc_nt_max(T), s);
        if (e == cudaSuccess) e = launch_tc_requant(q, s);
        if (e == cudaSuccess) e = mark(2);
        if (e == cudaSuccess) e = launch_tc_expert(q, 1, tc_nt_max(T), s);
        if (e == cudaSuccess) e = launch_combine(q, s);
        if (e == cudaSuccess) e = mark(3);
        if (opts) {
            opts->n_launches = (T <= 8 ? 1 : cfg->n_experts <= 256 ? 3 : 4) + 5 + (x_host ? 1 : 0);
            opts->path_ran = MOE_PATH_TC;
        }
        return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_layer (tensor cores)");
    }
    if (e == cudaSuccess) e = launch_router_any(p, x, dtype, 1, 1, s);
    if (e == cudaSuccess) e = mark(1);
    if (e == cudaSuccess) e = launch_gate_up(p, tl, false, s);
    if (e == cudaSuccess) e = mark(2);
    if (e == cudaSuccess) e = launch_down(p, tl, false, s);
    if (e == cudaSuccess) e = mark(3);
    if (opts) {
        opts->n_launches = (T <= 8 ? 1 : cfg->n_experts <= 256 ? 3 : 4) + 2 + (x_host ? 1 : 0);
        opts->path_ran = MOE_PATH_MULTI;
    }
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_layer");
}

moe_status moe_layer(const moe_config* cfg, const moe_pool* pool, const float* w_router, const float* bias,
                     const void* x, moe_dtype dtype, int32_t T, float* out, int32_t accumulate, int32_t* topk_idx_out,
                     float* topk_w_out, void* ws, size_t ws_bytes, moe_stream_t stream) {
    return moe_layer_ex(cfg, pool, w_router, bias, x, dtype, T, out, accumulate, topk_idx_out, topk_w_out, ws,
                        ws_bytes, stream, nullptr);
}

moe_status moe_rmsnorm(const void* x, moe_dtype dtype, int32_t T, int32_t d, float eps, float* x_in, float* x_copy,
                       moe_stream_t stream) {
    MOE_TRY(check_dtype(dtype));
    if (T < 0 || d <= 0 || d % 4) return fail(MOE_EINVAL, "T >= 0 and d > 0, a multiple of 4, required");
    if (T == 0) return MOE_OK;
    MOE_TRY(check_ptr(x, "x"));
    MOE_TRY(check_ptr(x_in, "x_in"));
    MOE_TRY(check_ptr(x_copy, "x_copy", true));
    cudaStream_t s = (cudaStream_t)stream;
    const int grid = std::min((int)T, 65535);
    if (dtype == MOE_BF16)
        k_rmsnorm<__nv_bfloat16><<<grid, kThreads, 0, s>>>(static_cast<const __nv_bfloat16*>(x), T, d, eps, x_in,
                                                           x_copy);
    else
        k_rmsnorm<float><<<grid, kThreads, 0, s>>>(static_cast<const float*>(x), T, d, eps, x_in, x_copy);
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_rmsnorm");
}

moe_status moe_poll_status(const void* ws, int32_t* info, moe_stream_t stream) {
    MOE_TRY(check_ptr(ws, "ws"));
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "moe_poll_status sync");
    int32_t hv[2] = {0, 0};
    e = cudaMemcpy(hv, ws, sizeof(hv), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "moe_poll_status copy");
    if (info) *info = hv[1];
    if (hv[0] != 0) return fail((moe_status)hv[0], "a kernel reported an error (info " + std::to_string(hv[1]) + ")");
    return MOE_OK;
}

const char* moe_status_string(moe_status st) {
    switch (st) {
        case MOE_OK: return "MOE_OK";
        case MOE_EINVAL: return "MOE_EINVAL: invalid argument";
        case MOE_EALIGN: return "MOE_EALIGN: pointer not 16-byte aligned";
        case MOE_ENOSPACE: return "MOE_ENOSPACE: workspace too small";
        case MOE_ECUDA: return "MOE_ECUDA: CUDA error";
        case MOE_ETIMEOUT: return "MOE_ETIMEOUT: bounded device wait expired";
        case MOE_EDEVICE: return "MOE_EDEVICE: a kernel found an invalid value";
        default: return "unknown moe_status";
    }
}

const char* moe_last_error(void) { return g_last_error.c_str(); }

}  // extern "C"
