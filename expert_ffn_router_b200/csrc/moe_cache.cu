// HBM expert cache with host-memory overflow: the layer's pool stays in
// pinned host memory, n_slots blobs are resident in device memory, and
// moe_cache_fetch makes the experts a call selects resident, evicting the
// least recently used others.  The book-keeping is host code over memory the
// caller provides; the device sees only the slot table (expert -> slot), which
// the fetch updates with small kernels whose (expert, slot) pairs travel as
// kernel arguments, so no host buffer has to outlive an asynchronous copy.
#include <cuda_runtime.h>

#include <cstring>
#include <string>

#include "moe.h"
#include "moe_launch.h"

namespace moe {

namespace {

constexpr uint64_t kCacheMagic = 0x4d4f45434143484bull;  // "MOECACHK"
constexpr uint64_t kPinned = ~0ull;                      // last-use stamp of a slot never evicted
constexpr int kPairsPerLaunch = 512;

struct CacheHdr {
    uint64_t magic;
    int32_t n_slots, n_exp;
    uint64_t clock;
};

// Views of the caller's state memory: header, then slot -> expert, expert ->
// slot (host mirror), slot -> last use, expert -> 2 * (the last call that
// selected it) + 1 once that call has placed it.
struct CacheView {
    CacheHdr* h;
    int32_t* slot_expert;
    int32_t* slot_of;
    uint64_t* last_use;
    uint64_t* need;
};

size_t align8(size_t v) { return (v + 7) & ~size_t(7); }

size_t state_bytes(int n_slots, int n_exp) {
    return align8(sizeof(CacheHdr)) + align8((size_t)n_slots * 4) + align8((size_t)n_exp * 4) + 8 * (size_t)n_slots +
           8 * (size_t)n_exp;
}

CacheView view(void* state, int n_slots, int n_exp) {
    char* b = static_cast<char*>(state);
    CacheView v;
    v.h = reinterpret_cast<CacheHdr*>(b);
    b += align8(sizeof(CacheHdr));
    v.slot_expert = reinterpret_cast<int32_t*>(b);
    b += align8((size_t)n_slots * 4);
    v.slot_of = reinterpret_cast<int32_t*>(b);
    b += align8((size_t)n_exp * 4);
    v.last_use = reinterpret_cast<uint64_t*>(b);
    b += 8 * (size_t)n_slots;
    v.need = reinterpret_cast<uint64_t*>(b);
    return v;
}

struct SlotPairs {
    int n;
    int expert[kPairsPerLaunch];
    int slot[kPairsPerLaunch];
};

// slot_of[expert[i]] = slot[i] for the pairs of one launch, in order (an
// eviction's -1 precedes the new owner's entry only for different experts,
// so the order never matters for one expert).
__global__ void k_cache_update(int32_t* slot_of, const SlotPairs pairs) {
    for (int i = threadIdx.x; i < pairs.n; i += blockDim.x) slot_of[pairs.expert[i]] = pairs.slot[i];
}

__global__ void k_cache_fill(int32_t* slot_of, int n, int32_t v) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) slot_of[i] = v;
}

moe_status flush_pairs(int32_t* slot_of, SlotPairs& pairs, cudaStream_t s) {
    if (pairs.n == 0) return MOE_OK;
    k_cache_update<<<1, 256, 0, s>>>(slot_of, pairs);
    const cudaError_t e = cudaGetLastError();
    pairs.n = 0;
    if (e != cudaSuccess) return fail(MOE_ECUDA, std::string("moe_cache: slot table update: ") + cudaGetErrorString(e));
    return MOE_OK;
}

moe_status add_pair(int32_t* slot_of, SlotPairs& pairs, int e, int sl, cudaStream_t s) {
    pairs.expert[pairs.n] = e;
    pairs.slot[pairs.n] = sl;
    if (++pairs.n == kPairsPerLaunch) return flush_pairs(slot_of, pairs, s);
    return MOE_OK;
}

moe_status check_cache(const moe_config* cfg, const moe_cache* c) {
    const moe_status st = check_cfg(cfg);
    if (st != MOE_OK) return st;
    if (!c) return fail(MOE_EINVAL, "cache is NULL");
    if (!c->host_w || !c->slots || !c->slot_of || !c->state)
        return fail(MOE_EINVAL, "cache: host_w, slots, slot_of and state must be set");
    if (c->n_slots < 1) return fail(MOE_EINVAL, "cache: n_slots must be >= 1");
    if (reinterpret_cast<uintptr_t>(c->slots) % 16 || reinterpret_cast<uintptr_t>(c->slot_of) % 4 ||
        reinterpret_cast<uintptr_t>(c->state) % 8)
        return fail(MOE_EALIGN, "cache: slots must be 16-byte, slot_of 4-byte and state 8-byte aligned");
    if (cfg->has_shared && c->n_slots < 2) return fail(MOE_EINVAL, "cache: n_slots must be >= 2 with a shared expert");
    return MOE_OK;
}

}  // namespace

}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_cache_state_bytes(const moe_config* cfg, int32_t n_slots) {
    if (check_cfg(cfg) != MOE_OK || n_slots < 1) return 0;
    return state_bytes(n_slots, cfg->n_experts + cfg->has_shared);
}

moe_status moe_cache_init(const moe_config* cfg, moe_cache* c, moe_stream_t stream) {
    const moe_status st = check_cache(cfg, c);
    if (st != MOE_OK) return st;
    const int n_exp = cfg->n_experts + cfg->has_shared;
    CacheView v = view(c->state, c->n_slots, n_exp);
    std::memset(c->state, 0, state_bytes(c->n_slots, n_exp));
    v.h->magic = kCacheMagic;
    v.h->n_slots = c->n_slots;
    v.h->n_exp = n_exp;
    v.h->clock = 0;
    for (int i = 0; i < c->n_slots; ++i) v.slot_expert[i] = -1;
    for (int e = 0; e < n_exp; ++e) v.slot_of[e] = -1;
    cudaStream_t s = (cudaStream_t)stream;
    const size_t B = 3ull * cfg->d * cfg->f * cfg->wbits / 8;
    k_cache_fill<<<(n_exp + 255) / 256, 256, 0, s>>>(c->slot_of, n_exp, -1);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess && cfg->has_shared) {  // the shared expert: slot 0, for good
        const int sh = cfg->n_experts;
        e = cudaMemcpyAsync(c->slots, c->host_w + (size_t)sh * B, B, cudaMemcpyHostToDevice, s);
        v.slot_expert[0] = sh;
        v.slot_of[sh] = 0;
        v.last_use[0] = kPinned;
        if (e == cudaSuccess) {
            SlotPairs pairs;
            pairs.n = 0;
            const moe_status st2 = add_pair(c->slot_of, pairs, sh, 0, s);
            if (st2 != MOE_OK) return st2;
            return flush_pairs(c->slot_of, pairs, s);
        }
    }
    if (e != cudaSuccess) return fail(MOE_ECUDA, std::string("moe_cache_init: ") + cudaGetErrorString(e));
    return MOE_OK;
}

moe_status moe_cache_fetch(const moe_config* cfg, moe_cache* c, const int32_t* idx, int32_t T, moe_stream_t stream,
                           moe_cache_stats* stats) {
    moe_status st = check_cache(cfg, c);
    if (st != MOE_OK) return st;
    if (T < 0 || (T > 0 && !idx)) return fail(MOE_EINVAL, "moe_cache_fetch: idx is NULL or T < 0");
    const int E = cfg->n_experts, k = cfg->top_k, n_exp = E + cfg->has_shared;
    CacheView v = view(c->state, c->n_slots, n_exp);
    if (v.h->magic != kCacheMagic || v.h->n_slots != c->n_slots || v.h->n_exp != n_exp)
        return fail(MOE_EINVAL, "moe_cache_fetch: the cache was not initialised for this config (moe_cache_init)");
    const uint64_t now = ++v.h->clock;
    auto selected = [&](int e) { return (v.need[e] >> 1) == now; };
    // the call's distinct experts
    int n_need = 0, n_miss = 0;
    for (int64_t i = 0; i < (int64_t)T * k; ++i) {
        const int e = idx[i];
        if (e == -1) continue;  // a slot the router's truncation dropped
        if (e < 0 || e >= E) return fail(MOE_EINVAL, "moe_cache_fetch: expert index out of range in idx");
        if (!selected(e)) {
            v.need[e] = now << 1;
            ++n_need;
            n_miss += v.slot_of[e] < 0;
        }
    }
    // enough slots that this call does not select (free or evictable)?
    int avail = 0;
    for (int s2 = 0; s2 < c->n_slots; ++s2) {
        const int o = v.slot_expert[s2];
        avail += o < 0 || (v.last_use[s2] != kPinned && !selected(o));
    }
    if (n_miss > avail)
        return fail(MOE_ENOSPACE, "moe_cache_fetch: " + std::to_string(c->n_slots) + " slots cannot hold the call's " +
                                      std::to_string(n_need) + " experts");
    cudaStream_t s = (cudaStream_t)stream;
    const size_t B = 3ull * cfg->d * cfg->f * cfg->wbits / 8;
    SlotPairs pairs;
    pairs.n = 0;
    int64_t hits = 0, misses = 0;
    for (int64_t i = 0; i < (int64_t)T * k; ++i) {
        const int e = idx[i];
        if (e < 0 || (v.need[e] & 1)) continue;  // dropped, or placed already
        v.need[e] |= 1;
        const int sl = v.slot_of[e];
        if (sl >= 0) {
            ++hits;
            v.last_use[sl] = now;
            continue;
        }
        // a free slot, else the least recently used slot whose expert this call does not select
        int victim = -1;
        uint64_t best = ~0ull;
        for (int s2 = 0; s2 < c->n_slots; ++s2) {
            const int o = v.slot_expert[s2];
            if (o < 0) {
                victim = s2;
                break;
            }
            if (v.last_use[s2] == kPinned || selected(o)) continue;
            if (v.last_use[s2] < best) {
                best = v.last_use[s2];
                victim = s2;
            }
        }
        if (victim < 0) return fail(MOE_ENOSPACE, "moe_cache_fetch: no slot left");  // (excluded above)
        const int old = v.slot_expert[victim];
        if (old >= 0) {
            v.slot_of[old] = -1;
            if ((st = add_pair(c->slot_of, pairs, old, -1, s)) != MOE_OK) return st;
        }
        const cudaError_t e2 =
            cudaMemcpyAsync(c->slots + (size_t)victim * B, c->host_w + (size_t)e * B, B, cudaMemcpyHostToDevice, s);
        if (e2 != cudaSuccess) return fail(MOE_ECUDA, std::string("moe_cache_fetch: ") + cudaGetErrorString(e2));
        v.slot_expert[victim] = e;
        v.slot_of[e] = victim;
        v.last_use[victim] = now;
        ++misses;
        if ((st = add_pair(c->slot_of, pairs, e, victim, s)) != MOE_OK) return st;
    }
    if ((st = flush_pairs(c->slot_of, pairs, s)) != MOE_OK) return st;
    if (stats) {
        stats->hits = hits;
        stats->misses = misses;
        stats->bytes = misses * (int64_t)B;
    }
    return MOE_OK;
}

}  // extern "C"
