// Internal launchers shared by the translation units of libmoe (host side).
#pragma once

#include <cuda_runtime.h>

#include <string>

#include "moe_common.cuh"

namespace moe {

// Tiling choices of the expert kernels for a given shape.
struct ExpertTiling {
    int ncl3, rpw3;  // gate/up: 16-byte chunks per lane per row, rows per warp per item
    int ncl4, rpw4;  // down: the same
};

ExpertTiling expert_tiling(int d, int f, int wb);

// Persistent-grid size for a kernel: SMs x resident CTAs (cached per kernel).
int persistent_grid(const void* func, size_t smem, int threads = kThreads);
// Resident CTAs per SM (0 if the configuration does not fit), cached.
int blocks_per_sm(const void* func, size_t smem, int threads);
// Raise the dynamic shared-memory limit of a kernel once (cached).
cudaError_t allow_smem(const void* func, size_t smem);

struct DecPlan;
// Persistent single-launch decode kernel (T <= 8): plan (false if the shape
// does not fit) and cooperative launch.
bool decode_plan(const Dims& m, DecPlan* pl);
cudaError_t launch_decode(const Params& p, const DecPlan& pl, const void* x, bool bf16, cudaStream_t s);

cudaError_t launch_gate_up(const Params& p, const ExpertTiling& tl, bool dbg, cudaStream_t s);

// Router launch sequence (a0 + a1 (+ a2)) and the host-side checks the entry
// points share (moe_capi.cu).
cudaError_t launch_router_any(Params& p, const void* x, moe_dtype dt, int do_quant, int bucket, cudaStream_t s);
moe_status fail(moe_status st, const std::string& msg);
moe_status check_cfg(const moe_config* c);
moe_status check_ptr(const void* p, const char* name, bool nullable = false);
moe_status check_dtype(moe_dtype dt);
cudaError_t launch_down(const Params& p, const ExpertTiling& tl, bool dbg, cudaStream_t s);

// Tensor-core expert path (moe_ktc.cu).  nt_max: bound on the tokens of one
// task in this call (<= kTcNT).
bool tc_shape_ok(const Dims& m);
// stage 0: gate/up, 1: down.
cudaError_t launch_tc_expert(const Params& p, int stage, int nt_max, cudaStream_t s);
// h -> the down operand (int8 codes in the MMA layout), scales, code sums.
cudaError_t launch_tc_requant(const Params& p, cudaStream_t s);
// Operand B of every task from int8 rows `src` (row = assignment id / key_div).
cudaError_t launch_tc_gather(const Params& p, const int8_t* src, int ld, int key_div, int K, uint8_t* dst,
                             cudaStream_t s);
// out (+)= weighted sum of the per-assignment down outputs, over the grid.
cudaError_t launch_combine(const Params& p, cudaStream_t s);

}  // namespace moe
