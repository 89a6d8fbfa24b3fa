// Internal declarations shared by the CUDA sources of libmoonep (not installed).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moonep.h"

namespace moonep {

// Planner launch shape: one histogram block per chunk of kChunkTokens tokens
// of one source rank; the last block to finish also lays the plan out.
constexpr int kChunkTokens = 512;
constexpr int kPlanThreads = 512;
constexpr int kPlanWarps = kPlanThreads / 32;
constexpr int kDstThreads = 256;

struct Dims {
    int S, H, K, E, R, B, tp, mode;
    int G;    // E / R
    int nch;  // chunks per rank = ceil(S / kChunkTokens)
    int NR;   // rows per rank = E + B
    int nvs;  // NvS
};

// Planning workspace, carved out of one device allocation owned by the handle.
struct Workspace {
    int32_t *hist;      // [R*nch][E]: chunk histograms, then their exclusive prefix over (r, chunk)
    uint32_t *arrive;   // [1] blocks of the counting kernel that finished (reset by the last)
    int32_t *status;    // [1] error bits gathered while counting (reset by the last block)
    int32_t *estart;    // [E] start of each expert inside its group's sequence
    int32_t *keep;      // [R] picks each home group keeps
    int32_t *don;       // [4][R]: donor, recipient, start, length of each donation
    int32_t *ndon;      // [1]
    int32_t *rowmap;    // [R][G]: row, on rank s, of the j-th expert of the group s takes from
    int32_t *rowstart;  // [R][E+B]: first slot of each row
};

size_t workspace_bytes(const Dims &d);
void carve_workspace(const Dims &d, void *base, Workspace *ws);

struct PlanArgs {
    Dims d;
    const int32_t *topk;
    const int32_t *tpe;
    moonep_plan_t plan;
    Workspace ws;
};

size_t plan_count_smem_bytes(const Dims &d);
cudaError_t launch_plan(const PlanArgs &a, int sms, cudaStream_t st);

struct CopyArgs {
    Dims d;
    const int32_t *dst;
    const int32_t *status;
    int32_t *status_rw;
    const void *src;  // dispatch: hidden [R,S,H]; combine: y [R,NvS,H]
    const float *w;   // dispatch: route_weights [R,S,K]; combine: route_weights_nvs
    void *out;        // dispatch: hidden_nvs; combine: out [R,S,H]
    float *w_out;     // dispatch: route_weights_nvs; combine: gathered weights [R,S,K]
};

cudaError_t launch_dispatch(const CopyArgs &a, int grid, cudaStream_t st);
cudaError_t launch_combine(const CopyArgs &a, int grid, cudaStream_t st);
int dispatch_blocks_per_sm();
int combine_blocks_per_sm(int K);

struct WeightArgs {
    Dims d;
    const int32_t *slot_expert;  // [R*B]
    int32_t *status;             // plan status (read; BAD_PLAN may be OR-ed in)
    int n_proj;
    int64_t hhp;                 // H * Hp elements per expert
    const void *src[MOONEP_MAX_PROJ];
    void *dst[MOONEP_MAX_PROJ];
};

cudaError_t launch_prefetch(const WeightArgs &a, int grid, cudaStream_t st);
cudaError_t launch_reduce_grad(const WeightArgs &a, int grid, cudaStream_t st);
int weights_blocks_per_sm();

// ---- small device helpers ------------------------------------------------
__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Programmatic dependent launch: wait for the grid this launch depends on
// (a no-op when the launch has no such dependency) / let the dependent grid
// start its prologue.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ int ld_cg(const int32_t *p) { return __ldcg(p); }

}  // namespace moonep
