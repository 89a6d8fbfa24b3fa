// Internal declarations shared by the CUDA sources of libmoonep (not installed).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moonep.h"

namespace moonep {

// Planner launch shape: one cooperative block per chunk of `ct` tokens of one
// source rank (all blocks resident), kPlanThreads threads each.
constexpr int kPlanThreads = 1024;
constexpr int kPlanWarps = kPlanThreads / 32;
constexpr int kChunkTokensMin = 256;
constexpr int kMaxDevices = 64;
constexpr uint32_t kBarrierPolls = 1u << 22;  // each poll is an L2 round trip: ~2 s, then MOONEP_STATUS_TIMEOUT

struct Dims {
    int S, H, K, E, R, B, tp, mode;
    int G;    // E / R
    int ct;   // tokens per planner chunk
    int cw;   // planner warps that count picks (each keeps per-expert counters)
    int nch;  // chunks per rank = ceil(S / ct)
    int NR;   // rows per rank = E + B
    int nvs;  // NvS
    int fast2;  // planner keeps second-recipient dst bases (when shared memory allows)
    int xtab;   // planner keeps the split column pass's and the rank pass's dst-base tables (when they fit)
};

// Planning workspace (one device allocation owned by the handle).
struct Workspace {
    int32_t *hist;                // [R*nch][E] picks per (chunk, expert)
    int32_t *cnt;                 // [2][R][E] picks per (source rank, expert), by call parity
    int32_t *gload;               // [2][R] picks per home group (group planning), by call parity
    unsigned long long *arrive;   // planner blocks that ever reached the grid barrier
    int32_t *status;              // [2] error bits of the counting phase, by call parity
};

size_t workspace_bytes(const Dims &d);
void carve_workspace(const Dims &d, void *base, Workspace *ws);

struct PlanArgs {
    Dims d;
    const int32_t *topk;        // [R,S,K], or [S,K] of src_rank
    const int32_t *tpe;         // [R,E] router counts to check, or NULL (group planning)
    int src_rank;               // -1: plan the whole group; else this rank's picks only
    const int32_t *counts_all;  // [R,E] every rank's counts (src_rank >= 0)
    moonep_plan_t plan;
    Workspace ws;
    uint32_t polls;     // grid-barrier poll limit (kBarrierPolls unless a test lowers it)
    uint32_t withheld;  // arrivals the barrier waits for beyond the grid (0; a test hook sets it)
};

size_t plan_smem_bytes(const Dims &d);
int plan_blocks_per_sm(const Dims &d);
cudaError_t plan_set_smem_limit(size_t bytes);
size_t plan_static_smem_bytes();
cudaError_t launch_plan(const PlanArgs &a, int grid, cudaStream_t st);

struct CopyArgs {
    Dims d;
    const int32_t *dst;
    const int32_t *status;
    int32_t *status_rw;
    int64_t ntok;     // token rows: R*S (the group), S (one rank)
    const void *src;  // dispatch: hidden [ntok,H]; combine: y [R,NvS,H] (unless peered)
    const float *w;   // dispatch: route_weights [ntok,K]; combine: route_weights_nvs (unless peered)
    void *out;        // dispatch: hidden_nvs (unless peered); combine: out [ntok,H]
    float *w_out;     // dispatch: route_weights_nvs (unless peered); combine: gathered weights [ntok,K]
    // peered: slot dst = q*NvS + i lives at row i of rank q's own buffer
    // peer[q] (dispatch writes it, combine reads it), its route weight at
    // peer_w[q][i] (all NULL: no weights)
    int peered;
    void *peer[MOONEP_MAX_R];
    float *peer_w[MOONEP_MAX_R];
};

// 1 when p lives on a device other than `device` (a peer GPU's memory), 0
// when on `device` (or host-visible), -1 when CUDA cannot tell (ipc.cu)
int on_other_device(const void *p, int device);

cudaError_t launch_dispatch(const CopyArgs &a, int grid, cudaStream_t st);
cudaError_t launch_dispatch_bulk(const CopyArgs &a, int grid, cudaStream_t st);
cudaError_t dispatch_bulk_set_smem_limit(size_t bytes);
int dispatch_bulk_blocks_per_sm(const Dims &d);
bool dispatch_use_bulk(const Dims &d);
cudaError_t launch_combine(const CopyArgs &a, int grid, cudaStream_t st);
int dispatch_blocks_per_sm(int K);
int combine_blocks_per_sm(int K);

struct WeightArgs {
    Dims d;
    const int32_t *slot_expert;  // [R*B]
    int32_t *status;             // plan status (read; BAD_PLAN may be OR-ed in)
    int n_proj;
    int64_t hhp;                 // H * Hp elements per expert
    const void *src[MOONEP_MAX_PROJ];
    void *dst[MOONEP_MAX_PROJ];
    // rank < 0: the group (src/dst span all experts [E,..] and all slots
    // [R*B,..]).  rank >= 0: that rank's share.  Its own side is dst (prefetch:
    // its slots [B,..]) or dst (reduce_grad: its home experts [G,..]); the
    // other side is every rank's tensor, peer[p][q] = rank q's home experts
    // [G,..] (prefetch) or slots [B,..] (reduce_grad).
    int rank;
    const void *peer[MOONEP_MAX_PROJ][MOONEP_MAX_R];
    int remote;  // some peer tensor lives on another GPU: plain loads and stores only, no bulk copies
};

cudaError_t launch_prefetch(const WeightArgs &a, int grid, int sms, cudaStream_t st);
cudaError_t launch_reduce_grad(const WeightArgs &a, int grid, int sms, cudaStream_t st);
int weights_blocks_per_sm();

// group GEMM (gemm.cu)
int gemm_supported(const Dims &d, int64_t Hp);
cudaError_t gemm_set_smem_limit();
int launch_group_gemm(const Dims &d, const moonep_plan_t *plan, const void *x, const void *W, const void *pool,
                      void *y, int64_t Hp, int32_t *pairs, cudaStream_t st);
int gemm_pair_slots(const Dims &d);
size_t gemm_table_bytes(const Dims &d);  // the pair table in the handle workspace

// ---- host helpers shared by the entry points (api.cu) ----------------------
int fail_cuda(cudaError_t e);                  // records the error text, returns MOONEP_ERR_CUDA
int64_t nvs_of(const moonep_config_t &c);
int check_config(const moonep_config_t &c);
int prepare_device(int device);                // kernel attributes, once per device
int plan_dims(const moonep_config_t &c, int device, Dims *d, int *grid);
bool plan_ok(const moonep_plan_t *p);

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

#include "bulk.cuh"


}  // namespace moonep
