/*
 * moonep.h -- C ABI of the balanced expert-parallel (EP) hot path, one B200.
 *
 * The operations are those of MoonEP ("MoonEP: A Perfectly Balanced Expert
 * Parallelism Library via Dynamic Redundant Experts", the project's GitHub
 * README, and the MarkTechPost article "Moonshot AI Open-Sources MoonEP").
 * An EP group of R ranks is emulated on one GPU: every per-rank tensor carries
 * a leading [R] dimension and the R partitions live in one device allocation.
 * A remote access of the original design is an offset into that allocation.
 *
 * Notation (README, "Usage > Integration"): S input tokens per rank, K experts
 * per token, E routed experts in the group, R ranks, B prefetch slots per rank,
 * H hidden size, H' expert FFN intermediate size, NvS dispatched token slots
 * per rank (S*K real slots plus the padding of every row), G = E/R experts per
 * home group.  bf16 tensors are passed as void pointers to 16-bit values.
 *
 * Conventions for every call:
 *  - All tensor arguments are DEVICE pointers on the device that was current
 *    when the handle was created, row-major and densely packed.  The caller
 *    owns every tensor, including the plan arrays; the library owns only the
 *    handle and a small planning workspace inside it.
 *  - Every call is asynchronous on `stream` (NULL = legacy default stream) and
 *    never synchronises the host, except moonep_read_status and
 *    moonep_plan_status.
 *  - Return value: MOONEP_OK, or a negative MOONEP_ERR_* for errors detected
 *    on the host before anything is launched.  Data-dependent errors are found
 *    on the device and reported as MOONEP_STATUS_* bits in plan->status; every
 *    later call that takes that plan then does nothing.
 *  - Every call can be captured in a CUDA graph (stream capture), the
 *    planner's cooperative launch included; a replayed plan reads the inputs
 *    the captured pointers hold at replay time.
 *  - Calls that share a handle must be ordered on one stream (they share the
 *    planning workspace).  Calls that overlap on the GPU and write the same
 *    caller buffers race.
 */
#ifndef MOONEP_H
#define MOONEP_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MOONEP_API __attribute__((visibility("default")))
#else
#define MOONEP_API
#endif

/* Same type as cudaStream_t; declared here so callers need no CUDA header. */
typedef struct CUstream_st *moonep_stream_t;

/* host-side error codes (return values) */
#define MOONEP_OK 0
#define MOONEP_ERR_NULL (-1)   /* a required pointer is NULL */
#define MOONEP_ERR_CONFIG (-2) /* the configuration is rejected (see moonep_create) */
#define MOONEP_ERR_ALIGN (-3)  /* a tensor pointer is not 16-byte aligned */
#define MOONEP_ERR_CUDA (-4)   /* a CUDA runtime call failed (allocation or launch) */
#define MOONEP_ERR_SIZE (-5)   /* a size argument is outside the supported range */
#define MOONEP_ERR_DEVICE (-6) /* an operand is not memory of the handle's own GPU */

/* device-side status bits, OR-ed into plan->status */
#define MOONEP_STATUS_BAD_EXPERT 1     /* an expert id outside [0, E) (e.g. a -1 mask) */
#define MOONEP_STATUS_DUP_EXPERT 2     /* an expert picked twice by one token */
#define MOONEP_STATUS_COUNT_MISMATCH 4 /* tokens_per_expert differs from the picks */
#define MOONEP_STATUS_BAD_PLAN 8       /* a plan index pointed outside its buffer; skipped */
#define MOONEP_STATUS_TIMEOUT 16       /* the planner's grid barrier gave up waiting (see moonep_set_plan_barrier) */

/* Supported ranges (moonep_create checks them). */
#define MOONEP_MAX_R 64
#define MOONEP_MAX_E 4096
#define MOONEP_MAX_K 32
#define MOONEP_MAX_PROJ 8

/*
 * Construction parameters; they follow the README's
 * Buffer(S, H, K, E, num_ep_ranks, num_sms, token_padding, B) ("API guide").
 *   S, H, K, E, R, B : as in the notation above.  H % 8 == 0 (rows move as
 *                      16-byte vectors).  E % R == 0.  1 <= K <= min(E, 32).
 *   token_padding    : every non-empty row is padded to a multiple of it.
 *   num_sms          : SMs the copy kernels may occupy; 0 = all of them.
 *   mode             : 0 = training, which needs B >= E/R because copies come
 *                      from at most one remote home group per rank; 1 =
 *                      inference, any B >= 0, copied experts past the first B
 *                      are read from their home rows ("How to set B"); 2 =
 *                      inference where the B slots go to the received experts
 *                      with the most picks on the rank (ties: lower id), so
 *                      the home-row overflow carries the fewest tokens (the
 *                      README leaves this choice open); 3 = training with
 *                      the fewest copies: a home group's picks are ordered
 *                      by expert pick count (ascending, ties by id) instead
 *                      of by id, so a donor gives away its largest experts
 *                      and every recipient's range spans as few experts as
 *                      the donation allows (B >= E/R, as in mode 0).  Slots
 *                      are in ascending expert id in every mode.
 */
typedef struct {
    int32_t S, H, K, E, R, B, token_padding, num_sms, mode;
} moonep_config_t;

/*
 * A plan: caller-owned DEVICE arrays, written by moonep_plan and read by every
 * other call.  The README keeps the plan ("MoonEPCommPlan") for prefetch,
 * combine and both backward passes ("dispatch fwd").
 *   dst         [R,S,K] int32  slot of pick (r,t,k): dest_rank*NvS + row start + position
 *   cu_seqlens  [R,E+B] int32  inclusive padded end offset of each row of each rank
 *   row_counts  [R,E+B] int32  real picks per row
 *   slot_expert [R,B]   int32  expert held by prefetch slot b of rank r, -1 = unused
 *   counts      [R,E]   int32  picks of expert e made on source rank r
 *   assign      [R,4]   int32  per rank: picks of its own group it keeps, donor
 *                              group it takes copies from (-1 none), start and
 *                              length of the range it takes in that group's
 *                              sequence
 *   maxvio      [1]     float  max_e(T_e / T_bar) - 1 ("Performance")
 *   status      [1]     int32  0 or MOONEP_STATUS_* bits
 */
typedef struct {
    int32_t *dst;
    int32_t *cu_seqlens;
    int32_t *row_counts;
    int32_t *slot_expert;
    int32_t *counts;
    int32_t *assign;
    float *maxvio;
    int32_t *status;
} moonep_plan_t;

typedef struct moonep_handle *moonep_handle_t;

/*
 * Element counts of the plan arrays for a configuration, so that a caller can
 * allocate a moonep_plan_t before any handle exists (the README's
 * "MoonEPCommPlan", "dispatch fwd", is kept by the caller for the later
 * calls).  Every count is in elements of the array's own type:
 *   dst          R*S*K (group plan) or S*K (one rank's plan, one_rank != 0)
 *   cu_seqlens   R*(E+B)            row_counts  R*(E+B)
 *   slot_expert  R*B (0 when B = 0; the pointer may then be NULL)
 *   counts       R*E                assign      R*4
 *   maxvio       1 float            status      1 int32
 *   nvs          NvS, the slots of one rank's dispatch buffer (moonep_nvs):
 *                hidden_nvs holds R*NvS rows of H bf16, route_weights_nvs
 *                R*NvS floats (one rank's buffers: NvS each)
 * Host only: no device is touched.  Returns MOONEP_ERR_NULL for a NULL
 * argument, or cfg's moonep_create error (MOONEP_ERR_CONFIG) with *out
 * zeroed.
 */
typedef struct {
    int64_t dst, cu_seqlens, row_counts, slot_expert, counts, assign, maxvio, status, nvs;
} moonep_plan_sizes_t;
MOONEP_API int moonep_plan_sizes(const moonep_config_t *cfg, int32_t one_rank, moonep_plan_sizes_t *out);

/*
 * Validate cfg and create a handle on the current device; allocates the
 * planning workspace (cudaMalloc, a few hundred KB).  Rejects (ERR_CONFIG):
 * E % R != 0, K > E, H % 8 != 0, training with B < E/R, sizes past the
 * MOONEP_MAX_* limits, R*S*K or R*NvS at or above 2^31, a mode outside 0..3.
 * *out is NULL on error.
 */
MOONEP_API int moonep_create(const moonep_config_t *cfg, moonep_handle_t *out);

/* Free the handle and its workspace.  NULL is accepted.  The caller makes sure
 * no call on the handle is still running on the GPU. */
MOONEP_API int moonep_destroy(moonep_handle_t h);

/* NvS = roundup(S*K + 2*(E/R)*(token_padding-1), token_padding): the slots of
 * one rank's static buffer (README notation "NvS").  Negative on a NULL handle. */
MOONEP_API int64_t moonep_nvs(moonep_handle_t h);

/* Copy the handle's configuration into *out. */
MOONEP_API int moonep_get_config(moonep_handle_t h, moonep_config_t *out);

/*
 * Plan one layer: read the router output of all R ranks and write *plan.
 * README "dispatch fwd" (planning part), "Performance" item 2 (online
 * planning); the planning rule itself is this library's reading of the pages
 * (documented in the repository's design notes and in oracle/moonep_oracle.c).
 *   topk              [R,S,K] int32  expert ids picked by each token
 *   tokens_per_expert [R,E]   int32  the router's local counts, or NULL; when
 *                                    given, checked against the picks
 * Every rank ends with exactly S*K real slots.  Device-side errors: BAD_EXPERT,
 * DUP_EXPERT, COUNT_MISMATCH (then the other plan arrays are unspecified).
 */
MOONEP_API int moonep_plan(moonep_handle_t h, const int32_t *topk, const int32_t *tokens_per_expert,
                const moonep_plan_t *plan, moonep_stream_t stream);

/*
 * Fused-permute dispatch (README "dispatch fwd"; "combine bwd" is the same call
 * on the output gradient with the saved plan): every token row is written
 * straight into its K expert-grouped slots.
 *   hidden            [R,S,H]  bf16   token rows
 *   route_weights     [R,S,K]  fp32   or NULL
 *   hidden_nvs        [R,NvS,H] bf16  written at the real slots only; padding
 *                                     slots are left as they were
 *   route_weights_nvs [R,NvS]  fp32   or NULL; written at the real slots
 * hidden, hidden_nvs: 16-byte aligned.
 */
MOONEP_API int moonep_dispatch(moonep_handle_t h, const moonep_plan_t *plan, const void *hidden,
                    const float *route_weights, void *hidden_nvs, float *route_weights_nvs,
                    moonep_stream_t stream);

/*
 * Combine (README "combine fwd"; "dispatch bwd" calls it with
 * route_weights_nvs = NULL): out[r,t,:] = bf16(sum_k w_k * y[dst[r,t,k],:]),
 * accumulated in fp32 in k order, rounded to nearest even.
 *   hidden_nvs        [R,NvS,H] bf16  expert output y
 *   route_weights_nvs [R,NvS]   fp32  or NULL for the unweighted sum (w_k = 1)
 *   out               [R,S,H]   bf16
 *   gathered_weights  [R,S,K]   fp32  or NULL; = route_weights_nvs[dst]
 * hidden_nvs, out: 16-byte aligned.
 */
MOONEP_API int moonep_combine(moonep_handle_t h, const moonep_plan_t *plan, const void *hidden_nvs,
                   const float *route_weights_nvs, void *out, float *gathered_weights,
                   moonep_stream_t stream);

/*
 * Weight prefetch (README "Weight buffer", "dispatch fwd" prefetch_weight):
 * for each projection p and each used slot (r,b), pool[p][r][b] = W[p][e] with
 * e = slot_expert[r][b].  Each expert is read once and written to every slot
 * holding it.
 *   weights[p] [E,H,Hp]   bf16  the home experts (rows [0,E) of the pages'
 *                               [E+B,H,H'] tensor)
 *   pool[p]    [R,B,H,Hp] bf16  rank r's rows [E,E+B)
 * 1 <= n_proj <= MOONEP_MAX_PROJ; all pointers 16-byte aligned.
 */
MOONEP_API int moonep_prefetch_weight(moonep_handle_t h, const moonep_plan_t *plan, int32_t n_proj,
                           const void *const *weights, void *const *pool, int64_t Hp,
                           moonep_stream_t stream);

/*
 * Grad-slot reduction (README "Grad buffer", "dispatch bwd" reduce_grad): for
 * each projection and each expert e held by at least one slot,
 * grads[p][e] += sum of reduce_buffers[p][r][b] over the slots holding e, in
 * ascending (r,b) order in fp32; then every consumed slot is set to +0.0 for
 * the next microbatch.  Unused slots are untouched.
 *   grads[p]          [E,H,Hp]   fp32  the home experts' parameter gradients
 *   reduce_buffers[p] [R,B,H,Hp] fp32  all ranks' slot gradients
 * 1 <= n_proj <= MOONEP_MAX_PROJ; all pointers 16-byte aligned.
 */
MOONEP_API int moonep_reduce_grad(moonep_handle_t h, const moonep_plan_t *plan, int32_t n_proj,
                       float *const *grads, float *const *reduce_buffers, int64_t Hp,
                       moonep_stream_t stream);

/*
 * The VM group GEMM that consumes a dispatched layer (README "Integration":
 * one [E+B, H, H'] weight tensor per projection, with cu_seqlens selecting
 * the expert row of every token segment; "Weight buffer": rows [0, E) are the
 * home experts, rows [E, E+B) the rank's prefetch slots).  For every rank r
 * and every row i of its plan with row_counts[r][i] > 0:
 *   y_nvs[r, s_i : s_i + pad(n_i), :] = x_nvs[r, s_i : s_i + pad(n_i), :] @ Wi
 * where s_i = cu_seqlens[r][i] - pad(n_i) is the row's first slot, and
 * Wi = weights[i] for i < E (home rows, and inference overflow rows, which
 * read the home expert), pool[r][i - E] for slot rows.  fp32 accumulation on
 * the tensor cores, bf16 output rounded to nearest even.  Padding slots are
 * multiplied too (their contents are unspecified); slots after a rank's last
 * row are not written.
 *   x_nvs   [R,NvS,H]  bf16  the dispatched buffer
 *   weights [E,H,Hp]   bf16  the home experts
 *   pool    [R,B,H,Hp] bf16  every rank's prefetch slots (NULL allowed if B=0)
 *   y_nvs   [R,NvS,Hp] bf16  output
 * Requires token_padding % 128 == 0 (a 128-row tile never spans two rows),
 * H % 64 == 0 and Hp % 256 == 0, else MOONEP_ERR_SIZE; pointers 16-byte
 * aligned.  Every operand must be memory of the handle's own GPU: the kernel
 * feeds its tiles through TMA into two-SM clusters, which never read another
 * GPU's memory.  A pointer that CUDA reports on another device (a peer or
 * IPC mapping) gives MOONEP_ERR_DEVICE before anything is launched.  A failed
 * plan (plan->status != 0) computes nothing.
 */
MOONEP_API int moonep_group_gemm(moonep_handle_t h, const moonep_plan_t *plan, const void *x_nvs,
                                 const void *weights, const void *pool, void *y_nvs, int64_t Hp,
                                 moonep_stream_t stream);

/*
 * ---- One rank of a real EP group ----
 *
 * On R GPUs each rank holds only its own router output, and the R dispatched
 * buffers live on R devices.  README "dispatch fwd" gives every rank its
 * local tokens_per_expert [E]; gathered from all ranks (an all-gather of
 * R*E int32, which the caller runs, e.g. with NCCL), they are all the
 * planner needs besides the rank's own picks: every rank then derives the
 * same layout, and each writes dst for its own picks only.  Dispatch and
 * combine take the R ranks' buffers as a table of device pointers (peer
 * mappings of the other ranks' memory on a real group; R separate
 * allocations on one GPU).  The slot encoding is the group one: dst =
 * q*NvS + i is row i of rank q's buffer.  The calls share the handle's
 * conventions; moonep_plan_rank has its own planning workspace in the
 * handle, so it may alternate with moonep_plan on one stream.
 */

/*
 * Plan rank `rank`'s share of one layer.
 *   topk        [S,K] int32  the rank's own picks
 *   counts_all  [R,E] int32  every rank's router counts, row q = rank q's
 *                            tokens_per_expert (the gathered table)
 *   plan        as for moonep_plan, except dst: [S,K], the slots of this
 *               rank's picks.  cu_seqlens, row_counts, slot_expert, assign
 *               and maxvio hold the whole group's layout (identical on every
 *               rank, and equal to moonep_plan's for the same routing);
 *               counts is a copy of counts_all.
 * Result: equal to the rank's slice of moonep_plan's plan for the group's
 * picks.  Device-side errors: BAD_EXPERT and DUP_EXPERT in the rank's picks;
 * COUNT_MISMATCH when row `rank` of counts_all differs from the picks, or
 * when any row holds a negative count or does not sum to S*K (then the other
 * plan arrays are unspecified).  A rank sees only its own picks: a group is consistent
 * when every rank's status is 0 (combine them, e.g. with an all-reduce).
 * ERR_SIZE when rank is outside [0, R).
 */
MOONEP_API int moonep_plan_rank(moonep_handle_t h, int32_t rank, const int32_t *topk, const int32_t *counts_all,
                                const moonep_plan_t *plan, moonep_stream_t stream);

/*
 * Dispatch of one rank's tokens with a plan from moonep_plan_rank: every row
 * goes straight to its K slots in the destination ranks' buffers.
 *   hidden            [S,H] bf16   the rank's token rows (16-byte aligned)
 *   route_weights     [S,K] fp32   or NULL
 *   hidden_nvs        R device pointers (host array): rank q's [NvS,H] bf16
 *                     buffer, each 16-byte aligned; written at real slots only
 *   route_weights_nvs R device pointers to rank q's [NvS] fp32, or NULL; with
 *                     route_weights given, written at the real slots
 * The tables are read on the host at the call; the buffers they name must
 * stay valid until the launch completes.
 */
MOONEP_API int moonep_dispatch_rank(moonep_handle_t h, const moonep_plan_t *plan, const void *hidden,
                                    const float *route_weights, void *const *hidden_nvs,
                                    float *const *route_weights_nvs, moonep_stream_t stream);

/*
 * Combine of one rank's tokens with a plan from moonep_plan_rank:
 * out[t,:] = bf16(sum_k w_k * y[dst[t,k]]) in fp32, k order, as moonep_combine.
 *   hidden_nvs        R device pointers: rank q's expert output [NvS,H] bf16
 *   route_weights_nvs R device pointers to rank q's [NvS] fp32, or NULL for
 *                     the unweighted sum
 *   out               [S,H] bf16 (16-byte aligned)
 *   gathered_weights  [S,K] fp32 or NULL; = the weight of each slot read
 */
MOONEP_API int moonep_combine_rank(moonep_handle_t h, const moonep_plan_t *plan, const void *const *hidden_nvs,
                                   const float *const *route_weights_nvs, void *out, float *gathered_weights,
                                   moonep_stream_t stream);

/*
 * Weight prefetch of one rank (README "Weight buffer"): for each projection p
 * and each used slot b of rank `rank`, pool[p][b] = the home copy of expert
 * e = slot_expert[rank][b], read from its home rank q = e / G.
 *   weights[p*R + q] [G,H,Hp] bf16  rank q's home experts of projection p
 *                                   (peer mappings on a real group)
 *   pool[p]          [B,H,Hp] bf16  this rank's prefetch slots
 * The plan is this rank's (moonep_plan_rank) or the group's: only its
 * slot_expert is read.  Same checks as moonep_prefetch_weight; ERR_SIZE when
 * rank is outside [0, R).  Bit-identical to rank `rank`'s slots after
 * moonep_prefetch_weight.
 */
MOONEP_API int moonep_prefetch_weight_rank(moonep_handle_t h, const moonep_plan_t *plan, int32_t rank, int32_t n_proj,
                                           const void *const *weights, void *const *pool, int64_t Hp,
                                           moonep_stream_t stream);

/*
 * Grad-slot reduction of one home rank (README "Grad buffer"): for each
 * projection and each home expert e of rank `rank` held by at least one slot
 * of any rank, grads[p][e - rank*G] += the slots holding e, in ascending
 * (rank, slot) order in fp32; then those slots are set to +0.0.
 *   grads[p]                 [G,H,Hp] fp32  this rank's home experts' gradients
 *   reduce_buffers[p*R + q]  [B,H,Hp] fp32  rank q's slot gradients (peer
 *                                           mappings on a real group); read,
 *                                           and the consumed slots zeroed
 * The R ranks' calls touch disjoint slots (each slot holds one expert, whose
 * home is one rank).  Bit-identical to the home rank's share of
 * moonep_reduce_grad.
 */
MOONEP_API int moonep_reduce_grad_rank(moonep_handle_t h, const moonep_plan_t *plan, int32_t rank, int32_t n_proj,
                                       float *const *grads, float *const *reduce_buffers, int64_t Hp,
                                       moonep_stream_t stream);

/*
 * ---- Sharing rank buffers between processes ----
 *
 * With one process per rank, every rank's dispatch buffer, weight rows and
 * grad slots must be mapped into its peers (the README's ranks reach them
 * through one symmetric device mapping: "Weight buffer", "Grad buffer";
 * MarkTechPost, "Memory contract").  A rank exports the device allocation
 * behind each of its buffers; the other ranks import it and put the pointer
 * in the tables of the per-rank calls above.  Works between processes on one
 * GPU and between GPUs of a node (CUDA IPC; the importer's current device is
 * the one that accesses the memory).
 *
 * The per-rank calls keep bulk (TMA) copies to this GPU's own memory: when a
 * table holds another GPU's memory, moonep_dispatch_rank,
 * moonep_prefetch_weight_rank and moonep_reduce_grad_rank use their
 * plain-load/store kernels for that call (the answer per table is cached on
 * the handle).  No call waits on another rank: the caller orders the ranks'
 * phases (e.g. a barrier after every rank's dispatch, before any combine).
 */
typedef struct {
    unsigned char handle[64]; /* the exporting allocation's IPC handle */
    int64_t offset;           /* the exported pointer's offset in that allocation */
    int64_t bytes;            /* the allocation's size */
} moonep_ipc_handle_t;

/* Export the allocation holding the device pointer `ptr` (memory from
 * cudaMalloc, e.g. a caching allocator's block; not VMM memory).  The handle
 * is plain bytes: send it to the other processes by any channel. */
MOONEP_API int moonep_ipc_export(const void *ptr, moonep_ipc_handle_t *out);

/* Map another process's export into this process, on the current device:
 * *out = the exported pointer here.  Exports from one allocation share one
 * mapping (reference-counted).  Not for this process's own exports (CUDA
 * cannot reopen them; use the pointer itself).  ERR_SIZE for an offset
 * outside the allocation; ERR_CUDA when CUDA refuses the mapping. */
MOONEP_API int moonep_ipc_import(const moonep_ipc_handle_t *h, void **out);

/* Release one import (the pointer moonep_ipc_import returned); the mapping
 * closes with its last import.  No kernel may still use it.  ERR_SIZE when
 * ptr is not an import of this process. */
MOONEP_API int moonep_ipc_close(void *ptr);

/*
 * moonep_plan without a handle and without allocating: the same plan as
 * moonep_plan for the same cfg and inputs.  (This entry point has no
 * counterpart on the pages; it exists for callers that cannot call cudaMalloc
 * in the layer path, e.g. when a caching allocator or a start-up reservation
 * owns all device memory, where a raw cudaMalloc would break that budget and
 * may synchronise the device.)
 *
 * Its planning workspace is one fixed array of MOONEP_NOALLOC_SCRATCH_BYTES in
 * device memory, part of the library image: every GPU that loads the library
 * holds it until the process exits.  A cfg whose workspace does not fit is
 * rejected with MOONEP_ERR_SIZE (the training shape R=8, S=4096, K=8, E=256
 * needs about 150 KB).  The call allocates nothing (no cudaMalloc, cudaFree or
 * allocating library routine); it clears the part of the array that must
 * start at zero with cudaMemsetAsync on `stream`.
 *
 * The first call on a device looks the array's device address up
 * (cudaGetSymbolAddress, with that device current) and keeps it for the
 * life of the process; make that first call before any stream capture, and
 * do not use the library across a cudaDeviceReset (the kept address, like
 * the kernel attributes every entry point sets once per device, would be
 * stale).  All calls share the one array: calls that
 * overlap on the GPU race, so order them on one stream.  Arguments, layouts
 * and status bits are those of moonep_plan; cfg is checked as moonep_create
 * checks it.
 */
#define MOONEP_NOALLOC_SCRATCH_BYTES (1 << 20)
MOONEP_API int moonep_plan_noalloc(const moonep_config_t *cfg, const int32_t *topk,
                                   const int32_t *tokens_per_expert, const moonep_plan_t *plan,
                                   moonep_stream_t stream);

/* Read plan->status into *status (host).  Synchronises `stream`.  This is
 * the status read of the library's scope (named moonep_plan_status there),
 * with the stream made explicit; moonep_plan_status below is the stream-less
 * form. */
MOONEP_API int moonep_read_status(const moonep_plan_t *plan, int32_t *status, moonep_stream_t stream);

/* Read plan->status into *status after waiting for all work on the current
 * device (cudaDeviceSynchronize), whatever stream wrote it. */
MOONEP_API int moonep_plan_status(const moonep_plan_t *plan, int32_t *status);

/*
 * Fault injection for tests, on the host side (nothing faults on the GPU).
 * The planner's grid barrier of handle h (moonep_plan and moonep_plan_rank)
 * gives up after max_polls polls (0 restores the default, about 2 s of
 * polling) and, with missing > 0, also waits for `missing` block arrivals
 * that never come, so that every block gives up.  The call then sets
 * MOONEP_STATUS_TIMEOUT in plan->status and writes no other plan array;
 * later calls on the plan do nothing.  A timeout caused this way leaves the
 * handle usable: restore (0, 0) and plan again.  After a timeout of any other
 * cause, destroy the handle.  ERR_SIZE when missing is outside [0, 2^20].
 */
MOONEP_API int moonep_set_plan_barrier(moonep_handle_t h, uint32_t max_polls, int32_t missing);

/* Static description of a MOONEP_ERR_* code. */
MOONEP_API const char *moonep_error_string(int code);

/* Name and text of the CUDA error behind the calling thread's last
 * MOONEP_ERR_CUDA ("no error" if none yet).  Valid until the next failing call
 * on this thread. */
MOONEP_API const char *moonep_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* MOONEP_H */
