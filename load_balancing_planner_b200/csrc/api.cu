// C ABI of libmoonep: host-side validation, the handle, and kernel launches.
// Every entry point is declared and documented in include/moonep.h.
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>
#include <new>

#include "moonep_internal.cuh"

namespace moonep {
cudaError_t weights_set_smem_limit(size_t bytes);
size_t weights_static_smem_bytes();
}  // namespace moonep

using namespace moonep;

struct moonep_handle {
    moonep_config_t cfg;
    Dims d;
    int device;
    int sms;            // SMs the copy kernels may occupy
    int grid_plan;      // planner blocks (all resident)
    int grid_dispatch;  // whole waves over those SMs
    bool bulk_dispatch; // rows moved with bulk copies through shared memory
    int grid_combine;
    int grid_weights;
    void *ws_mem;
    Workspace ws;
    Workspace ws_rank;  // one-rank planning (moonep_plan_rank): its own barrier counter and parity slots
    uint32_t barrier_polls;     // the planner's grid-barrier poll limit
    uint32_t barrier_withheld;  // arrivals that never come (fault injection for tests; normally 0)
    int grid_dispatch_vec;      // the vector dispatch kernel's grid (rank tables on other GPUs)
    // the last pointer tables checked for memory on other GPUs, and the answers
    static constexpr int kRemoteCache = 4;
    std::mutex remote_mu;
    int remote_next;
    int remote_n[kRemoteCache];
    const void *remote_tab[kRemoteCache][MOONEP_MAX_PROJ * MOONEP_MAX_R];
    int remote_ans[kRemoteCache];
};

// Does any pointer of a rank call's table live on another GPU?  Such tables
// (peer mappings of a real group on several GPUs) are served with plain
// loads and stores; bulk copies are kept to this GPU's own memory.  The
// answers for the last few tables are kept, so a caller that passes the same
// tables every layer pays for the pointer queries once.
static bool table_is_remote(moonep_handle_t h, const void *const *tab, int n) {
    std::lock_guard<std::mutex> lock(h->remote_mu);
    for (int c = 0; c < moonep_handle::kRemoteCache; ++c)
        if (n == h->remote_n[c] && memcmp(tab, h->remote_tab[c], sizeof(void *) * (size_t)n) == 0)
            return h->remote_ans[c] != 0;
    int remote = 0;
    for (int i = 0; i < n; ++i)
        if (on_other_device(tab[i], h->device) == 1) remote = 1;
    const int c = h->remote_next;
    h->remote_next = (c + 1) % moonep_handle::kRemoteCache;
    h->remote_n[c] = n;
    memcpy(h->remote_tab[c], tab, sizeof(void *) * (size_t)n);
    h->remote_ans[c] = remote;
    return remote != 0;
}

// Handle workspace: [group planning][group GEMM pair table][one-rank planning]
static size_t pair_table_offset(const Dims &d) { return (workspace_bytes(d) + 255) / 256 * 256; }
static size_t rank_ws_offset(const Dims &d) {
    return (pair_table_offset(d) + gemm_table_bytes(d) + 255) / 256 * 256;
}

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static thread_local char g_last_error[256] = "no error";

namespace moonep {
int fail_cuda(cudaError_t e) {
    snprintf(g_last_error, sizeof(g_last_error), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
    return MOONEP_ERR_CUDA;
}
}  // namespace moonep

extern "C" const char *moonep_last_error(void) { return g_last_error; }

extern "C" const char *moonep_error_string(int code) {
    switch (code) {
        case MOONEP_OK: return "ok";
        case MOONEP_ERR_NULL: return "a required pointer is NULL";
        case MOONEP_ERR_CONFIG: return "configuration rejected";
        case MOONEP_ERR_ALIGN: return "tensor pointer not 16-byte aligned";
        case MOONEP_ERR_CUDA: return "CUDA runtime call failed";
        case MOONEP_ERR_SIZE: return "size argument out of the supported range";
        case MOONEP_ERR_DEVICE: return "operand not in the handle's own GPU memory";
        default: return "unknown moonep error";
    }
}

namespace moonep {
int64_t nvs_of(const moonep_config_t &c) {
    const int64_t C = (int64_t)c.S * c.K, G = c.E / c.R, tp = c.token_padding;
    const int64_t n = C + 2 * G * (tp - 1);
    return (n + tp - 1) / tp * tp;
}

int check_config(const moonep_config_t &c) {
    if (c.R < 1 || c.R > MOONEP_MAX_R) return MOONEP_ERR_CONFIG;
    if (c.E < 1 || c.E > MOONEP_MAX_E || c.E % c.R != 0) return MOONEP_ERR_CONFIG;
    if (c.K < 1 || c.K > MOONEP_MAX_K || c.K > c.E) return MOONEP_ERR_CONFIG;
    if (c.S < 1 || c.H < 8 || c.H % 8 != 0) return MOONEP_ERR_CONFIG;
    if (c.B < 0 || c.token_padding < 1 || c.num_sms < 0) return MOONEP_ERR_CONFIG;
    if (c.mode < 0 || c.mode > 3) return MOONEP_ERR_CONFIG;
    if ((c.mode == 0 || c.mode == 3) && c.B < c.E / c.R) return MOONEP_ERR_CONFIG;
    if ((int64_t)c.R * c.B > 4096 || c.E + (int64_t)c.B > (int64_t)1 << 20) return MOONEP_ERR_CONFIG;
    if ((int64_t)c.R * c.S * c.K >= ((int64_t)1 << 31)) return MOONEP_ERR_CONFIG;
    if (c.token_padding > (1 << 20)) return MOONEP_ERR_CONFIG;
    if ((int64_t)c.R * nvs_of(c) >= ((int64_t)1 << 31)) return MOONEP_ERR_CONFIG;
    return MOONEP_OK;
}

// Raise the dynamic shared-memory limit of the kernels that need more than
// 48 KB to the device's maximum, once per device (a per-function attribute:
// setting it per handle would let a later small handle lower it below an
// earlier large handle's need).
int prepare_device(int device) {
    static std::mutex mu;
    static bool done[kMaxDevices] = {};
    if (device < 0 || device >= kMaxDevices) return MOONEP_ERR_SIZE;
    std::lock_guard<std::mutex> lock(mu);
    if (done[device]) return MOONEP_OK;
    int optin = 0;
    cudaError_t e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device);
    if (e == cudaSuccess) e = plan_set_smem_limit((size_t)optin - plan_static_smem_bytes());
    if (e == cudaSuccess) e = weights_set_smem_limit((size_t)optin - weights_static_smem_bytes());
    if (e == cudaSuccess) e = dispatch_bulk_set_smem_limit((size_t)optin - 1024);
    if (e == cudaSuccess) e = gemm_set_smem_limit();
    if (e != cudaSuccess) return fail_cuda(e);
    done[device] = true;
    return MOONEP_OK;
}

// Planner dimensions for cfg on `device`: every block of the cooperative
// launch must be resident, so the chunk grows until R * ceil(S / ct) blocks
// fit; the counting warps shrink until their per-expert tables fit.
int plan_dims(const moonep_config_t &cfg, int device, Dims *out, int *grid) {
    Dims d;
    memset(&d, 0, sizeof(d));
    d.S = cfg.S; d.H = cfg.H; d.K = cfg.K; d.E = cfg.E; d.R = cfg.R; d.B = cfg.B;
    d.tp = cfg.token_padding; d.mode = cfg.mode;
    d.G = d.E / d.R;
    d.NR = d.E + d.B;
    d.nvs = (int)nvs_of(cfg);
    int sms = 0, optin = 0;
    cudaError_t e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device);
    if (e != cudaSuccess) return fail_cuda(e);
    const size_t smem_max = (size_t)optin - plan_static_smem_bytes();
    d.ct = d.S < kChunkTokensMin ? d.S : kChunkTokensMin;
    for (int iter = 0; iter < 8; ++iter) {
        d.nch = (d.S + d.ct - 1) / d.ct;
        // the optional layout tables only where they still fit
        d.cw = 1;
        d.fast2 = 1;
        d.xtab = 1;
        if (plan_smem_bytes(d) > smem_max) d.xtab = 0;
        if (plan_smem_bytes(d) > smem_max) d.fast2 = 0;
        d.cw = kPlanWarps;
        while (d.cw > 1 && plan_smem_bytes(d) > smem_max) d.cw /= 2;
        if (plan_smem_bytes(d) > smem_max || (int64_t)d.ct * d.K > 65535) return MOONEP_ERR_CONFIG;
        const int cap = plan_blocks_per_sm(d) * sms;
        if (d.R * d.nch <= cap) {
            *out = d;
            *grid = d.R * d.nch;
            return MOONEP_OK;
        }
        if (cap < d.R) return MOONEP_ERR_CONFIG;
        const int per_rank = cap / d.R;
        int ct = (d.S + per_rank - 1) / per_rank;
        ct = (ct + 31) / 32 * 32;
        d.ct = ct > d.ct ? ct : d.ct + 32;
    }
    return MOONEP_ERR_CONFIG;
}

bool plan_ok(const moonep_plan_t *p) {
    return p && p->dst && p->cu_seqlens && p->row_counts && p->counts && p->assign && p->maxvio && p->status;
}
}  // namespace moonep


extern "C" int moonep_create(const moonep_config_t *cfg, moonep_handle_t *out) {
    if (!out) return MOONEP_ERR_NULL;
    *out = nullptr;
    if (!cfg) return MOONEP_ERR_NULL;
    const int rc = check_config(*cfg);
    if (rc != MOONEP_OK) return rc;

    moonep_handle *h = new (std::nothrow) moonep_handle();
    if (!h) return MOONEP_ERR_CUDA;
    h->cfg = *cfg;
    Dims &d = h->d;
    cudaError_t e = cudaGetDevice(&h->device);
    int sms = 0;
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, h->device);
    if (e != cudaSuccess) { delete h; return fail_cuda(e); }
    h->sms = (cfg->num_sms > 0 && cfg->num_sms < sms) ? cfg->num_sms : sms;
    int rc2 = prepare_device(h->device);
    if (rc2 == MOONEP_OK) rc2 = plan_dims(*cfg, h->device, &d, &h->grid_plan);
    if (rc2 != MOONEP_OK) { delete h; return rc2; }

    h->bulk_dispatch = dispatch_use_bulk(d);
    h->grid_dispatch = h->sms * (h->bulk_dispatch ? dispatch_bulk_blocks_per_sm(d) : dispatch_blocks_per_sm(d.K));
    h->grid_dispatch_vec = h->sms * dispatch_blocks_per_sm(d.K);
    h->grid_combine = h->sms * combine_blocks_per_sm(d.K);
    h->grid_weights = h->sms * weights_blocks_per_sm();

    const size_t wsb = rank_ws_offset(d) + workspace_bytes(d);
    if ((e = cudaMalloc(&h->ws_mem, wsb)) != cudaSuccess) { delete h; return fail_cuda(e); }
    if ((e = cudaMemset(h->ws_mem, 0, wsb)) != cudaSuccess) {
        cudaFree(h->ws_mem);
        delete h;
        return fail_cuda(e);
    }
    carve_workspace(d, h->ws_mem, &h->ws);
    carve_workspace(d, static_cast<char *>(h->ws_mem) + rank_ws_offset(d), &h->ws_rank);
    h->barrier_polls = kBarrierPolls;
    h->barrier_withheld = 0;
    *out = h;
    return MOONEP_OK;
}

extern "C" int moonep_destroy(moonep_handle_t h) {
    if (!h) return MOONEP_OK;
    cudaError_t e = cudaSuccess;
    if (h->ws_mem) e = cudaFree(h->ws_mem);
    delete h;
    return e == cudaSuccess ? MOONEP_OK : MOONEP_ERR_CUDA;
}

extern "C" int moonep_set_plan_barrier(moonep_handle_t h, uint32_t max_polls, int32_t missing) {
    if (!h) return MOONEP_ERR_NULL;
    if (missing < 0 || missing > (1 << 20)) return MOONEP_ERR_SIZE;
    h->barrier_polls = max_polls ? max_polls : kBarrierPolls;
    h->barrier_withheld = (uint32_t)missing;
    return MOONEP_OK;
}

extern "C" int64_t moonep_nvs(moonep_handle_t h) { return h ? (int64_t)h->d.nvs : MOONEP_ERR_NULL; }

extern "C" int moonep_get_config(moonep_handle_t h, moonep_config_t *out) {
    if (!h || !out) return MOONEP_ERR_NULL;
    *out = h->cfg;
    return MOONEP_OK;
}

extern "C" int moonep_plan(moonep_handle_t h, const int32_t *topk, const int32_t *tokens_per_expert,
                           const moonep_plan_t *plan, moonep_stream_t stream) {
    if (!h || !topk || !plan_ok(plan)) return MOONEP_ERR_NULL;
    if (h->d.B > 0 && !plan->slot_expert) return MOONEP_ERR_NULL;
    PlanArgs a;
    a.d = h->d;
    a.topk = topk;
    a.tpe = tokens_per_expert;
    a.src_rank = -1;
    a.counts_all = nullptr;
    a.plan = *plan;
    a.ws = h->ws;
    a.polls = h->barrier_polls;
    a.withheld = h->barrier_withheld;
    const cudaError_t e = launch_plan(a, h->grid_plan, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOONEP_OK : fail_cuda(e);
}

extern "C" int moonep_plan_rank(moonep_handle_t h, int32_t rank, const int32_t *topk, const int32_t *counts_all,
                                const moonep_plan_t *plan, moonep_stream_t stream) {
    if (!h || !topk || !counts_all || !plan_ok(plan)) return MOONEP_ERR_NULL;
    if (h->d.B > 0 && !plan->slot_expert) return MOONEP_ERR_NULL;
    if (rank < 0 || rank >= h->d.R) return MOONEP_ERR_SIZE;
    PlanArgs a;
    a.d = h->d;
    a.topk = topk;
    a.tpe = nullptr;
    a.src_rank = rank;
    a.counts_all = counts_all;
    a.plan = *plan;
    a.ws = h->ws_rank;
    a.polls = h->barrier_polls;
    a.withheld = h->barrier_withheld;
    const cudaError_t e = launch_plan(a, h->d.nch, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOONEP_OK : fail_cuda(e);
}

static CopyArgs copy_args(moonep_handle_t h, const moonep_plan_t *plan) {
    CopyArgs a;
    memset(&a, 0, sizeof(a));
    a.d = h->d;
    a.dst = plan->dst;
    a.status = plan->status;
    a.status_rw = plan->status;
    a.ntok = (int64_t)h->d.R * h->d.S;
    return a;
}

// One rank's call: its own S tokens, the R ranks' buffers through tables.
// Every buffer pointer is required and 16-byte aligned; the weight tables
// are all given or all NULL.
static int peer_tables(moonep_handle_t h, void *const *bufs, float *const *wbufs, CopyArgs *a) {
    if (!bufs) return MOONEP_ERR_NULL;
    a->ntok = h->d.S;
    a->peered = 1;
    for (int q = 0; q < h->d.R; ++q) {
        if (!bufs[q] || (wbufs && !wbufs[q])) return MOONEP_ERR_NULL;
        if (!aligned16(bufs[q])) return MOONEP_ERR_ALIGN;
        a->peer[q] = bufs[q];
        a->peer_w[q] = wbufs ? wbufs[q] : nullptr;
    }
    return MOONEP_OK;
}

extern "C" int moonep_dispatch(moonep_handle_t h, const moonep_plan_t *plan, const void *hidden,
                               const float *route_weights, void *hidden_nvs, float *route_weights_nvs,
                               moonep_stream_t stream) {
    if (!h || !plan || !plan->dst || !plan->status || !hidden || !hidden_nvs) return MOONEP_ERR_NULL;
    if (!aligned16(hidden) || !aligned16(hidden_nvs)) return MOONEP_ERR_ALIGN;
    CopyArgs a = copy_args(h, plan);
    a.src = hidden;
    a.w = route_weights;
    a.out = hidden_nvs;
    a.w_out = route_weights_nvs;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const cudaError_t e = h->bulk_dispatch ? launch_dispatch_bulk(a, h->grid_dispatch, st)
                                           : launch_dispatch(a, h->grid_dispatch, st);
    return e == cudaSuccess ? MOONEP_OK : fail_cuda(e);
}

extern "C" int moonep_dispatch_rank(moonep_handle_t h, const moonep_plan_t *plan, const void *hidden,
                                    const float *route_weights, void *const *hidden_nvs,
                                    float *const *route_weights_nvs, moonep_stream_t stream) {
    if (!h || !plan || !plan->dst || !plan->status || !hidden) return MOONEP_ERR_NULL;
    if (!aligned16(hidden)) return MOONEP_ERR_ALIGN;
    CopyArgs a = copy_args(h, plan);
    const int rc = peer_tables(h, hidden_nvs, route_weights_nvs, &a);
    if (rc != MOONEP_OK) return rc;
    a.src = hidden;
    a.w = route_weights;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // bulk stores only into this GPU's memory; rows for other GPUs go as
    // plain 16-byte stores
    const bool remote = table_is_remote(h, reinterpret_cast<const void *const *>(a.peer), h->d.R);
    const cudaError_t e = (h->bulk_dispatch && !remote) ? launch_dispatch_bulk(a, h->grid_dispatch, st)
                                                        : launch_dispatch(a, h->grid_dispatch_vec, st);
    return e == cudaSuccess ? MOONEP_OK : fail_cuda(e);
}

extern "C" int moonep_combine_rank(moonep_handle_t h, const moonep_plan_t *plan, const void *const *hidden_nvs,
                                   const float *const *route_weights_nvs, void *out, float *gathered_weights,
                                   moonep_stream_t stream) {
    if (!h || !plan || !plan->dst || !plan->status || !out) return MOONEP_ERR_NULL;
    if (!aligned16(out)) return MOONEP_ERR_ALIGN;
    CopyArgs a = copy_args(h, plan);
    // the kernel only reads through these tables
    const int rc = peer_tables(h, const_cast<void *const *>(hidden_nvs),
                               const_cast<float *const *>(route_weights_nvs), &a);
    if (rc != MOONEP_OK) return rc;
    a.out = out;
    a.w_out = route_weights_nvs ? gathered_weights : nullptr;
    const cudaError_t e = launch_combine(a, h->grid_combine, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOONEP_OK : fail_cuda(e);
}

extern "C" int moonep_combine(moonep_handle_t h, const moonep_plan_t *plan, const void *hidden_nvs,
                              const float *route_weights_nvs, void *out, float *gathered_weights,
                              moonep_stream_t stream) {
    if (!h || !plan || !plan->dst || !plan->status || !hidden_nvs || !out) return MOONEP_ERR_NULL;
    if (!aligned16(hidden_nvs) || !aligned16(out)) return MOONEP_ERR_ALIGN;
    CopyArgs a = copy_args(h, plan);
    a.src = hidden_nvs;
    a.w = route_weights_nvs;
    a.out = out;
    a.w_out = route_weights_nvs ? gathered_weights : nullptr;
    const cudaError_t e = launch_combine(a, h->grid_combine, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOONEP_OK : fail_cuda(e);
}

static int weight_args(moonep_handle_t h, const moonep_plan_t *plan, int32_t n_proj, const void *const *src,
                       void *const *dst, int64_t Hp, WeightArgs *a) {
    if (!h || !plan || !plan->status || !src || !dst) return MOONEP_ERR_NULL;
    if (n_proj < 1 || n_proj > MOONEP_MAX_PROJ || Hp < 1) return MOONEP_ERR_SIZE;
    if (h->d.B > 0 && !plan->slot_expert) return MOONEP_ERR_NULL;
    memset(a, 0, sizeof(*a));
    a->d = h->d;
    a->slot_expert = plan->slot_expert;
    a->status = plan->status;
    a->n_proj = n_proj;
    a->hhp = (int64_t)h->d.H * Hp;
    a->rank = -1;
    for (int p = 0; p < n_proj; ++p) {
        if (!src[p] || !dst[p]) return MOONEP_ERR_NULL;
        if (!aligned16(src[p]) || !aligned16(dst[p])) return MOONEP_ERR_ALIGN;
        a->src[p] = src[p];
        a->dst[p] = dst[p];
    }
    return MOONEP_OK;
}

extern "C" int moonep_prefetch_weight(moonep_handle_t h, const moonep_plan_t *plan, int32_t n_proj,
                                      const void *const *weights, void *const *pool, int64_t Hp,
                                      moonep_stream_t stream) {
    WeightArgs a;
    const int rc = weight_args(h, plan, n_proj, weights, pool, Hp, &a);
    if (rc != MOONEP_OK) return rc;
    if (h->d.B == 0) return MOONEP_OK;  // no slots: nothing to copy
    const cudaError_t e = launch_prefetch(a, h->grid_weights, h->sms, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOONEP_OK : fail_cuda(e);
}

extern "C" int moonep_reduce_grad(moonep_handle_t h, const moonep_plan_t *plan, int32_t n_proj,
                                  float *const *grads, float *const *reduce_buffers, int64_t Hp,
                                  moonep_stream_t stream) {
    WeightArgs a;
    // the reduce buffers are the source (read, then zeroed), the grads the destination
    const int rc = weight_args(h, plan, n_proj, reinterpret_cast<const void *const *>(reduce_buffers),
                               reinterpret_cast<void *const *>(grads), Hp, &a);
    if (rc != MOONEP_OK) return rc;
    if (h->d.B == 0) return MOONEP_OK;
    const cudaError_t e = launch_reduce_grad(a, h->grid_weights, h->sms, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOONEP_OK : fail_cuda(e);
}

// One rank's weight call: its own tensors (own[p]) and every rank's tensor
// of the other side (peers[p*R + q]).
static int weight_args_rank(moonep_handle_t h, const moonep_plan_t *plan, int32_t rank, int32_t n_proj,
                            void *const *own, const void *const *peers, int64_t Hp, WeightArgs *a) {
    if (!h || !plan || !plan->status || !own || !peers) return MOONEP_ERR_NULL;
    if (n_proj < 1 || n_proj > MOONEP_MAX_PROJ || Hp < 1 || rank < 0 || rank >= h->d.R) return MOONEP_ERR_SIZE;
    if (h->d.B > 0 && !plan->slot_expert) return MOONEP_ERR_NULL;
    memset(a, 0, sizeof(*a));
    a->d = h->d;
    a->slot_expert = plan->slot_expert;
    a->status = plan->status;
    a->n_proj = n_proj;
    a->hhp = (int64_t)h->d.H * Hp;
    a->rank = rank;
    for (int p = 0; p < n_proj; ++p) {
        if (!own[p]) return MOONEP_ERR_NULL;
        if (!aligned16(own[p])) return MOONEP_ERR_ALIGN;
        a->dst[p] = own[p];
        for (int q = 0; q < h->d.R; ++q) {
            const void *x = peers[(size_t)p * h->d.R + q];
            if (!x) return MOONEP_ERR_NULL;
            if (!aligned16(x)) return MOONEP_ERR_ALIGN;
            a->peer[p][q] = x;
        }
    }
    a->remote = table_is_remote(h, peers, n_proj * h->d.R) ? 1 : 0;
    return MOONEP_OK;
}

extern "C" int moonep_prefetch_weight_rank(moonep_handle_t h, const moonep_plan_t *plan, int32_t rank, int32_t n_proj,
                                           const void *const *weights, void *const *pool, int64_t Hp,
                                           moonep_stream_t stream) {
    WeightArgs a;
    const int rc = weight_args_rank(h, plan, rank, n_proj, pool, weights, Hp, &a);
    if (rc != MOONEP_OK) return rc;
    if (h->d.B == 0) return MOONEP_OK;
    const cudaError_t e = launch_prefetch(a, h->grid_weights, h->sms, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOONEP_OK : fail_cuda(e);
}

extern "C" int moonep_reduce_grad_rank(moonep_handle_t h, const moonep_plan_t *plan, int32_t rank, int32_t n_proj,
                                       float *const *grads, float *const *reduce_buffers, int64_t Hp,
                                       moonep_stream_t stream) {
    WeightArgs a;
    const int rc = weight_args_rank(h, plan, rank, n_proj, reinterpret_cast<void *const *>(grads),
                                    reinterpret_cast<const void *const *>(reduce_buffers), Hp, &a);
    if (rc != MOONEP_OK) return rc;
    if (h->d.B == 0) return MOONEP_OK;
    const cudaError_t e = launch_reduce_grad(a, h->grid_weights, h->sms, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOONEP_OK : fail_cuda(e);
}

extern "C" int moonep_group_gemm(moonep_handle_t h, const moonep_plan_t *plan, const void *x_nvs,
                                 const void *weights, const void *pool, void *y_nvs, int64_t Hp,
                                 moonep_stream_t stream) {
    if (!h || !plan || !plan->cu_seqlens || !plan->status || !x_nvs || !weights || !y_nvs) return MOONEP_ERR_NULL;
    if (h->d.B > 0 && !pool) return MOONEP_ERR_NULL;
    if (!aligned16(x_nvs) || !aligned16(weights) || !aligned16(y_nvs) || (pool && !aligned16(pool)))
        return MOONEP_ERR_ALIGN;
    const int rc = gemm_supported(h->d, Hp);
    if (rc != MOONEP_OK) return rc;
    // the GEMM reads its operands with TMA into two-SM clusters: local memory only
    const void *ops[4] = {x_nvs, weights, pool, y_nvs};
    for (const void *p : ops)
        if (p && on_other_device(p, h->device) == 1) return MOONEP_ERR_DEVICE;
    int32_t *pairs = reinterpret_cast<int32_t *>(static_cast<char *>(h->ws_mem) + pair_table_offset(h->d));
    return launch_group_gemm(h->d, plan, x_nvs, weights, pool, y_nvs, Hp, pairs, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int moonep_plan_sizes(const moonep_config_t *cfg, int32_t one_rank, moonep_plan_sizes_t *out) {
    if (!cfg || !out) return MOONEP_ERR_NULL;
    memset(out, 0, sizeof(*out));
    const int rc = check_config(*cfg);
    if (rc != MOONEP_OK) return rc;
    const int64_t R = cfg->R, S = cfg->S, K = cfg->K, E = cfg->E, B = cfg->B;
    out->dst = one_rank ? S * K : R * S * K;
    out->cu_seqlens = R * (E + B);
    out->row_counts = R * (E + B);
    out->slot_expert = R * B;
    out->counts = R * E;
    out->assign = R * 4;
    out->maxvio = 1;
    out->status = 1;
    out->nvs = nvs_of(*cfg);
    return MOONEP_OK;
}

extern "C" int moonep_plan_status(const moonep_plan_t *plan, int32_t *status) {
    if (!plan || !plan->status || !status) return MOONEP_ERR_NULL;
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess) e = cudaMemcpy(status, plan->status, sizeof(int32_t), cudaMemcpyDeviceToHost);
    return e == cudaSuccess ? MOONEP_OK : fail_cuda(e);
}

extern "C" int moonep_read_status(const moonep_plan_t *plan, int32_t *status, moonep_stream_t stream) {
    if (!plan || !plan->status || !status) return MOONEP_ERR_NULL;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(status, plan->status, sizeof(int32_t), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    return e == cudaSuccess ? MOONEP_OK : fail_cuda(e);
}
