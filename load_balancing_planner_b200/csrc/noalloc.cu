// moonep_plan_noalloc: the planner without a handle and without any device
// allocation.  Its planning workspace is a fixed-size array in device memory
// that the library image itself carries (every GPU that loads the library
// holds MOONEP_NOALLOC_SCRATCH_BYTES for it until the process exits).
//
// Who needs it: callers that must not call cudaMalloc in the layer path --
// a framework whose caching allocator owns the device memory, or a server
// that reserved all of it at start-up -- because a raw cudaMalloc there
// breaks their memory budget and can synchronise the device.
#include <mutex>

#include "moonep_internal.cuh"

namespace moonep {

// The scratch array.  In host code its name is a host-side stand-in, not a
// device address; the address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MOONEP_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch array, looked up once per device with that
// device current (the first call on a device does this).
static int scratch_address(int device, void **out) {
    static std::mutex mu;
    static void *addr[kMaxDevices] = {};
    if (device < 0 || device >= kMaxDevices) return MOONEP_ERR_SIZE;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[device]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return fail_cuda(e);
        addr[device] = p;
    }
    *out = addr[device];
    return MOONEP_OK;
}

}  // namespace moonep

using namespace moonep;

extern "C" int moonep_plan_noalloc(const moonep_config_t *cfg, const int32_t *topk,
                                   const int32_t *tokens_per_expert, const moonep_plan_t *plan,
                                   moonep_stream_t stream) {
    if (!cfg || !topk || !plan_ok(plan)) return MOONEP_ERR_NULL;
    int rc = check_config(*cfg);
    if (rc != MOONEP_OK) return rc;
    if (cfg->B > 0 && !plan->slot_expert) return MOONEP_ERR_NULL;
    int device = 0;
    const cudaError_t e0 = cudaGetDevice(&device);
    if (e0 != cudaSuccess) return fail_cuda(e0);
    if ((rc = prepare_device(device)) != MOONEP_OK) return rc;
    Dims d;
    int grid = 0;
    if ((rc = plan_dims(*cfg, device, &d, &grid)) != MOONEP_OK) return rc;
    if (workspace_bytes(d) > MOONEP_NOALLOC_SCRATCH_BYTES) return MOONEP_ERR_SIZE;
    void *base = nullptr;
    if ((rc = scratch_address(device, &base)) != MOONEP_OK) return rc;

    PlanArgs a;
    a.d = d;
    a.topk = topk;
    a.tpe = tokens_per_expert;
    a.src_rank = -1;
    a.counts_all = nullptr;
    a.plan = *plan;
    a.polls = kBarrierPolls;
    a.withheld = 0;
    carve_workspace(d, base, &a.ws);
    // The array keeps the previous call's contents.  What must start at zero
    // -- the per-rank count tables, the barrier counter and the error slots,
    // laid out contiguously after the chunk histograms -- is cleared here, on
    // the caller's stream, so every call starts like a fresh handle's first.
    const size_t clear = workspace_bytes(d) - (size_t)(reinterpret_cast<char *>(a.ws.cnt) - static_cast<char *>(base));
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(a.ws.cnt, 0, clear, st);
    if (e == cudaSuccess) e = launch_plan(a, grid, st);
    return e == cudaSuccess ? MOONEP_OK : fail_cuda(e);
}
