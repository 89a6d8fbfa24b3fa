// Sharing rank buffers between processes (CUDA IPC), for one rank of a real
// EP group per process.  MoonEP's ranks reach each other's dispatch buffers,
// weight rows and grad slots through one symmetric device mapping (README,
// "Weight buffer", "Grad buffer"; MarkTechPost, "Memory contract"); a process
// here exports the allocation behind each of its buffers, and every peer
// imports it, on the same GPU or on another GPU of the node.  Host code only.
#include <cuda.h>
#include <string.h>

#include <mutex>
#include <vector>

#include "moonep_internal.cuh"

namespace moonep {

typedef CUresult (*AddressRangeFn)(CUdeviceptr *, size_t *, CUdeviceptr);

// The driver's cuMemGetAddressRange (the allocation holding a pointer),
// found through the runtime so the library needs no link against libcuda.
static int address_range(const void *p, char **base, size_t *bytes) {
    static std::once_flag once;
    static AddressRangeFn fn = nullptr;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<AddressRangeFn>(f);
    });
    if (!fn) return fail_cuda(cudaErrorNotSupported);
    CUdeviceptr b = 0;
    size_t n = 0;
    if (fn(&b, &n, reinterpret_cast<CUdeviceptr>(p)) != CUDA_SUCCESS) return fail_cuda(cudaErrorInvalidValue);
    *base = reinterpret_cast<char *>(b);
    *bytes = n;
    return MOONEP_OK;
}

// Mappings this process opened: one per distinct exported allocation, shared
// by every import of a pointer inside it.
struct Mapping {
    unsigned char key[64];
    char *base;
    size_t bytes;
    int refs;
};
static std::mutex g_mu;
static std::vector<Mapping> g_maps;

}  // namespace moonep

using namespace moonep;

static_assert(sizeof(cudaIpcMemHandle_t) == 64, "a CUDA IPC handle is 64 bytes");

extern "C" int moonep_ipc_export(const void *ptr, moonep_ipc_handle_t *out) {
    if (!ptr || !out) return MOONEP_ERR_NULL;
    memset(out, 0, sizeof(*out));
    char *base = nullptr;
    size_t bytes = 0;
    int rc = address_range(ptr, &base, &bytes);
    if (rc != MOONEP_OK) return rc;
    cudaIpcMemHandle_t h;
    const cudaError_t e = cudaIpcGetMemHandle(&h, base);
    if (e != cudaSuccess) return fail_cuda(e);
    memcpy(out->handle, &h, sizeof(h));
    out->offset = static_cast<const char *>(ptr) - base;
    out->bytes = (int64_t)bytes;
    return MOONEP_OK;
}

extern "C" int moonep_ipc_import(const moonep_ipc_handle_t *h, void **out) {
    if (!h || !out) return MOONEP_ERR_NULL;
    *out = nullptr;
    if (h->offset < 0 || h->bytes <= 0 || h->offset >= h->bytes) return MOONEP_ERR_SIZE;
    std::lock_guard<std::mutex> lock(g_mu);
    for (Mapping &m : g_maps)
        if (memcmp(m.key, h->handle, 64) == 0) {
            if ((size_t)h->offset >= m.bytes) return MOONEP_ERR_SIZE;
            ++m.refs;
            *out = m.base + h->offset;
            return MOONEP_OK;
        }
    cudaIpcMemHandle_t ih;
    memcpy(&ih, h->handle, sizeof(ih));
    void *base = nullptr;
    const cudaError_t e = cudaIpcOpenMemHandle(&base, ih, cudaIpcMemLazyEnablePeerAccess);
    if (e != cudaSuccess) return fail_cuda(e);
    Mapping m;
    memcpy(m.key, h->handle, 64);
    m.base = static_cast<char *>(base);
    m.bytes = (size_t)h->bytes;
    m.refs = 1;
    g_maps.push_back(m);
    *out = m.base + h->offset;
    return MOONEP_OK;
}

extern "C" int moonep_ipc_close(void *ptr) {
    if (!ptr) return MOONEP_ERR_NULL;
    std::lock_guard<std::mutex> lock(g_mu);
    for (size_t i = 0; i < g_maps.size(); ++i) {
        Mapping &m = g_maps[i];
        char *p = static_cast<char *>(ptr);
        if (p >= m.base && p < m.base + m.bytes) {
            if (--m.refs > 0) return MOONEP_OK;
            const cudaError_t e = cudaIpcCloseMemHandle(m.base);
            g_maps.erase(g_maps.begin() + (long)i);
            return e == cudaSuccess ? MOONEP_OK : fail_cuda(e);
        }
    }
    return MOONEP_ERR_SIZE;  // not a pointer this process imported
}

namespace moonep {
// 1 when `p` lives on a device other than `device` (a peer GPU's memory,
// e.g. imported from another process), else 0; -1 when CUDA cannot tell.
int on_other_device(const void *p, int device) {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();
        return -1;
    }
    return (at.type == cudaMemoryTypeDevice && at.device != device) ? 1 : 0;
}
}  // namespace moonep
