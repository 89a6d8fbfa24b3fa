// Fused-permute dispatch and combine (MoonEP README, "dispatch fwd",
// "combine fwd", "dispatch bwd", "combine bwd"; MarkTechPost, "Core idea:
// dynamic redundant experts", property 3: tokens are written straight into
// their expert-grouped positions and the buffer views go to the compute).
//
// Both kernels are HBM-bound gathers/scatters of whole bf16 rows.  One warp
// owns one token: lane k (< K) holds the token's k-th destination slot, and
// the row moves as 16-byte vectors, U vectors per lane in flight, with
// streaming cache hints (every byte is touched once).  The grid is a whole
// number of waves over the SMs and walks the tokens in a grid-stride loop.
#include "moonep_internal.cuh"

namespace moonep {

__device__ __forceinline__ uint4 ld_stream(const uint4 *p) { return __ldcs(p); }
__device__ __forceinline__ void st_stream(uint4 *p, const uint4 &v) { __stcs(p, v); }

// Slot dk = q*NvS + i of the group: row dk of the one buffer `base`, or row i
// of rank q's own buffer when the call is peered.  `row` is in units of T.
template <typename T>
__device__ __forceinline__ T *slot_row(const CopyArgs &a, T *base, int dk, int64_t row) {
    if (!a.peered) return base + (int64_t)dk * row;
    const int q = dk / a.d.nvs;
    return static_cast<T *>(a.peer[q]) + (int64_t)(dk - q * a.d.nvs) * row;
}
// the route weight of slot dk, or NULL when the call carries none
__device__ __forceinline__ float *slot_weight(const CopyArgs &a, float *base, int dk) {
    if (!a.peered) return base ? base + dk : nullptr;
    const int q = dk / a.d.nvs;
    return a.peer_w[q] ? a.peer_w[q] + (dk - q * a.d.nvs) : nullptr;
}
template <typename T>
__device__ __forceinline__ T *shfl_ptr(T *p, int src) {
    return reinterpret_cast<T *>(__shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(p), src));
}

// ---- dispatch ----------------------------------------------------------------
// KT > 0: K known at compile time, the K destination rows are broadcast into
// registers once per token; KT == 0: any K, one shuffle per row and step.
template <int KT, int U>
__global__ void __launch_bounds__(256) dispatch_kernel(const __grid_constant__ CopyArgs a) {
    pdl_wait();
    if (*a.status != 0) return;
    const Dims &d = a.d;
    const int K = KT > 0 ? KT : d.K;
    const int lane = threadIdx.x & 31;
    const int HV = d.H >> 3;
    const int64_t ntok = a.ntok;
    const int64_t nslots = (int64_t)d.R * d.nvs;
    const uint4 *src = static_cast<const uint4 *>(a.src);
    uint4 *buf = static_cast<uint4 *>(a.out);
    const int64_t wstride = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t tok = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; tok < ntok; tok += wstride) {
        uint4 *mine = nullptr;  // lane k: the row of the token's k-th slot
        if (lane < K) {
            const int dk = a.dst[tok * K + lane];
            if (dk < 0 || dk >= nslots) {
                atomicOr(a.status_rw, MOONEP_STATUS_BAD_PLAN);
            } else {
                mine = slot_row(a, buf, dk, HV);
                float *wo = slot_weight(a, a.w_out, dk);
                if (a.w != nullptr && wo != nullptr) *wo = __ldcs(a.w + tok * K + lane);
            }
        }
        const uint4 *row = src + tok * HV;
        if constexpr (KT > 0) {
            uint4 *orow[KT];
#pragma unroll
            for (int k = 0; k < KT; ++k) orow[k] = shfl_ptr(mine, k);
            for (int v0 = 0; v0 < HV; v0 += 32 * U) {
                uint4 x[U];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int v = v0 + u * 32 + lane;
                    if (v < HV) x[u] = ld_stream(row + v);
                }
#pragma unroll
                for (int k = 0; k < KT; ++k) {
                    if (orow[k] == nullptr) continue;
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const int v = v0 + u * 32 + lane;
                        if (v < HV) st_stream(orow[k] + v, x[u]);
                    }
                }
            }
        } else {
            for (int v0 = 0; v0 < HV; v0 += 32 * U) {
                uint4 x[U];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int v = v0 + u * 32 + lane;
                    if (v < HV) x[u] = ld_stream(row + v);
                }
                for (int k = 0; k < K; ++k) {
                    uint4 *o = shfl_ptr(mine, k);
                    if (o == nullptr) continue;
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const int v = v0 + u * 32 + lane;
                        if (v < HV) st_stream(o + v, x[u]);
                    }
                }
            }
        }
    }
}

// ---- dispatch with bulk (TMA) copies -----------------------------------------
// Rows of at least kBulkMinRow bytes move through shared memory with the bulk
// copy engine: each warp runs a ring of NS row stages.  Lane 0 loads a token's
// row with one bulk global->shared copy (completion on an mbarrier), then
// writes it to its K slots with K bulk shared->global copies (one bulk group
// per token); a stage is refilled once the previous token's stores have read
// it.  Waits are bounded: on a timeout the kernel flags MOONEP_STATUS_TIMEOUT,
// drains what it issued and returns.
constexpr int kBulkMinRow = 2048;
constexpr int kBulkStages = 3;
// one warp per block; NS stages of `rowbytes` each, then NS mbarriers
template <int KT>
__global__ void __launch_bounds__(32) dispatch_bulk_kernel(const __grid_constant__ CopyArgs a) {
    extern __shared__ __align__(128) uint8_t sm[];
    pdl_wait();
    if (*a.status != 0) return;
    const Dims &d = a.d;
    const int K = KT > 0 ? KT : d.K;
    const int lane = threadIdx.x;
    const uint32_t rowbytes = (uint32_t)d.H * 2u;
    const int64_t ntok = a.ntok;
    const int64_t nslots = (int64_t)d.R * d.nvs;
    const uint8_t *src = static_cast<const uint8_t *>(a.src);
    uint8_t *buf = static_cast<uint8_t *>(a.out);
    const uint32_t stage0 = smem_addr(sm);
    const uint32_t bar0 = smem_addr(sm + (size_t)kBulkStages * rowbytes);
    const int64_t first = blockIdx.x, step = gridDim.x;
    auto tok_of = [&](int64_t i) { return first + i * step; };
    const uint64_t pol = l2_evict_first_policy();

    if (lane == 0) {
        for (int s = 0; s < kBulkStages; ++s) mbar_init(bar0 + 8u * s);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        for (int s = 0; s < kBulkStages; ++s)
            if (tok_of(s) < ntok)
                bulk_load(stage0 + s * rowbytes, src + tok_of(s) * rowbytes, rowbytes, bar0 + 8u * s);
    }
    __syncwarp();
    bool ok = true;
    int64_t i = 0;
    for (; tok_of(i) < ntok; ++i) {
        const int64_t tok = tok_of(i);
        const int s = (int)(i % kBulkStages);
        const uint32_t parity = (uint32_t)((i / kBulkStages) & 1);
        uint8_t *mine = nullptr;  // lane k: the row of the token's k-th slot
        if (lane < K) {
            const int dk = a.dst[tok * K + lane];
            if (dk < 0 || dk >= nslots) {
                atomicOr(a.status_rw, MOONEP_STATUS_BAD_PLAN);
            } else {
                mine = slot_row(a, buf, dk, rowbytes);
                float *wo = slot_weight(a, a.w_out, dk);
                if (a.w != nullptr && wo != nullptr) *wo = __ldcs(a.w + tok * K + lane);
            }
        }
        if (lane == 0) ok = mbar_wait(bar0 + 8u * s, parity);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        for (int k = 0; k < K; ++k) {
            uint8_t *o = shfl_ptr(mine, k);
            if (lane == 0 && o != nullptr) bulk_store(o, stage0 + s * rowbytes, rowbytes, pol);
        }
        if (lane == 0) {
            bulk_commit();
            // refill the previous token's stage once its stores have read it
            if (i >= 1 && tok_of(i - 1 + kBulkStages) < ntok) {
                bulk_wait_read1();
                const int sp = (int)((i - 1) % kBulkStages);
                bulk_load(stage0 + sp * rowbytes, src + tok_of(i - 1 + kBulkStages) * rowbytes, rowbytes,
                          bar0 + 8u * sp);
            }
        }
        __syncwarp();
    }
    if (lane == 0) {
        if (!ok) {
            atomicOr(a.status_rw, MOONEP_STATUS_TIMEOUT);
            // loads still in flight: tokens i .. i + kBulkStages - 2 (bounded waits)
            for (int64_t j = i; j < i + kBulkStages - 1 && tok_of(j) < ntok; ++j)
                mbar_wait(bar0 + 8u * (uint32_t)(j % kBulkStages), (uint32_t)((j / kBulkStages) & 1));
        }
        bulk_wait_all();  // every issued load was consumed; the stores must finish reading
    }
    __syncwarp();
}

// ---- dispatch through a deep ring, one producer and one consumer warp --------
// Warp 0 (lane 0) streams the block's token rows into a ring of NS row stages
// with bulk loads; warp 1 waits for each row, its lanes k < K resolve the K
// destination slots (and copy the route weight), and lane 0 writes the row
// to them with K bulk stores, one bulk group per token.  A stage goes back
// to the producer once its stores have read it: after committing token i,
// the consumer waits until at most D groups still read (token i - D is done)
// and arrives on that stage's "empty" barrier.  So up to D tokens' stores and
// NS - D loads are in flight per block at any time, and no load waits behind
// the stores of the token just before it.  Every wait is bounded; a timeout
// sets MOONEP_STATUS_TIMEOUT, both warps stop, and the block drains the copies
// it issued before it exits.
#ifndef MOONEP_RING_NS
#define MOONEP_RING_NS 14
#endif
#ifndef MOONEP_RING_D
#define MOONEP_RING_D 6
#endif
constexpr int kRingNS = MOONEP_RING_NS;
constexpr int kRingD = MOONEP_RING_D;
static_assert(kRingD >= 1 && kRingD < kRingNS, "stores in flight must leave a stage for loads");

template <int KT>
__global__ void __launch_bounds__(64) dispatch_ring_kernel(const __grid_constant__ CopyArgs a) {
    extern __shared__ __align__(128) uint8_t sm[];
    __shared__ volatile int s_abort;
    __shared__ int s_status;
    pdl_wait();
    // one read of the plan's status for the whole block (another block may
    // set BAD_PLAN meanwhile; both warps must take the same branch)
    if (threadIdx.x == 0) s_status = *a.status;
    __syncthreads();
    if (s_status != 0) return;
    const Dims &d = a.d;
    const int K = KT > 0 ? KT : d.K;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t rowbytes = (uint32_t)d.H * 2u;
    const int64_t ntok = a.ntok;
    const int64_t nslots = (int64_t)d.R * d.nvs;
    const uint8_t *src = static_cast<const uint8_t *>(a.src);
    uint8_t *buf = static_cast<uint8_t *>(a.out);
    const uint32_t stage0 = smem_addr(sm);
    const uint32_t full0 = smem_addr(sm + (size_t)kRingNS * rowbytes);
    const uint32_t empty0 = full0 + 8u * kRingNS;
    const int64_t first = blockIdx.x, step = gridDim.x;
    const int64_t mine_n = first < ntok ? (ntok - 1 - first) / step + 1 : 0;  // tokens of this block

    if (threadIdx.x == 0) {
        for (int s = 0; s < kRingNS; ++s) {
            mbar_init(full0 + 8u * s);
            mbar_init(empty0 + 8u * s);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        s_abort = 0;
    }
    __syncthreads();

    int64_t issued = 0;  // producer: loads issued
    if (warp == 0) {
        if (lane == 0) {
            for (int64_t i = 0; i < mine_n; ++i) {
                const int s = (int)(i % kRingNS);
                if (i >= kRingNS && !mbar_wait(empty0 + 8u * s, (uint32_t)(((i / kRingNS) - 1) & 1))) {
                    s_abort = 1;
                    break;
                }
                if (s_abort) break;
                bulk_load(stage0 + s * rowbytes, src + (first + i * step) * rowbytes, rowbytes, full0 + 8u * s);
                issued = i + 1;
            }
        }
    } else {
        const uint64_t pol = l2_evict_first_policy();
        for (int64_t i = 0; i < mine_n; ++i) {
            const int64_t tok = first + i * step;
            const int s = (int)(i % kRingNS);
            uint8_t *mine = nullptr;  // lane k: the row of the token's k-th slot
            if (lane < K) {
                const int dk = a.dst[tok * K + lane];
                if (dk < 0 || dk >= nslots) {
                    atomicOr(a.status_rw, MOONEP_STATUS_BAD_PLAN);
                } else {
                    mine = slot_row(a, buf, dk, rowbytes);
                    float *wo = slot_weight(a, a.w_out, dk);
                    if (a.w != nullptr && wo != nullptr) *wo = __ldcs(a.w + tok * K + lane);
                }
            }
            bool ok = true;
            if (lane == 0) ok = !s_abort && mbar_wait(full0 + 8u * s, (uint32_t)((i / kRingNS) & 1));
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) {
                if (lane == 0) s_abort = 1;
                break;
            }
            for (int k = 0; k < K; ++k) {
                uint8_t *o = shfl_ptr(mine, k);
                if (lane == 0 && o != nullptr) bulk_store(o, stage0 + s * rowbytes, rowbytes, pol);
            }
            if (lane == 0) {
                bulk_commit();
                if (i >= kRingD) {
                    bulk_wait_read<kRingD>();  // token i - D's stores have read its stage
                    mbar_arrive(empty0 + 8u * (uint32_t)((i - kRingD) % kRingNS));
                }
            }
            __syncwarp();
        }
        if (lane == 0) bulk_wait_all();  // the stores must finish before the block's shared memory goes
    }
    __syncthreads();
    if (threadIdx.x == 0 && s_abort) {
        atomicOr(a.status_rw, MOONEP_STATUS_TIMEOUT);
        // every load still in flight lands before exit: the last one issued
        // into each stage (the earlier ones completed before it was issued)
        for (int64_t j = issued - 1; j >= 0 && j >= issued - kRingNS; --j)
            mbar_wait(full0 + 8u * (uint32_t)(j % kRingNS), (uint32_t)((j / kRingNS) & 1));
    }
}

size_t dispatch_ring_smem(const Dims &d) { return (size_t)kRingNS * d.H * 2 + 16 * kRingNS; }

size_t dispatch_bulk_smem(const Dims &d) { return (size_t)kBulkStages * d.H * 2 + 8 * kBulkStages; }
bool dispatch_use_bulk(const Dims &d) { return (size_t)d.H * 2 >= kBulkMinRow && dispatch_bulk_smem(d) <= 200 * 1024; }
#ifndef MOONEP_DISPATCH_RING
#define MOONEP_DISPATCH_RING 1
#endif
// the deep ring where its NS row stages fit one block's shared memory
static bool dispatch_use_ring(const Dims &d) {
    return MOONEP_DISPATCH_RING && (size_t)d.H * 2 >= kBulkMinRow && dispatch_ring_smem(d) <= 220 * 1024;
}

// ---- combine -----------------------------------------------------------------
__device__ __forceinline__ void fma_bf16x8(float (&acc)[8], const uint4 &y, float w) {
    const uint32_t q[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        acc[2 * i] = fmaf(w, __uint_as_float(q[i] << 16), acc[2 * i]);
        acc[2 * i + 1] = fmaf(w, __uint_as_float(q[i] & 0xffff0000u), acc[2 * i + 1]);
    }
}

__device__ __forceinline__ uint4 pack_bf16x8(const float (&acc)[8]) {
    uint32_t q[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
        q[i] = *reinterpret_cast<const uint32_t *>(&h);
    }
    return make_uint4(q[0], q[1], q[2], q[3]);
}

// KT > 0: K known at compile time (all K*U loads of a step in flight);
// KT == 0: any K, loads issued in groups of 4 rows.
template <int KT, int U>
__global__ void __launch_bounds__(256) combine_kernel(const __grid_constant__ CopyArgs a) {
    pdl_wait();
    if (*a.status != 0) return;
    const Dims &d = a.d;
    const int K = KT > 0 ? KT : d.K;
    const int lane = threadIdx.x & 31;
    const int HV = d.H >> 3;
    const int64_t ntok = a.ntok;
    const int64_t nslots = (int64_t)d.R * d.nvs;
    const uint4 *y = static_cast<const uint4 *>(a.peered ? a.peer[0] : a.src);
    // weighted: route_weights_nvs given (one buffer, or every rank's when peered)
    const bool weighted = a.peered ? a.peer_w[0] != nullptr : a.w != nullptr;
    uint4 *out = static_cast<uint4 *>(a.out);
    const int64_t wstride = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t tok = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; tok < ntok; tok += wstride) {
        const uint4 *mine = y;  // lane k: the row of the token's k-th slot (a valid row on every lane)
        float wk = 1.0f;
        if (lane < K) {
            const int dk = a.dst[tok * K + lane];
            if (dk < 0 || dk >= nslots) {
                atomicOr(a.status_rw, MOONEP_STATUS_BAD_PLAN);
                wk = 0.0f;
            } else {
                mine = slot_row(a, y, dk, HV);
                if (weighted) {
                    wk = *slot_weight(a, const_cast<float *>(a.w), dk);
                    if (a.w_out != nullptr) a.w_out[tok * K + lane] = wk;
                }
            }
        }
        uint4 *orow = out + tok * HV;
        for (int v0 = 0; v0 < HV; v0 += 32 * U) {
            float acc[U][8];
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[u][i] = 0.0f;
            if constexpr (KT > 0) {
                uint4 yv[KT][U];
#pragma unroll
                for (int k = 0; k < KT; ++k) {
                    const uint4 *yrow = shfl_ptr(mine, k);
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const int v = v0 + u * 32 + lane;
                        yv[k][u] = v < HV ? ld_stream(yrow + v) : make_uint4(0, 0, 0, 0);
                    }
                }
#pragma unroll
                for (int k = 0; k < KT; ++k) {
                    const float ww = __shfl_sync(0xffffffffu, wk, k);
#pragma unroll
                    for (int u = 0; u < U; ++u) fma_bf16x8(acc[u], yv[k][u], ww);
                }
            } else {
                for (int k0 = 0; k0 < K; k0 += 4) {
                    uint4 yv[4][U];
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint4 *yrow = shfl_ptr(mine, (k0 + kk) & 31);
#pragma unroll
                        for (int u = 0; u < U; ++u) {
                            const int v = v0 + u * 32 + lane;
                            yv[kk][u] = (v < HV && k0 + kk < K) ? ld_stream(yrow + v) : make_uint4(0, 0, 0, 0);
                        }
                    }
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const float ww = __shfl_sync(0xffffffffu, wk, (k0 + kk) & 31);
                        if (k0 + kk < K) {
#pragma unroll
                            for (int u = 0; u < U; ++u) fma_bf16x8(acc[u], yv[kk][u], ww);
                        }
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int v = v0 + u * 32 + lane;
                if (v < HV) st_stream(orow + v, pack_bf16x8(acc[u]));
            }
        }
    }
}

// ---- launch ------------------------------------------------------------------
static cudaLaunchAttribute pdl_attr() {
    cudaLaunchAttribute at;
    at.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at.val.programmaticStreamSerializationAllowed = 1;
    return at;
}

template <typename Kern>
static cudaError_t launch_pdl(Kern kern, int grid, cudaStream_t st, const CopyArgs &a) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    cudaLaunchAttribute at[1] = {pdl_attr()};
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a);
}

#ifndef MOONEP_DISPATCH_U
#define MOONEP_DISPATCH_U 4
#endif
constexpr int kDispatchU = MOONEP_DISPATCH_U;

#define MOONEP_DISPATCH_CASES(X) X(1) X(2) X(4) X(6) X(8)

template <typename Kern>
static cudaError_t launch_pdl_smem(Kern kern, int grid, int block, size_t smem, cudaStream_t st, const CopyArgs &a) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1] = {pdl_attr()};
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a);
}

cudaError_t launch_dispatch(const CopyArgs &a, int grid, cudaStream_t st) {
    switch (a.d.K) {
#define X(k) case k: return launch_pdl(dispatch_kernel<k, kDispatchU>, grid, st, a);
        MOONEP_DISPATCH_CASES(X)
#undef X
        default: return launch_pdl(dispatch_kernel<0, kDispatchU>, grid, st, a);
    }
}

cudaError_t launch_dispatch_bulk(const CopyArgs &a, int grid, cudaStream_t st) {
    if (dispatch_use_ring(a.d)) {
        const size_t smem = dispatch_ring_smem(a.d);
        switch (a.d.K) {
#define X(k) case k: return launch_pdl_smem(dispatch_ring_kernel<k>, grid, 64, smem, st, a);
            MOONEP_DISPATCH_CASES(X)
#undef X
            default: return launch_pdl_smem(dispatch_ring_kernel<0>, grid, 64, smem, st, a);
        }
    }
    const size_t smem = dispatch_bulk_smem(a.d);
    switch (a.d.K) {
#define X(k) case k: return launch_pdl_smem(dispatch_bulk_kernel<k>, grid, 32, smem, st, a);
        MOONEP_DISPATCH_CASES(X)
#undef X
        default: return launch_pdl_smem(dispatch_bulk_kernel<0>, grid, 32, smem, st, a);
    }
}

cudaError_t dispatch_bulk_set_smem_limit(size_t bytes) {
    cudaError_t e = cudaSuccess;
#define X(k) if (e == cudaSuccess) e = cudaFuncSetAttribute(dispatch_bulk_kernel<k>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    MOONEP_DISPATCH_CASES(X)
    X(0)
#undef X
#define X(k) if (e == cudaSuccess) e = cudaFuncSetAttribute(dispatch_ring_kernel<k>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    MOONEP_DISPATCH_CASES(X)
    X(0)
#undef X
    return e;
}

int dispatch_bulk_blocks_per_sm(const Dims &d) {
    int n = 0;
    if (dispatch_use_ring(d)) {
        const size_t smem = dispatch_ring_smem(d);
        switch (d.K) {
#define X(k) case k: cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, dispatch_ring_kernel<k>, 64, smem); break;
            MOONEP_DISPATCH_CASES(X)
#undef X
            default: cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, dispatch_ring_kernel<0>, 64, smem); break;
        }
        return n > 0 ? n : 1;
    }
    const size_t smem = dispatch_bulk_smem(d);
    switch (d.K) {
#define X(k) case k: cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, dispatch_bulk_kernel<k>, 32, smem); break;
        MOONEP_DISPATCH_CASES(X)
#undef X
        default: cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, dispatch_bulk_kernel<0>, 32, smem); break;
    }
    return n > 0 ? n : 1;
}

int dispatch_blocks_per_sm(int K) {
    int n = 0;
    switch (K) {
#define X(k) case k: cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, dispatch_kernel<k, kDispatchU>, 256, 0); break;
        MOONEP_DISPATCH_CASES(X)
#undef X
        default: cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, dispatch_kernel<0, kDispatchU>, 256, 0); break;
    }
    return n > 0 ? n : 1;
}

cudaError_t launch_combine(const CopyArgs &a, int grid, cudaStream_t st) {
    switch (a.d.K) {
        case 1: return launch_pdl(combine_kernel<1, 4>, grid, st, a);
        case 2: return launch_pdl(combine_kernel<2, 4>, grid, st, a);
        case 4: return launch_pdl(combine_kernel<4, 2>, grid, st, a);
        case 6: return launch_pdl(combine_kernel<6, 2>, grid, st, a);
        case 8: return launch_pdl(combine_kernel<8, 2>, grid, st, a);
        default: return launch_pdl(combine_kernel<0, 2>, grid, st, a);
    }
}

int combine_blocks_per_sm(int K) {
    int n = 0;
    switch (K) {
        case 1: cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, combine_kernel<1, 4>, 256, 0); break;
        case 2: cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, combine_kernel<2, 4>, 256, 0); break;
        case 4: cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, combine_kernel<4, 2>, 256, 0); break;
        case 6: cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, combine_kernel<6, 2>, 256, 0); break;
        case 8: cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, combine_kernel<8, 2>, 256, 0); break;
        default: cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, combine_kernel<0, 2>, 256, 0); break;
    }
    return n > 0 ? n : 1;
}

}  // namespace moonep
