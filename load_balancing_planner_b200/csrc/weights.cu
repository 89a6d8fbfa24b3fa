// Weight prefetch and grad-slot reduction (MoonEP README, "Weight buffer",
// "Grad buffer", "dispatch fwd" prefetch_weight, "dispatch bwd" reduce_grad;
// MarkTechPost, "Memory contract").
//
// Both walk the used prefetch slots of all ranks grouped by expert: the first
// slot (in (rank, slot) order) that holds an expert leads, and a linked list
// in shared memory chains the later slots holding the same expert.  Work is
// cut into (projection, leading slot, tile of the [H, H'] matrix) units taken
// by a grid-stride loop, so every expert matrix is read once:
//   prefetch:    load a bf16 tile of W[e], store it to every slot holding e;
//   reduce_grad: load the fp32 tile of G[e], add every holder's tile in
//                ascending slot order, store G[e], store zeros to the holders.
#include "moonep_internal.cuh"

namespace moonep {

constexpr int kWThreads = 256;
constexpr int kWVec = 4;                          // 16-byte vectors per thread per tile
constexpr int kWTile = kWThreads * kWVec;         // vectors per tile
constexpr int kWMaxWarps = 9;                     // warps of the largest block that builds slot lists

// Binary search for expert e in one rank's slot row: used slots first, in
// ascending expert order, then -1s (the layout moonep_plan writes).
__device__ __forceinline__ int find_slot(const int32_t *row, int B, int e) {
    int lo = 0, hi = B;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        const int v = row[mid];
        if (v >= 0 && v < e) lo = mid + 1;
        else hi = mid;
    }
    return (lo < B && row[lo] == e) ? lo : -1;
}

// Where the matrices live (mb = bytes per matrix).  The group: expert e is
// row e of an [E,..] tensor, slot j = q*B + b row j of an [R*B,..] tensor.
// One rank: its own side is a [G,..] (home experts) or [B,..] (its slots)
// tensor at `own`; the other side is rank q's tensor peer[p][q].
__device__ __forceinline__ char *expert_at(const WeightArgs &a, const void *own, int p, int e, size_t mb,
                                           bool via_peers) {
    const char *m;
    if (a.rank < 0) {
        m = static_cast<const char *>(own) + (size_t)e * mb;
    } else {
        const int G = a.d.G, q = e / G;
        m = via_peers ? static_cast<const char *>(a.peer[p][q]) + (size_t)(e - q * G) * mb
                      : static_cast<const char *>(own) + (size_t)(e - a.rank * G) * mb;
    }
    return const_cast<char *>(m);
}

__device__ __forceinline__ char *slot_at(const WeightArgs &a, const void *own, int p, int j, size_t mb,
                                         bool via_peers) {
    const char *m;
    if (a.rank < 0) {
        m = static_cast<const char *>(own) + (size_t)j * mb;
    } else {
        const int B = a.d.B, q = j / B;
        m = via_peers ? static_cast<const char *>(a.peer[p][q]) + (size_t)(j - q * B) * mb
                      : static_cast<const char *>(own) + (size_t)(j - a.rank * B) * mb;
    }
    return const_cast<char *>(m);
}

__device__ __forceinline__ int warp_incl_scan_w(int v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    return v;
}

// Shared-memory slot tables: se[RB] expert or -1, nxt[RB] next slot holding
// the same expert (-1 = last), lead[] leading slots in ascending order.
// One rank's share keeps only its own slots (prefetch) or the slots holding
// its home experts (by_home, reduce_grad).  Returns the number of leaders, or
// -1 after flagging a malformed slot table.
__device__ int build_slot_lists(const WeightArgs &a, int32_t *se, int32_t *nxt, int32_t *lead, bool by_home,
                                int nthreads = kWThreads) {
    __shared__ int s_bad;
    __shared__ int s_warp[kWMaxWarps];
    const int R = a.d.R, B = a.d.B, E = a.d.E, RB = R * B;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    if (tid == 0) s_bad = 0;
    __syncthreads();
    for (int s = tid; s < RB; s += nthreads) {
        const int e = a.slot_expert[s];
        if (e < -1 || e >= E) s_bad = 1;
        se[s] = e;
    }
    __syncthreads();
    for (int s = tid; s < RB; s += nthreads) {
        const int e = se[s];
        if (s % B != 0 && e >= 0) {
            const int prev = se[s - 1];
            if (prev < 0 || prev >= e) s_bad = 1;  // used slots first, ascending, distinct
            if (prev >= 0 && prev / a.d.G != e / a.d.G) s_bad = 1;  // copies of one home group per rank
        }
    }
    __syncthreads();
    if (s_bad) {
        if (tid == 0) atomicOr(a.status, MOONEP_STATUS_BAD_PLAN);
        return -1;
    }
    if (a.rank >= 0) {  // whole rows are kept or dropped, so rows stay sorted
        for (int s = tid; s < RB; s += nthreads) {
            const int e = se[s];
            if (e >= 0 && (by_home ? e / a.d.G != a.rank : s / B != a.rank)) se[s] = -1;
        }
        __syncthreads();
    }
    const int per = (RB + nthreads - 1) / nthreads;  // <= 32 (RB <= 8192)
    const int s0 = min(RB, tid * per), s1 = min(RB, s0 + per);
    unsigned mask = 0;
    int cnt = 0;
    for (int s = s0; s < s1; ++s) {
        const int e = se[s];
        const int r = s / B;
        int next = -1;
        bool leader = e >= 0;
        if (e >= 0) {
            for (int r2 = 0; r2 < r && leader; ++r2)
                if (find_slot(se + r2 * B, B, e) >= 0) leader = false;
            for (int r2 = r + 1; r2 < R; ++r2) {
                const int j = find_slot(se + r2 * B, B, e);
                if (j >= 0) {
                    next = r2 * B + j;
                    break;
                }
            }
        }
        nxt[s] = next;
        if (leader) {
            mask |= 1u << (s - s0);
            ++cnt;
        }
    }
    // leaders in ascending slot order: block-wide exclusive scan of the counts
    const int incl = warp_incl_scan_w(cnt);
    if (lane == 31) s_warp[w] = incl;
    __syncthreads();
    const int nw = nthreads / 32;
    if (w == 0) {
        const int x = lane < nw ? s_warp[lane] : 0;
        const int xi = warp_incl_scan_w(x);
        if (lane < nw) s_warp[lane] = xi;
    }
    __syncthreads();
    int pos = (w > 0 ? s_warp[w - 1] : 0) + incl - cnt;
    const int total = s_warp[nw - 1];
    for (int s = s0; s < s1; ++s)
        if (mask & (1u << (s - s0))) lead[pos++] = s;
    __syncthreads();
    return total;
}

__global__ void __launch_bounds__(kWThreads) prefetch_kernel(const __grid_constant__ WeightArgs a) {
    pdl_wait();
    if (*a.status != 0) return;
    extern __shared__ int32_t wsm[];
    const int RB = a.d.R * a.d.B;
    int32_t *se = wsm, *nxt = wsm + RB, *lead = wsm + 2 * RB;
    const int nlead = build_slot_lists(a, se, nxt, lead, false);
    if (nlead <= 0) return;
    const int64_t nvec = a.hhp / 8;  // bf16: 8 per 16 bytes
    const size_t mb = (size_t)a.hhp * 2;
    const int64_t ntiles = (nvec + kWTile - 1) / kWTile;
    const int64_t units = (int64_t)a.n_proj * nlead * ntiles;
    for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
        const int p = (int)(u / ((int64_t)nlead * ntiles));
        const int64_t rem = u - (int64_t)p * nlead * ntiles;
        const int s = lead[rem / ntiles];
        const int64_t t0 = (rem % ntiles) * kWTile;
        const uint4 *src = reinterpret_cast<const uint4 *>(expert_at(a, a.src[p], p, se[s], mb, true)) + t0;
        uint4 x[kWVec];
#pragma unroll
        for (int i = 0; i < kWVec; ++i) {
            const int64_t v = t0 + i * kWThreads + threadIdx.x;
            if (v < nvec) x[i] = __ldcs(src + i * kWThreads + threadIdx.x);
        }
        for (int j = s; j >= 0; j = nxt[j]) {
            uint4 *dst = reinterpret_cast<uint4 *>(slot_at(a, a.dst[p], p, j, mb, false)) + t0;
#pragma unroll
            for (int i = 0; i < kWVec; ++i) {
                const int64_t v = t0 + i * kWThreads + threadIdx.x;
                if (v < nvec) __stcs(dst + i * kWThreads + threadIdx.x, x[i]);
            }
        }
    }
}

// Bulk variant of the prefetch: after the block has built the slot lists,
// one thread moves 32 KB pieces of each expert matrix through a 3-stage ring
// in shared memory with the TMA engine: one bulk load per piece, then one
// bulk store per slot holding the expert, and the stage is refilled as soon
// as those stores have read it.  Every expert piece is read once.
constexpr int kPfStages = 3;
#ifndef MOONEP_PF_TILE_KB
#define MOONEP_PF_TILE_KB 32
#endif
constexpr uint32_t kPfTile = MOONEP_PF_TILE_KB * 1024;

__global__ void __launch_bounds__(kWThreads) prefetch_bulk_kernel(const __grid_constant__ WeightArgs a) {
    pdl_wait();
    if (*a.status != 0) return;
    extern __shared__ __align__(128) int32_t wsm[];
    const int RB = a.d.R * a.d.B;
    int32_t *se = wsm, *nxt = wsm + RB, *lead = wsm + 2 * RB;
    const int nlead = build_slot_lists(a, se, nxt, lead, false);
    if (nlead <= 0 || threadIdx.x != 0) return;
    uint8_t *stages = reinterpret_cast<uint8_t *>(wsm) + ((sizeof(int32_t) * 3 * (size_t)RB + 127) & ~(size_t)127);
    const uint32_t stage0 = smem_addr(stages);
    const uint32_t bar0 = stage0 + kPfStages * kPfTile;
    const uint64_t bytes_per = (uint64_t)a.hhp * 2;  // one expert matrix, bf16
    const int64_t ntiles = (int64_t)((bytes_per + kPfTile - 1) / kPfTile);
    const int64_t units = (int64_t)a.n_proj * nlead * ntiles;
    const int64_t first = blockIdx.x, step = gridDim.x;
    const uint64_t pol = l2_evict_first_policy();
    // unit i of this block -> projection, leading slot, byte offset, size
    auto piece = [&](int64_t i, int &p, int &s, uint64_t &off, uint32_t &n) {
        const int64_t u = first + i * step;
        p = (int)(u / ((int64_t)nlead * ntiles));
        const int64_t rem = u - (int64_t)p * nlead * ntiles;
        s = lead[rem / ntiles];
        off = (uint64_t)(rem % ntiles) * kPfTile;
        n = (uint32_t)min((uint64_t)kPfTile, bytes_per - off);
    };
    auto load = [&](int64_t i, int st) {
        int p, s;
        uint64_t off;
        uint32_t n;
        piece(i, p, s, off, n);
        bulk_load(stage0 + st * kPfTile,
                  reinterpret_cast<const uint8_t *>(expert_at(a, a.src[p], p, se[s], bytes_per, true)) + off, n,
                  bar0 + 8u * st);
    };
    for (int st = 0; st < kPfStages; ++st) mbar_init(bar0 + 8u * st);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    for (int st = 0; st < kPfStages; ++st)
        if (first + st * step < units) load(st, st);
    bool ok = true;
    int64_t i = 0;
    for (; first + i * step < units; ++i) {
        const int st = (int)(i % kPfStages);
        if (!(ok = mbar_wait(bar0 + 8u * st, (uint32_t)((i / kPfStages) & 1)))) break;
        int p, s;
        uint64_t off;
        uint32_t n;
        piece(i, p, s, off, n);
        for (int j = s; j >= 0; j = nxt[j])
            bulk_store(reinterpret_cast<uint8_t *>(slot_at(a, a.dst[p], p, j, bytes_per, false)) + off,
                       stage0 + st * kPfTile, n, pol);
        bulk_commit();
        // refill the previous unit's stage once its stores have read it
        if (i >= 1 && first + (i - 1 + kPfStages) * step < units) {
            bulk_wait_read1();
            load(i - 1 + kPfStages, (int)((i - 1) % kPfStages));
        }
    }
    if (!ok) {
        atomicOr(a.status, MOONEP_STATUS_TIMEOUT);
        // loads still in flight: units i .. i + kPfStages - 2 (bounded waits)
        for (int64_t j = i; j < i + kPfStages - 1 && first + j * step < units; ++j)
            mbar_wait(bar0 + 8u * (uint32_t)(j % kPfStages), (uint32_t)((j / kPfStages) & 1));
    }
    bulk_wait_all();
}

// Deep-ring variant of the bulk prefetch, one block per SM: after the block
// has built the slot lists, warp 0 (lane 0) streams the block's 32 KB pieces
// into a ring of kPfRing stages with bulk loads, and warp 1 (lane 0) writes
// each piece to every slot holding its expert with bulk stores, one bulk
// group per piece, handing a stage back once its stores have read it (up to
// kPfInFlight pieces' stores in flight).  No load waits behind the stores of
// the piece before it.  Waits are bounded; a timeout sets
// MOONEP_STATUS_TIMEOUT, both warps stop, and the loads in flight land
// before the block exits.
#ifndef MOONEP_PF_RING
#define MOONEP_PF_RING 4
#endif
#ifndef MOONEP_PF_INFLIGHT
#define MOONEP_PF_INFLIGHT (MOONEP_PF_RING / 2)
#endif
constexpr int kPfRing = MOONEP_PF_RING;
constexpr int kPfInFlight = MOONEP_PF_INFLIGHT;
static_assert(kPfInFlight >= 1 && kPfInFlight < kPfRing, "stores in flight must leave a stage for loads");

__global__ void __launch_bounds__(kWThreads) prefetch_ring_kernel(const __grid_constant__ WeightArgs a) {
    __shared__ volatile int s_abort;
    __shared__ int s_status;
    pdl_wait();
    // one read of the plan's status for the whole block (another block may
    // flag BAD_PLAN meanwhile; every thread must take the same branch)
    if (threadIdx.x == 0) s_status = *a.status;
    __syncthreads();
    if (s_status != 0) return;
    extern __shared__ __align__(128) int32_t wsm[];
    const int RB = a.d.R * a.d.B;
    int32_t *se = wsm, *nxt = wsm + RB, *lead = wsm + 2 * RB;
    const int nlead = build_slot_lists(a, se, nxt, lead, false);  // block-uniform result
    if (nlead <= 0) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp > 1) return;
    uint8_t *stages = reinterpret_cast<uint8_t *>(wsm) + ((sizeof(int32_t) * 3 * (size_t)RB + 127) & ~(size_t)127);
    const uint32_t stage0 = smem_addr(stages);
    const uint32_t full0 = stage0 + kPfRing * kPfTile;
    const uint32_t empty0 = full0 + 8u * kPfRing;
    const uint64_t bytes_per = (uint64_t)a.hhp * 2;  // one expert matrix, bf16
    const int64_t ntiles = (int64_t)((bytes_per + kPfTile - 1) / kPfTile);
    const int64_t units = (int64_t)a.n_proj * nlead * ntiles;
    const int64_t first = blockIdx.x, step = gridDim.x;
    const int64_t mine_n = first < units ? (units - 1 - first) / step + 1 : 0;
    auto piece = [&](int64_t i, int &p, int &s, uint64_t &off, uint32_t &n) {
        const int64_t u = first + i * step;
        p = (int)(u / ((int64_t)nlead * ntiles));
        const int64_t rem = u - (int64_t)p * nlead * ntiles;
        s = lead[rem / ntiles];
        off = (uint64_t)(rem % ntiles) * kPfTile;
        n = (uint32_t)min((uint64_t)kPfTile, bytes_per - off);
    };
    if (threadIdx.x == 0) {
        for (int st = 0; st < kPfRing; ++st) {
            mbar_init(full0 + 8u * st);
            mbar_init(empty0 + 8u * st);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        s_abort = 0;
    }
    // warps 0 and 1 only: named barrier 1 over 64 threads
    asm volatile("bar.sync 1, 64;" ::: "memory");
    int64_t issued = 0;
    if (warp == 0 && lane == 0) {
        for (int64_t i = 0; i < mine_n; ++i) {
            const int st = (int)(i % kPfRing);
            if (i >= kPfRing && !mbar_wait(empty0 + 8u * st, (uint32_t)(((i / kPfRing) - 1) & 1))) {
                s_abort = 1;
                break;
            }
            if (s_abort) break;
            int p, s;
            uint64_t off;
            uint32_t n;
            piece(i, p, s, off, n);
            bulk_load(stage0 + st * kPfTile,
                      reinterpret_cast<const uint8_t *>(expert_at(a, a.src[p], p, se[s], bytes_per, true)) + off, n,
                      full0 + 8u * st);
            issued = i + 1;
        }
    } else if (warp == 1 && lane == 0) {
        const uint64_t pol = l2_evict_first_policy();
        for (int64_t i = 0; i < mine_n; ++i) {
            const int st = (int)(i % kPfRing);
            if (s_abort || !mbar_wait(full0 + 8u * st, (uint32_t)((i / kPfRing) & 1))) {
                s_abort = 1;
                break;
            }
            int p, s;
            uint64_t off;
            uint32_t n;
            piece(i, p, s, off, n);
            for (int j = s; j >= 0; j = nxt[j])
                bulk_store(reinterpret_cast<uint8_t *>(slot_at(a, a.dst[p], p, j, bytes_per, false)) + off,
                           stage0 + st * kPfTile, n, pol);
            bulk_commit();
            if (i >= kPfInFlight) {
                bulk_wait_read<kPfInFlight>();  // piece i - kPfInFlight's stores have read its stage
                mbar_arrive(empty0 + 8u * (uint32_t)((i - kPfInFlight) % kPfRing));
            }
        }
        bulk_wait_all();  // the stores finish before the block's shared memory goes
    }
    asm volatile("bar.sync 1, 64;" ::: "memory");
    if (threadIdx.x == 0 && s_abort) {
        atomicOr(a.status, MOONEP_STATUS_TIMEOUT);
        // the last load issued into each stage lands before exit
        for (int64_t j = issued - 1; j >= 0 && j >= issued - kPfRing; --j)
            mbar_wait(full0 + 8u * (uint32_t)(j % kPfRing), (uint32_t)((j / kPfRing) & 1));
    }
}

// a.src[p] = reduce buffer [R*B, H*Hp] (read, then zeroed), a.dst[p] = grads [E, H*Hp].
__global__ void __launch_bounds__(kWThreads) reduce_grad_kernel(const __grid_constant__ WeightArgs a) {
    pdl_wait();
    if (*a.status != 0) return;
    extern __shared__ int32_t wsm[];
    const int RB = a.d.R * a.d.B;
    int32_t *se = wsm, *nxt = wsm + RB, *lead = wsm + 2 * RB;
    const int nlead = build_slot_lists(a, se, nxt, lead, true);
    if (nlead <= 0) return;
    const int64_t nvec = a.hhp / 4;  // fp32: 4 per 16 bytes
    const size_t mb = (size_t)a.hhp * 4;
    const int64_t ntiles = (nvec + kWTile - 1) / kWTile;
    const int64_t units = (int64_t)a.n_proj * nlead * ntiles;
    const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
        const int p = (int)(u / ((int64_t)nlead * ntiles));
        const int64_t rem = u - (int64_t)p * nlead * ntiles;
        const int s = lead[rem / ntiles];
        const int64_t t0 = (rem % ntiles) * kWTile;
        float4 *g = reinterpret_cast<float4 *>(expert_at(a, a.dst[p], p, se[s], mb, false)) + t0;
        float4 acc[kWVec];
#pragma unroll
        for (int i = 0; i < kWVec; ++i) {
            const int64_t v = t0 + i * kWThreads + threadIdx.x;
            acc[i] = v < nvec ? __ldcs(g + i * kWThreads + threadIdx.x) : zero;
        }
        for (int j = s; j >= 0; j = nxt[j]) {
            const float4 *slot = reinterpret_cast<const float4 *>(slot_at(a, a.src[p], p, j, mb, true)) + t0;
#pragma unroll
            for (int i = 0; i < kWVec; ++i) {
                const int64_t v = t0 + i * kWThreads + threadIdx.x;
                if (v < nvec) {
                    const float4 x = __ldcs(slot + i * kWThreads + threadIdx.x);
                    acc[i].x = __fadd_rn(acc[i].x, x.x);
                    acc[i].y = __fadd_rn(acc[i].y, x.y);
                    acc[i].z = __fadd_rn(acc[i].z, x.z);
                    acc[i].w = __fadd_rn(acc[i].w, x.w);
                }
            }
        }
#pragma unroll
        for (int i = 0; i < kWVec; ++i) {
            const int64_t v = t0 + i * kWThreads + threadIdx.x;
            if (v < nvec) __stcs(g + i * kWThreads + threadIdx.x, acc[i]);
        }
        for (int j = s; j >= 0; j = nxt[j]) {
            float4 *slot = reinterpret_cast<float4 *>(slot_at(a, a.src[p], p, j, mb, true)) + t0;
#pragma unroll
            for (int i = 0; i < kWVec; ++i) {
                const int64_t v = t0 + i * kWThreads + threadIdx.x;
                if (v < nvec) __stcs(slot + i * kWThreads + threadIdx.x, zero);
            }
        }
    }
}

// Bulk variant of the grad-slot reduction.  Warp 0 streams, one 16 KB fp32
// piece at a time, each unit's grad piece and then its holders' pieces in
// ascending slot order through a 6-slot ring in shared memory (bulk loads
// completing on mbarriers); the other 8 warps add them up in registers (16
// floats a thread), in that order, store the sum to the grad and zeros to
// the holders, and hand each ring slot back as soon as they have read it.
#ifndef MOONEP_RG_RING
#define MOONEP_RG_RING 6
#endif
#ifndef MOONEP_RG_BPS
#define MOONEP_RG_BPS 2
#endif
constexpr int kRgRing = MOONEP_RG_RING;
constexpr int kRgTile = 4096;                  // floats per piece (16 KB)
constexpr int kRgThreads = 32 + 256;           // producer warp + 8 summing warps
constexpr int kRgPer = kRgTile / 256;          // floats per summing thread

__global__ void __launch_bounds__(kRgThreads) reduce_grad_bulk_kernel(const __grid_constant__ WeightArgs a) {
    pdl_wait();
    if (*a.status != 0) return;
    extern __shared__ __align__(128) int32_t wsm[];
    const int RB = a.d.R * a.d.B;
    int32_t *se = wsm, *nxt = wsm + RB, *lead = wsm + 2 * RB;
    const int nlead = build_slot_lists(a, se, nxt, lead, true, kRgThreads);
    const size_t mb = (size_t)a.hhp * 4;
    if (nlead <= 0) return;
    uint8_t *ring = reinterpret_cast<uint8_t *>(wsm) + ((sizeof(int32_t) * 3 * (size_t)RB + 127) & ~(size_t)127);
    const uint32_t ring0 = smem_addr(ring);
    const uint32_t full0 = ring0 + kRgRing * kRgTile * 4, empty0 = full0 + 8 * kRgRing;
    const int64_t npiece = (a.hhp + kRgTile - 1) / kRgTile;
    const int64_t units = (int64_t)a.n_proj * nlead * npiece;
    const int64_t first = blockIdx.x, step = gridDim.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    __shared__ int s_err;
    if (tid == 0) {
        s_err = 0;
        for (int k = 0; k < kRgRing; ++k) {
            mbar_init(full0 + 8u * k);
            asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(empty0 + 8u * k), "r"(8) : "memory");
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    volatile int *err = &s_err;
    auto unit = [&](int64_t i, int &p, int &s, int64_t &off, int &n) {
        const int64_t u = first + i * step;
        p = (int)(u / ((int64_t)nlead * npiece));
        const int64_t rem = u - (int64_t)p * nlead * npiece;
        s = lead[rem / npiece];
        off = (rem % npiece) * kRgTile;
        n = (int)min((int64_t)kRgTile, a.hhp - off);
    };

    if (warp == 0) {
        if (lane == 0) {
            int64_t seq = 0;  // pieces issued: ring slot seq % kRgRing, round seq / kRgRing
            for (int64_t i = 0; first + i * step < units && !*err; ++i) {
                int p, s, n;
                int64_t off;
                unit(i, p, s, off, n);
                const float *g = reinterpret_cast<const float *>(expert_at(a, a.dst[p], p, se[s], mb, false)) + off;
                // the unit's pieces: its grad (j = -1), then every holder in slot order
                for (int j = -1;;) {
                    const int k = (int)(seq % kRgRing);
                    if (seq >= kRgRing && !mbar_wait(empty0 + 8u * k, (uint32_t)(((seq / kRgRing) - 1) & 1))) {
                        atomicOr(a.status, MOONEP_STATUS_TIMEOUT);
                        *err = 1;
                        break;
                    }
                    const float *src =
                        j < 0 ? g : reinterpret_cast<const float *>(slot_at(a, a.src[p], p, j, mb, true)) + off;
                    bulk_load(ring0 + k * kRgTile * 4, src, (uint32_t)n * 4u, full0 + 8u * k);
                    ++seq;
                    j = j < 0 ? s : nxt[j];
                    if (j < 0) break;
                }
            }
            // the last load issued into each ring slot has landed before anyone leaves
            for (int64_t q = max((int64_t)0, seq - kRgRing); q < seq; ++q)
                if (!mbar_wait(full0 + 8u * (uint32_t)(q % kRgRing), (uint32_t)((q / kRgRing) & 1)))
                    atomicOr(a.status, MOONEP_STATUS_TIMEOUT);
        }
        return;
    }
    const int t = tid - 32;  // summing thread 0..255
    int64_t seq = 0;
    for (int64_t i = 0; first + i * step < units && !*err; ++i) {
        int p, s, n;
        int64_t off;
        unit(i, p, s, off, n);
        float acc[kRgPer];
        bool ok = true;
        for (int j = -1;;) {  // the grad piece, then every holder in slot order
            const int k = (int)(seq % kRgRing);
            ok = __all_sync(0xffffffffu, mbar_wait(full0 + 8u * k, (uint32_t)((seq / kRgRing) & 1)));
            if (!ok) break;
            const float4 *v = reinterpret_cast<const float4 *>(ring + (size_t)k * kRgTile * 4);
#pragma unroll
            for (int q = 0; q < kRgPer / 4; ++q) {
                const int idx = q * 256 + t;  // float4 index inside the piece
                const float4 x = idx * 4 < n ? v[idx] : make_float4(0.f, 0.f, 0.f, 0.f);
                if (j < 0) {
                    acc[4 * q] = x.x, acc[4 * q + 1] = x.y, acc[4 * q + 2] = x.z, acc[4 * q + 3] = x.w;
                } else {
                    acc[4 * q] = __fadd_rn(acc[4 * q], x.x);
                    acc[4 * q + 1] = __fadd_rn(acc[4 * q + 1], x.y);
                    acc[4 * q + 2] = __fadd_rn(acc[4 * q + 2], x.z);
                    acc[4 * q + 3] = __fadd_rn(acc[4 * q + 3], x.w);
                }
            }
            __syncwarp();
            if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(empty0 + 8u * k) : "memory");
            ++seq;
            j = j < 0 ? s : nxt[j];
            if (j < 0) break;
        }
        if (!ok) {
            if (lane == 0) atomicOr(a.status, MOONEP_STATUS_TIMEOUT);
            *err = 1;
            break;
        }
        float4 *g = reinterpret_cast<float4 *>(reinterpret_cast<float *>(expert_at(a, a.dst[p], p, se[s], mb, false)) + off);
#pragma unroll
        for (int q = 0; q < kRgPer / 4; ++q) {
            const int idx = q * 256 + t;
            if (idx * 4 < n) __stcs(g + idx, make_float4(acc[4 * q], acc[4 * q + 1], acc[4 * q + 2], acc[4 * q + 3]));
        }
        const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = s; j >= 0; j = nxt[j]) {
            float4 *z = reinterpret_cast<float4 *>(reinterpret_cast<float *>(slot_at(a, a.src[p], p, j, mb, true)) + off);
#pragma unroll
            for (int q = 0; q < kRgPer / 4; ++q) {
                const int idx = q * 256 + t;
                if (idx * 4 < n) __stcs(z + idx, zero);
            }
        }
    }
}

static size_t weights_smem(const WeightArgs &a) { return sizeof(int32_t) * 3 * (size_t)a.d.R * a.d.B; }

template <typename Kern>
static cudaError_t launch_w(Kern kern, const WeightArgs &a, int grid, cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kWThreads);
    cfg.dynamicSmemBytes = weights_smem(a);
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a);
}

static size_t prefetch_bulk_smem(const WeightArgs &a) {
    return ((weights_smem(a) + 127) & ~(size_t)127) + kPfStages * (size_t)kPfTile + 8 * kPfStages;
}

// The bulk prefetch kernels need 16-byte aligned matrices of whole 16-byte
// units, at least one piece long.
static bool prefetch_bulk_fits(const WeightArgs &a) {
    bool aligned = ((a.hhp * 2) % 16) == 0;
    for (int p = 0; p < a.n_proj; ++p)
        aligned = aligned && (reinterpret_cast<uintptr_t>(a.src[p]) % 16) == 0 &&
                  (reinterpret_cast<uintptr_t>(a.dst[p]) % 16) == 0;
    return aligned && a.hhp * 2 >= kPfTile;
}

// ... and the older kernel room for its ring next to the slot tables
bool prefetch_use_bulk(const WeightArgs &a) { return prefetch_bulk_fits(a) && prefetch_bulk_smem(a) <= 110 * 1024; }

static size_t prefetch_ring_smem(const WeightArgs &a) {
    return ((weights_smem(a) + 127) & ~(size_t)127) + kPfRing * (size_t)kPfTile + 16 * kPfRing;
}

#ifndef MOONEP_PF_USE_RING
#define MOONEP_PF_USE_RING 1
#endif

cudaError_t launch_prefetch(const WeightArgs &a, int grid, int sms, cudaStream_t st) {
    if (a.remote || !prefetch_bulk_fits(a)) return launch_w(prefetch_kernel, a, grid, st);
    if (MOONEP_PF_USE_RING && prefetch_ring_smem(a) <= 220 * 1024) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)sms);  // one deep ring per SM
        cfg.blockDim = dim3(kWThreads);
        cfg.dynamicSmemBytes = prefetch_ring_smem(a);
        cfg.stream = st;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        at[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, prefetch_ring_kernel, a);
    }
    if (!prefetch_use_bulk(a)) return launch_w(prefetch_kernel, a, grid, st);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * sms));  // two rings per SM
    cfg.blockDim = dim3(kWThreads);
    cfg.dynamicSmemBytes = prefetch_bulk_smem(a);
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, prefetch_bulk_kernel, a);
}

static size_t reduce_bulk_smem(const WeightArgs &a) {
    return ((weights_smem(a) + 127) & ~(size_t)127) + kRgRing * (size_t)kRgTile * 4 + 16 * kRgRing;
}

bool reduce_grad_use_bulk(const WeightArgs &a) {
    bool aligned = (a.hhp % 4) == 0;
    for (int p = 0; p < a.n_proj; ++p)
        aligned = aligned && (reinterpret_cast<uintptr_t>(a.src[p]) % 16) == 0 &&
                  (reinterpret_cast<uintptr_t>(a.dst[p]) % 16) == 0;
    return aligned && a.hhp >= kRgTile && reduce_bulk_smem(a) <= (MOONEP_RG_BPS == 1 ? 220 : 110) * 1024;
}

cudaError_t launch_reduce_grad(const WeightArgs &a, int grid, int sms, cudaStream_t st) {
    if (a.remote || !reduce_grad_use_bulk(a)) return launch_w(reduce_grad_kernel, a, grid, st);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(MOONEP_RG_BPS * sms));  // rings per SM
    cfg.blockDim = dim3(kRgThreads);
    cfg.dynamicSmemBytes = reduce_bulk_smem(a);
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, reduce_grad_bulk_kernel, a);
}

int weights_blocks_per_sm() {
    int n = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, reduce_grad_kernel, kWThreads, 0);
    return n > 0 ? n : 1;
}

size_t weights_static_smem_bytes() {
    cudaFuncAttributes fa;
    size_t m = 0;
    if (cudaFuncGetAttributes(&fa, prefetch_kernel) == cudaSuccess) m = fa.sharedSizeBytes;
    if (cudaFuncGetAttributes(&fa, reduce_grad_kernel) == cudaSuccess && fa.sharedSizeBytes > m) m = fa.sharedSizeBytes;
    if (cudaFuncGetAttributes(&fa, prefetch_bulk_kernel) == cudaSuccess && fa.sharedSizeBytes > m) m = fa.sharedSizeBytes;
    if (cudaFuncGetAttributes(&fa, prefetch_ring_kernel) == cudaSuccess && fa.sharedSizeBytes > m) m = fa.sharedSizeBytes;
    if (cudaFuncGetAttributes(&fa, reduce_grad_bulk_kernel) == cudaSuccess && fa.sharedSizeBytes > m)
        m = fa.sharedSizeBytes;
    return m;
}

cudaError_t weights_set_smem_limit(size_t bytes) {
    cudaError_t e = cudaFuncSetAttribute(prefetch_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(prefetch_bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(prefetch_ring_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(reduce_grad_bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(reduce_grad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

}  // namespace moonep
