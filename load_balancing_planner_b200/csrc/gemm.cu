// The VM group GEMM that consumes a dispatched layer (MoonEP README,
// "Integration": one [E+B, H, H'] weight tensor per projection, with the
// planner's cu_seqlens selecting which expert row each token segment uses;
// "Weight buffer": rows [0, E) are the home experts, rows [E, E+B) this rank's
// prefetch slots).  For every rank r and every non-empty row i of its plan,
//   y[r, rows of i, :] = x[r, rows of i, :] @ Wrow(r, i),
// Wrow = W[i] for i < E (home rows, and inference overflow rows read from the
// home expert), pool[r][i - E] for slot rows.
//
// sm_100a design: a cluster of two CTAs (one per SM) computes 256 x 256
// output tiles with tcgen05.mma.cta_group::2 (bf16 x bf16 -> fp32, M=256,
// N=256, K=16).  Each CTA holds 128 rows of A and 128 of the 256 columns of
// B in shared memory, so an SM reads 16 KB of operands per MMA instead of the
// 24 KB a one-SM 128 x 256 tile needs; the one-SM design was bound by shared
// memory bandwidth (operand reads plus TMA fills) at about 70 % of the bf16
// peak.
//
// The clusters are persistent, one per pair of SMs, and claim tiles in order
// from a global counter (column tile fastest, then the live 256-row pairs in
// (rank, plan row) order), so the clusters working at one time share A rows
// and weights in L2.  In each CTA, warp 4 streams its A and B halves through a
// 6-stage ring with 2-D TMA loads (128-byte swizzle, no multicast) that
// complete on the leader's mbarriers; one thread of the leader (warp 5)
// issues the MMAs into one of two 256-column accumulators in each CTA's
// tensor memory, and its commits free the stages and signal the accumulators
// in both CTAs; warps 0-3 read the other accumulator back (tcgen05.ld), round
// to bf16 and store, overlapping the next tile's main loop.
//
// Tiles: rows are padded to token_padding, a multiple of 128, so every
// 128-row tile lies in one plan row; pair_map_kernel pairs consecutive tiles
// of the same plan row, so both halves of a pair share one weight, and an odd
// tile count leaves a dead second half that is computed on valid rows and not
// stored.  Every mbarrier wait is bounded; a timeout sets
// MOONEP_STATUS_TIMEOUT.
#include <cuda.h>

#include "moonep_internal.cuh"

namespace moonep {

constexpr int kGBM = 128, kGBN = 256, kGBK = 64;  // per-CTA rows, tile columns, K per stage
constexpr int kGThreads = 192;  // warps 0-3 epilogue, 4 TMA producer, 5 MMA issuer
constexpr int kGBoxB = kGBK * 64 * 2;              // 8 KB: one TMA box of B (64 K-rows x 64 columns)
constexpr uint32_t kGPolls = 1u << 22;             // bounded mbarrier waits (try_wait suspends between polls)

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// Wait until the phase with parity `parity` of `bar` has completed; false
// after kGPolls polls.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
    const uint32_t a = smem_u32(bar);
    for (uint32_t it = 0; it < kGPolls; ++it) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(a), "r"(parity)
            : "memory");
        if (done) return true;
    }
    return false;
}

// The same wait with cluster-scope acquire: for barriers that CTAs of the
// cluster other than this one arrive on, and data they wrote before arriving.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t *bar, uint32_t parity) {
    const uint32_t a = smem_u32(bar);
    for (uint32_t it = 0; it < kGPolls; ++it) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(a), "r"(parity)
            : "memory");
        if (done) return true;
    }
    return false;
}

// Shared-memory matrix descriptors (tcgen05), 128-byte swizzle, version 1.
// A: K-major rows of 128 bytes, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_k_sw128(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// B: N-major; 64-column atoms (one TMA box) 8 KB apart, 8-row K groups 1024
// bytes apart.
__device__ __forceinline__ uint64_t desc_mn_sw128(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)(kGBoxB >> 4) << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}


constexpr int kGStages = 6;
constexpr int kGTileA = kGBM * kGBK * 2;        // 16 KB: this CTA's 128 rows
constexpr int kGTileB = kGBK * (kGBN / 2) * 2;  // 16 KB: this CTA's 128 columns (2 boxes)
constexpr int kGSmem = 1024 + kGStages * (kGTileA + kGTileB) + 512;
constexpr uint32_t kGIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((uint32_t)(kGBN >> 3) << 17) |
                              ((uint32_t)(256 >> 4) << 24);

struct GemmArgs {
    CUtensorMap tx, tw, tp;
    const int32_t *cu_seqlens;  // [R, E+B]
    const int32_t *pairs;       // [R, pmax]: (plan row << 12) | pair index in the row, or -1; then [R] counts
    int *tile_ctr;              // next unclaimed tile (zeroed by pair_map_kernel)
    int32_t *status;
    void *y;
    int R, E, B, H, Hp, nvs, NR, pmax, ntiles;
};

// pairs[r][q]: the q-th 256-row pair of rank r, in plan-row order; -1 past
// the last pair, and everywhere for a failed plan.  pairs[R][r] (after the R
// rows): the number of pairs of rank r; then the GEMM's tile counter, reset.
__global__ void __launch_bounds__(256) pair_map_kernel(const int32_t *cu_seqlens, const int32_t *status,
                                                        int32_t *pairs, int NR, int pmax) {
    pdl_wait();
    const int r = blockIdx.x, tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    __shared__ int s_warp[8], s_carry;
    const int32_t *cu = cu_seqlens + (int64_t)r * NR;
    int32_t *out = pairs + (int64_t)r * pmax;
    const bool failed = ld_cg(status) != 0;
    if (tid == 0) s_carry = 0;
    __syncthreads();
    for (int i0 = 0; i0 < NR && !failed; i0 += 256) {
        const int i = i0 + tid;
        int np = 0;
        if (i < NR) {
            const int lp = ld_cg(cu + i) - (i > 0 ? ld_cg(cu + i - 1) : 0);  // padded rows, a multiple of 128
            np = (lp / kGBM + 1) / 2;
        }
        int incl = np;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        if (lane == 31) s_warp[w] = incl;
        __syncthreads();
        int before = s_carry;
        for (int k = 0; k < w; ++k) before += s_warp[k];
        const int first = before + incl - np;
        for (int j = 0; j < np; ++j)
            if (first + j < pmax) out[first + j] = (i << 12) | j;
        __syncthreads();
        if (tid == 0)
            for (int k = 0; k < 8; ++k) s_carry += s_warp[k];
        __syncthreads();
    }
    const int used = failed ? 0 : min(s_carry, pmax);
    for (int q = used + tid; q < pmax; q += 256) out[q] = -1;
    if (tid == 0) pairs[(int64_t)gridDim.x * pmax + r] = used;  // the live pairs of rank r
    if (r == 0 && tid == 0) pairs[(int64_t)gridDim.x * (pmax + 1)] = 0;  // the GEMM's tile counter
}

__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
    uint32_t out;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(addr), "r"(rank));
    return out;
}

__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *map, int c0, int c1,
                                                 uint32_t bar_cluster) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
        "%3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar_cluster)
        : "memory");
}

__device__ __forceinline__ void umma_bf16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(kGIdesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_commit_pair(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"((uint16_t)3)
        : "memory");
}

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Where tile t of the compact work list lies.  Tiles run column tile fastest
// over the live pairs in (rank, pair) order, so the clusters working at one
// time share A rows and, pair after pair, one expert's weight in L2.  Both
// CTAs of a cluster derive the same tile; `live` is this CTA's half.
struct GemmTile {
    int r, nt, row0, brow0;
    bool live, slot;
};

__device__ __forceinline__ GemmTile gemm_tile(const GemmArgs &a, const int *s_pre, int t, uint32_t crank) {
    GemmTile g;
    const int gp = t / a.ntiles;
    g.nt = t - gp * a.ntiles;
    int r = 0;
    while (r + 1 < a.R && s_pre[r + 1] <= gp) ++r;
    g.r = r;
    const int v = ld_cg(a.pairs + (int64_t)r * a.pmax + (gp - s_pre[r]));
    if (v < 0) {  // not written for a live index: read row 0, store nothing
        g.row0 = 0, g.brow0 = 0, g.live = false, g.slot = false;
        return g;
    }
    const int i = v >> 12, pj = v & 4095;
    const int32_t *cu = a.cu_seqlens + (int64_t)r * a.NR;
    const int end = ld_cg(cu + i), beg = i > 0 ? ld_cg(cu + i - 1) : 0;
    const int off = 2 * kGBM * pj + kGBM * (int)crank;
    g.live = off < end - beg;
    g.row0 = beg + (g.live ? off : 2 * kGBM * pj);
    g.slot = i >= a.E;
    g.brow0 = (i < a.E ? i : r * a.B + (i - a.E)) * a.H;
    return g;
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

constexpr int kGTQ = 4;  // tile queue depth

// Persistent, with tiles handed out in order from a global counter: the
// leader's producer thread claims the next tile for its cluster and posts it
// to a small queue in both CTAs' shared memory.  Warp 4 (lane 0) of each CTA
// streams its A and B halves of the posted tiles through the stage ring;
// warp 5 (lane 0) of the leader issues every tile's MMAs into one of two
// 256-column accumulators; warps 0-3 (one tensor-memory lane quadrant each)
// drain the other accumulator meanwhile, so a tile's epilogue overlaps the
// next tile's main loop.  Claiming in order keeps the clusters working at one
// time on neighbouring tiles (shared A rows and weights in L2), and a cluster
// that starts late finds the work taken.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGThreads, 1)
    group_gemm_kernel(const __grid_constant__ GemmArgs a) {
    extern __shared__ uint8_t gsm_raw[];
    uint8_t *gsm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(gsm_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *sA = gsm;
    uint8_t *sB = gsm + kGStages * kGTileA;
    uint64_t *full = reinterpret_cast<uint64_t *>(sB + kGStages * kGTileB);
    uint64_t *empty = full + kGStages;
    uint64_t *tfull = empty + kGStages;  // [2] accumulator b holds a finished tile (both CTAs)
    uint64_t *tempty = tfull + 2;        // [2] accumulator b drained by both CTAs (leader; 8 warp arrivals)
    uint64_t *mdone = tempty + 2;        // every MMA issued has completed (both CTAs)
    uint64_t *qfull = mdone + 1;         // [kGTQ] queue entry posted (both CTAs)
    uint64_t *qempty = qfull + kGTQ;     // [kGTQ] queue entry read by every consumer (leader; 10 arrivals)
    int *tq = reinterpret_cast<int *>(qempty + kGTQ);  // [kGTQ] posted tile, or >= ntile to stop
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tq + kGTQ);
    __shared__ int s_pre[MOONEP_MAX_R + 1];
    __shared__ int s_err;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint32_t crank;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(crank));

    pdl_wait();
    // The pair table is written before this kernel and only read here, so
    // both CTAs of a cluster see the same work list.
    if (tid == 0) {
        int acc = 0;
        for (int r = 0; r < a.R; ++r) {
            s_pre[r] = acc;
            acc += ld_cg(a.pairs + (int64_t)a.R * a.pmax + r);
        }
        s_pre[a.R] = acc;
        s_err = 0;
        for (int s = 0; s < kGStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 8);
        }
        mbar_init(mdone, 1);
        for (int j = 0; j < kGTQ; ++j) {
            mbar_init(&qfull[j], 1);
            mbar_init(&qempty[j], 10);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    const int ntile = s_pre[a.R] * a.ntiles;
    if (ntile == 0) return;  // both CTAs of the cluster
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(2 * kGBN));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    cluster_sync();  // both CTAs' barriers are initialised before either signals the other
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *tmem_slot;
    const int nk = a.H / kGBK;
    volatile int *err = &s_err;
    const uint32_t lead_qempty = mapa_shared(smem_u32(qempty), 0);
    // the n-th posted tile, read by a consumer (which then frees the entry);
    // -1 after a timeout
    auto take = [&](int n, bool release) -> int {
        const int j = n % kGTQ;
        if (!mbar_wait_cluster(&qfull[j], (uint32_t)((n / kGTQ) & 1))) return -1;
        const int t = *reinterpret_cast<volatile int *>(&tq[j]);
        if (release) mbar_arrive_cluster(lead_qempty + 8u * (uint32_t)j);
        return t;
    };

    if (warp == 4) {
        if (lane == 0) {
            uint32_t kit = 0;  // k-blocks loaded over all tiles: stage kit % kGStages
            for (int n = 0;; ++n) {
                int t;
                if (crank == 0) {  // claim and post the cluster's next tile
                    const int j = n % kGTQ;
                    if (n >= kGTQ && !mbar_wait_cluster(&qempty[j], (uint32_t)(((n / kGTQ) - 1) & 1))) {
                        atomicOr(a.status, MOONEP_STATUS_TIMEOUT);
                        *err = 1;
                        break;
                    }
                    t = atomicAdd(a.tile_ctr, 1);
                    const uint32_t q0 = smem_u32(&tq[j]), q1 = mapa_shared(q0, 1);
                    asm volatile("st.shared::cta.u32 [%0], %1;" ::"r"(q0), "r"(t) : "memory");
                    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(q1), "r"(t) : "memory");
                    const uint32_t b0 = smem_u32(&qfull[j]);
                    mbar_arrive_cluster(mapa_shared(b0, 0));
                    mbar_arrive_cluster(mapa_shared(b0, 1));
                } else {
                    t = take(n, true);
                    if (t < 0) {
                        atomicOr(a.status, MOONEP_STATUS_TIMEOUT);
                        *err = 1;
                        break;
                    }
                }
                if (t >= ntile) break;
                const GemmTile g = gemm_tile(a, s_pre, t, crank);
                const CUtensorMap *tb = g.slot ? &a.tp : &a.tw;
                bool ok = true;
                for (int kb = 0; kb < nk; ++kb, ++kit) {
                    const int s = (int)(kit % kGStages);
                    if (kit >= kGStages && !mbar_wait(&empty[s], ((kit / kGStages) - 1) & 1)) {
                        ok = false;
                        break;
                    }
                    const uint32_t bar = mapa_shared(smem_u32(&full[s]), 0);  // the leader's barrier
                    if (crank == 0) mbar_expect_tx(&full[s], 2 * (kGTileA + kGTileB));
                    tma_load_2d_pair(smem_u32(sA + s * kGTileA), &a.tx, kb * kGBK, g.r * a.nvs + g.row0, bar);
#pragma unroll
                    for (int qb = 0; qb < 2; ++qb)
                        tma_load_2d_pair(smem_u32(sB + s * kGTileB + qb * kGBoxB), tb,
                                         g.nt * kGBN + (int)crank * (kGBN / 2) + qb * 64, g.brow0 + kb * kGBK, bar);
                }
                if (!ok) {
                    atomicOr(a.status, MOONEP_STATUS_TIMEOUT);
                    *err = 1;
                    break;
                }
            }
        }
    } else if (warp == 5) {
        if (lane == 0 && crank == 0) {
            uint32_t kit = 0;
            for (int n = 0;; ++n) {
                const int t = take(n, true);
                if (t < 0 || t >= ntile) {
                    if (t < 0) atomicOr(a.status, MOONEP_STATUS_TIMEOUT);
                    break;
                }
                const int b = n & 1;
                if (n >= 2 && !mbar_wait(&tempty[b], ((n >> 1) - 1) & 1)) {
                    atomicOr(a.status, MOONEP_STATUS_TIMEOUT);
                    *err = 1;
                    break;
                }
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const uint32_t d = tmem + (uint32_t)(b * kGBN);
                bool ok = true;
                for (int kb = 0; kb < nk; ++kb, ++kit) {
                    const int s = (int)(kit % kGStages);
                    if (!mbar_wait(&full[s], (kit / kGStages) & 1)) {
                        ok = false;
                        break;
                    }
                    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                    const uint32_t a0 = smem_u32(sA + s * kGTileA), b0 = smem_u32(sB + s * kGTileB);
#pragma unroll
                    for (int k = 0; k < kGBK / 16; ++k)
                        umma_bf16_pair(d, desc_k_sw128(a0 + k * 32), desc_mn_sw128(b0 + k * 16 * 128), (kb | k) != 0);
                    umma_commit_pair(&empty[s]);  // frees stage s in both CTAs once these MMAs have read it
                }
                if (!ok) {
                    atomicOr(a.status, MOONEP_STATUS_TIMEOUT);
                    *err = 1;
                    break;
                }
                umma_commit_pair(&tfull[b]);  // both CTAs' accumulators b hold tile t
            }
            umma_commit_pair(mdone);  // after every MMA issued above has completed
        }
    } else {
        const uint32_t lead_tempty = mapa_shared(smem_u32(tempty), 0);
        for (int n = 0;; ++n) {
            const int t = __shfl_sync(0xffffffffu, lane == 0 ? take(n, true) : 0, 0);
            if (t < 0 || t >= ntile) {
                if (t < 0 && lane == 0) atomicOr(a.status, MOONEP_STATUS_TIMEOUT);
                break;
            }
            const int b = n & 1;
            const bool ok = __all_sync(0xffffffffu, mbar_wait(&tfull[b], (n >> 1) & 1));
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            if (!ok) {
                if (lane == 0) atomicOr(a.status, MOONEP_STATUS_TIMEOUT);
                *err = 1;
                break;
            }
            const GemmTile g = gemm_tile(a, s_pre, t, crank);
            if (g.live) {
                const int row = g.row0 + warp * 32 + lane;
                uint4 *yrow = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.y) +
                                                        ((int64_t)g.r * a.nvs + row) * a.Hp + g.nt * kGBN);
#pragma unroll 1
                for (int cc = 0; cc < kGBN / 32; ++cc) {
                    uint32_t v32[32];
                    const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(b * kGBN + cc * 32);
                    asm volatile(
                        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
                        "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
                        : "=r"(v32[0]), "=r"(v32[1]), "=r"(v32[2]), "=r"(v32[3]), "=r"(v32[4]), "=r"(v32[5]),
                          "=r"(v32[6]), "=r"(v32[7]), "=r"(v32[8]), "=r"(v32[9]), "=r"(v32[10]), "=r"(v32[11]),
                          "=r"(v32[12]), "=r"(v32[13]), "=r"(v32[14]), "=r"(v32[15]), "=r"(v32[16]), "=r"(v32[17]),
                          "=r"(v32[18]), "=r"(v32[19]), "=r"(v32[20]), "=r"(v32[21]), "=r"(v32[22]), "=r"(v32[23]),
                          "=r"(v32[24]), "=r"(v32[25]), "=r"(v32[26]), "=r"(v32[27]), "=r"(v32[28]), "=r"(v32[29]),
                          "=r"(v32[30]), "=r"(v32[31])
                        : "r"(taddr));
                    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                    uint32_t pk[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const __nv_bfloat162 h2 =
                            __floats2bfloat162_rn(__uint_as_float(v32[2 * j]), __uint_as_float(v32[2 * j + 1]));
                        pk[j] = *reinterpret_cast<const uint32_t *>(&h2);
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        yrow[cc * 4 + j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
                }
            }
            // this warp's quadrant of accumulator b may be overwritten
            asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(lead_tempty + 8u * (uint32_t)b);
        }
    }
    __syncwarp();
    // No CTA frees its tensor memory while MMAs of the pair may still write it.
    if (warp == 0 && lane == 0 && !mbar_wait(mdone, 0)) atomicOr(a.status, MOONEP_STATUS_TIMEOUT);
    __syncwarp();
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    cluster_sync();
    if (warp == 0) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * kGBN));
    }
}

// ---- host side ---------------------------------------------------------------

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 2-D bf16 tensor map over [rows, cols] (cols contiguous), box {64, box_rows}.
static bool make_map(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int gemm_supported(const Dims &d, int64_t Hp) {
    if (d.tp % kGBM != 0 || d.H % kGBK != 0 || Hp % kGBN != 0 || Hp <= 0) return MOONEP_ERR_SIZE;
    if ((int64_t)d.E * d.H > INT32_MAX || (int64_t)d.R * d.B * d.H > INT32_MAX ||
        (int64_t)d.R * d.nvs > INT32_MAX)
        return MOONEP_ERR_SIZE;
    return MOONEP_OK;
}

cudaError_t gemm_set_smem_limit() {
    return cudaFuncSetAttribute(group_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kGSmem);
}

int launch_group_gemm(const Dims &d, const moonep_plan_t *plan, const void *x, const void *W, const void *pool,
                      void *y, int64_t Hp, int32_t *pairs, cudaStream_t st) {
    GemmArgs a;
    memset(&a, 0, sizeof(a));
    if (!make_map(&a.tx, x, (uint64_t)d.R * d.nvs, d.H, kGBM) ||
        !make_map(&a.tw, W, (uint64_t)d.E * d.H, Hp, kGBK) ||
        !make_map(&a.tp, d.B > 0 ? pool : W, d.B > 0 ? (uint64_t)d.R * d.B * d.H : (uint64_t)d.E * d.H, Hp, kGBK))
        return MOONEP_ERR_CUDA;
    a.cu_seqlens = plan->cu_seqlens;
    a.pairs = pairs;
    a.status = plan->status;
    a.y = y;
    a.R = d.R;
    a.E = d.E;
    a.B = d.B;
    a.H = d.H;
    a.Hp = (int)Hp;
    a.nvs = d.nvs;
    a.NR = d.NR;
    a.pmax = gemm_pair_slots(d);
    a.tile_ctr = pairs + (int64_t)d.R * (a.pmax + 1);  // after the table and the per-rank counts
    a.ntiles = (int)(Hp / kGBN);
    pair_map_kernel<<<d.R, 256, 0, st>>>(plan->cu_seqlens, plan->status, pairs, d.NR, a.pmax);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail_cuda(e);
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kGThreads);
    cfg.dynamicSmemBytes = kGSmem;
    cfg.stream = st;
    // one cluster per pair of SMs; a cluster that cannot start until others
    // finish finds every tile claimed and leaves
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) == cudaSuccess)
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return fail_cuda(e);
    cfg.gridDim = dim3((unsigned)(sms < 2 ? 2 : sms & ~1));
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, group_gemm_kernel, a);
    return e == cudaSuccess ? MOONEP_OK : fail_cuda(e);
}

int gemm_pair_slots(const Dims &d) { return (d.nvs / kGBM + d.NR + 1) / 2; }

size_t gemm_table_bytes(const Dims &d) { return sizeof(int32_t) * ((size_t)d.R * (gemm_pair_slots(d) + 1) + 1); }

}  // namespace moonep
