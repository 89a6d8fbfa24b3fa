// The VM group GEMM that consumes a dispatched layer (MoonEP README,
// "Integration": one [E+B, H, H'] weight tensor per projection, with the
// planner's cu_seqlens selecting which expert row each token segment uses;
// "Weight buffer": rows [0, E) are the home experts, rows [E, E+B) this rank's
// prefetch slots).  For every rank r and every non-empty row i of its plan,
//   y[r, rows of i, :] = x[r, rows of i, :] @ Wrow(r, i),
// Wrow = W[i] for i < E (home rows, and inference overflow rows read from the
// home expert), pool[r][i - E] for slot rows.
//
// sm_100a design: a cluster of two CTAs (one per SM) computes a 256 x 256
// output tile with tcgen05.mma.cta_group::2 (bf16 x bf16 -> fp32, M=256,
// N=256, K=16).  Each CTA holds 128 rows of A and 128 of the 256 columns of
// B in shared memory, so an SM reads 16 KB of operands per MMA instead of the
// 24 KB a one-SM 128 x 256 tile needs; the one-SM design was bound by shared
// memory bandwidth (operand reads plus TMA fills) at about 70 % of the bf16
// peak.  Warp 0 of each CTA streams its halves through a 6-stage ring with
// 2-D TMA loads (128-byte swizzle, no multicast) that complete on the pair
// leader's mbarriers; one thread of the leader issues the MMAs into a
// 256-column accumulator in each CTA's tensor memory, and its commits free
// the stages and signal the accumulators in both CTAs; all four warps of each
// CTA read their 128 rows back (tcgen05.ld), round to bf16 and store.
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
constexpr int kGThreads = 128;
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
constexpr int kGSmem = 1024 + kGStages * (kGTileA + kGTileB) + 256;
constexpr uint32_t kGIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((uint32_t)(kGBN >> 3) << 17) |
                              ((uint32_t)(256 >> 4) << 24);

struct GemmArgs {
    CUtensorMap tx, tw, tp;
    const int32_t *cu_seqlens;  // [R, E+B]
    const int32_t *pairs;       // [R, pmax]: (plan row << 12) | pair index in the row, or -1
    int32_t *status;
    void *y;
    int R, E, B, H, Hp, nvs, NR, pmax, ntiles;
};

// pairs[r][q]: the q-th 256-row pair of rank r, in plan-row order; -1 past
// the last pair, and everywhere for a failed plan.
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
    const int used = failed ? 0 : s_carry;
    for (int q = used + tid; q < pmax; q += 256) out[q] = -1;
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

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGThreads, 1)
    group_gemm_kernel(const __grid_constant__ GemmArgs a) {
    extern __shared__ uint8_t gsm_raw[];
    uint8_t *gsm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(gsm_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *sA = gsm;
    uint8_t *sB = gsm + kGStages * kGTileA;
    uint64_t *full = reinterpret_cast<uint64_t *>(sB + kGStages * kGTileB);
    uint64_t *empty = full + kGStages;
    uint64_t *accum = empty + kGStages;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(accum + 1);
    __shared__ int s_v, s_start, s_lp, s_err;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint32_t crank;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(crank));
    const int c = blockIdx.x >> 1;
    const int nt = c % a.ntiles, rq = c / a.ntiles;
    const int r = rq / a.pmax, q = rq - r * a.pmax;

    pdl_wait();
    // The pair table is written before this kernel and read only here, so
    // both CTAs of a pair take the same decision.
    if (tid == 0) {
        const int v = ld_cg(a.pairs + (int64_t)r * a.pmax + q);
        s_v = v;
        s_err = 0;
        if (v >= 0) {
            const int i = v >> 12;
            const int32_t *cu = a.cu_seqlens + (int64_t)r * a.NR;
            const int end = ld_cg(cu + i), beg = i > 0 ? ld_cg(cu + i - 1) : 0;
            s_start = beg;
            s_lp = end - beg;
        }
    }
    __syncthreads();
    const int v = s_v;
    if (v < 0) return;  // both CTAs of the pair
    const int wrow = v >> 12, pj = v & 4095;
    const int off = 2 * kGBM * pj + kGBM * (int)crank;
    const bool live = off < s_lp;
    const int row0 = s_start + (live ? off : 2 * kGBM * pj);
    const CUtensorMap *tb = wrow < a.E ? &a.tw : &a.tp;
    const int brow0 = (wrow < a.E ? wrow : r * a.B + (wrow - a.E)) * a.H;

    if (tid == 0) {
        for (int s = 0; s < kGStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accum, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(kGBN));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    cluster_sync();  // both CTAs' barriers are initialised before either signals the other
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *tmem_slot;
    const int nk = a.H / kGBK;
    volatile int *err = &s_err;

    if (warp == 0 && lane == 0) {
        for (int kb = 0; kb < nk; ++kb) {
            const int s = kb % kGStages;
            if (kb >= kGStages && !mbar_wait(&empty[s], ((kb / kGStages) - 1) & 1)) {
                atomicOr(a.status, MOONEP_STATUS_TIMEOUT);
                *err = 1;
                break;
            }
            const uint32_t bar = mapa_shared(smem_u32(&full[s]), 0);  // the leader's barrier
            if (crank == 0) mbar_expect_tx(&full[s], 2 * (kGTileA + kGTileB));
            tma_load_2d_pair(smem_u32(sA + s * kGTileA), &a.tx, kb * kGBK, r * a.nvs + row0, bar);
#pragma unroll
            for (int qb = 0; qb < 2; ++qb)
                tma_load_2d_pair(smem_u32(sB + s * kGTileB + qb * kGBoxB), tb,
                                 nt * kGBN + (int)crank * (kGBN / 2) + qb * 64, brow0 + kb * kGBK, bar);
        }
    } else if (warp == 1 && lane == 0 && crank == 0) {
        for (int kb = 0; kb < nk; ++kb) {
            const int s = kb % kGStages;
            if (!mbar_wait(&full[s], (kb / kGStages) & 1)) {
                atomicOr(a.status, MOONEP_STATUS_TIMEOUT);
                *err = 1;
                break;
            }
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const uint32_t a0 = smem_u32(sA + s * kGTileA), b0 = smem_u32(sB + s * kGTileB);
#pragma unroll
            for (int k = 0; k < kGBK / 16; ++k)
                umma_bf16_pair(tmem, desc_k_sw128(a0 + k * 32), desc_mn_sw128(b0 + k * 16 * 128), (kb | k) != 0);
            umma_commit_pair(&empty[s]);  // frees stage s in both CTAs once these MMAs have read it
        }
        umma_commit_pair(accum);  // both CTAs' accumulators are complete
    }
    __syncwarp();

    const bool ok = __all_sync(0xffffffffu, mbar_wait(accum, 0));
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (!ok) {
        if (lane == 0) atomicOr(a.status, MOONEP_STATUS_TIMEOUT);
    } else if (live && !*err) {
        const int row = row0 + warp * 32 + lane;
        uint4 *yrow = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.y) +
                                                ((int64_t)r * a.nvs + row) * a.Hp + nt * kGBN);
#pragma unroll 1
        for (int cc = 0; cc < kGBN / 32; ++cc) {
            uint32_t v32[32];
            const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16) + cc * 32;
            asm volatile(
                "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
                "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
                : "=r"(v32[0]), "=r"(v32[1]), "=r"(v32[2]), "=r"(v32[3]), "=r"(v32[4]), "=r"(v32[5]), "=r"(v32[6]),
                  "=r"(v32[7]), "=r"(v32[8]), "=r"(v32[9]), "=r"(v32[10]), "=r"(v32[11]), "=r"(v32[12]),
                  "=r"(v32[13]), "=r"(v32[14]), "=r"(v32[15]), "=r"(v32[16]), "=r"(v32[17]), "=r"(v32[18]),
                  "=r"(v32[19]), "=r"(v32[20]), "=r"(v32[21]), "=r"(v32[22]), "=r"(v32[23]), "=r"(v32[24]),
                  "=r"(v32[25]), "=r"(v32[26]), "=r"(v32[27]), "=r"(v32[28]), "=r"(v32[29]), "=r"(v32[30]),
                  "=r"(v32[31])
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
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    cluster_sync();  // neither CTA frees its memory while the pair's MMAs may still read it
    if (warp == 0) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kGBN));
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
    a.ntiles = (int)(Hp / kGBN);
    pair_map_kernel<<<d.R, 256, 0, st>>>(plan->cu_seqlens, plan->status, pairs, d.NR, a.pmax);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail_cuda(e);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * (int64_t)d.R * a.pmax * a.ntiles));
    cfg.blockDim = dim3(kGThreads);
    cfg.dynamicSmemBytes = kGSmem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, group_gemm_kernel, a);
    return e == cudaSuccess ? MOONEP_OK : fail_cuda(e);
}

int gemm_pair_slots(const Dims &d) { return (d.nvs / kGBM + d.NR + 1) / 2; }

}  // namespace moonep
