// The VM group GEMM that consumes a dispatched layer (MoonEP README,
// "Integration": one [E+B, H, H'] weight tensor per projection, with the
// planner's cu_seqlens selecting which expert row each token segment uses;
// "Weight buffer": rows [0, E) are the home experts, rows [E, E+B) this rank's
// prefetch slots).  For every rank r and every non-empty row i of its plan,
//   y[r, rows of i, :] = x[r, rows of i, :] @ Wrow(r, i),
// Wrow = W[i] for i < E (home rows, and inference overflow rows read from the
// home expert), pool[r][i - E] for slot rows.
//
// sm_100a design: one CTA per 128 x 256 output tile.  Warp 0 streams A (the
// tile's 128 buffer rows) and B (the row's weight) through a 4-stage ring in
// shared memory with TMA, 128-byte swizzled; warp 1 issues tcgen05.mma
// (bf16 x bf16 -> fp32, M=128, N=256, K=16) into a 256-column accumulator in
// tensor memory and frees each stage with tcgen05.commit; then all four warps
// read the accumulator back (tcgen05.ld, one warp per 32 lanes), round to
// bf16 and store.  Rows are 128-aligned inside their segments because the
// padding unit token_padding is a multiple of 128, so a tile never straddles
// two weight rows.  Every mbarrier wait is bounded; a timeout sets
// MOONEP_STATUS_TIMEOUT and the CTA drains what it issued before it frees the
// tensor memory.
#include <cuda.h>

#include "moonep_internal.cuh"

namespace moonep {

constexpr int kGBM = 128, kGBN = 256, kGBK = 64, kGStages = 4;
constexpr int kGThreads = 128;
constexpr int kGTileA = kGBM * kGBK * 2;     // 16 KB
constexpr int kGTileB = kGBK * kGBN * 2;     // 32 KB: 4 boxes of 64 K-rows x 64 columns
constexpr int kGBoxB = kGBK * 64 * 2;        // 8 KB
constexpr uint32_t kGPolls = 1u << 22;       // bounded mbarrier waits (try_wait suspends between polls)
constexpr int kGSmem = 1024 + kGStages * (kGTileA + kGTileB) + 256;

struct GemmArgs {
    CUtensorMap tx;  // x [R*NvS, H], box {64, 128}
    CUtensorMap tw;  // W [E*H, Hp], box {64, 64}
    CUtensorMap tp;  // pool [R*B*H, Hp], box {64, 64} (== tw when B == 0)
    const int32_t *cu_seqlens;  // [R, E+B]
    int32_t *status;            // plan status: read, TIMEOUT OR-ed in
    void *y;                    // [R*NvS, Hp] bf16
    int E, B, H, Hp, nvs, NR, mtiles;
};

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

// 2-D TMA tile load into this CTA's shared memory, completion on `bar`.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int c0, int c1, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
        : "memory");
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

// kind::f16 instruction descriptor: D fp32, A and B bf16, A K-major, B
// N-major, N = 256, M = 128.
constexpr uint32_t kGIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((uint32_t)(kGBN >> 3) << 17) |
                             ((uint32_t)(kGBM >> 4) << 24);

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(kGIdesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__global__ void __launch_bounds__(kGThreads, 1) group_gemm_kernel(const __grid_constant__ GemmArgs a) {
    extern __shared__ uint8_t gsm_raw[];
    // 1024-byte alignment for the swizzled tiles
    uint8_t *gsm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(gsm_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *sA = gsm;
    uint8_t *sB = gsm + kGStages * kGTileA;
    uint64_t *full = reinterpret_cast<uint64_t *>(sB + kGStages * kGTileB);
    uint64_t *empty = full + kGStages;
    uint64_t *accum = empty + kGStages;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(accum + 1);
    __shared__ int s_row, s_err;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nt = blockIdx.x;
    const int r = blockIdx.y / a.mtiles, row0 = (blockIdx.y - r * a.mtiles) * kGBM;

    pdl_wait();
    // the weight row of this tile: the first row i whose inclusive end
    // cu_seqlens[r][i] lies past row0 (none: the tile is past the used rows;
    // a failed plan: nothing to compute)
    if (tid == 0) {
        s_row = ld_cg(a.status) != 0 ? -1 : a.NR;
        s_err = 0;
    }
    __syncthreads();
    const int32_t *cu = a.cu_seqlens + (int64_t)r * a.NR;
    if (s_row >= 0)
        for (int i = tid; i < a.NR; i += kGThreads)
            if (ld_cg(cu + i) > row0) atomicMin(&s_row, i);
    __syncthreads();
    const int wrow = s_row;
    if (wrow < 0 || wrow >= a.NR) return;  // uniform over the block
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
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(kGBN));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *tmem_slot;
    const int nk = a.H / kGBK;

    if (warp == 0 && lane == 0) {
        // producer
        int issued = 0;
        for (int kb = 0; kb < nk; ++kb) {
            const int s = kb % kGStages;
            if (kb >= kGStages && !mbar_wait(&empty[s], ((kb / kGStages) - 1) & 1)) {
                atomicOr(a.status, MOONEP_STATUS_TIMEOUT);
                s_err = 1;
                break;
            }
            if (*(volatile int *)&s_err) break;
            mbar_expect_tx(&full[s], kGTileA + kGTileB);
            tma_load_2d(sA + s * kGTileA, &a.tx, kb * kGBK, r * a.nvs + row0, &full[s]);
#pragma unroll
            for (int q = 0; q < kGBN / 64; ++q)
                tma_load_2d(sB + s * kGTileB + q * kGBoxB, tb, nt * kGBN + q * 64, brow0 + kb * kGBK, &full[s]);
            issued = kb + 1;
        }
        // the last load issued into each stage has landed before anyone leaves
        for (int kb = max(0, issued - kGStages); kb < issued; ++kb)
            if (!mbar_wait(&full[kb % kGStages], (kb / kGStages) & 1)) atomicOr(a.status, MOONEP_STATUS_TIMEOUT);
    } else if (warp == 1 && lane == 0) {
        // MMA issuer
        for (int kb = 0; kb < nk; ++kb) {
            const int s = kb % kGStages;
            if (!mbar_wait(&full[s], (kb / kGStages) & 1)) {
                atomicOr(a.status, MOONEP_STATUS_TIMEOUT);
                s_err = 1;
                break;
            }
            if (*(volatile int *)&s_err) break;
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const uint32_t a0 = smem_u32(sA + s * kGTileA), b0 = smem_u32(sB + s * kGTileB);
#pragma unroll
            for (int k = 0; k < kGBK / 16; ++k)
                umma_bf16(tmem, desc_k_sw128(a0 + k * 32), desc_mn_sw128(b0 + k * 16 * 128), (kb | k) != 0);
            umma_commit(&empty[s]);  // the stage is free once these MMAs have read it
        }
        umma_commit(accum);  // every MMA issued above has completed
    }
    __syncwarp();

    // epilogue: warp w owns accumulator lanes (tile rows) 32w .. 32w+31
    const bool ok = __all_sync(0xffffffffu, mbar_wait(accum, 0));  // warp-uniform: tcgen05.ld is .aligned
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (!ok) {
        if (lane == 0) atomicOr(a.status, MOONEP_STATUS_TIMEOUT);
    } else if (!*(volatile int *)&s_err) {
        const int row = row0 + warp * 32 + lane;
        uint4 *yrow = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.y) +
                                                ((int64_t)r * a.nvs + row) * a.Hp + nt * kGBN);
#pragma unroll 1
        for (int c = 0; c < kGBN / 32; ++c) {
            uint32_t v[32];
            const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16) + c * 32;
            asm volatile(
                "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
                "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
                : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
                  "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
                  "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]),
                  "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]),
                  "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
                : "r"(taddr));
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
            uint32_t p[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
                p[j] = *reinterpret_cast<const uint32_t *>(&h2);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j)
                yrow[c * 4 + j] = make_uint4(p[4 * j], p[4 * j + 1], p[4 * j + 2], p[4 * j + 3]);
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 0) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kGBN));
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
                      void *y, int64_t Hp, cudaStream_t st) {
    GemmArgs a;
    memset(&a, 0, sizeof(a));
    if (!make_map(&a.tx, x, (uint64_t)d.R * d.nvs, d.H, kGBM) ||
        !make_map(&a.tw, W, (uint64_t)d.E * d.H, Hp, kGBK) ||
        !make_map(&a.tp, d.B > 0 ? pool : W, d.B > 0 ? (uint64_t)d.R * d.B * d.H : (uint64_t)d.E * d.H, Hp, kGBK))
        return MOONEP_ERR_CUDA;
    a.cu_seqlens = plan->cu_seqlens;
    a.status = plan->status;
    a.y = y;
    a.E = d.E;
    a.B = d.B;
    a.H = d.H;
    a.Hp = (int)Hp;
    a.nvs = d.nvs;
    a.NR = d.NR;
    a.mtiles = d.nvs / kGBM;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(Hp / kGBN), (unsigned)(d.R * a.mtiles));
    cfg.blockDim = dim3(kGThreads);
    cfg.dynamicSmemBytes = kGSmem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, group_gemm_kernel, a);
    return e == cudaSuccess ? MOONEP_OK : fail_cuda(e);
}

}  // namespace moonep
