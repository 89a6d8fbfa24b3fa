// The online planner (MoonEP README, "Performance" item 2 and "dispatch fwd";
// MarkTechPost, "Core idea: dynamic redundant experts").  The pages fix what
// the plan must satisfy -- exactly S*K slots per rank, copies from at most one
// remote home group per rank in training, overflow experts read from their
// home rows in inference, padded cu_seqlens[E+B] -- but print no rule.  The
// rule implemented here (alias chain over home-group loads, donors keep the
// prefix of their expert-ordered sequence) is documented with the C oracle.
//
// Two launches:
//   plan_count_kernel  one block per (source rank, chunk of kChunkTokens
//                      tokens): histogram of the chunk and the stable rank of
//                      every pick among the chunk's picks of its expert, by
//                      warp match/popc.  The last block to arrive (an atomic
//                      counter, no spinning) lays the plan out: prefix of the
//                      histograms over (rank, chunk), T_e, maxvio, the alias
//                      chain, rows, cu_seqlens.
//   plan_dst_kernel    one thread per pick: position in its group's sequence
//                      -> destination rank, row and slot.  Launched with
//                      programmatic dependent launch so its launch overlaps the
//                      layout step.
#include "moonep_internal.cuh"

namespace moonep {

static inline size_t align256(size_t b) { return (b + 255) / 256 * 256; }

size_t workspace_bytes(const Dims &d) {
    size_t n = 0;
    n += align256(sizeof(int32_t) * (size_t)d.R * d.nch * d.E);  // hist
    n += align256(sizeof(uint32_t));                               // arrive
    n += align256(sizeof(int32_t));                                // status
    n += align256(sizeof(int32_t) * (size_t)d.E);                  // estart
    n += align256(sizeof(int32_t) * (size_t)d.R);                  // keep
    n += align256(sizeof(int32_t) * 4 * (size_t)d.R);              // don
    n += align256(sizeof(int32_t));                                // ndon
    n += align256(sizeof(int32_t) * (size_t)d.R * d.G);            // rowmap
    n += align256(sizeof(int32_t) * (size_t)d.R * d.NR);           // rowstart
    return n;
}

void carve_workspace(const Dims &d, void *base, Workspace *ws) {
    char *p = static_cast<char *>(base);
    auto take = [&](size_t bytes) { char *q = p; p += align256(bytes); return q; };
    ws->hist = reinterpret_cast<int32_t *>(take(sizeof(int32_t) * (size_t)d.R * d.nch * d.E));
    ws->arrive = reinterpret_cast<uint32_t *>(take(sizeof(uint32_t)));
    ws->status = reinterpret_cast<int32_t *>(take(sizeof(int32_t)));
    ws->estart = reinterpret_cast<int32_t *>(take(sizeof(int32_t) * (size_t)d.E));
    ws->keep = reinterpret_cast<int32_t *>(take(sizeof(int32_t) * (size_t)d.R));
    ws->don = reinterpret_cast<int32_t *>(take(sizeof(int32_t) * 4 * (size_t)d.R));
    ws->ndon = reinterpret_cast<int32_t *>(take(sizeof(int32_t)));
    ws->rowmap = reinterpret_cast<int32_t *>(take(sizeof(int32_t) * (size_t)d.R * d.G));
    ws->rowstart = reinterpret_cast<int32_t *>(take(sizeof(int32_t) * (size_t)d.R * d.NR));
}

size_t plan_count_smem_bytes(const Dims &d) {
    const size_t count = sizeof(uint16_t) * ((size_t)kPlanWarps * d.E + 2 * (size_t)kChunkTokens * d.K);
    const size_t layout = sizeof(int32_t) * 3 * (size_t)d.E;
    return count > layout ? count : layout;
}

// ---- block-wide exclusive scan (kPlanThreads threads) -----------------------
__device__ __forceinline__ int warp_incl_scan(int v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    return v;
}

__device__ int block_excl_scan(int v, int *s_warp) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int incl = warp_incl_scan(v);
    if (lane == 31) s_warp[w] = incl;
    __syncthreads();
    if (w == 0) {
        const int x = lane < kPlanWarps ? s_warp[lane] : 0;
        const int xi = warp_incl_scan(x);
        if (lane < kPlanWarps) s_warp[lane] = xi - x;
    }
    __syncthreads();
    const int r = s_warp[w] + incl - v;
    __syncthreads();
    return r;
}

// ---- layout step, run by the last counting block ---------------------------
__device__ void plan_layout(const PlanArgs &a, uint8_t *smem) {
    const Dims &d = a.d;
    const int E = d.E, R = d.R, G = d.G, NR = d.NR, B = d.B;
    const int RN = R * d.nch;
    const int C = d.S * d.K;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;

    int32_t *T = reinterpret_cast<int32_t *>(smem);  // [E] picks per expert
    int32_t *ex = T + E;                             // [E] exclusive prefix of T over all experts
    int32_t *es = ex + E;                            // [E] start inside the group's sequence

    __shared__ int s_L[MOONEP_MAX_R], s_keep[MOONEP_MAX_R], s_cur[MOONEP_MAX_R];
    __shared__ int s_from[MOONEP_MAX_R], s_to[MOONEP_MAX_R], s_start[MOONEP_MAX_R], s_amt[MOONEP_MAX_R];
    __shared__ int s_rfrom[MOONEP_MAX_R], s_rstart[MOONEP_MAX_R], s_rlen[MOONEP_MAX_R];
    __shared__ int s_smallq[2 * MOONEP_MAX_R], s_largeq[MOONEP_MAX_R];
    __shared__ int s_ndon, s_maxT, s_status;
    __shared__ int s_warp[kPlanWarps];

    if (tid < R) s_L[tid] = 0;
    if (tid == 0) {
        s_maxT = 0;
        s_status = ld_cg(a.ws.status);
    }
    __syncthreads();

    // Step 1: per expert, exclusive prefix of the chunk histograms over
    // (source rank, chunk) -- the offset of each chunk's picks inside the
    // expert's run of its group sequence -- plus counts[r][e] and T_e.
    bool mismatch = false;
    for (int e = tid; e < E; e += kPlanThreads) {
        int run = 0, rsum = 0;
        for (int j0 = 0; j0 < RN; j0 += 16) {
            int v[16];
#pragma unroll
            for (int u = 0; u < 16; ++u)
                v[u] = (j0 + u < RN) ? ld_cg(a.ws.hist + (int64_t)(j0 + u) * E + e) : 0;
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int j = j0 + u;
                if (j < RN) {
                    __stcg(a.ws.hist + (int64_t)j * E + e, run);
                    run += v[u];
                    rsum += v[u];
                    if ((j + 1) % d.nch == 0) {
                        const int rr = j / d.nch;
                        a.plan.counts[(int64_t)rr * E + e] = rsum;
                        if (a.tpe && __ldg(a.tpe + (int64_t)rr * E + e) != rsum) mismatch = true;
                        rsum = 0;
                    }
                }
            }
        }
        T[e] = run;
        atomicAdd(&s_L[e / G], run);
        atomicMax(&s_maxT, run);
    }
    if (mismatch) atomicOr(&s_status, MOONEP_STATUS_COUNT_MISMATCH);
    __syncthreads();
    if (s_status != 0) {
        if (tid == 0) {
            *a.plan.status = s_status;
            *a.ws.status = 0;
            *a.ws.arrive = 0;
        }
        return;
    }

    // Step 2: maxvio and the alias chain over the group loads (one thread;
    // at most 2R iterations: every pass retires one under-loaded rank).
    if (tid == 0) {
        const double tbar = (double)((int64_t)R * d.S * d.K) / (double)E;
        *a.plan.maxvio = (float)((double)s_maxT / tbar - 1.0);
        int sh = MOONEP_MAX_R, st = MOONEP_MAX_R, lh = 0, lt = 0, nd = 0;
        for (int h = 0; h < R; ++h) {
            s_cur[h] = s_L[h];
            if (s_L[h] < C) s_smallq[st++] = h;
            if (s_L[h] > C) s_largeq[lt++] = h;
            s_rfrom[h] = -1;
            s_rstart[h] = 0;
            s_rlen[h] = 0;
        }
        while (sh < st && lh < lt) {
            const int s = s_smallq[sh++];
            const int l = s_largeq[lh];
            const int dd = C - s_cur[s];
            s_from[nd] = l;
            s_to[nd] = s;
            s_amt[nd] = dd;
            ++nd;
            s_cur[s] = C;
            s_cur[l] -= dd;
            if (s_cur[l] < C) {
                ++lh;
                s_smallq[--sh] = l;
            } else if (s_cur[l] == C) {
                ++lh;
            }
        }
        for (int h = 0; h < R; ++h) s_keep[h] = s_L[h];
        for (int j = 0; j < nd; ++j) s_keep[s_from[j]] -= s_amt[j];
        for (int h = 0; h < R; ++h) {
            int next = s_keep[h];
            for (int j = 0; j < nd; ++j)
                if (s_from[j] == h) {
                    s_start[j] = next;
                    next += s_amt[j];
                }
        }
        for (int j = 0; j < nd; ++j) {
            s_rfrom[s_to[j]] = s_from[j];
            s_rstart[s_to[j]] = s_start[j];
            s_rlen[s_to[j]] = s_amt[j];
        }
        s_ndon = nd;
        *a.ws.ndon = nd;
    }

    // Step 3: start of every expert inside its group's sequence.
    {
        const int per = (E + kPlanThreads - 1) / kPlanThreads;
        const int e0 = min(E, tid * per), e1 = min(E, e0 + per);
        int sum = 0;
        for (int e = e0; e < e1; ++e) sum += T[e];
        int run = block_excl_scan(sum, s_warp);
        for (int e = e0; e < e1; ++e) {
            ex[e] = run;
            run += T[e];
        }
    }
    __syncthreads();
    for (int e = tid; e < E; e += kPlanThreads) {
        es[e] = ex[e] - ex[(e / G) * G];
        a.ws.estart[e] = es[e];
    }
    for (int j = tid; j < R; j += kPlanThreads) {
        a.ws.keep[j] = s_keep[j];
        a.plan.assign[4 * j + 0] = s_keep[j];
        a.plan.assign[4 * j + 1] = s_rfrom[j];
        a.plan.assign[4 * j + 2] = s_rstart[j];
        a.plan.assign[4 * j + 3] = s_rlen[j];
    }
    for (int j = tid; j < s_ndon; j += kPlanThreads) {
        a.ws.don[j] = s_from[j];
        a.ws.don[R + j] = s_to[j];
        a.ws.don[2 * R + j] = s_start[j];
        a.ws.don[3 * R + j] = s_amt[j];
    }
    __syncthreads();

    // Step 4: rows of every rank (one warp per rank).
    for (int s = w; s < R; s += kPlanWarps) {
        int32_t *rc = a.plan.row_counts + (int64_t)s * NR;
        int32_t *se = a.plan.slot_expert + (int64_t)s * B;
        const int keep_s = s_keep[s];
        for (int i = lane; i < NR; i += 32) {
            int n = 0;
            if (i < E && i / G == s) n = max(0, min(es[i] + T[i], keep_s) - es[i]);
            rc[i] = n;
        }
        for (int b = lane; b < B; b += 32) se[b] = -1;
        __syncwarp();
        const int h = s_rfrom[s];
        if (h >= 0) {
            const int a0 = s_rstart[s], a1 = a0 + s_rlen[s];
            int q0 = 0;
            for (int j0 = 0; j0 < G; j0 += 32) {
                const int j = j0 + lane;
                const int e = h * G + j;
                int ov = 0;
                if (j < G) ov = max(0, min(es[e] + T[e], a1) - max(es[e], a0));
                const unsigned has = __ballot_sync(0xffffffffu, ov > 0);
                const int q = q0 + __popc(has & lanemask_lt());
                if (j < G) {
                    int row = -1;
                    if (ov > 0 && q < B) {
                        row = E + q;
                        se[q] = e;
                        rc[E + q] = ov;
                    } else if (ov > 0) {
                        row = e;  // inference overflow: the expert's home row
                        rc[e] = ov;
                    }
                    a.ws.rowmap[(int64_t)s * G + j] = row;
                }
                q0 += __popc(has);
            }
        }
        __syncwarp();
        int carry = 0;
        for (int i0 = 0; i0 < NR; i0 += 32) {
            const int i = i0 + lane;
            const int n = i < NR ? rc[i] : 0;
            const int p = n ? (n + d.tp - 1) / d.tp * d.tp : 0;
            const int incl = warp_incl_scan(p);
            if (i < NR) {
                a.plan.cu_seqlens[(int64_t)s * NR + i] = carry + incl;
                a.ws.rowstart[(int64_t)s * NR + i] = carry + incl - p;
            }
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
    }
    if (tid == 0) {
        *a.plan.status = 0;
        *a.ws.status = 0;
        *a.ws.arrive = 0;
    }
}

// ---- counting kernel ---------------------------------------------------------
__global__ void __launch_bounds__(kPlanThreads, 1) plan_count_kernel(PlanArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    const Dims &d = a.d;
    const int E = d.E, K = d.K;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    uint16_t *wcnt = reinterpret_cast<uint16_t *>(smem);  // [kPlanWarps][E] per-warp counts
    uint16_t *ent_e = wcnt + kPlanWarps * E;              // [kChunkTokens*K] expert of each pick
    uint16_t *ent_rank = ent_e + kChunkTokens * K;        // [kChunkTokens*K] rank inside its warp's run
    __shared__ int s_bad, s_last;

    const int r = blockIdx.x / d.nch, c = blockIdx.x - (blockIdx.x / d.nch) * d.nch;
    const int t0 = c * kChunkTokens;
    const int t1 = min(d.S, t0 + kChunkTokens);
    const int n_ent = (t1 - t0) * K;
    const int64_t base = ((int64_t)r * d.S + t0) * K;

    int bad = 0;
    for (int i = tid; i < kPlanWarps * E; i += kPlanThreads) wcnt[i] = 0;
    for (int i = tid; i < n_ent; i += kPlanThreads) {
        const int e = __ldg(a.topk + base + i);
        const bool good = e >= 0 && e < E;
        if (!good) bad |= MOONEP_STATUS_BAD_EXPERT;
        ent_e[i] = good ? (uint16_t)e : (uint16_t)0xFFFF;
    }
    if (tid == 0) s_bad = 0;
    __syncthreads();

    // Each warp walks a contiguous run of the chunk, 32 picks at a time, in
    // (token, k) order; peers with the same expert are found with match_any
    // and ranked by lane, so ranks follow token order (experts are distinct
    // within a token).
    const int per_warp = (n_ent + kPlanWarps * 32 - 1) / (kPlanWarps * 32) * 32;
    const int w0 = w * per_warp, w1 = min(n_ent, w0 + per_warp);
    uint16_t *mine = wcnt + w * E;
    for (int i0 = w0; i0 < w1; i0 += 32) {
        const int i = i0 + lane;
        const int e = i < w1 ? (int)ent_e[i] : 0xFFFF;
        const bool good = e != 0xFFFF;
        const unsigned peers = __match_any_sync(0xffffffffu, good ? e : E + lane);
        const int before = __popc(peers & lanemask_lt());
        const int prior = good ? (int)mine[e] : 0;
        __syncwarp();
        if (good && before == 0) mine[e] = (uint16_t)(prior + __popc(peers));
        __syncwarp();
        if (i < w1) ent_rank[i] = (uint16_t)(prior + before);
    }
    __syncthreads();

    // duplicate experts within a token
    for (int tt = tid; tt < t1 - t0; tt += kPlanThreads) {
        const uint16_t *tok = ent_e + tt * K;
        for (int k = 1; k < K; ++k) {
            const uint16_t ek = tok[k];
            if (ek == 0xFFFF) continue;
            for (int k2 = 0; k2 < k; ++k2)
                if (tok[k2] == ek) bad |= MOONEP_STATUS_DUP_EXPERT;
        }
    }
    // per-expert exclusive prefix over the warps; the chunk's histogram row
    int32_t *hrow = a.ws.hist + (int64_t)(r * d.nch + c) * E;
    for (int e = tid; e < E; e += kPlanThreads) {
        int run = 0;
#pragma unroll
        for (int w2 = 0; w2 < kPlanWarps; ++w2) {
            const int v = wcnt[w2 * E + e];
            wcnt[w2 * E + e] = (uint16_t)run;
            run += v;
        }
        __stcg(hrow + e, run);
    }
    __syncthreads();
    // stable rank of each pick inside the chunk, parked in dst until the
    // destination kernel replaces it
    for (int i = tid; i < n_ent; i += kPlanThreads) {
        const int e = ent_e[i];
        if (e != 0xFFFF) a.plan.dst[base + i] = (int)wcnt[(i / per_warp) * E + e] + (int)ent_rank[i];
    }

    bad = __reduce_or_sync(0xffffffffu, bad);
    if (lane == 0 && bad) atomicOr(&s_bad, bad);
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        if (s_bad) atomicOr(a.ws.status, s_bad);
        __threadfence();
        const unsigned prev = atomicAdd(a.ws.arrive, 1u);
        s_last = prev == gridDim.x - 1;
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    pdl_trigger();
    plan_layout(a, smem);
}

// ---- destination of every pick ---------------------------------------------
__global__ void __launch_bounds__(kDstThreads) plan_dst_kernel(PlanArgs a) {
    pdl_wait();
    if (ld_cg(a.plan.status) != 0) return;
    const Dims &d = a.d;
    const int64_t total = (int64_t)d.R * d.S * d.K;
    const int SK = d.S * d.K;
    const int nd = ld_cg(a.ws.ndon);
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int e = __ldg(a.topk + idx);
        const int r = (int)(idx / SK);
        const int t = (int)(idx - (int64_t)r * SK) / d.K;
        const int c = t / kChunkTokens;
        const int es = ld_cg(a.ws.estart + e);
        const int g = es + ld_cg(a.ws.hist + (int64_t)(r * d.nch + c) * d.E + e) + ld_cg(a.plan.dst + idx);
        const int h = e / d.G;
        int dest = h, row = e, off = g - es;
        if (g >= ld_cg(a.ws.keep + h)) {
            dest = -1;
            for (int j = 0; j < nd; ++j) {
                const int st = ld_cg(a.ws.don + 2 * d.R + j);
                if (ld_cg(a.ws.don + j) == h && g >= st && g < st + ld_cg(a.ws.don + 3 * d.R + j)) {
                    dest = ld_cg(a.ws.don + d.R + j);
                    off = g - max(es, st);
                    break;
                }
            }
            row = dest >= 0 ? ld_cg(a.ws.rowmap + (int64_t)dest * d.G + (e - h * d.G)) : -1;
            if (row < 0) {  // cannot happen for a consistent layout; never index with it
                atomicOr(a.plan.status, MOONEP_STATUS_BAD_PLAN);
                continue;
            }
        }
        a.plan.dst[idx] = dest * d.nvs + ld_cg(a.ws.rowstart + (int64_t)dest * d.NR + row) + off;
    }
}

cudaError_t launch_plan(const PlanArgs &a, int sms, cudaStream_t st) {
    const int grid = a.d.R * a.d.nch;
    const size_t smem = plan_count_smem_bytes(a.d);
    plan_count_kernel<<<grid, kPlanThreads, smem, st>>>(a);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;

    const int64_t total = (int64_t)a.d.R * a.d.S * a.d.K;
    int64_t blocks = (total + kDstThreads - 1) / kDstThreads;
    if (blocks > (int64_t)sms * 8) blocks = (int64_t)sms * 8;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(kDstThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, plan_dst_kernel, a);
}

cudaError_t plan_set_smem_limit(size_t bytes) {
    return cudaFuncSetAttribute(plan_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

}  // namespace moonep
