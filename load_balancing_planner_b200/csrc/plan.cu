// The online planner (MoonEP README, "Performance" item 2 and "dispatch fwd";
// MarkTechPost, "Core idea: dynamic redundant experts").  The pages fix what
// the plan must satisfy -- exactly S*K slots per rank, copies from at most one
// remote home group per rank in training, overflow experts read from their
// home rows in inference, padded cu_seqlens[E+B] -- but print no rule.  The
// rule implemented here is this library's reading: the group sequence of home
// rank h lists its picks by (expert, source rank, token), experts in id order
// (or, in the fewest-copies mode, by pick count); an alias chain over
// the group loads decides who gives how much to whom; a donor keeps the prefix
// of its sequence and gives consecutive ranges after it; a recipient's copied
// experts take its slots in ascending id, overflow rows past B (inference).
//
// One cooperative launch, one block per (source rank, chunk of `ct` tokens),
// all blocks resident:
//   A. count: the chunk's picks go to shared memory; each warp ranks its runs
//      of 32 picks per expert with lane masks (shared-memory atomicOr, then
//      popc below the lane: token order), which also finds an expert picked
//      twice by one token; per-warp counts are scanned into the chunk's
//      histogram row (global), its per-rank counts and its picks per home
//      group, and every pick gets its stable rank inside the chunk.
//   -- grid barrier: one 64-bit arrive counter that only grows; bounded spin.
//   B. layout, computed by every block from the histograms (no second
//      barrier): T_e, maxvio, the alias chain (one warp, in closed form over
//      prefix sums of deficits and excesses; it runs on a spare warp during
//      the column pass, from the group loads the count phase summed), expert
//      starts, and per rank a compact row table with inclusive running sums.
//   C. every block writes a slice of cu_seqlens / row_counts / slot_expert,
//      then dst for its own picks from per-expert bases (one shared-memory
//      read per pick in the common case).
// One rank's share (src_rank >= 0) runs the same kernel over that rank's
// chunks only: the other ranks' counts come from the gathered table, which
// every block validates first, and the alias chain follows the column pass.
#include "moonep_internal.cuh"

#ifndef MOONEP_PLAN_COLSPLIT
#define MOONEP_PLAN_COLSPLIT 1
#endif
#ifndef MOONEP_PLAN_FOLDRANK
#define MOONEP_PLAN_FOLDRANK 1
#endif

namespace moonep {

__host__ __device__ static inline size_t align256(size_t b) { return (b + 255) / 256 * 256; }

size_t workspace_bytes(const Dims &d) {
    return align256(sizeof(int32_t) * (size_t)d.R * d.nch * d.E) +
           align256(sizeof(int32_t) * 2 * (size_t)d.R * d.E) + align256(sizeof(int32_t) * 2 * (size_t)d.R) +
           align256(4 * sizeof(uint64_t));
}

void carve_workspace(const Dims &d, void *base, Workspace *ws) {
    char *p = static_cast<char *>(base);
    ws->hist = reinterpret_cast<int32_t *>(p);
    p += align256(sizeof(int32_t) * (size_t)d.R * d.nch * d.E);
    ws->cnt = reinterpret_cast<int32_t *>(p);
    p += align256(sizeof(int32_t) * 2 * (size_t)d.R * d.E);
    ws->gload = reinterpret_cast<int32_t *>(p);
    p += align256(sizeof(int32_t) * 2 * (size_t)d.R);
    ws->arrive = reinterpret_cast<unsigned long long *>(p);        // [0] blocks arrived, ever
    ws->status = reinterpret_cast<int32_t *>(p + sizeof(uint64_t));  // [2] error bits, by call parity
}

// Shared memory: [region 1: max(per-warp counts, layout tables)] [picks: expert u16, rank i32]
__host__ __device__ static inline size_t counts_bytes(const Dims &d) {
    return align256(sizeof(uint16_t) * (size_t)d.cw * d.E);
}

__host__ __device__ static size_t region1_bytes(const Dims &d) {
    // counting phase: per-warp counts + per-warp lane masks; layout phase reuses it
    const size_t counts = counts_bytes(d) + sizeof(uint32_t) * (size_t)d.cw * d.E;
    // int32: T, pre, es, nhome, kbase, nrecv, ovfincl, recvstart, ebase, eend
    // (10 E), ebase2, eend2 (2 E, when fast2) + slotincl (R B) + pre2, dbase,
    // dlim (3 E, when xtab); int16: qidx (E) + slotj (R B)
    const size_t layout = sizeof(int32_t) * ((10 + 2 * (size_t)d.fast2 + 3 * (size_t)d.xtab) * d.E + (size_t)d.R * d.B) +
                          sizeof(int16_t) * ((size_t)d.E + (size_t)d.R * d.B + 2);
    return align256(counts > layout ? counts : layout);
}

// Block 0 keeps a copy of the router's local counts (loaded at kernel start,
// checked after the barrier) when they are small enough.
__host__ __device__ static inline bool tpe_in_smem(const Dims &d) { return (size_t)d.R * d.E <= 16384; }

// picks of the block's chunk: expert (u16) and rank inside the chunk (u16, < ct*K <= 65535)
__host__ __device__ static inline size_t ent_bytes(const Dims &d) {
    return 2 * align256(sizeof(uint16_t) * (size_t)d.ct * d.K);
}

size_t plan_smem_bytes(const Dims &d) {
    return region1_bytes(d) + ent_bytes(d) + (tpe_in_smem(d) ? sizeof(int32_t) * (size_t)d.R * d.E : 0);
}

// Phase timestamps for profiling builds (-DMOONEP_PLAN_TRACE); no code otherwise.
#ifdef MOONEP_PLAN_TRACE
__device__ unsigned long long g_plan_trace[1024][16];
#define PLAN_TRACE(k) PLAN_TRACE_BY(k, 0)
#define PLAN_TRACE_BY(k, t)                                                                \
    do {                                                                                   \
        if (threadIdx.x == (t) && blockIdx.x < 1024) {                                     \
            unsigned long long t_;                                                         \
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                         \
            g_plan_trace[blockIdx.x][k] = t_;                                              \
        }                                                                                  \
    } while (0)
extern "C" __attribute__((visibility("default"))) int moonep_plan_trace(unsigned long long *host, int n) {
    return (int)cudaMemcpyFromSymbol(host, g_plan_trace, sizeof(unsigned long long) * 16 * (size_t)n);
}
#else
#define PLAN_TRACE(k) \
    do {              \
    } while (0)
#define PLAN_TRACE_BY(k, t) \
    do {                    \
    } while (0)
#endif

// ---- warp / block helpers -------------------------------------------------
__device__ __forceinline__ int warp_incl_scan(int v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    return v;
}

__device__ __forceinline__ int warp_sum(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ int warp_max(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ int pad_to(int n, int tp) { return n ? (n + tp - 1) / tp * tp : 0; }

// Grid barrier over all blocks of a cooperative launch, split into arrive and
// wait so a block can do local work in between.  The counter only grows: at
// kernel start it holds k * gridDim.x (k calls done), every block adds one,
// and all wait until it reaches (k + 1) * gridDim.x, with a bounded number of
// polls (the handle's limit; a test hook can also add arrivals that never
// come, so every block gives up while the counter stays a multiple of the
// grid).  Both are called by every thread of the block.
__device__ void grid_arrive(unsigned long long *ctr) {
    __syncthreads();
    // release at GPU scope: the block's writes ordered before it by the
    // barrier above are visible to whoever acquires the counter
    if (threadIdx.x == 0) asm volatile("red.release.gpu.global.add.u64 [%0], 1;" ::"l"(ctr) : "memory");
}

__device__ bool grid_wait(unsigned long long *ctr, unsigned long long target, uint32_t polls) {
    __shared__ int s_ok;
    __syncthreads();
    if (threadIdx.x == 0) {
        int ok = 0;
        for (uint32_t it = 0; it < polls; ++it) {
            unsigned long long v;
            asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(ctr) : "memory");
            if (v >= target) {
                ok = 1;
                break;
            }
            if (it > 64) __nanosleep(32);
        }
        s_ok = ok;
    }
    __syncthreads();
    return s_ok != 0;
}

// Shared-memory outputs of the alias chain, indexed by rank.
struct AliasOut {
    int *keep, *rfrom, *rstart, *rlen, *doff, *dlist;
};

// The balancing assignment in closed form, run by one warp: rank h lives on
// lane h % 32, slot h / 32 (NS slots cover R <= 32 * NS ranks).  Out of line:
// its call sites (group and one-rank planning, both rank-slot counts) share
// one copy of the code.
template <int NS>
__device__ __noinline__ void alias_chain(int R, int C, const int *s_L, const AliasOut o) {
    const int lane = threadIdx.x & 31;
    int Lv[NS], D[NS], X[NS], Pin[NS], Qin[NS], Pex[NS], Qex[NS];
    int carryP = 0, carryQ = 0;
#pragma unroll
    for (int sl = 0; sl < NS; ++sl) {
        const int h = lane + 32 * sl;
        Lv[sl] = h < R ? s_L[h] : C;
        D[sl] = max(C - Lv[sl], 0);
        X[sl] = max(Lv[sl] - C, 0);
        Pin[sl] = warp_incl_scan(D[sl]) + carryP;
        Qin[sl] = warp_incl_scan(X[sl]) + carryQ;
        carryP = __shfl_sync(0xffffffffu, Pin[sl], 31);
        carryQ = __shfl_sync(0xffffffffu, Qin[sl], 31);
        Pex[sl] = Pin[sl] - D[sl];
        Qex[sl] = Qin[sl] - X[sl];
    }
    unsigned smallb[NS], largeb[NS];
#pragma unroll
    for (int sl = 0; sl < NS; ++sl) {
        smallb[sl] = __ballot_sync(0xffffffffu, D[sl] > 0);
        largeb[sl] = __ballot_sync(0xffffffffu, X[sl] > 0);
    }
    int donor[NS], off[NS], amt[NS];
#pragma unroll
    for (int sl = 0; sl < NS; ++sl) donor[sl] = -1, off[sl] = 0, amt[sl] = 0;
    // small ranks: the large rank whose excess interval holds Pex
#pragma unroll
    for (int sl2 = 0; sl2 < NS; ++sl2)
        for (unsigned m = largeb[sl2]; m; m &= m - 1) {
            const int l = __ffs(m) - 1;
            const int qe = __shfl_sync(0xffffffffu, Qex[sl2], l);
            const int qi = __shfl_sync(0xffffffffu, Qin[sl2], l);
#pragma unroll
            for (int sl = 0; sl < NS; ++sl)
                if (D[sl] > 0 && qe <= Pex[sl] && Pex[sl] < qi) {
                    donor[sl] = l + 32 * sl2;
                    off[sl] = Pex[sl] - qe;
                    amt[sl] = D[sl];
                }
        }
    // drained large ranks: a small demand interval strictly holds Qin; the
    // rest comes from the next large rank
#pragma unroll
    for (int sl2 = 0; sl2 < NS; ++sl2)
        for (unsigned m = smallb[sl2]; m; m &= m - 1) {
            const int s = __ffs(m) - 1;
            const int pe = __shfl_sync(0xffffffffu, Pex[sl2], s);
            const int pi = __shfl_sync(0xffffffffu, Pin[sl2], s);
#pragma unroll
            for (int sl = 0; sl < NS; ++sl)
                if (X[sl] > 0 && pe < Qin[sl] && Qin[sl] < pi) {
                    int nxt = -1;
                    const unsigned above_mask = ~((2u << lane) - 1u);  // lanes above this one (0 for lane 31)
#pragma unroll
                    for (int t = NS - 1; t >= sl; --t) {
                        const unsigned cand = t == sl ? (largeb[t] & above_mask) : largeb[t];
                        if (cand) nxt = 32 * t + __ffs(cand) - 1;
                    }
                    donor[sl] = nxt;
                    off[sl] = 0;
                    amt[sl] = pi - Qin[sl];
                }
        }
    int keep[NS], start[NS];
#pragma unroll
    for (int sl = 0; sl < NS; ++sl) keep[sl] = D[sl] > 0 ? Lv[sl] : C - (X[sl] > 0 ? amt[sl] : 0);
#pragma unroll
    for (int sl = 0; sl < NS; ++sl) {
        const int dl = donor[sl] < 0 ? 0 : donor[sl];
        int kd = 0;
#pragma unroll
        for (int t = 0; t < NS; ++t) {
            const int k = __shfl_sync(0xffffffffu, keep[t], dl & 31);
            if ((dl >> 5) == t) kd = k;
        }
        start[sl] = donor[sl] < 0 ? 0 : kd + off[sl];
    }
    PLAN_TRACE(9);
    // recipients of each donor in increasing start order
    int pos[NS], cnt[NS];
#pragma unroll
    for (int sl = 0; sl < NS; ++sl) pos[sl] = 0, cnt[sl] = 0;
#pragma unroll
    for (int sl2 = 0; sl2 < NS; ++sl2) {
        const unsigned rb = __ballot_sync(0xffffffffu, donor[sl2] >= 0);
        for (unsigned m = rb; m; m &= m - 1) {
            const int s = __ffs(m) - 1;
            const int dn = __shfl_sync(0xffffffffu, donor[sl2], s);
            const int st = __shfl_sync(0xffffffffu, start[sl2], s);
#pragma unroll
            for (int sl = 0; sl < NS; ++sl) {
                if (donor[sl] == dn && st < start[sl]) ++pos[sl];
                if (dn == lane + 32 * sl) ++cnt[sl];
            }
        }
    }
    int doff[NS], carry = 0;
#pragma unroll
    for (int sl = 0; sl < NS; ++sl) {
        const int incl = warp_incl_scan(cnt[sl]) + carry;
        carry = __shfl_sync(0xffffffffu, incl, 31);
        doff[sl] = incl - cnt[sl];
    }
#pragma unroll
    for (int sl = 0; sl < NS; ++sl) {
        const int h = lane + 32 * sl;
        if (h < R) {
            o.keep[h] = keep[sl];
            o.rfrom[h] = donor[sl];
            o.rstart[h] = start[sl];
            o.rlen[h] = amt[sl];
            o.doff[h] = doff[sl];
        }
        if (h == R) o.doff[R] = doff[sl];
    }
    if (R == 32 * NS && lane == 0) o.doff[R] = carry;
    __syncwarp();
#pragma unroll
    for (int sl = 0; sl < NS; ++sl) {
        const int h = lane + 32 * sl;
        if (h < R && donor[sl] >= 0) o.dlist[o.doff[donor[sl]] + pos[sl]] = h;
    }
}

// Expert starts inside their group sequences in the fewest-copies order
// (pick count ascending, ties by id): an expert starts after every expert of
// its group that sorts before it.  Warps 1.. of the block; out of line, so
// the kernel's own code is laid out the same in every mode.
__device__ __noinline__ void expert_starts_by_count(const int32_t *T, int32_t *es, int E, int R, int G) {
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    if (G <= 32) {
        // one warp per group, expert j on lane j: the counts go round the warp once
        for (int h = w - 1; w >= 1 && h < R; h += kPlanWarps - 1) {
            const int te = lane < G ? T[h * G + lane] : 0;
            int sum = 0;
#pragma unroll 8
            for (int m = 0; m < 32; ++m) {
                const int tm = __shfl_sync(0xffffffffu, te, m);
                sum += (m < G && (tm < te || (tm == te && m < lane))) ? tm : 0;
            }
            if (lane < G) es[h * G + lane] = sum;
        }
    } else {
        for (int e = tid - 32; w >= 1 && e < E; e += kPlanThreads - 32) {
            const int g0 = e - e % G, te = T[e];
            int sum = 0;
            for (int m = g0; m < g0 + G; ++m) {
                const int tm = T[m];
                if (tm < te || (tm == te && m < e)) sum += tm;
            }
            es[e] = sum;
        }
    }
}

// The helpers below hold paths that the common configurations never take (or
// take on a few threads), kept out of line with the alias chain: the planner
// is latency-bound, its warps fetch their code cold after the streaming
// kernels of a layer, and every cache line of code on the way costs time, so
// the kernel's own path stays compact.

// Duplicate picks token by token, for K that does not divide 32 (a token's
// picks then straddle the counting warps' runs of 32).  Out of line: the
// common K keep it off the kernel's own code path.
__device__ __noinline__ int dup_by_token(const uint16_t *ent_e, int ntok, int K) {
    int bad = 0;
    for (int tt = threadIdx.x; tt < ntok; tt += kPlanThreads) {
        const uint16_t *tok = ent_e + tt * K;
        for (int k = 1; k < K; ++k) {
            const uint16_t ek = tok[k];
            if (ek == 0xFFFF) continue;
            for (int k2 = 0; k2 < k; ++k2)
                if (tok[k2] == ek) bad |= MOONEP_STATUS_DUP_EXPERT;
        }
    }
    return bad;
}

// The column pass in one loop per expert (rows of the per-rank counts, then
// this rank's earlier chunk rows), for configurations whose layout tables
// leave no room for the split form.  Returns this thread's count mismatch.
__device__ __noinline__ bool column_pass_one_loop(const PlanArgs &a, const int32_t *cnt, const int32_t *own,
                                                  const int32_t *mine_rows, const int32_t *tpe_s, int32_t *T,
                                                  int32_t *pre, int r, int c, bool checker, bool one_rank) {
    const Dims &d = a.d;
    const int E = d.E, R = d.R, nrows = R + c;
    bool mismatch = false;
    for (int e = threadIdx.x; e < E; e += kPlanThreads) {
        int tot = 0, mypre = 0, myv = 0;
        for (int q0 = 0; q0 < nrows; q0 += 16) {
            int v[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int q = q0 + u;
                const int32_t *src = q < R ? cnt + (int64_t)q * E + e : mine_rows + (int64_t)(q - R) * E + e;
                v[u] = q < nrows ? ld_cg(src) : 0;
            }
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int q = q0 + u;
                if (q < R) {
                    tot += v[u];
                    if (q < r) mypre += v[u];
                    if (q == r) myv = v[u];
                    if (checker && !one_rank) {
                        const int t = tpe_in_smem(d) ? tpe_s[q * E + e] : __ldg(a.tpe + (int64_t)q * E + e);
                        if (t != v[u]) mismatch = true;
                    }
                } else {
                    mypre += v[u];  // 0 past the last row
                }
            }
        }
        T[e] = tot;
        pre[e] = mypre;
        if (c == 0 && !one_rank) a.plan.counts[(int64_t)r * E + e] = myv;
        if (checker && one_rank && ld_cg(own + e) != myv) mismatch = true;  // the rank's own row
    }
    return mismatch;
}

// One rank's planning: the gathered counts must hold S*K non-negative picks
// per rank, or the layout is undefined.  Every block checks every row (so all
// take the same decision); block 0 copies the rows into the plan.
__device__ __noinline__ void check_gathered_counts(const PlanArgs &a, int *s_cbad) {
    const Dims &d = a.d;
    const int E = d.E, R = d.R, lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    for (int q = w; q < R; q += kPlanWarps) {
        const int32_t *row = a.counts_all + (int64_t)q * E;
        long long sum = 0;
        bool neg = false;
        for (int e0 = 0; e0 < E; e0 += 32 * 8) {
            int v[8];  // all loads of a batch in flight before any store
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int e = e0 + 32 * u + lane;
                v[u] = e < E ? ld_cg(row + e) : 0;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int e = e0 + 32 * u + lane;
                neg |= v[u] < 0;
                sum += v[u];
                if (blockIdx.x == 0 && e < E) a.plan.counts[(int64_t)q * E + e] = v[u];
            }
        }
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        const bool rowbad = __any_sync(0xffffffffu, neg) || sum != (long long)d.S * d.K;
        if (lane == 0 && rowbad) atomicOr(s_cbad, MOONEP_STATUS_COUNT_MISMATCH);
    }
}

// Block 0 of group planning: the router's local counts against the counts of
// this call, every (rank, expert) once.  Run by the threads that have no
// column-pass work, so it stays off the other threads' path; thread t of n
// takes entries t, t + n, ..., 8 loads in flight per batch, so the check
// costs one round of loads like the column pass beside it.
__device__ __noinline__ bool check_router_counts(const PlanArgs &a, const int32_t *cnt, const int32_t *tpe_s,
                                                 int t, int n) {
    const Dims &d = a.d;
    const int tot = d.R * d.E;
    bool mismatch = false;
    for (int i0 = t; i0 < tot; i0 += 8 * n) {
        int v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = i0 + u * n;
            v[u] = i < tot ? ld_cg(cnt + i) : 0;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = i0 + u * n;
            if (i < tot && v[u] != (tpe_in_smem(d) ? tpe_s[i] : __ldg(a.tpe + i))) mismatch = true;
        }
    }
    return mismatch;
}

// Mode 2: rank s takes into its B slots the received experts with the most
// picks (ties to the lower index).  nrecv_s holds every received expert's
// picks; expert j with ov picks is taken when fewer than B beat it.
__device__ __noinline__ bool take_by_count(const int32_t *nrecv_s, int G, int j, int ov, int B) {
    int better = 0;
    for (int m = 0; m < G; ++m) {
        const int om = nrecv_s[m];
        better += (om > ov) || (om == ov && m < j);
    }
    return better < B;
}

// Fold this block's offset of each expert (its start in the group sequence
// plus the picks of earlier chunks) into the kept-pick base and limit, so a
// pick of rank rk inside the chunk needs only rk: its position in the group
// sequence is g = off + rk.  T and pre are rewritten (the outputs never read
// them).  Used when the layout tables have no room for the rank pass to do it.
__device__ __noinline__ void fold_chunk_offsets(int32_t *T, int32_t *pre, const int32_t *es, const int32_t *pre2,
                                                const int32_t *kbase, const int *s_keep, int E, int G, int t, int n) {
    for (int e = t; e < E; e += n) {
        const int off = es[e] + pre[e] + (pre2 ? pre2[e] : 0);
        T[e] = kbase[e] + off;          // kept pick: dst = T[e] + rk ...
        pre[e] = s_keep[e / G] - off;   // ... while rk < pre[e]
    }
}

// ---- the planner kernel ----------------------------------------------------
// 1024 threads per block: the register budget is 64 per thread.
__global__ void __launch_bounds__(kPlanThreads, 1) plan_kernel(const __grid_constant__ PlanArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    const Dims &d = a.d;
    const int E = d.E, K = d.K, R = d.R, G = d.G, B = d.B, NR = d.NR, tp = d.tp;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;

    uint8_t *region1 = smem;
    uint16_t *ent_e = reinterpret_cast<uint16_t *>(smem + region1_bytes(d));
    uint16_t *ent_rank = reinterpret_cast<uint16_t *>(reinterpret_cast<uint8_t *>(ent_e) +
                                                      align256(sizeof(uint16_t) * (size_t)d.ct * K));
    int32_t *tpe_s = reinterpret_cast<int32_t *>(smem + region1_bytes(d) + ent_bytes(d));  // [R][E], block 0
    // one_rank: the grid covers one source rank's chunks, and the per-rank
    // counts come from the caller (every rank's router counts, gathered)
    const bool one_rank = a.src_rank >= 0;
    const bool checker = blockIdx.x == 0 && (one_rank || a.tpe != nullptr);
    const int CW = d.cw;
    uint16_t *wcnt = reinterpret_cast<uint16_t *>(region1);                       // [CW][E]
    uint32_t *wmask = reinterpret_cast<uint32_t *>(region1 + counts_bytes(d));    // [CW][E]
    const int row = one_rank ? a.src_rank * d.nch + (int)blockIdx.x : (int)blockIdx.x;  // histogram row = r * nch + c
    const int r = row / d.nch, c = row - r * d.nch;
    const int t0 = c * d.ct;
    const int t1 = min(d.S, t0 + d.ct);
    const int n_ent = (t1 - t0) * K;
    // picks (and their dst) of this chunk: [R,S,K] for the group, [S,K] for one rank
    const int64_t base = ((one_rank ? 0 : (int64_t)r * d.S) + t0) * K;
    // the chunk's first picks are loaded before the clears below, so their
    // latency overlaps them
    int pk[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int i = tid + u * kPlanThreads;
        pk[u] = i < n_ent ? __ldg(a.topk + base + i) : 0;
    }
    for (int i = tid; i < CW * E; i += kPlanThreads) {
        wcnt[i] = 0;
        wmask[i] = 0u;
    }
    // the plan's status starts at 0 (block 0, before the grid barrier); every
    // later update is an atomicOr, so no error bit can be overwritten
    if (blockIdx.x == 0 && tid == 0) *a.plan.status = 0;
    if (checker && !one_rank && tpe_in_smem(d))
        for (int i = tid; i < R * E; i += kPlanThreads) tpe_s[i] = __ldg(a.tpe + i);

    __shared__ unsigned long long s_call;
    __shared__ int s_bad;
    __shared__ int s_gl[MOONEP_MAX_R];  // this chunk's picks per home group
    if (tid < MOONEP_MAX_R) s_gl[tid] = 0;
    if (tid == 0) {
        s_call = *reinterpret_cast<volatile unsigned long long *>(a.ws.arrive) / gridDim.x;
        s_bad = 0;
    }

    PLAN_TRACE(0);

    // ---------------- A. count ----------------
    int bad = 0;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int i = tid + u * kPlanThreads;
        if (i < n_ent) {
            const int e = pk[u];
            const bool good = e >= 0 && e < E;
            if (!good) bad |= MOONEP_STATUS_BAD_EXPERT;
            ent_e[i] = good ? (uint16_t)e : (uint16_t)0xFFFF;
        }
    }
    for (int i = tid + 2 * kPlanThreads; i < n_ent; i += kPlanThreads) {
        const int e = __ldg(a.topk + base + i);
        const bool good = e >= 0 && e < E;
        if (!good) bad |= MOONEP_STATUS_BAD_EXPERT;
        ent_e[i] = good ? (uint16_t)e : (uint16_t)0xFFFF;
    }
    __syncthreads();
    PLAN_TRACE(6);
    // Each counting warp walks a contiguous run of the chunk, 32 picks at a
    // time in (token, k) order.  The lanes holding the same expert find each
    // other through a per-warp lane-mask word per expert (shared-memory
    // atomicOr, read back, cleared), and are ranked by lane, so ranks follow
    // token order.  When K divides 32 every group of 32 holds whole tokens,
    // and a peer inside the lane's own token is a duplicate.  Runs are a
    // power of two long (>= 32) so a pick's warp is a shift away.
    int lg_run = 5;
    while ((CW << lg_run) < n_ent) ++lg_run;
    const int per_warp = 1 << lg_run;
    const bool whole_tokens = (32 % K) == 0;
    const unsigned tok_bits = K >= 32 ? 0xffffffffu : ((1u << K) - 1u);
    const unsigned tok_mask = whole_tokens ? tok_bits << (lane - lane % K) : 0u;
    if (w < CW) {
        const int w0 = w * per_warp, w1 = min(n_ent, w0 + per_warp);
        uint16_t *mine = wcnt + w * E;
        uint32_t *msk = wmask + w * E;
        for (int i0 = w0; i0 < w1; i0 += 32) {
            const int i = i0 + lane;
            const int e = i < w1 ? (int)ent_e[i] : 0xFFFF;
            const bool good = e != 0xFFFF;
            if (good) atomicOr(msk + e, 1u << lane);
            __syncwarp();
            const unsigned peers = good ? msk[e] : (1u << lane);
            __syncwarp();
            if (good) msk[e] = 0u;
            if (good && __popc(peers & tok_mask) > 1) bad |= MOONEP_STATUS_DUP_EXPERT;
            const int before = __popc(peers & lanemask_lt());
            const int prior = good ? (int)mine[e] : 0;
            __syncwarp();
            if (good && before == 0) mine[e] = (uint16_t)(prior + __popc(peers));
            __syncwarp();
            if (i < w1) ent_rank[i] = (uint16_t)(prior + before);
        }
    }
    if (!whole_tokens) bad |= dup_by_token(ent_e, t1 - t0, K);  // tokens straddle runs
    __syncthreads();
    PLAN_TRACE(7);
    // chunk totals: the histogram row (read back by this rank's later chunks)
    // and an exact integer add into the per-rank counts of this call
    const unsigned long long call = s_call;
    const int parity = (int)(call & 1);
    int32_t *hrow = a.ws.hist + (int64_t)row * E;
    int32_t *crow = a.ws.cnt + ((size_t)parity * R + r) * E;
    for (int e = tid; e < E; e += kPlanThreads) {
        int run = 0;
        for (int w2 = 0; w2 < CW; ++w2) {
            const int v = wcnt[w2 * E + e];
            wcnt[w2 * E + e] = (uint16_t)run;
            run += v;
        }
        __stcg(hrow + e, run);
        if (run) {
            atomicAdd(crow + e, run);
            if (!one_rank) atomicAdd(&s_gl[e / G], run);
        }
    }
    bad = __reduce_or_sync(0xffffffffu, bad);
    if (lane == 0 && bad) atomicOr(&s_bad, bad);
    __syncthreads();
    if (tid == 0 && s_bad) atomicOr(a.ws.status + parity, s_bad);
    // the group loads of this call, complete at the grid barrier
    if (!one_rank && tid < R && s_gl[tid]) atomicAdd(a.ws.gload + (size_t)parity * R + tid, s_gl[tid]);
    PLAN_TRACE(8);
    grid_arrive(a.ws.arrive);
    // while the other blocks arrive: each pick's rank inside the chunk
    for (int i = tid; i < n_ent; i += kPlanThreads) {
        const int e = ent_e[i];
        if (e != 0xFFFF) ent_rank[i] = (uint16_t)(ent_rank[i] + wcnt[(i >> lg_run) * E + e]);
    }
    // The next call's tables (the other parity) start at zero.  No block of
    // this call reads or writes them, and the next call starts after this
    // kernel ends, so they are cleared here, before the wait: a block that
    // gives up waiting still leaves them clean.
    if (blockIdx.x == 0 && tid == 0) a.ws.status[parity ^ 1] = 0;
    if (blockIdx.x == 0 && tid < R) a.ws.gload[(size_t)(parity ^ 1) * R + tid] = 0;
    {
        int32_t *next = a.ws.cnt + (size_t)(parity ^ 1) * R * E;
        const int64_t tot = (int64_t)R * E, per = (tot + gridDim.x - 1) / gridDim.x;
        for (int64_t i = (int64_t)blockIdx.x * per + tid; i < min(tot, (int64_t)(blockIdx.x + 1) * per);
             i += kPlanThreads)
            next[i] = 0;
    }
    PLAN_TRACE(5);
    if (!grid_wait(a.ws.arrive, (call + 1) * gridDim.x + a.withheld, a.polls)) {
        if (tid == 0) atomicOr(a.plan.status, MOONEP_STATUS_TIMEOUT);
        return;
    }
    PLAN_TRACE(1);

    // ---------------- B. layout (every block) ----------------
    // T and pre are rewritten, once the outputs no longer need them, into the
    // dst base and the rank limit of each expert's kept picks in this chunk
    int32_t *T = reinterpret_cast<int32_t *>(region1);  // [E] picks per expert
    int32_t *pre = T + E;               // [E] picks of each expert in histogram rows before this block's
    int32_t *es = pre + E;              // [E] start of each expert inside its group sequence
    int32_t *nhome = es + E;            // [E] kept picks of expert e on its home rank
    // [E] first the inclusive padded running sum over the home rows of e's
    // rank, then the dst base of a kept pick of e (dst = kbase[e] + position)
    int32_t *kbase = nhome + E;
    int32_t *nrecv = kbase + E;         // [R*G] picks of the j-th donor-group expert received by rank s
    int32_t *ovfincl = nrecv + E;       // [R*G] inclusive padded running sum over the overflow rows
    int32_t *recvstart = ovfincl + E;   // [R*G] first slot of the row holding that received expert
    // [E] e's donated picks at their first recipient: dst = ebase[e] + rk for
    // a pick of chunk rank rk below eend[e] (both relative to this chunk)
    int32_t *ebase = recvstart + E;
    int32_t *eend = ebase + E;
    int32_t *ebase2 = eend + E;         // [E] the same for the second recipient (fast2 only)
    int32_t *eend2 = ebase2 + E;        // [E]
    int32_t *slotincl = eend + E + (d.fast2 ? 2 * E : 0);  // [R*B] inclusive padded running sum over the slot rows
    // [E] picks of e in this rank's earlier chunks, when the column pass
    // sums those rows on warps of their own (pre then holds only the picks
    // of earlier ranks)
    int32_t *pre2 = slotincl + R * B;
    // [E] the dst base of a kept pick of e relative to this chunk, and the
    // chunk rank below which picks of e are kept (set in the rank pass)
    int32_t *dbase = pre2 + E;
    int32_t *dlim = dbase + E;
    // (pre2, dbase and dlim exist when the layout tables have room: d.xtab)
    int16_t *qidx = reinterpret_cast<int16_t *>(slotincl + R * B + (d.xtab ? 3 * E : 0));  // [R*G] received-expert index, -1 none
    int16_t *slotj = qidx + E;          // [R*B] donor-group index of the expert in slot b

    __shared__ int s_L[MOONEP_MAX_R], s_keep[MOONEP_MAX_R];
    __shared__ int s_rfrom[MOONEP_MAX_R], s_rstart[MOONEP_MAX_R], s_rlen[MOONEP_MAX_R];
    __shared__ int s_dlist[MOONEP_MAX_R], s_doff[MOONEP_MAX_R + 1];
    __shared__ int s_hsize[MOONEP_MAX_R], s_osize[MOONEP_MAX_R], s_nslot[MOONEP_MAX_R];
    __shared__ int s_status, s_wmax[kPlanWarps];

    if (tid == kPlanThreads - 1) s_status = ld_cg(a.ws.status + parity);
    // Group planning: the count phase summed the group loads, so one warp
    // with no column-pass work (when E < 32 * (kPlanWarps - 1)) runs the alias
    // chain while the others do the column pass.  One rank's planning gets
    // its loads from the column pass below.
    const int aw = min(kPlanWarps - 1, (E + 31) / 32);
    // the split column pass: experts on threads [0, E) and again on the
    // threads after the alias warp, [col2, col2 + E)
    const int col2 = 32 * (aw + 1);
    const bool colsplit = MOONEP_PLAN_COLSPLIT && d.xtab && col2 + E <= kPlanThreads;
    const bool foldrank = MOONEP_PLAN_FOLDRANK && d.xtab;
    // the router-count check of block 0 runs on the threads past the split
    // column pass when there is at least a warp of them
    const bool spare_check = colsplit && kPlanThreads - (col2 + E) >= 32;
    if (!one_rank && w == aw) {
        for (int h = lane; h < R; h += 32) s_L[h] = ld_cg(a.ws.gload + (size_t)parity * R + h);
        __syncwarp();
        AliasOut o{s_keep, s_rfrom, s_rstart, s_rlen, s_doff, s_dlist};
        if (R <= 32)
            alias_chain<1>(R, d.S * K, s_L, o);
        else
            alias_chain<2>(R, d.S * K, s_L, o);
    }
    // Column sums of the histogram: T_e, this block's prefix (rows before its
    // own), per-rank counts (checked against the router's, written by the
    // rank's first block).
    // Per expert: T_e from the per-rank counts, this block's prefix from the
    // counts of earlier ranks plus its own rank's earlier chunks, and the
    // router's counts checked against ours (all ranks, so every block takes
    // the same decision).  One round of loads per thread.
    // (Loads are batched into registers ahead of any global store, so the
    // compiler keeps them all in flight.)
    bool mismatch = false;
    {
        const int32_t *cnt = one_rank ? a.counts_all : a.ws.cnt + (size_t)parity * R * E;
        const int32_t *own = a.ws.cnt + ((size_t)parity * R + r) * E;  // this call's picks of rank r
        const int32_t *mine_rows = a.ws.hist + (int64_t)r * d.nch * E;
        // rows q < R are the per-rank counts, rows R <= q < R + c this rank's
        // earlier chunk histograms; 16 loads in flight per batch
        if (colsplit) {
            // warps 0.. sum the per-rank counts, the warps after the alias
            // warp this rank's earlier chunk rows: one batch of loads each
            // for up to 16 rows, where one thread per expert took two
            if (tid < E) {
                const int e = tid;
                int tot = 0, mypre = 0, myv = 0;
                for (int q0 = 0; q0 < R; q0 += 16) {
                    int v[16];
#pragma unroll
                    for (int u = 0; u < 16; ++u) v[u] = q0 + u < R ? ld_cg(cnt + (int64_t)(q0 + u) * E + e) : 0;
#pragma unroll
                    for (int u = 0; u < 16; ++u) {
                        const int q = q0 + u;
                        if (q >= R) continue;
                        tot += v[u];
                        if (q < r) mypre += v[u];
                        if (q == r) myv = v[u];
                    }
                }
                T[e] = tot;
                pre[e] = mypre;
                if (c == 0 && !one_rank) a.plan.counts[(int64_t)r * E + e] = myv;
                if (checker && one_rank && ld_cg(own + e) != myv) mismatch = true;  // the rank's own row
                if (checker && !one_rank && !spare_check) mismatch |= check_router_counts(a, cnt, tpe_s, e, E);
            } else if (checker && !one_rank && spare_check && tid >= col2 + E) {
                mismatch = check_router_counts(a, cnt, tpe_s, tid - (col2 + E), kPlanThreads - (col2 + E));
            } else if (tid >= col2 && tid < col2 + E) {
                const int e = tid - col2;
                int sum = 0;
                for (int q0 = 0; q0 < c; q0 += 16) {
                    int v[16];
#pragma unroll
                    for (int u = 0; u < 16; ++u) v[u] = q0 + u < c ? ld_cg(mine_rows + (int64_t)(q0 + u) * E + e) : 0;
#pragma unroll
                    for (int u = 0; u < 16; ++u) sum += v[u];
                }
                pre2[e] = sum;
            }
        } else {
            mismatch = column_pass_one_loop(a, cnt, own, mine_rows, tpe_s, T, pre, r, c, checker, one_rank);
        }
    }
    // the router's counts are checked by block 0 only, which writes the
    // plan's status at its end; the layout goes ahead either way
    __shared__ int s_mismatch;
    if (tid == 0) s_mismatch = 0;
    const int mm = __reduce_or_sync(0xffffffffu, mismatch ? 1 : 0);
    __shared__ int s_cbad;
    if (tid == 0) s_cbad = 0;
    __syncthreads();
    if (lane == 0 && mm) atomicOr(&s_mismatch, MOONEP_STATUS_COUNT_MISMATCH);
    // One rank: the gathered counts must hold S*K non-negative picks per rank,
    // or the layout below is undefined.  Every block checks every row, so all
    // take the same decision; block 0 copies the rows into the plan.
    if (one_rank) check_gathered_counts(a, &s_cbad);
    // group loads and the largest count
    int mx = 0;
    for (int e = tid; e < E; e += kPlanThreads) mx = max(mx, T[e]);
    mx = warp_max(mx);
    if (lane == 0) s_wmax[w] = mx;
    for (int h = w; one_rank && h < R; h += kPlanWarps) {
        int sum = 0;
        for (int j = lane; j < G; j += 32) sum += T[h * G + j];
        sum = warp_sum(sum);
        if (lane == 0) s_L[h] = sum;
    }
    __syncthreads();
    PLAN_TRACE(2);
    if (s_status != 0 || s_cbad != 0) {
        if (blockIdx.x == 0 && tid == 0) atomicOr(a.plan.status, s_status | s_mismatch | s_cbad);
        return;
    }

    // The alias chain in closed form (warp 0; ranks h = lane and lane + 32).
    // Under-loaded ranks ("small", deficit C - L) in ascending order lay their
    // deficits end to end on a demand line (prefixes P); over-loaded ranks
    // ("large", excess L - C) lay their excesses on the same line (prefixes
    // Q).  A small rank takes its whole deficit from the large rank whose
    // excess interval holds the start of its demand.  A large rank whose
    // excess ends strictly inside some small rank's demand interval is
    // drained below C by it and takes the rest from the next large rank.  A
    // donor's gifts leave in demand-line order, so a gift starts at the
    // donor's kept count plus its distance from the donor's excess start.
    // This equals the queue-driven chain step for step.
    if (one_rank && w == 0) {
        AliasOut o{s_keep, s_rfrom, s_rstart, s_rlen, s_doff, s_dlist};
        if (R <= 32)
            alias_chain<1>(R, d.S * K, s_L, o);
        else
            alias_chain<2>(R, d.S * K, s_L, o);
    }
    if (w == 1 && blockIdx.x == 0) {
        int mxw = lane < kPlanWarps ? s_wmax[lane] : 0;
        mxw = warp_max(mxw);
        if (lane == 0) {
            const double tbar = (double)((int64_t)R * d.S * K) / (double)E;
            *a.plan.maxvio = (float)((double)mxw / tbar - 1.0);
        }
    }
    PLAN_TRACE(10);
    // expert starts inside their group sequences (warps 1.., while warp 0
    // runs the alias chain).  Mode 3 (fewest copies) orders a group by pick
    // count, ties by id: an expert starts after every expert of its group
    // that sorts before it, one pass over the group per expert.
    if (d.mode == 3) {
        expert_starts_by_count(T, es, E, R, G);
    } else if (w >= 1) {
        for (int h = w - 1; h < R; h += kPlanWarps - 1) {
            int carry = 0;
            for (int j0 = 0; j0 < G; j0 += 32) {
                const int j = j0 + lane;
                const int t = j < G ? T[h * G + j] : 0;
                const int incl = warp_incl_scan(t) + carry;
                if (j < G) es[h * G + j] = incl - t;
                carry = __shfl_sync(0xffffffffu, incl, 31);
            }
        }
    }
    __syncthreads();
    PLAN_TRACE(11);
    // compact row table of every rank (one warp per rank)
    for (int s = w; s < R; s += kPlanWarps) {
        const int keep_s = s_keep[s];
        int carry = 0;
        for (int j0 = 0; j0 < G; j0 += 32) {
            const int j = j0 + lane;
            const int e = s * G + j;
            int n = 0;
            if (j < G) n = max(0, min(es[e] + T[e], keep_s) - es[e]);
            const int incl = warp_incl_scan(pad_to(n, tp)) + carry;
            if (j < G) {
                nhome[e] = n;
                kbase[e] = incl;  // home-row running sum for now
            }
            carry = __shfl_sync(0xffffffffu, incl, 31);
        }
        int nq = 0, nslot = 0, ocarry = 0, scarry = 0;
        const int h = s_rfrom[s];
        if (h >= 0) {
            const int a0 = s_rstart[s], a1 = a0 + s_rlen[s];
            // Which received experts take the B slots: the first B in id
            // order, or (mode 2) the B with the most picks here, ties to the
            // lower id; the slots themselves go in id order either way.
            const bool by_count = d.mode == 2;
            if (by_count) {
                for (int j = lane; j < G; j += 32) {
                    const int e = h * G + j;
                    nrecv[s * G + j] = max(0, min(es[e] + T[e], a1) - max(es[e], a0));
                }
                __syncwarp();
            }
            for (int j0 = 0; j0 < G; j0 += 32) {
                const int j = j0 + lane;
                const int e = h * G + j;
                int ov = 0;
                if (j < G) ov = max(0, min(es[e] + T[e], a1) - max(es[e], a0));
                const unsigned has = __ballot_sync(0xffffffffu, ov > 0);
                bool take = ov > 0 && nq + __popc(has & lanemask_lt()) < B;
                if (by_count && ov > 0) take = take_by_count(nrecv + s * G, G, j, ov, B);
                const unsigned tk = __ballot_sync(0xffffffffu, take);
                // slot index of a taken expert; B marks an overflow row
                const int q = take ? nslot + __popc(tk & lanemask_lt()) : B;
                const bool is_ovf = ov > 0 && !take;
                const int oincl = warp_incl_scan(is_ovf ? pad_to(ov, tp) : 0) + ocarry;
                const int sincl = warp_incl_scan(take ? pad_to(ov, tp) : 0) + scarry;
                if (j < G) {
                    nrecv[s * G + j] = ov;
                    qidx[s * G + j] = (int16_t)(ov > 0 ? q : -1);
                    ovfincl[s * G + j] = oincl;
                }
                if (take) {
                    slotj[s * B + q] = (int16_t)j;
                    slotincl[s * B + q] = sincl;
                }
                nq += __popc(has);
                nslot += __popc(tk);
                ocarry = __shfl_sync(0xffffffffu, oincl, 31);
                scarry = __shfl_sync(0xffffffffu, sincl, 31);
            }
        }
        for (int b = nslot + lane; b < B; b += 32) {
            slotj[s * B + b] = (int16_t)-1;
            slotincl[s * B + b] = scarry;
        }
        if (lane == 0) {
            s_hsize[s] = carry;
            s_osize[s] = ocarry;
            s_nslot[s] = nslot;
        }
        __syncwarp();
        // first slot of every row: rows come in index order, so the donor
        // group's overflow rows sit before or after the home rows, and the
        // slot rows E.. come last
        const int off_home = (h >= 0 && h < s) ? ocarry : 0;
        const int off_ovf = (h > s) ? carry : 0;
        const int off_slot = carry + ocarry;
        // this rank's place in its donor's list of recipients, and the
        // recipient just before it (whose range ends where this one starts)
        int prev = -1;
        if (h >= 0 && d.fast2)
            for (int k = s_doff[h]; k < s_doff[h + 1]; ++k)
                if (s_dlist[k] == s) prev = k > s_doff[h] ? s_dlist[k - 1] : -1;
        for (int j = lane; j < G; j += 32) {
            const int e = s * G + j;
            kbase[e] = s * d.nvs + off_home + kbase[e] - pad_to(nhome[e], tp) - es[e];
            if (foldrank) {
                // this block's offset of e (its start in the group sequence
                // plus the picks of earlier ranks and chunks): a kept pick of
                // chunk rank rk goes to dbase[e] + rk while rk < dlim[e]
                const int off = es[e] + pre[e] + (colsplit ? pre2[e] : 0);
                dbase[e] = kbase[e] + off;
                dlim[e] = keep_s - off;
            }
            if (h >= 0) {
                const int q = qidx[s * G + j];
                const int p = pad_to(nrecv[s * G + j], tp);
                const int st = q < 0 ? -1
                               : q < B ? off_slot + slotincl[s * B + q] - p
                                       : off_ovf + ovfincl[s * G + j] - p;
                recvstart[s * G + j] = st;
                // fast-path bases of expert eh's donated part, set by the
                // recipient whose range holds its start (first) and by the
                // recipient right after that one (second).  They are taken
                // relative to this block's chunk: a pick of chunk rank rk
                // sits at g = off + rk in the group sequence.
                const int eh = h * G + j;
                const int off = es[eh] + pre[eh] + (colsplit ? pre2[eh] : 0);
                const int lo = max(es[eh], s_keep[h]);
                const int a0 = s_rstart[s], a1 = a0 + s_rlen[s];
                if (q >= 0 && a0 <= lo && lo < a1) {
                    ebase[eh] = s * d.nvs + st - max(es[eh], a0) + off;
                    eend[eh] = a1 - off;
                } else if (d.fast2 && q >= 0 && prev >= 0 && s_rstart[prev] <= lo &&
                           lo < s_rstart[prev] + s_rlen[prev]) {
                    ebase2[eh] = s * d.nvs + st - a0 + off;
                    eend2[eh] = a1 - off;
                }
            }
        }
    }
    __syncthreads();
    PLAN_TRACE(3);

    // padded running total of rank s up to and including row i
    auto upto = [&](int s, int i) -> int {
        int v = 0;
        const int hs = s * G;
        const int h = s_rfrom[s];
        if (i >= hs) {
            if (i < hs + G) {  // the home-row running sum, recovered from kbase
                const int off_home = (h >= 0 && h < s) ? s_osize[s] : 0;
                v += kbase[i] - s * d.nvs - off_home + pad_to(nhome[i], tp) + es[i];
            } else {
                v += s_hsize[s];
            }
        }
        if (h >= 0) {
            const int hd = h * G;
            if (i >= hd) v += i < hd + G ? ovfincl[s * G + (i - hd)] : s_osize[s];
        }
        if (i >= E) v += slotincl[s * B + (i - E)];
        return v;
    };
    auto count_of = [&](int s, int i) -> int {
        if (i < E) {
            if (i / G == s) return nhome[i];
            const int h = s_rfrom[s];
            if (h >= 0 && i / G == h) {
                const int j = i - h * G;
                return qidx[s * G + j] >= B ? nrecv[s * G + j] : 0;
            }
            return 0;
        }
        const int b = i - E;
        return b < s_nslot[s] ? nrecv[s * G + slotj[s * B + b]] : 0;
    };

    // ---------------- C. outputs and dst ----------------
    // The first `ow` warps write this block's share of the per-rank outputs
    // (nothing below reads them) while the other warps fold the chunk
    // offsets into the bases and write dst, after a barrier of their own.
    const int total = R * NR;  // R*(E+B) and R*B are far below 2^31 under the config limits
    const int per = (total + (int)gridDim.x - 1) / (int)gridDim.x;
    const int ow = per <= 128 ? 1 : 4;
    if (w < ow) {
        const int ot = 32 * ow;
        if (blockIdx.x == 0) {
            for (int j = tid; j < R; j += ot) {
                a.plan.assign[4 * j + 0] = s_keep[j];
                a.plan.assign[4 * j + 1] = s_rfrom[j];
                a.plan.assign[4 * j + 2] = s_rstart[j];
                a.plan.assign[4 * j + 3] = s_rlen[j];
            }
        }
        const int i0 = (int)blockIdx.x * per, i1 = min(total, i0 + per);
        for (int idx = i0 + tid; idx < i1; idx += ot) {
            const int s = idx / NR, i = idx - s * NR;
            a.plan.cu_seqlens[idx] = upto(s, i);
            a.plan.row_counts[idx] = count_of(s, i);
        }
        const int tb = R * B;
        const int perb = (tb + (int)gridDim.x - 1) / (int)gridDim.x;
        const int b0 = (int)blockIdx.x * perb, b1 = min(tb, b0 + perb);
        for (int idx = b0 + tid; idx < b1; idx += ot) {
            const int s = idx / B, b = idx - s * B;
            a.plan.slot_expert[idx] = b < s_nslot[s] ? s_rfrom[s] * G + slotj[idx] : -1;
        }
        PLAN_TRACE(13);
    } else {
        const int t2 = tid - 32 * ow, n2 = kPlanThreads - 32 * ow;
        int32_t *kb = dbase, *kl = dlim;
        if (!foldrank) {
            fold_chunk_offsets(T, pre, es, colsplit ? pre2 : nullptr, kbase, s_keep, E, G, t2, n2);
            asm volatile("bar.sync 1, %0;" ::"r"(n2) : "memory");
            kb = T;
            kl = pre;
        }
        PLAN_TRACE_BY(12, 32 * ow);
        // destination of every pick of this block's chunk
        for (int i = t2; i < n_ent; i += n2) {
            const int e = ent_e[i];
            const int rk = ent_rank[i];
            int dst;
            if (rk < kl[e]) {
                dst = kb[e] + rk;
            } else if (rk < eend[e]) {
                dst = ebase[e] + rk;
            } else if (d.fast2 && rk < eend2[e]) {
                dst = ebase2[e] + rk;
            } else {  // the expert's donated run spans three or more recipients
                // (in line: a call inside this loop slows every pass of it
                // by more than the code it would move out)
                const int h = e / G;
                const int g = rk + s_keep[h] - kl[e];
                int dest = -1;
                for (int k = s_doff[h]; k < s_doff[h + 1]; ++k) {
                    const int s = s_dlist[k];
                    if (g >= s_rstart[s] && g < s_rstart[s] + s_rlen[s]) {
                        dest = s;
                        break;
                    }
                }
                const int st = dest < 0 ? -1 : recvstart[dest * G + (e - h * G)];
                if (st < 0) {  // unreachable for a consistent layout; never write with it
                    atomicOr(a.plan.status, MOONEP_STATUS_BAD_PLAN);
                    continue;
                }
                dst = dest * d.nvs + st + (g - max(es[e], s_rstart[dest]));
            }
            a.plan.dst[base + i] = dst;
        }
        PLAN_TRACE_BY(4, 32 * ow);
    }
    if (blockIdx.x == 0) {
        __syncthreads();
        if (tid == 0 && s_mismatch) atomicOr(a.plan.status, s_mismatch);
    }
}

cudaError_t launch_plan(const PlanArgs &a, int grid, cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kPlanThreads);
    cfg.dynamicSmemBytes = plan_smem_bytes(a.d);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, plan_kernel, a);
}

int plan_blocks_per_sm(const Dims &d) {
    int n = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, plan_kernel, kPlanThreads, plan_smem_bytes(d));
    return n;
}

size_t plan_static_smem_bytes() {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, plan_kernel) != cudaSuccess) return 0;
    return fa.sharedSizeBytes;
}

cudaError_t plan_set_smem_limit(size_t bytes) {
    return cudaFuncSetAttribute(plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

}  // namespace moonep
