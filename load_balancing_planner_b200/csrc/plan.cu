// The online planner (MoonEP README, "Performance" item 2 and "dispatch fwd";
// MarkTechPost, "Core idea: dynamic redundant experts").  The pages fix what
// the plan must satisfy -- exactly S*K slots per rank, copies from at most one
// remote home group per rank in training, overflow experts read from their
// home rows in inference, padded cu_seqlens[E+B] -- but print no rule.  The
// rule implemented here is this library's reading: the group sequence of home
// rank h lists its picks by (expert, source rank, token); an alias chain over
// the group loads decides who gives how much to whom; a donor keeps the prefix
// of its sequence and gives consecutive ranges after it; a recipient's copied
// experts take its slots in ascending id, overflow rows past B (inference).
//
// One cooperative launch, one block per (source rank, chunk of `ct` tokens),
// all blocks resident:
//   A. count: the chunk's picks go to shared memory; each warp ranks its runs
//      of 32 picks per expert with match_any/popc (token order), which also
//      finds an expert picked twice by one token; per-warp counts are scanned
//      into the chunk's histogram row (global) and every pick's stable rank
//      inside the chunk.
//   -- grid barrier: one 64-bit arrive counter that only grows; bounded spin.
//   B. layout, computed by every block from the histogram (no second
//      barrier): T_e, loads, maxvio, the alias chain (one warp, in closed form
//      over prefix sums of deficits and excesses), expert starts, and per rank
//      a compact row table with inclusive running sums.
//   C. every block writes a slice of cu_seqlens / row_counts / slot_expert,
//      then dst for its own picks from per-expert bases (one shared-memory
//      read per pick in the common case).
#include "moonep_internal.cuh"

namespace moonep {

__host__ __device__ static inline size_t align256(size_t b) { return (b + 255) / 256 * 256; }

size_t workspace_bytes(const Dims &d) {
    return align256(sizeof(int32_t) * (size_t)d.R * d.nch * d.E) +
           align256(sizeof(int32_t) * 2 * (size_t)d.R * d.E) + align256(4 * sizeof(uint64_t));
}

void carve_workspace(const Dims &d, void *base, Workspace *ws) {
    char *p = static_cast<char *>(base);
    ws->hist = reinterpret_cast<int32_t *>(p);
    p += align256(sizeof(int32_t) * (size_t)d.R * d.nch * d.E);
    ws->cnt = reinterpret_cast<int32_t *>(p);
    p += align256(sizeof(int32_t) * 2 * (size_t)d.R * d.E);
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
    const size_t layout = sizeof(int32_t) * (9 * (size_t)d.E + 2 * (size_t)d.R * d.B) +
                          sizeof(int16_t) * (2 * (size_t)d.E + 2);
    return align256(counts > layout ? counts : layout);
}

// Block 0 keeps a copy of the router's local counts (loaded at kernel start,
// checked after the barrier) when they are small enough.
__host__ __device__ static inline bool tpe_in_smem(const Dims &d) { return (size_t)d.R * d.E <= 16384; }

__host__ __device__ static inline size_t ent_bytes(const Dims &d) {
    return align256(sizeof(uint16_t) * (size_t)d.ct * d.K) + align256(sizeof(int32_t) * (size_t)d.ct * d.K);
}

size_t plan_smem_bytes(const Dims &d) {
    return region1_bytes(d) + ent_bytes(d) + (tpe_in_smem(d) ? sizeof(int32_t) * (size_t)d.R * d.E : 0);
}

// Phase timestamps for profiling builds (-DMOONEP_PLAN_TRACE); no code otherwise.
#ifdef MOONEP_PLAN_TRACE
__device__ unsigned long long g_plan_trace[1024][16];
#define PLAN_TRACE(k)                                                                      \
    do {                                                                                   \
        if (threadIdx.x == 0 && blockIdx.x < 1024) {                                       \
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

// Grid barrier over all blocks of a cooperative launch.  The counter only
// grows: at kernel start it holds k * gridDim.x (k calls done), every block
// adds one, and all wait until it reaches (k + 1) * gridDim.x, with a bounded
// number of polls.  Returns false on timeout.
__device__ bool grid_barrier(unsigned long long *ctr, unsigned long long target) {
    __shared__ int s_ok;
    __syncthreads();
    if (threadIdx.x == 0) {
        int ok = 0;
        __threadfence();
        const unsigned long long old = atomicAdd(ctr, 1ull);
        if (old + 1 >= target) {
            ok = 1;
        } else {
            const volatile unsigned long long *v = ctr;
            for (uint32_t it = 0; it < kBarrierPolls; ++it) {
                if (*v >= target) {
                    ok = 1;
                    break;
                }
                if (it > 64) __nanosleep(32);
            }
        }
        __threadfence();
        s_ok = ok;
    }
    __syncthreads();
    return s_ok != 0;
}

// ---- the planner kernel ----------------------------------------------------
// 1024 threads per block: the register budget is 64 per thread.
__global__ void __launch_bounds__(kPlanThreads, 1) plan_kernel(PlanArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    const Dims &d = a.d;
    const int E = d.E, K = d.K, R = d.R, G = d.G, B = d.B, NR = d.NR, tp = d.tp;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;

    uint8_t *region1 = smem;
    uint16_t *ent_e = reinterpret_cast<uint16_t *>(smem + region1_bytes(d));
    int32_t *ent_rank = reinterpret_cast<int32_t *>(reinterpret_cast<uint8_t *>(ent_e) +
                                                    align256(sizeof(uint16_t) * (size_t)d.ct * K));
    int32_t *tpe_s = reinterpret_cast<int32_t *>(smem + region1_bytes(d) + ent_bytes(d));  // [R][E], block 0
    const bool checker = blockIdx.x == 0 && a.tpe != nullptr;
    // the plan's status starts at 0 (block 0, before the grid barrier); every
    // later update is an atomicOr, so no error bit can be overwritten
    if (blockIdx.x == 0 && tid == 0) *a.plan.status = 0;
    if (checker && tpe_in_smem(d))
        for (int i = tid; i < R * E; i += kPlanThreads) tpe_s[i] = __ldg(a.tpe + i);

    __shared__ unsigned long long s_call;
    __shared__ int s_bad;
    if (tid == 0) {
        s_call = *reinterpret_cast<volatile unsigned long long *>(a.ws.arrive) / gridDim.x;
        s_bad = 0;
    }

    PLAN_TRACE(0);
    const int row = blockIdx.x;  // histogram row = r * nch + c
    const int r = row / d.nch, c = row - r * d.nch;
    const int t0 = c * d.ct;
    const int t1 = min(d.S, t0 + d.ct);
    const int n_ent = (t1 - t0) * K;
    const int64_t base = ((int64_t)r * d.S + t0) * K;

    // ---------------- A. count ----------------
    const int CW = d.cw;
    uint16_t *wcnt = reinterpret_cast<uint16_t *>(region1);                       // [CW][E]
    uint32_t *wmask = reinterpret_cast<uint32_t *>(region1 + counts_bytes(d));    // [CW][E]
    int bad = 0;
    for (int i = tid; i < CW * E; i += kPlanThreads) {
        wcnt[i] = 0;
        wmask[i] = 0u;
    }
    for (int i = tid; i < n_ent; i += kPlanThreads) {
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
            if (i < w1) ent_rank[i] = prior + before;
        }
    }
    if (!whole_tokens) {  // tokens straddle runs: check duplicates token by token
        for (int tt = tid; tt < t1 - t0; tt += kPlanThreads) {
            const uint16_t *tok = ent_e + tt * K;
            for (int k = 1; k < K; ++k) {
                const uint16_t ek = tok[k];
                if (ek == 0xFFFF) continue;
                for (int k2 = 0; k2 < k; ++k2)
                    if (tok[k2] == ek) bad |= MOONEP_STATUS_DUP_EXPERT;
            }
        }
    }
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
        if (run) atomicAdd(crow + e, run);
    }
    __syncthreads();
    PLAN_TRACE(8);
    for (int i = tid; i < n_ent; i += kPlanThreads) {
        const int e = ent_e[i];
        if (e != 0xFFFF) ent_rank[i] += wcnt[(i >> lg_run) * E + e];
    }
    bad = __reduce_or_sync(0xffffffffu, bad);
    if (lane == 0 && bad) atomicOr(&s_bad, bad);
    __syncthreads();
    if (tid == 0 && s_bad) atomicOr(a.ws.status + parity, s_bad);

    PLAN_TRACE(5);
    if (!grid_barrier(a.ws.arrive, (call + 1) * gridDim.x)) {
        if (tid == 0) atomicOr(a.plan.status, MOONEP_STATUS_TIMEOUT);
        return;
    }
    PLAN_TRACE(1);
    // the next call's error slot: every block of this call is past its last
    // write to the other slot's counterpart, and the next call starts after
    // this kernel ends
    if (blockIdx.x == 0 && tid == 0) a.ws.status[parity ^ 1] = 0;
    {
        int32_t *next = a.ws.cnt + (size_t)(parity ^ 1) * R * E;
        const int64_t tot = (int64_t)R * E, per = (tot + gridDim.x - 1) / gridDim.x;
        for (int64_t i = (int64_t)blockIdx.x * per + tid; i < min(tot, (int64_t)(blockIdx.x + 1) * per);
             i += kPlanThreads)
            next[i] = 0;
    }

    // ---------------- B. layout (every block) ----------------
    int32_t *T = reinterpret_cast<int32_t *>(region1);  // [E] picks per expert
    int32_t *pre = T + E;               // [E] picks of each expert in histogram rows before this block's
    int32_t *es = pre + E;              // [E] start of each expert inside its group sequence
    int32_t *nhome = es + E;            // [E] kept picks of expert e on its home rank
    int32_t *homeincl = nhome + E;      // [E] inclusive padded running sum over the home rows of e's rank
    int32_t *homestart = homeincl + E;  // [E] first slot of home row e; later: dst base of kept picks
    int32_t *nrecv = homestart + E;     // [R*G] picks of the j-th donor-group expert received by rank s; later: dst base
    int32_t *ovfincl = nrecv + E;       // [R*G] inclusive padded running sum over overflow rows; later: end of range
    int32_t *recvstart = ovfincl + E;   // [R*G] first slot of the row holding that received expert
    int32_t *slotincl = recvstart + E;  // [R*B] inclusive padded running sum over the slot rows
    int32_t *slotj = slotincl + R * B;  // [R*B] donor-group index of the expert in slot b
    int16_t *qidx = reinterpret_cast<int16_t *>(slotj + R * B);  // [R*G] received-expert index, -1 none
    int16_t *edon = qidx + E;           // [E] first recipient (in the donor's list) overlapping e's run
    __shared__ int s_L[MOONEP_MAX_R], s_keep[MOONEP_MAX_R];
    __shared__ int s_rfrom[MOONEP_MAX_R], s_rstart[MOONEP_MAX_R], s_rlen[MOONEP_MAX_R];
    __shared__ int s_dlist[MOONEP_MAX_R], s_doff[MOONEP_MAX_R + 1];
    __shared__ int s_hsize[MOONEP_MAX_R], s_osize[MOONEP_MAX_R], s_nslot[MOONEP_MAX_R];
    __shared__ int s_status, s_wmax[kPlanWarps];

    if (tid == kPlanThreads - 1) s_status = ld_cg(a.ws.status + parity);
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
        const int32_t *cnt = a.ws.cnt + (size_t)parity * R * E;
        const int32_t *mine_rows = a.ws.hist + (int64_t)r * d.nch * E;
        for (int e = tid; e < E; e += kPlanThreads) {
            int tot = 0, mypre = 0, myv = 0;
            for (int r0 = 0; r0 < R; r0 += 8) {
                int v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int rr = r0 + u;
                    v[u] = rr < R ? ld_cg(cnt + (int64_t)rr * E + e) : 0;
                }
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int rr = r0 + u;
                    if (rr < R) {
                        tot += v[u];
                        if (rr < r) mypre += v[u];
                        if (rr == r) myv = v[u];
                        if (checker) {
                            const int t = tpe_in_smem(d) ? tpe_s[rr * E + e] : __ldg(a.tpe + (int64_t)rr * E + e);
                            if (t != v[u]) mismatch = true;
                        }
                    }
                }
            }
            for (int c0 = 0; c0 < c; c0 += 8) {
                int v[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) v[u] = c0 + u < c ? ld_cg(mine_rows + (int64_t)(c0 + u) * E + e) : 0;
#pragma unroll
                for (int u = 0; u < 8; ++u) mypre += v[u];
            }
            T[e] = tot;
            pre[e] = mypre;
            if (c == 0) a.plan.counts[(int64_t)r * E + e] = myv;
        }
    }
    // the router's counts are checked by block 0 only, which writes the
    // plan's status at its end; the layout goes ahead either way
    __shared__ int s_mismatch;
    if (tid == 0) s_mismatch = 0;
    const int mm = __reduce_or_sync(0xffffffffu, mismatch ? 1 : 0);
    __syncthreads();
    if (lane == 0 && mm) atomicOr(&s_mismatch, MOONEP_STATUS_COUNT_MISMATCH);
    // group loads and the largest count
    int mx = 0;
    for (int e = tid; e < E; e += kPlanThreads) mx = max(mx, T[e]);
    mx = warp_max(mx);
    if (lane == 0) s_wmax[w] = mx;
    for (int h = w; h < R; h += kPlanWarps) {
        int sum = 0;
        for (int j = lane; j < G; j += 32) sum += T[h * G + j];
        sum = warp_sum(sum);
        if (lane == 0) s_L[h] = sum;
    }
    __syncthreads();
    PLAN_TRACE(2);
    if (s_status != 0) {
        if (blockIdx.x == 0 && tid == 0) atomicOr(a.plan.status, s_status | s_mismatch);
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
    if (w == 0) {
        const int C = d.S * K;
        int Lv[2], D[2], X[2], Pin[2], Qin[2], Pex[2], Qex[2];
        int carryP = 0, carryQ = 0;
#pragma unroll
        for (int sl = 0; sl < 2; ++sl) {
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
        unsigned smallb[2], largeb[2];
#pragma unroll
        for (int sl = 0; sl < 2; ++sl) {
            smallb[sl] = __ballot_sync(0xffffffffu, D[sl] > 0);
            largeb[sl] = __ballot_sync(0xffffffffu, X[sl] > 0);
        }
        int donor[2] = {-1, -1}, off[2] = {0, 0}, amt[2] = {0, 0};
        // small ranks: the large rank whose excess interval holds Pex
#pragma unroll
        for (int sl2 = 0; sl2 < 2; ++sl2)
            for (unsigned m = largeb[sl2]; m; m &= m - 1) {
                const int l = __ffs(m) - 1;
                const int qe = __shfl_sync(0xffffffffu, Qex[sl2], l);
                const int qi = __shfl_sync(0xffffffffu, Qin[sl2], l);
#pragma unroll
                for (int sl = 0; sl < 2; ++sl)
                    if (D[sl] > 0 && qe <= Pex[sl] && Pex[sl] < qi) {
                        donor[sl] = l + 32 * sl2;
                        off[sl] = Pex[sl] - qe;
                        amt[sl] = D[sl];
                    }
            }
        // drained large ranks: a small demand interval strictly holds Qin
#pragma unroll
        for (int sl2 = 0; sl2 < 2; ++sl2)
            for (unsigned m = smallb[sl2]; m; m &= m - 1) {
                const int s = __ffs(m) - 1;
                const int pe = __shfl_sync(0xffffffffu, Pex[sl2], s);
                const int pi = __shfl_sync(0xffffffffu, Pin[sl2], s);
#pragma unroll
                for (int sl = 0; sl < 2; ++sl)
                    if (X[sl] > 0 && pe < Qin[sl] && Qin[sl] < pi) {
                        // the next large rank after this one
                        const unsigned above = sl == 0 ? (largeb[0] & ~((2u << lane) - 1u)) : 0u;
                        const unsigned above1 = sl == 1 ? (largeb[1] & ~((2u << lane) - 1u)) : largeb[1];
                        donor[sl] = above ? __ffs(above) - 1 : 32 + __ffs(above1) - 1;
                        off[sl] = 0;
                        amt[sl] = pi - Qin[sl];
                    }
            }
        int keep[2], start[2];
#pragma unroll
        for (int sl = 0; sl < 2; ++sl) keep[sl] = D[sl] > 0 ? Lv[sl] : C - (X[sl] > 0 ? amt[sl] : 0);
#pragma unroll
        for (int sl = 0; sl < 2; ++sl) {
            const int dl = donor[sl] < 0 ? 0 : donor[sl];
            const int k0 = __shfl_sync(0xffffffffu, keep[0], dl & 31);
            const int k1 = __shfl_sync(0xffffffffu, keep[1], dl & 31);
            start[sl] = donor[sl] < 0 ? 0 : (dl < 32 ? k0 : k1) + off[sl];
        }
        // recipients of each donor in increasing start order
        int pos[2] = {0, 0}, cnt[2] = {0, 0};
#pragma unroll
        for (int sl2 = 0; sl2 < 2; ++sl2) {
            const unsigned rb = __ballot_sync(0xffffffffu, donor[sl2] >= 0);
            for (unsigned m = rb; m; m &= m - 1) {
                const int s = __ffs(m) - 1;
                const int dn = __shfl_sync(0xffffffffu, donor[sl2], s);
                const int st = __shfl_sync(0xffffffffu, start[sl2], s);
#pragma unroll
                for (int sl = 0; sl < 2; ++sl) {
                    if (donor[sl] == dn && st < start[sl]) ++pos[sl];
                    if (dn == lane + 32 * sl) ++cnt[sl];
                }
            }
        }
        int doff[2], carry = 0;
#pragma unroll
        for (int sl = 0; sl < 2; ++sl) {
            const int incl = warp_incl_scan(cnt[sl]) + carry;
            carry = __shfl_sync(0xffffffffu, incl, 31);
            doff[sl] = incl - cnt[sl];
        }
#pragma unroll
        for (int sl = 0; sl < 2; ++sl) {
            const int h = lane + 32 * sl;
            if (h < R) {
                s_keep[h] = keep[sl];
                s_rfrom[h] = donor[sl];
                s_rstart[h] = start[sl];
                s_rlen[h] = amt[sl];
                s_doff[h] = doff[sl];
            }
            if (h == R) s_doff[R] = doff[sl];
        }
        if (R == 64 && lane == 0) s_doff[R] = carry;
        __syncwarp();
#pragma unroll
        for (int sl = 0; sl < 2; ++sl) {
            const int h = lane + 32 * sl;
            if (h < R && donor[sl] >= 0) s_dlist[s_doff[donor[sl]] + pos[sl]] = h;
        }
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
    // expert starts inside their group sequences (warps 1.., one home group
    // each, while warp 0 runs the alias chain)
    if (w >= 1) {
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
    // first recipient, in the donor's list, whose range overlaps expert e's run
    for (int e = tid; e < E; e += kPlanThreads) {
        const int h = e / G;
        const int lo = max(es[e], s_keep[h]), hi = es[e] + T[e];
        int first = -1;
        if (lo < hi)
            for (int k = s_doff[h]; k < s_doff[h + 1]; ++k) {
                const int s = s_dlist[k];
                if (s_rstart[s] + s_rlen[s] > lo) {
                    first = k;
                    break;
                }
            }
        edon[e] = (int16_t)first;
    }
    PLAN_TRACE(12);

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
                homeincl[e] = incl;
            }
            carry = __shfl_sync(0xffffffffu, incl, 31);
        }
        int nq = 0, ocarry = 0, scarry = 0;
        const int h = s_rfrom[s];
        if (h >= 0) {
            const int a0 = s_rstart[s], a1 = a0 + s_rlen[s];
            for (int j0 = 0; j0 < G; j0 += 32) {
                const int j = j0 + lane;
                const int e = h * G + j;
                int ov = 0;
                if (j < G) ov = max(0, min(es[e] + T[e], a1) - max(es[e], a0));
                const unsigned has = __ballot_sync(0xffffffffu, ov > 0);
                const int q = nq + __popc(has & lanemask_lt());
                const bool is_slot = ov > 0 && q < B, is_ovf = ov > 0 && q >= B;
                const int oincl = warp_incl_scan(is_ovf ? pad_to(ov, tp) : 0) + ocarry;
                const int sincl = warp_incl_scan(is_slot ? pad_to(ov, tp) : 0) + scarry;
                if (j < G) {
                    nrecv[s * G + j] = ov;
                    qidx[s * G + j] = (int16_t)(ov > 0 ? q : -1);
                    ovfincl[s * G + j] = oincl;
                }
                if (is_slot) {
                    slotj[s * B + q] = j;
                    slotincl[s * B + q] = sincl;
                }
                nq += __popc(has);
                ocarry = __shfl_sync(0xffffffffu, oincl, 31);
                scarry = __shfl_sync(0xffffffffu, sincl, 31);
            }
        }
        const int nslot = min(nq, B);
        for (int b = nslot + lane; b < B; b += 32) {
            slotj[s * B + b] = -1;
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
        for (int j = lane; j < G; j += 32) {
            const int e = s * G + j;
            homestart[e] = off_home + homeincl[e] - pad_to(nhome[e], tp);
            if (h >= 0) {
                const int q = qidx[s * G + j];
                const int p = pad_to(nrecv[s * G + j], tp);
                recvstart[s * G + j] = q < 0 ? -1
                                       : q < B ? off_slot + slotincl[s * B + q] - p
                                               : off_ovf + ovfincl[s * G + j] - p;
            }
        }
    }
    __syncthreads();
    PLAN_TRACE(3);

    // padded running total of rank s up to and including row i
    auto upto = [&](int s, int i) -> int {
        int v = 0;
        const int hs = s * G;
        if (i >= hs) v += i < hs + G ? homeincl[i] : s_hsize[s];
        const int h = s_rfrom[s];
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

    // ---------------- C. outputs ----------------
    if (blockIdx.x == 0) {
        for (int j = tid; j < R; j += kPlanThreads) {
            a.plan.assign[4 * j + 0] = s_keep[j];
            a.plan.assign[4 * j + 1] = s_rfrom[j];
            a.plan.assign[4 * j + 2] = s_rstart[j];
            a.plan.assign[4 * j + 3] = s_rlen[j];
        }
    }
    {
        const int64_t total = (int64_t)R * NR;
        const int64_t per = (total + gridDim.x - 1) / gridDim.x;
        const int64_t i0 = (int64_t)blockIdx.x * per, i1 = min(total, i0 + per);
        for (int64_t idx = i0 + tid; idx < i1; idx += kPlanThreads) {
            const int s = (int)(idx / NR), i = (int)(idx - (int64_t)s * NR);
            a.plan.cu_seqlens[idx] = upto(s, i);
            a.plan.row_counts[idx] = count_of(s, i);
        }
        const int64_t tb = (int64_t)R * B;
        const int64_t perb = (tb + gridDim.x - 1) / gridDim.x;
        const int64_t b0 = (int64_t)blockIdx.x * perb, b1 = min(tb, b0 + perb);
        for (int64_t idx = b0 + tid; idx < b1; idx += kPlanThreads) {
            const int s = (int)(idx / B), b = (int)(idx - (int64_t)s * B);
            a.plan.slot_expert[idx] = b < s_nslot[s] ? s_rfrom[s] * G + slotj[idx] : -1;
        }
    }
    __syncthreads();
    PLAN_TRACE(13);
    // per-expert dst bases: kept picks land at kbase + g; donated picks of the
    // first recipient overlapping the expert land at ebase + g while g < eend
    int32_t *kbase = homestart, *ebase = nrecv, *eend = ovfincl;
    for (int e = tid; e < E; e += kPlanThreads) {
        const int h = e / G;
        kbase[e] = h * d.nvs + homestart[e] - es[e];
        const int k = edon[e];
        if (k >= 0) {
            const int s = s_dlist[k];
            ebase[e] = s * d.nvs + recvstart[s * G + (e - h * G)] - max(es[e], s_rstart[s]);
            eend[e] = s_rstart[s] + s_rlen[s];
        } else {
            ebase[e] = 0;
            eend[e] = 0;
        }
    }
    __syncthreads();
    PLAN_TRACE(14);
    // destination of every pick of this block's chunk
    for (int i = tid; i < n_ent; i += kPlanThreads) {
        const int e = ent_e[i];
        const int h = e / G;
        const int g = es[e] + pre[e] + ent_rank[i];
        int dst;
        if (g < s_keep[h]) {
            dst = kbase[e] + g;
        } else if (g < eend[e]) {
            dst = ebase[e] + g;
        } else {  // the expert's donated run spans several recipients
            int dest = -1;
            for (int k = edon[e] + 1; k >= 1 && k < s_doff[h + 1]; ++k) {
                const int s = s_dlist[k];
                if (g < s_rstart[s] + s_rlen[s]) {
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
    PLAN_TRACE(4);
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
